/*
 * stepq.h -- C ABI of the packed-state gated Delta-rule decode step (STEPQuant).
 *
 * The method (pages: ai.info summary "STEPQuant: When and Where Errors Matter
 * in Delta-Rule Recurrent State Quantization", sections "Key Contributions" and
 * "Methodology in Plain English"; ai-papers.net article, section
 * "STEPQuantの仕組み"; ai-trend.me review, sections "방법" and "핵심 용어"):
 * every concurrent request keeps one recurrent state S [dk x dv] per head.  The
 * state is stored packed -- key-row scale x value-column scale x integer code,
 * with a bit width per unit (a head for Gated-DeltaNet, a key row for KDA) and
 * a few FP16 "pivot" units -- and one decode step reconstructs it, applies the
 * gated Delta update, reads out o = S^T q, refits the scales and writes the
 * packed state back.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are CUDA device pointers on the current device;
 *     "host" pointers are read during the call only.  All device tensors are
 *     contiguous fp32, row-major in the shapes given, and 16-byte aligned,
 *     except the [batch, heads] tensors (beta, and alpha of Gated-DeltaNet),
 *     which need 4-byte alignment only.
 *   - The caller owns every buffer passed in.  The library allocates no device
 *     memory and never frees a caller buffer.
 *   - Kernels are enqueued on the pool's stream (or the stream argument) and
 *     the call returns without synchronising; results are ready when that
 *     stream reaches the point of the call.
 *   - Arguments are validated on the host before any launch; an invalid call
 *     returns an error status and enqueues nothing.  A failed launch returns
 *     STEPQ_ERR_CUDA.  No call throws or aborts.  stepq_last_error() returns a
 *     one-line description of the last failure on the calling thread.
 *   - Only dk = dv = 128 is implemented (other sizes: STEPQ_ERR_UNSUPPORTED).
 */
#ifndef STEPQ_H
#define STEPQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the shared library (built with hidden default visibility). */
#if defined(__GNUC__)
#define STEPQ_API __attribute__((visibility("default")))
#else
#define STEPQ_API
#endif

typedef enum {
    STEPQ_OK = 0,
    STEPQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad table entry, misalignment */
    STEPQ_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement */
    STEPQ_ERR_CUDA = 3,        /* a CUDA call or kernel launch failed */
    STEPQ_ERR_STATE = 4        /* the pool handle is not usable (e.g. destroyed) */
} stepq_status;

/* Gate kinds.  Gated-DeltaNet: one retention gate per (request, head), and the
 * unit of bit allocation is the head.  KDA (Kimi Delta Attention): one gate per
 * key row, and the unit of bit allocation is the key row (ai.info summary,
 * "Future Directions"; ai-papers.net, "STEPQuantの仕組み"). */
#define STEPQ_GDN 0
#define STEPQ_KDA 1

/* Row width meaning "FP16 pivot": the row is stored as dv binary16 values and
 * takes no part in the scale fit (ai.info summary, "Key Contributions"). */
#define STEPQ_PIVOT_BITS 16

/* Scale fits (stepq_pool_set_scale_mode).  STEPQ_SCALE_DUAL is the method;
 * the others are the ablation variants the pages compare it with. */
#define STEPQ_SCALE_DUAL 0
#define STEPQ_SCALE_ROW 1
#define STEPQ_SCALE_COL 2
#define STEPQ_SCALE_HEAD 3

/* Largest batch * heads a pool may hold. */
#define STEPQ_MAX_ITEMS (1 << 24)

typedef struct {
    int variant;  /* STEPQ_GDN or STEPQ_KDA */
    int batch;    /* requests, >= 0 (0 gives an empty pool; every call is a no-op) */
    int heads;    /* heads per request, >= 1 */
    int dk, dv;   /* key and value dimension; 128 and 128 */
    int ls_iters; /* least-squares rounds of the column-scale fit, 0..8 (1 is the default) */
    /* host [heads * dk]: width of key row i of head h, in bits: 2..8, or 16 for
     * an FP16 pivot row.  Gated-DeltaNet requires one width per head. */
    const uint8_t *bits;
    /* host [heads * dk]: calibrated row-impact weight of key row i of head h,
     * finite and > 0 (pivot rows: ignored).  Fixed for all requests.  It
     * enters the row scale as max(rho_i, rho_max / 4)^(-1/2), rho_max the
     * largest weight among the head's quantised rows (a row is coarsened by
     * at most a factor 2 against the head's highest-impact row), and the
     * column-scale fit as the weight of the row's squared error. */
    const float *rho;
} stepq_desc;

typedef struct stepq_pool stepq_pool; /* opaque handle */

/*
 * Device bytes the caller must provide for a pool: the packed states of all
 * batch * heads items followed by the library's small per-head tables.
 * Returns 0 if the descriptor is invalid or unsupported.
 *
 * Packed state layout (offsets in bytes from the start of the buffer):
 *   item (b, h) starts at b * R + P_h, R = sum over heads of the item sizes,
 *   P_h = sum of the item sizes of heads 0..h-1;
 *   item = r[dk] fp32 | c[dv] fp32 | slab 0 | ... | slab dv/16 - 1.
 *   Slab s covers value columns 16s .. 16s+15 of all dk key rows and holds
 *   32 interleaved streams: stream l (rg = l % 8, cg = l / 8) carries the
 *   fields of key rows 16rg .. 16rg+15 and value columns 16s + 4cg .. +3,
 *   row-major (row 16rg, its 4 columns first), packed little-endian into
 *   32-bit words and zero-padded to W words.  The fields of row 16rg + p
 *   (position p) are F_p bits wide, F_p = the largest width at position p
 *   over the 8 row groups, so every stream of a head has the same layout and
 *   W = ceil(4 * (F_0 + ... + F_15) / 32); for a head of one width b,
 *   F_p = b and W = 2b.  Word m of stream l sits at slab byte offset
 *   4 * (32 m + l), so a slab takes 128 W bytes and an item
 *   4 dk + 4 dv + 1024 W bytes.  "Key row" above means storage row: a head
 *   whose rows all have one width stores them in key order; otherwise the key
 *   rows are sorted by width (widest first, a pivot row counting 16, ties by
 *   key index) and the j-th sorted row is storage row
 *   16 (j % (dk/16)) + j / (dk/16).  r[] is in storage order too.  A field
 *   of a quantised row holds the offset-binary code (code + 2^(F_p - 1));
 *   a field of a pivot row (F_p = 16) holds the binary16 bits of the
 *   element.  The stored element is r_i * c_j * code_ij (ai-papers.net,
 *   "STEPQuantの仕組み"); pivot rows keep r_i = 0, and a Gated-DeltaNet
 *   pivot head keeps c_j = 0 as well.  The interleave lets the 32 lanes of a
 *   warp that own one slab read and write it in whole 128-byte lines.
 */
STEPQ_API size_t stepq_pool_bytes(const stepq_desc *desc);

/* Bytes of the packed states alone (the prefix of the pool buffer that holds
 * the items); 0 if the descriptor is invalid. */
STEPQ_API size_t stepq_state_bytes(const stepq_desc *desc);

/*
 * Where a pool buffer's regions lie (byte offsets from its start), for
 * inspection and tests; the pages describe no counterpart.  The packed states
 * come first, then the library's tables: the per-head records, the item
 * offsets within a request and the item sizes per head, the device status
 * word, the item order and the staging records (one per item, 16 bytes:
 * item, item bytes | head << 16, item offset / 1024, request).  Every region
 * is followed by a guard region of guard_bytes bytes (guards[0] after the
 * states, then one after each table in that order) that pool creation fills
 * with a fixed pattern and stepq_pool_check_guards compares.
 * STEPQ_ERR_INVALID_ARG / STEPQ_ERR_UNSUPPORTED for an invalid descriptor.
 */
typedef struct {
    size_t states, state_bytes;
    size_t head_records, head_offsets, item_sizes, status_word, item_order, staging_records;
    size_t guards[7];
    size_t guard_bytes;
    size_t total; /* == stepq_pool_bytes(desc) */
} stepq_pool_regions;
STEPQ_API stepq_status stepq_pool_layout(const stepq_desc *desc, stepq_pool_regions *out);

/*
 * Create a pool over a caller-owned device buffer of at least
 * stepq_pool_bytes(desc) bytes (16-byte aligned).  Copies the descriptor and
 * the host tables, writes the derived per-head tables into the tail of the
 * buffer, and synchronises the given stream once before returning (creation is
 * not on the decode path).  The packed states are left uninitialised: call
 * stepq_pack before the first decode step.  cuda_stream is a cudaStream_t
 * (NULL = the legacy default stream); it can be changed with
 * stepq_pool_set_stream.  On success *out receives the handle.
 */
STEPQ_API stepq_status stepq_pool_create(const stepq_desc *desc, void *dev_buf, size_t bytes,
                               void *cuda_stream, stepq_pool **out);

/* Release the handle (host memory only; the device buffer stays the caller's).
 * Passing NULL returns STEPQ_ERR_INVALID_ARG. */
STEPQ_API stepq_status stepq_pool_destroy(stepq_pool *pool);

/* The scale fit of the pool's later stepq_pack, stepq_decode_step and
 * stepq_decode_step_split calls (default STEPQ_SCALE_DUAL, the method: row
 * scales from magnitude and impact, least-squares column scales).  The
 * ablation variants (ai.info, "Main Findings": the method against
 * spatial-only, temporal-only and uniform settings; state outliers lie along
 * key rows and value columns at once) keep the stored form r_i c_j code_ij
 * with plain absolute-maximum scales, no impact weights and no least squares:
 *   STEPQ_SCALE_ROW : c_j = 1, r_i = max_j |S_ij| / Q_i (a zero row: 1 / Q_i);
 *   STEPQ_SCALE_COL : r_i = 1 / Q_i, c_j = max_i |S_ij| (a zero column: 1);
 *   STEPQ_SCALE_HEAD: r_i = 1 / Q_i, every c_j the largest |S_ij| of the
 *                     state (one scale per (request, head)).
 * Pivot rows are kept in binary16 in every mode.  Host-only; takes effect on
 * the next call.  STEPQ_ERR_INVALID_ARG for another mode. */
STEPQ_API stepq_status stepq_pool_set_scale_mode(stepq_pool *pool, int mode);

/* Stream on which the pool's later calls enqueue their kernels. */
STEPQ_API stepq_status stepq_pool_set_stream(stepq_pool *pool, void *cuda_stream);

/*
 * Restrict the pool's later decode steps to the requests active[0 ..
 * n_active) (host array of distinct request indices in 0 .. batch-1, read
 * during the call; NULL = every request, n_active ignored) -- the slot-indexed
 * pool of a serving runtime, where requests come and go between steps and
 * each keeps its slot of the state pool, as in a KV-cache allocation
 * (ai.info summary, "Why This Matters": the packed state replaces the
 * runtime's per-request state storage).  stepq_decode_step keeps its
 * [batch, heads, ...] tensor shapes, indexed by request slot: it reads the
 * rows of q, k, v, alpha, beta and writes the rows of out of the active
 * requests only, and updates only their states; the other rows and states
 * are neither read nor written.  The item order and staging tables in the
 * pool buffer's tail are rebuilt on the host (heaviest heads first) and
 * uploaded on the pool's stream (no sync).  stepq_pack, stepq_unpack and
 * stepq_decode_step_split always cover every request (split returns
 * STEPQ_ERR_UNSUPPORTED while a subset is active).
 */
STEPQ_API stepq_status stepq_pool_set_active(stepq_pool *pool, const int *active, int n_active);

/*
 * Fit and quantise full-precision states into the pool (the initial state of
 * every item, or a restore from a checkpoint).  S: device fp32
 * [batch, heads, dk, dv].  Per item: row scales from the row's root-mean-square
 * magnitude and impact weight (r_i = rms_i max(rho_i, rho_max / 4)^(-1/2) /
 * Q_i), column scales by least squares, codes by
 * round-half-even with clamping -- the same fit the decode step performs after
 * its update (ai.info summary, "Methodology in Plain English").
 */
STEPQ_API stepq_status stepq_pack(stepq_pool *pool, const float *S);

/* Dequantise every item into S_out: device fp32 [batch, heads, dk, dv],
 * S_ij = (r_i * c_j) * code_ij, or the stored binary16 value on pivot rows. */
STEPQ_API stepq_status stepq_unpack(stepq_pool *pool, float *S_out);

/*
 * One decode step for every (request, head) item of the pool, in one fused
 * kernel: reconstruct the state from the packed pool, apply the gated Delta
 * update, read out, refit the scales, requantise and write the packed state
 * back in place (ai.info summary, "Key Contributions" and "Methodology in
 * Plain English"; ai-trend.me, "핵심 용어: Gated Delta Rule").
 *   S'   = diag(alpha) S      (one alpha per item for GDN, per key row for KDA)
 *   vold = S'^T k
 *   S    = S' + beta k (v - vold)^T
 *   out  = S^T q              (from the updated, unquantised state)
 * Inputs (device fp32): q, k [batch, heads, dk]; v [batch, heads, dv];
 * alpha [batch, heads] (GDN) or [batch, heads, dk] (KDA), each in (0, 1];
 * beta [batch, heads].  Output: out [batch, heads, dv] (device fp32; must not
 * alias an input).  Values are not range-checked on the device.
 */
STEPQ_API stepq_status stepq_decode_step(stepq_pool *pool, const float *q, const float *k, const float *v,
                               const float *alpha, const float *beta, float *out);

/*
 * The same decode step as stepq_decode_step computed the way the pages'
 * serving kernels split it (ai.info summary, "Key Contributions": the
 * reconstruction, Delta update and readout fused, with scale fitting and
 * packed writeback on a separate CUDA stream): one kernel reconstructs,
 * updates and reads out, writing the updated unquantised state to S_work;
 * then the fit and packed writeback (the stepq_pack kernel on S_work) run on
 * side_stream, which waits for the first kernel, and the pool's stream waits
 * for them.  Kept to measure the split against the single fused pass; the
 * results agree with stepq_decode_step within rounding.  S_work: device fp32
 * [batch, heads, dk, dv], 16-byte aligned, caller-owned, overwritten; must not
 * overlap the pool or the step tensors.  side_stream: cudaStream_t; NULL or the
 * pool's stream runs both halves on the pool's stream.  Other arguments as in
 * stepq_decode_step.
 */
STEPQ_API stepq_status stepq_decode_step_split(stepq_pool *pool, float *S_work, const float *q, const float *k,
                                               const float *v, const float *alpha, const float *beta, float *out,
                                               void *side_stream);

/*
 * The same update and readout on an unquantised fp32 state, in place: the
 * full-precision baseline the packed step is measured against.  S: device fp32
 * [batch, heads, dk, dv]; other tensors as in stepq_decode_step.  Uses only
 * desc->variant, batch, heads, dk, dv.  cuda_stream: cudaStream_t or NULL.
 */
STEPQ_API stepq_status stepq_fp32_step(const stepq_desc *desc, float *S, const float *q, const float *k,
                             const float *v, const float *alpha, const float *beta, float *out,
                             void *cuda_stream);

/*
 * Synchronise the pool's stream and read the pool's device status word.  The
 * fused decode kernel stages items with asynchronous copies and waits for them
 * with a bounded wait; if a wait ever gave up (the copy did not land within
 * about two seconds), the kernel records it there and stops, leaving the
 * remaining items of that step un-updated.  Returns STEPQ_OK if no kernel
 * reported an error since the last check, else STEPQ_ERR_CUDA (and clears the
 * word).
 */
STEPQ_API stepq_status stepq_pool_check(stepq_pool *pool);

/*
 * Failure-detection self-test (no counterpart on the pages): one CTA runs the
 * bounded barrier wait the decode kernel uses for its staged copies, on a
 * barrier that needs one arrival.  With arrive != 0 the thread arrives first
 * and the wait completes; with arrive == 0 nothing arrives and the wait gives
 * up after limit_cycles SM clock cycles, as a wait for a copy that never lands
 * would.  result: device int[2], written with result[0] = 0 (completed) or 1
 * (gave up: the decode kernel's timeout status) and result[1] = cycles spent
 * waiting (saturated at 2^31 - 1).  limit_cycles in [0, 2^34] (up to about 8 s
 * at the B200's clock), else STEPQ_ERR_INVALID_ARG.  Asynchronous on
 * cuda_stream (cudaStream_t or NULL); nothing else is touched, so the context
 * stays usable after a wait that gave up.
 */
STEPQ_API stepq_status stepq_selftest_bounded_wait(int *result, long long limit_cycles, int arrive,
                                                   void *cuda_stream);

/*
 * Memory-safety aid (no counterpart on the pages): synchronise the pool's
 * stream and compare the guard regions that follow every region of the pool
 * buffer (see stepq_pool_layout) with the pattern pool creation wrote.  A
 * kernel write beyond the packed states or a table shows up here.  Returns
 * STEPQ_OK, or STEPQ_ERR_STATE naming the first changed guard word in
 * stepq_last_error(); STEPQ_ERR_CUDA if the copy back fails.  Host memory
 * only on the stack; the guards are not rewritten.
 *
 * A library built with STEPQ_CHECK=1 (libstepq_check.so, loaded by the Python
 * binding when the environment variable STEPQ_CHECK is 1) also validates, in a
 * kernel launched before every kernel that reads the pool's tables, each head
 * record and staging record against the layout: item and head in range, the
 * item's size equal to its head's, its offset equal to request x request bytes
 * + the head's offset and inside the packed states, the order table equal to
 * the staging records.  A violation sets the status word (reported by
 * stepq_pool_check) and the dependent kernels return without touching memory;
 * while the word is set, later launches do nothing.
 */
STEPQ_API stepq_status stepq_pool_check_guards(stepq_pool *pool);

/*
 * The fused decode step of stepq_decode_step without a pool, allocating
 * nothing.  The pages describe no counterpart: it is a deployment variant of
 * the same kernel and computes exactly what stepq_decode_step computes.
 *
 * For callers that keep the packed states in memory they manage themselves
 * and may not allocate at decode time -- e.g. a serving runtime that gives all
 * free HBM to its own caching allocator, where a cudaMalloc would fail or
 * synchronise the device.  The kernel's scratch tables (per-head records, item
 * order, staging records, status word) live in a fixed file-scope device
 * array of 256 KiB inside the library instead of a pool buffer's tail; every
 * call rebuilds them on the host and uploads them on the stream before its
 * launch.  No device or host memory is allocated on the success path (an
 * error message may be formatted into the library's per-thread error string).
 *
 * The upload is a cudaMemcpyAsync from a static, pageable host image, and CUDA
 * starts a copy from pageable host memory only after the work queued earlier
 * on the stream has finished: each call therefore blocks the calling thread
 * until the stream has drained up to it, then returns with its own kernel
 * queued (unlike the pool entry points, which return without waiting).
 *
 * desc: as for stepq_pool_create, with heads <= 64 and tables that fit the
 * scratch (about 10 000 items at 32 heads, 7 500 at 64); larger descriptors
 * return STEPQ_ERR_UNSUPPORTED with the sizes in stepq_last_error().
 * states: device, state_bytes >= stepq_state_bytes(desc), 16-byte aligned,
 * laid out as a pool's packed states (e.g. packed by stepq_pack of a pool
 * with the same descriptor, then copied); updated in place.  q, k, v, alpha,
 * beta, out: as for stepq_decode_step.  cuda_stream: cudaStream_t or NULL.
 *
 * Calls share the one scratch array per device: two calls in flight at the
 * same time (on different streams or threads) race on it, so order them on
 * one stream.  The first call on a device looks up the scratch address
 * (cudaGetSymbolAddress).  The status word the kernel writes when a staged copy never lands is cleared by
 * the next call and not reported here; use a pool and stepq_pool_check where
 * that report is needed.
 */
STEPQ_API stepq_status stepq_decode_step_noalloc(const stepq_desc *desc, void *states, size_t state_bytes,
                                                 const float *q, const float *k, const float *v,
                                                 const float *alpha, const float *beta, float *out,
                                                 void *cuda_stream);

/* ---- calibration: the offline step that makes a pool's tables ------------ *
 * The pages fix a unit's width, once for all requests, from its quantisation
 * distortion at candidate widths and its mean log retention under an average
 * bit budget, keep the riskiest few units as FP16 pivots, and give every key
 * row an impact score, the expected squared weight of its error in the
 * readout (ai.info, "Methodology in Plain English" and "Key Contributions";
 * ai-papers.net, "STEPQuantの仕組み"; ai-trend.me, "방법").  Units: heads
 * (Gated-DeltaNet) or key rows (KDA).  This library's readings:
 *   rho_i = mean over calibration requests and steps of q_i^2 (floored at
 *   1e-30); lifetime weight w_u = 1 / (1 - abar_u^2) with abar_u =
 *   exp(mean log alpha_u) (1 - abar^2 floored at 1e-12); distortion D_u(b) =
 *   sum over sampled fp32 rollout states of sum_(rows i of u) rho_i
 *   sum_j (S_ij - r_i c_j code_ij)^2, all rows of the head fitted at width b;
 *   allocation: all units at the narrowest width, the ceil(pivot_frac * units)
 *   units of largest w_u D_u(narrowest) made pivots (16 bits, in the budget),
 *   then repeatedly the upgrade to the next candidate width with the largest
 *   w_u (D_u(b) - D_u(b')) / (b' - b) > 0 that fits the remaining budget
 *   round(avg_bits * units); ties go to the lower unit index.
 * dk = dv = 128.  The piecewise calls below are what stepq_calibrate runs;
 * they are exported for inspection and tests. */
typedef struct {
    int variant;        /* STEPQ_GDN or STEPQ_KDA */
    int batch, heads, dk, dv;  /* calibration requests; dk = dv = 128 */
    int steps;          /* rollout length T >= 1 */
    int sample_every;   /* states sampled after steps t with (t + 1) % sample_every == 0 */
    int ls_iters;       /* least-squares rounds of the fits (as the pool's) */
    int n_widths;       /* 1 .. 8 candidate widths */
    const int *widths;  /* host, strictly ascending, each in 2..8 */
    double avg_bits;    /* average width budget per unit, pivots counted at 16 */
    double pivot_frac;  /* share of units kept as FP16 pivots (ceil) */
} stepq_calib_desc;

/* Device scratch bytes stepq_calibrate needs for cd (0 if cd is invalid). */
STEPQ_API size_t stepq_calib_scratch_bytes(const stepq_calib_desc *cd);

/* The whole calibration, synchronous on cuda_stream (cudaStream_t or NULL):
 * the impact scores from every step's q and the retention sums from every
 * step's alpha; then the unquantised fp32 rollout from S0 (device,
 * [batch][heads][dk][dv], not modified) over the same inputs, the per-row
 * errors of every candidate width measured on the states after each sampled
 * step; then the widths.  q, k: device [steps][batch][heads][dk]; v: device
 * [steps][batch][heads][dv]; alpha: device [steps][batch][heads] (GDN) or
 * [steps][batch][heads][dk] (KDA); beta: device [steps][batch][heads]; all
 * fp32, 16-byte aligned (alpha and beta 4-byte for GDN).  scratch: device,
 * at least stepq_calib_scratch_bytes, 256-byte aligned, caller-owned.
 * Outputs (host): rho_out [heads*dk] and bits_out [heads*dk] (16 = pivot;
 * every row of a Gated-DeltaNet head alike), ready for stepq_desc.
 * STEPQ_ERR_INVALID_ARG when the pivots and the narrowest width alone exceed
 * the budget. */
STEPQ_API stepq_status stepq_calibrate(const stepq_calib_desc *cd, const float *S0, const float *q,
                                       const float *k, const float *v, const float *alpha, const float *beta,
                                       void *scratch, size_t scratch_bytes, void *cuda_stream, float *rho_out,
                                       uint8_t *bits_out);

/* One step's inputs into the running sums (asynchronous): acc_q2[h*dk+i] +=
 * sum_b q[b][h][i]^2 and acc_loga[u] += sum_b log alpha[b][u] (u = h, or
 * h*dk+i for KDA), in fp64, requests in order.  q: device [batch][heads][dk];
 * alpha: device [batch][heads] (GDN) or [batch][heads][dk]; acc_q2: device
 * fp64 [heads*dk]; acc_loga: device fp64 [heads] or [heads*dk]. */
STEPQ_API stepq_status stepq_calib_accumulate(int variant, int batch, int heads, const float *q,
                                              const float *alpha, double *acc_q2, double *acc_loga,
                                              void *cuda_stream);

/* Per-row squared errors of batch*heads fp32 states (asynchronous): state s
 * = (request, head s % heads) fitted and quantised with every row at
 * widths[x] (as stepq_pack would, rho = rho[head]) gives err[(s*n_widths +
 * x)*dk + i] = r'_i^2 sum_j (p_ij - c_j code_ij)^2 (fp32) and its r' and c in
 * rc[(s*n_widths + x)*(dk + dv) ..].  S: device [batch*heads][dk][dv]; rho:
 * device [heads*dk]; widths: host, as in stepq_calib_desc; err, rc: device. */
STEPQ_API stepq_status stepq_calib_row_error(int batch, int heads, const float *S, const float *rho,
                                             int n_widths, const int *widths, int ls_iters, float *err,
                                             float *rc, void *cuda_stream);

/* err_sum[(h*n_widths + x)*dk + i] += err of request b, for b = 0, 1, ... in
 * turn (fp64, asynchronous).  err: device, as written by
 * stepq_calib_row_error; err_sum: device fp64 [heads][n_widths][dk]. */
STEPQ_API stepq_status stepq_calib_reduce(int batch, int heads, int n_widths, const float *err,
                                          double *err_sum, void *cuda_stream);

/* Host: rho[u] = fp32(max(acc_q2[u] / n_samples, 1e-30)), u < heads*dk. */
STEPQ_API stepq_status stepq_calib_rho(int heads, double n_samples, const double *acc_q2, float *rho);

/* Host: the widths bits [heads*dk] from the sums (n_samples terms per unit in
 * acc_loga; err_sum [heads][n_widths][dk]) and rho [heads*dk], by the
 * allocation above.  STEPQ_ERR_INVALID_ARG when the budget is infeasible. */
STEPQ_API stepq_status stepq_calib_bits(int variant, int heads, double n_samples, const double *acc_loga,
                                        const float *rho, const double *err_sum, int n_widths,
                                        const int *widths, double avg_bits, double pivot_frac,
                                        uint8_t *bits);

/* Human-readable name of a status; never NULL. */
STEPQ_API const char *stepq_status_string(stepq_status s);

/* One-line description of the last failure on this thread ("" if none). */
STEPQ_API const char *stepq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* STEPQ_H */
