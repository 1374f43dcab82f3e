// Internal declarations shared by the host library and the kernels of the
// packed-state gated Delta-rule decode step.  Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace stepq {

constexpr int kDK = 128;          // key dimension (rows of a state)
constexpr int kDV = 128;          // value dimension (columns of a state)
constexpr int kThreads = 256;     // threads per item (8 warps)
constexpr int kRowsPerGroup = 16; // key rows of a stream's row group = rows a thread holds
constexpr int kRowGroups = kDK / kRowsPerGroup;
constexpr int kSlabCols = 16;     // value columns of a slab = columns a warp owns
constexpr int kSlabs = kDV / kSlabCols;
constexpr int kStreams = 32;      // streams per slab: 8 row groups x 4 column groups of 4
constexpr int kPivotBits = 16;
// scale fits: the method, and the ablation variants (row scales only, column
// scales only, one scale per state); the values of STEPQ_SCALE_*
constexpr int kScaleDual = 0, kScaleRow = 1, kScaleCol = 2, kScaleHead = 3;
constexpr int kHeaderBytes = 4 * kDK + 4 * kDV;  // r[dk] | c[dv]
constexpr int kMaxSlots = 8;

// Head kinds.
constexpr int kHeadQuant = 0;     // every row quantised
constexpr int kHeadAllPivot = 1;  // every row a binary16 pivot
constexpr int kHeadMixed = 2;     // some rows pivots

// Per-head record (host-built, staged with every item): the fit constants and
// the tile layout of the head's items.
struct HeadRec {
    float s[kDK];                // fp32(max(rho_i, rho_max / 4)^-1/2), rounded once from fp64 (0 on pivot rows), by storage row
    float rho[kDK];              // row-impact weights (0 on pivot rows)
    float rq[kDK];               // fp32(1 / Q_i), Q_i = 2^(b_i - 1) - 1 (0 on pivot rows)
    // per storage row (key order for a one-width head; otherwise the key rows
    // sorted by width and dealt to the row groups in turn):
    uint8_t bits[kDK];           // row widths (16 = pivot)
    uint8_t key_row[kDK];        // the key row stored as this row
    // field width of each row position p (storage rows 16 g + p): the widest
    // row at that position over the row groups; every stream of the head
    // lays out its fields alike.  Positions of 16-bit fields (pivot rows)
    // come first: n16 of them.
    uint8_t pos_bits[kRowsPerGroup];
    // bit offset of row position p in every stream: 4 x the sum of the
    // widths of the positions before it (a per-head constant)
    uint16_t pos_off[kRowsPerGroup];
    long long head_off;          // byte offset of the head's item inside a request
    int head_b;                  // common row width, 0 if the rows differ
    int head_kind;               // kHeadQuant / kHeadAllPivot / kHeadMixed
    int head_bytes;              // bytes of one item
    int slab_words;              // 32-bit words per stream (W)
    int n16;
    int pad;
};
static_assert(offsetof(HeadRec, pos_bits) % 16 == 0, "pos_bits is read as one 16-byte vector");
static_assert(sizeof(HeadRec) % 16 == 0, "head record must be a multiple of 16 bytes");

// Per-head tables derived on the host at pool creation, resident in the tail
// of the caller's pool buffer.
struct Tables {
    const HeadRec *rowrec;      // [H] head records
    const long long *head_off;  // [H] byte offset of head h's item inside a request
    const int *head_bytes;      // [H] bytes of an item of head h
    const int *order;           // [B*H] item processing order: all-pivot heads' items first
    // [B*H] per position: {item, item bytes | head << 16, state offset / 1024, request}
    const int4 *stage;
    int *status;                // device status word: 0 ok, else an error code
};

struct StepArgs {
    uint8_t *pool;
    Tables t;
    long long req_bytes;  // bytes of one request's items
    int heads;
    int n_items;
    int ls_iters;
    int kda;
    // staging ring of the fused decode kernel
    int nslots;
    int slot_bytes;
    int off_q, off_k, off_v, off_alpha, off_ab, off_rec;  // offsets inside a slot
    int n_pivot_items;  // items of all-pivot heads, placed first in the order
    int max_n16;        // the most leading 16-bit field positions of any other head
    int scale_mode;     // kScaleDual (the method) or an ablation variant
    int batch;                // requests of the pool (the layout's, also for an active subset)
    long long state_bytes;    // bytes of the packed states (the checking build validates against it)
    const float *q, *k, *v, *alpha, *beta;
    float *out;
    const float *S_in;  // pack
    float *S_out;       // unpack
};

// Device status codes.
constexpr int kStatusWaitTimeout = 1;
constexpr int kStatusBadHead = 2;
constexpr int kStatusBadTable = 3;  // the checking build (STEPQ_CHECK) found an inconsistent table entry

cudaError_t launch_decode_step(const StepArgs &a, cudaStream_t s);
cudaError_t launch_pack(const StepArgs &a, cudaStream_t s);
cudaError_t launch_unpack(const StepArgs &a, cudaStream_t s);
// The pages' split pipeline, first half: reconstruct, update, read out; the
// updated unquantised state goes to a.S_in (a work buffer), for launch_pack.
cudaError_t launch_split_update(const StepArgs &a, cudaStream_t s);
// Self-test of the bounded barrier wait the kernels use (one CTA): result[0] =
// 0 or kStatusWaitTimeout, result[1] = cycles waited (saturated).
cudaError_t launch_wait_selftest(int *result, long long limit, int arrive, cudaStream_t s);
// Calibration kernels (the offline step that makes a pool's tables).
constexpr int kCalibMaxWidths = 8;
struct CalibArgs {
    int batch, heads, kda;
    int n_widths;
    int widths[kCalibMaxWidths];   // candidate widths, 2..8
    int ls_iters;
    const float *S;                // [batch*heads][dk][dv] fp32 states
    const float *rho;              // [heads*dk] impact scores
    float *err;                    // [batch*heads][n_widths][dk] per-row squared errors
    float *rc;                     // [batch*heads][n_widths][dk + dv] fitted r', c
    double *err_sum;               // [heads][n_widths][dk]
    const float *q, *alpha;        // one step's inputs
    double *acc_q2, *acc_loga;     // [heads*dk], [heads] or [heads*dk]
};
cudaError_t launch_calib_accumulate(const CalibArgs &c, cudaStream_t s);
cudaError_t launch_calib_error(const CalibArgs &c, cudaStream_t s);
cudaError_t launch_calib_reduce(const CalibArgs &c, cudaStream_t s);

cudaError_t launch_fp32_step(float *S, const float *q, const float *k, const float *v,
                             const float *alpha, const float *beta, float *out, int n_items,
                             int kda, cudaStream_t s);
// CTAs the fused decode kernel runs per SM and the dynamic shared memory it
// gets for nslots staging slots of slot_bytes each; 0 if it cannot run.
int decode_ctas_per_sm(int nslots, int slot_bytes);

}  // namespace stepq
