// Kernels of the packed-state gated Delta-rule decode step (sm_100a).
//
// Thread mapping (every kernel): a CTA of 256 threads owns one (request,
// head) item at a time; warp w owns key rows 16w .. 16w+15 (= packed tile w),
// lane l owns value columns 4l .. 4l+3 (= column group l), so a thread holds
// 64 state elements in registers and reads / writes exactly one column-group
// stream of one tile: the pool layout is built around this mapping.  The
// elements are kept as float2 pairs (columns 4l, 4l+1 and 4l+2, 4l+3) so that
// every floating-point operation on the state is one packed f32x2 instruction;
// per-row factors are stored duplicated, (x, x), so that broadcasting them
// costs nothing.
//
// Method (ai.info summary of STEPQuant, "Key Contributions" and "Methodology in
// Plain English"; ai-papers.net, "STEPQuantの仕組み"; ai-trend.me, "핵심 용어"):
//   reconstruct  S_ij = r_i c_j code_ij   (pivot rows: binary16 values)
//   gate         S'   = diag(alpha) S
//   update       S    = S' + (beta k)(v - S'^T k)^T
//   readout      o    = S^T q
//   refit        r_i  = rms_i rho_i^-1/2 / Q_i ; p = S / r ;
//                c_j  = max_i |p_ij| / Q_i, then least squares for fixed codes
//   requantise   code = clamp(rne(p / c)); pack; store.
//
// The fused decode kernel never forms S: with a_i = alpha_i r_i it carries the
// state in old-scale units, U_ij = S_ij / (a_i c_j) = code_ij + gamma_i dt_j
// (gamma_i = beta k_i / a_i, dt_j = d_j / c_j, d = v - v_old), then
// P_ij = c_j U_ij = S_ij / a_i, and the fit's p_ij = P_ij h_i with
// h_i = a_i / r'_i.  The key projection is v_old_j = c_j sum_i (a_i k_i) code_ij
// and the readout o_j = c_j sum_i (a_i q_i) code_ij + (beta k.q) d_j.
#include "stepq_device.cuh"

namespace stepq {
namespace {

using namespace dev;

constexpr long long kWaitLimit = 4000000000LL;  // SM clock cycles before a wait gives up
constexpr float kRoundMagic = 12582912.0f;      // 1.5 * 2^23: x + it rounds x to an integer

struct alignas(16) ItemSmem {
    float2 rk2[kDK], rl2[kDK], rg2[kDK], ra2[kDK];  // update factors per row, duplicated
    float2 rh2[kDK], rw2[kDK], rq2[kDK];            // fit factors per row, duplicated
    float ra[kDK], rs[kDK], rrho[kDK];              // a_i, s_i, rho_i
    int rb[kDK];                                    // row widths
    float cc[kDV], cv[kDV], cd[kDV], cdt[kDV], cu[kDV];
    float cc0[kDV], cnew[kDV], ci[kDV], crat[kDV];
    float red[2][8][kDV];
    float rowt[8][16][36];  // per-warp transposition for row sums
    float kq[4];
    float beta_item;
    uint32_t tile_off[kTiles];
    int head_b, head_kind;
    long long head_off;
    uint64_t bar[kMaxSlots];
    int4 prod_rec;          // producer (thread 0): staging record of position prod_n
    int prod_n;             // producer: next position to stage
    uint32_t prod_issued;   // producer: items staged so far
};

using X2 = float2[kRowsPerWarp][2];  // the thread's 16 x 4 block as float2 pairs

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float2 ld2(const float2 *p) { return *p; }

// Call-free reciprocal, quotient and square root (within 2 ulp of the correctly
// rounded results) for the per-row and per-column factors computed while the
// thread's state is live in registers: the correctly rounded forms branch to a
// slow-path subroutine whose call would force the state out to local memory.
__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float div_approx(float a, float b) { return a * rcp_approx(b); }
__device__ __forceinline__ float sqrt_approx(float x)
{
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 3-input maximum of a, |b| and |c|.
__device__ __forceinline__ float max_abs3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
    return r;
}

// ---------------------------------------------------------------------------
// Column sums over the 8 warps of per-thread partials.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void stash(ItemSmem &sm, int vec, float2 a, float2 b)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    *reinterpret_cast<float4 *>(&sm.red[vec][w][4 * l]) = make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float sum_partials(const ItemSmem &sm, int vec, int j)
{
    float acc = sm.red[vec][0][j];
#pragma unroll
    for (int w = 1; w < 8; w++) acc += sm.red[vec][w][j];
    return acc;
}

__device__ __forceinline__ float max_partials(const ItemSmem &sm, int vec, int j)
{
    float acc = sm.red[vec][0][j];
#pragma unroll
    for (int w = 1; w < 8; w++) acc = fmaxf(acc, sm.red[vec][w][j]);
    return acc;
}

// Half of a column reduction: the partials of warps 4 half .. 4 half + 3.
__device__ __forceinline__ float sum_partials4(const ItemSmem &sm, int vec, int j, int half)
{
    const float a = sm.red[vec][4 * half][j], b = sm.red[vec][4 * half + 1][j];
    const float c = sm.red[vec][4 * half + 2][j], d = sm.red[vec][4 * half + 3][j];
    return (a + b) + (c + d);
}

__device__ __forceinline__ float max_partials4(const ItemSmem &sm, int vec, int j, int half)
{
    const float a = sm.red[vec][4 * half][j], b = sm.red[vec][4 * half + 1][j];
    const float c = sm.red[vec][4 * half + 2][j], d = sm.red[vec][4 * half + 3][j];
    return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// The duplicated factors of two consecutive rows (p 16-byte aligned) in one load.
__device__ __forceinline__ void ld_pairs(const float2 *p, float2 (&out)[2])
{
    const float4 v = *reinterpret_cast<const float4 *>(p);
    out[0] = make_float2(v.x, v.y);
    out[1] = make_float2(v.z, v.w);
}

// ---------------------------------------------------------------------------
// Decode the thread's column-group stream of its tile into X (code values as
// floats; pivot rows: their binary16 values).  Fixed width B > 0 keeps the
// stream in registers; B == 0 reads widths per row from sm.rb.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void decode_stream(const ItemSmem &sm, const uint32_t *words, int stride, X2 &X)
{
    const int w = threadIdx.x >> 5;
    if constexpr (B > 0) {
        uint32_t wd[2 * B];
#pragma unroll
        for (int m = 0; m < 2 * B; m++) wd[m] = words[m * stride];
        const float mz = -(kMagic + (float)(1 << (B - 1)));
        const float2 mz2 = f2(mz, mz);
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++)
#pragma unroll
            for (int hh = 0; hh < 2; hh++) {
                const uint32_t u0 = field_at<B>(wd, 4 * rr + 2 * hh) | kMagicBits;
                const uint32_t u1 = field_at<B>(wd, 4 * rr + 2 * hh + 1) | kMagicBits;
                X[rr][hh] = __fadd2_rn(f2(__uint_as_float(u0), __uint_as_float(u1)), mz2);
            }
    } else {
        BitReader br;
        br.init(words, stride);
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++) {
            const int b = sm.rb[kRowsPerWarp * w + rr];
            if (b == kPivotBits) {
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    const uint32_t hv = br.take(32);
                    X[rr][hh] = __half22float2(*reinterpret_cast<const __half2 *>(&hv));
                }
            } else {
                const uint32_t f = br.take(4 * b);
                const uint32_t mask = (1u << b) - 1u;
                const float mz = -(kMagic + (float)(1 << (b - 1)));
                const float2 mz2 = f2(mz, mz);
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    const uint32_t u0 = ((f >> (2 * hh * b)) & mask) | kMagicBits;
                    const uint32_t u1 = ((f >> ((2 * hh + 1) * b)) & mask) | kMagicBits;
                    X[rr][hh] = __fadd2_rn(f2(__uint_as_float(u0), __uint_as_float(u1)), mz2);
                }
            }
        }
    }
}

// One least-squares round's partial sums over the thread's rows, stashed for
// the column reduction: with n = rne(p / c) (clipped to the row's range when
// CLIP), N_j = sum w_i n_ij p_ij and D_j = sum w_i n_ij^2.
template <int B, bool ROWWISE, bool CLIP>
__device__ __forceinline__ void ls_partials(ItemSmem &sm, const X2 &X)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int r0 = kRowsPerWarp * w;
    const float2 rm2 = f2(kRoundMagic, kRoundMagic), nrm2 = f2(-kRoundMagic, -kRoundMagic);
    const float4 i4 = ld4(&sm.ci[4 * l]);
    const float2 ic0 = f2(i4.x, i4.y), ic1 = f2(i4.z, i4.w);
    float2 N0 = f2(0.f, 0.f), N1 = N0, D0 = N0, D1 = N0;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr += 2) {
        float2 wp[2];
        ld_pairs(&sm.rw2[r0 + rr], wp);
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const int i = r0 + rr + u;
            if (ROWWISE && sm.rb[i] == kPivotBits) continue;
            // round to the nearest integer, ties to even: x + 1.5 * 2^23 - 1.5 * 2^23;
            // clipping acts on the biased value (for a fixed width the bounds are
            // immediates)
            float2 m0 = __ffma2_rn(X[rr + u][0], ic0, rm2);
            float2 m1 = __ffma2_rn(X[rr + u][1], ic1, rm2);
            if (CLIP) {
                const float Q = (float)qmax_of(ROWWISE ? sm.rb[i] : B);
                const float lo = kRoundMagic - Q, hi = kRoundMagic + Q;
                m0 = f2(fminf(fmaxf(m0.x, lo), hi), fminf(fmaxf(m0.y, lo), hi));
                m1 = f2(fminf(fmaxf(m1.x, lo), hi), fminf(fmaxf(m1.y, lo), hi));
            }
            const float2 n0 = __fadd2_rn(m0, nrm2), n1 = __fadd2_rn(m1, nrm2);
            const float2 wn0 = __fmul2_rn(wp[u], n0), wn1 = __fmul2_rn(wp[u], n1);
            N0 = __ffma2_rn(wn0, X[rr + u][0], N0);
            N1 = __ffma2_rn(wn1, X[rr + u][1], N1);
            D0 = __ffma2_rn(wn0, n0, D0);
            D1 = __ffma2_rn(wn1, n1, D1);
        }
    }
    stash(sm, 0, N0, N1);
    stash(sm, 1, D0, D1);
}

// The least-squares column scales from the stashed partials, two threads per
// column: c_j = N_j / D_j (kept when D_j = 0), its reciprocal, and c0_j / c_j.
__device__ __forceinline__ void ls_update_columns(ItemSmem &sm)
{
    const int j = threadIdx.x >> 1, half = threadIdx.x & 1;
    float nn = sum_partials4(sm, 0, j, half), dd = sum_partials4(sm, 1, j, half);
    nn += __shfl_xor_sync(0xffffffffu, nn, 1);
    dd += __shfl_xor_sync(0xffffffffu, dd, 1);
    if (half == 0) {
        const float c = (dd > 0.f) ? div_approx(nn, dd) : sm.cnew[j];
        const float icn = rcp_approx(c);
        sm.cnew[j] = c;
        sm.ci[j] = icn;
        sm.crat[j] = sm.cc0[j] * icn;
    }
}

// Final codes of a fixed-width tile stream and their store: u = z + clip(rne(p / c))
// taken from the low mantissa bits of p / c + 2^23 + z; each 32-bit word is
// stored as soon as its last code is placed.
template <int B, bool CLIP>
__device__ __forceinline__ void pack_fixed(const X2 &X, float2 ic0, float2 ic1, uint32_t *words)
{
    constexpr int Qb = (1 << (B - 1)) - 1;
    const float mz = kMagic + (float)(1 << (B - 1));
    const float2 mz2 = f2(mz, mz);
    uint32_t ow[2 * B + 1];
#pragma unroll
    for (int m = 0; m <= 2 * B; m++) ow[m] = 0u;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++)
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
            float2 mm;
            if (!CLIP) {
                mm = __ffma2_rn(X[rr][hh], hh ? ic1 : ic0, mz2);
            } else {
                float2 t = __fmul2_rn(X[rr][hh], hh ? ic1 : ic0);
                t = f2(fminf(fmaxf(t.x, -(float)Qb), (float)Qb), fminf(fmaxf(t.y, -(float)Qb), (float)Qb));
                mm = __fadd2_rn(t, mz2);
            }
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int c = 4 * rr + 2 * hh + e;
                field_put_bits<B>(ow, c, __float_as_uint(e ? mm.y : mm.x));
#pragma unroll
                for (int m = (c * B) / 32; m < ((c + 1) * B) / 32; m++) words[m * kGroups] = ow[m];
            }
        }
}

// ---------------------------------------------------------------------------
// The fit (row scales, column scales, least squares), requantisation and the
// packed store.  On entry X holds P_ij = S_ij / a_i on quantised rows and S_ij
// on pivot rows; sm.ra, rs, rrho, rb, rq2 and sm.head_b / head_kind are set.
// Writes r', c and the item's streams at item_g.  Contains __syncthreads.
// ROWWISE: rows may differ in width and may be pivots.
// ---------------------------------------------------------------------------
template <int B, bool ROWWISE, bool MULTI>
__device__ __forceinline__ void fit_and_store(ItemSmem &sm, X2 &X, uint8_t *item_g, int ls_iters,
                                              bool store_c = true)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int r0 = kRowsPerWarp * w;
    // read now: the next item's phase 0 may rewrite them while this item's last
    // phase still runs
    const uint32_t tile_off = sm.tile_off[w];
    // ---- row magnitudes: sum over the 128 columns of P^2 -------------------
    {
        float *t = &sm.rowt[w][0][0];
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++) {
            float2 s2 = __fmul2_rn(X[rr][0], X[rr][0]);
            s2 = __ffma2_rn(X[rr][1], X[rr][1], s2);
            t[rr * 36 + l] = s2.x + s2.y;
        }
        __syncwarp();
        const int rr = l >> 1, hf = l & 1;
        float ss = 0.f;
#pragma unroll
        for (int m = 0; m < 4; m++) {
            const float4 x = ld4(t + rr * 36 + 16 * hf + 4 * m);
            ss += (x.x + x.y) + (x.z + x.w);
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (hf == 0) {
            const int i = r0 + rr;
            const int b = sm.rb[i];
            float rnew = 0.f, h = 1.f, wt = 0.f;  // pivot rows: p = S, not part of any fit
            if (b != kPivotBits) {
                const float a = sm.ra[i];
                float m = a * sqrt_approx(ss * (1.0f / kDV));
                if (m == 0.f) m = 1.f;
                rnew = (m * sm.rs[i]) * sm.rq2[i].x;
                h = div_approx(a, rnew);
                wt = (sm.rrho[i] * rnew) * rnew;
            }
            sm.rh2[i] = f2(h, h);
            sm.rw2[i] = f2(wt, wt);
            reinterpret_cast<float *>(item_g)[i] = rnew;
        }
        __syncwarp();
    }
    // ---- p = P h; column maxima (of |p| / Q_i for row-wise widths) ----------
    {
        float mx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr += 2) {
            float2 p[2][2], hh[2], qq[2];
            ld_pairs(&sm.rh2[r0 + rr], hh);
            if (ROWWISE) ld_pairs(&sm.rq2[r0 + rr], qq);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                p[u][0] = __fmul2_rn(X[rr + u][0], hh[u]);
                p[u][1] = __fmul2_rn(X[rr + u][1], hh[u]);
                X[rr + u][0] = p[u][0];
                X[rr + u][1] = p[u][1];
                if (ROWWISE) {  // pivot rows have rq2 = 0 and do not count
                    p[u][0] = __fmul2_rn(p[u][0], qq[u]);
                    p[u][1] = __fmul2_rn(p[u][1], qq[u]);
                }
            }
            mx[0] = max_abs3(mx[0], p[0][0].x, p[1][0].x);
            mx[1] = max_abs3(mx[1], p[0][0].y, p[1][0].y);
            mx[2] = max_abs3(mx[2], p[0][1].x, p[1][1].x);
            mx[3] = max_abs3(mx[3], p[0][1].y, p[1][1].y);
        }
        stash(sm, 0, f2(mx[0], mx[1]), f2(mx[2], mx[3]));
    }
    __syncthreads();
    {
        // two threads per column, each over four warps' partials
        const int j = tid >> 1, half = tid & 1;
        float m = max_partials4(sm, 0, j, half);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        if (half == 0) {
            if (!ROWWISE) m = m * sm.rq2[0].x;  // every row has the head's width
            const float c0 = (m > 0.f) ? m : 1.f;
            sm.cc0[j] = c0;
            sm.cnew[j] = c0;
            sm.ci[j] = rcp_approx(c0);
            sm.crat[j] = 1.f;
        }
    }
    __syncthreads();
    // ---- impact-weighted least squares for the column scales ---------------
    // |p / c0| <= Q, so the first round needs no clipping; later rounds clip to
    // the row's range.  More than one round is a separate instantiation (MULTI)
    // so that the one-round code holds a single round body.
    if (!MULTI) {
        if (ls_iters > 0) {
            ls_partials<B, ROWWISE, false>(sm, X);
            __syncthreads();
            ls_update_columns(sm);
            __syncthreads();
        }
    } else {
        for (int it = 0; it < ls_iters; it++) {
            if (it == 0)
                ls_partials<B, ROWWISE, false>(sm, X);
            else
                ls_partials<B, ROWWISE, true>(sm, X);
            __syncthreads();
            ls_update_columns(sm);
            __syncthreads();
        }
    }
    // ---- requantise, pack, store -------------------------------------------
    const float4 i4 = ld4(&sm.ci[4 * l]);
    const float2 ic0 = f2(i4.x, i4.y), ic1 = f2(i4.z, i4.w);
    float rat;
    {
        const float4 r = ld4(&sm.crat[4 * l]);
        rat = fmaxf(fmaxf(r.x, r.y), fmaxf(r.z, r.w));
    }
    // the largest |p / c| of a column is at most Q c0 / c: clip only where that
    // can reach Q + 1/2
    rat = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(rat)));
    uint32_t *words = reinterpret_cast<uint32_t *>(item_g + tile_off) + l;
    if constexpr (B > 0) {
        constexpr int Qb = (1 << (B - 1)) - 1;
        if ((float)Qb * (rat - 1.f) >= 0.49f)
            pack_fixed<B, true>(X, ic0, ic1, words);
        else
            pack_fixed<B, false>(X, ic0, ic1, words);
    } else {
        BitWriter bw;
        bw.init(words, kGroups);
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++) {
            const int b = sm.rb[r0 + rr];
            if (b == kPivotBits) {
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    const __half2 hv = __floats2half2_rn(X[rr][hh].x, X[rr][hh].y);
                    bw.put(*reinterpret_cast<const uint32_t *>(&hv), 32);
                }
            } else {
                const int Qb = qmax_of(b);
                const bool clip = (float)Qb * (rat - 1.f) >= 0.49f;
                const float mz = kMagic + (float)(1 << (b - 1));
                const float2 mz2 = f2(mz, mz);
                const uint32_t mask = (1u << b) - 1u;
                uint32_t f = 0;
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    float2 mm;
                    if (!clip) {
                        mm = __ffma2_rn(X[rr][hh], hh ? ic1 : ic0, mz2);
                    } else {
                        float2 t = __fmul2_rn(X[rr][hh], hh ? ic1 : ic0);
                        t = f2(fminf(fmaxf(t.x, -(float)Qb), (float)Qb), fminf(fmaxf(t.y, -(float)Qb), (float)Qb));
                        mm = __fadd2_rn(t, mz2);
                    }
                    f |= (__float_as_uint(mm.x) & mask) << (2 * hh * b);
                    f |= (__float_as_uint(mm.y) & mask) << ((2 * hh + 1) * b);
                }
                bw.put(f, 4 * b);
            }
        }
        bw.flush();
    }
    if (tid < kDV) reinterpret_cast<float *>(item_g)[kDK + tid] = store_c ? sm.cnew[tid] : 0.f;
}

// ---------------------------------------------------------------------------
// The fused decode step: persistent CTAs walk the item order.  Items of heads
// whose rows are all FP16 pivots come first in the order and are processed
// straight from global memory; every other item is staged into a ring of
// shared-memory slots by bulk copies (one mbarrier per slot) several items
// ahead of the compute.
// ---------------------------------------------------------------------------

// An item of an all-pivot head: binary16 state, update and readout, no fit.
__device__ void pivot_item(ItemSmem &sm, const StepArgs &a, int item)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int rq = item / a.heads, h = item - rq * a.heads;
    const HeadRec *rec = a.t.rowrec + h;
    uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + a.t.head_off[h];
    const long long vec = (long long)item * kDK;
    const float beta = a.beta[item];
    if (tid < kDK) {
        const int i = tid;
        const float al = a.kda ? a.alpha[vec + i] : a.alpha[item];
        const float k = a.k[vec + i], q = a.q[vec + i];
        sm.rk2[i] = f2(al * k, al * k);
        sm.rl2[i] = f2(al * q, al * q);
        sm.rg2[i] = f2(beta * k, beta * k);
        sm.ra2[i] = f2(al, al);
        float kq = k * q;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
        if (l == 0) sm.kq[w] = kq;
    } else {
        sm.cv[tid - kDK] = a.v[vec + tid - kDK];
    }
    __syncthreads();
    uint32_t *words = reinterpret_cast<uint32_t *>(item_g + rec->tile_off[w]) + l;
    X2 X;
    float2 V0 = f2(0.f, 0.f), V1 = V0, U0 = V0, U1 = V0;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const int i = kRowsPerWarp * w + rr;
        const uint32_t w0 = words[(2 * rr) * kGroups], w1 = words[(2 * rr + 1) * kGroups];
        const float2 h0 = __half22float2(*reinterpret_cast<const __half2 *>(&w0));
        const float2 h1 = __half22float2(*reinterpret_cast<const __half2 *>(&w1));
        const float2 kk = ld2(&sm.rk2[i]), ll = ld2(&sm.rl2[i]), aa = ld2(&sm.ra2[i]);
        X[rr][0] = __fmul2_rn(aa, h0);
        X[rr][1] = __fmul2_rn(aa, h1);
        V0 = __ffma2_rn(kk, h0, V0);
        V1 = __ffma2_rn(kk, h1, V1);
        U0 = __ffma2_rn(ll, h0, U0);
        U1 = __ffma2_rn(ll, h1, U1);
    }
    stash(sm, 0, V0, V1);
    stash(sm, 1, U0, U1);
    __syncthreads();
    if (tid < kDV) {
        sm.cd[tid] = sm.cv[tid] - sum_partials(sm, 0, tid);
    } else {
        sm.cu[tid - kDK] = sum_partials(sm, 1, tid - kDK);
    }
    __syncthreads();
    if (tid < kDV) {
        const float kq = (sm.kq[0] + sm.kq[1]) + (sm.kq[2] + sm.kq[3]);
        a.out[(long long)item * kDV + tid] = fmaf(beta * kq, sm.cd[tid], sm.cu[tid]);
    }
    const float4 d4 = ld4(&sm.cd[4 * l]);
    const float2 d0 = f2(d4.x, d4.y), d1 = f2(d4.z, d4.w);
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const int i = kRowsPerWarp * w + rr;
        const float2 gg = ld2(&sm.rg2[i]);
        const float2 s0 = __ffma2_rn(gg, d0, X[rr][0]), s1 = __ffma2_rn(gg, d1, X[rr][1]);
        const __half2 h0 = __floats2half2_rn(s0.x, s0.y);
        const __half2 h1 = __floats2half2_rn(s1.x, s1.y);
        words[(2 * rr) * kGroups] = *reinterpret_cast<const uint32_t *>(&h0);
        words[(2 * rr + 1) * kGroups] = *reinterpret_cast<const uint32_t *>(&h1);
    }
    __syncthreads();
}

// Issue the bulk copies that stage one item into slot buffer sb.  st = the
// item's staging record {item, item bytes, byte offset in the pool (lo, hi)}.
template <bool KDA>
__device__ __forceinline__ void stage_item(const StepArgs &a, int4 st, uint8_t *sb, uint64_t *bar)
{
    const int item = st.x, h = item % a.heads;
    const uint32_t bytes = (uint32_t)st.y;
    const uint8_t *src = a.pool + (long long)(((unsigned long long)(uint32_t)st.w << 32) | (uint32_t)st.z);
    const long long vec = (long long)item * kDK;
    const uint32_t tx = bytes + 3u * 4u * kDK + (KDA ? 4u * kDK : 0u) + (uint32_t)sizeof(HeadRec);
    mbar_arrive_expect_tx(bar, tx);
    bulk_g2s(sb, src, bytes, bar);
    bulk_g2s(sb + a.off_q, a.q + vec, 4 * kDK, bar);
    bulk_g2s(sb + a.off_k, a.k + vec, 4 * kDK, bar);
    bulk_g2s(sb + a.off_v, a.v + (long long)item * kDV, 4 * kDV, bar);
    if (KDA) bulk_g2s(sb + a.off_alpha, a.alpha + vec, 4 * kDK, bar);
    bulk_g2s(sb + a.off_rec, a.t.rowrec + h, sizeof(HeadRec), bar);
    // the per-item scalars (GDN alpha, beta) are 4-byte copies tracked by the same barrier
    const uint32_t dab = smem_addr(sb + a.off_ab);
    if (!KDA) asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dab), "l"(a.alpha + item) : "memory");
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dab + 4), "l"(a.beta + item) : "memory");
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Producer state, used by thread 0 only and kept in shared memory so that it
// costs no registers in the other threads: the next position to stage, the
// number staged so far, and that position's staging record, fetched one issue
// ahead with an asynchronous copy so that no global load stalls the thread.
__device__ __forceinline__ void prefetch_stage_rec(ItemSmem &sm, const StepArgs &a)
{
    if (sm.prod_n < a.n_items)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_addr(&sm.prod_rec)),
                     "l"(a.t.stage + sm.prod_n)
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Stage the next position into slot buffer sb (thread 0).
template <bool KDA>
__device__ __forceinline__ void produce(ItemSmem &sm, const StepArgs &a, uint8_t *sb, uint64_t *bar)
{
    asm volatile("cp.async.wait_all;" ::: "memory");
    stage_item<KDA>(a, sm.prod_rec, sb, bar);
    sm.prod_n += gridDim.x;
    sm.prod_issued++;
    prefetch_stage_rec(sm, a);
}

// Phase 0 of a staged item: per-row and per-column factors from the slot.
template <bool KDA>
__device__ __forceinline__ void phase0(ItemSmem &sm, const StepArgs &a, const uint8_t *sb)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const HeadRec *rec = reinterpret_cast<const HeadRec *>(sb + a.off_rec);
    const float *s_r = reinterpret_cast<const float *>(sb);
    const float *s_c = s_r + kDK;
    const float beta = *reinterpret_cast<const float *>(sb + a.off_ab + 4);
    if (tid < kDK) {
        const int i = tid;
        const int b = rec->bits[i];
        const float al = KDA ? reinterpret_cast<const float *>(sb + a.off_alpha)[i]
                             : *reinterpret_cast<const float *>(sb + a.off_ab);
        const float k = reinterpret_cast<const float *>(sb + a.off_k)[i];
        const float q = reinterpret_cast<const float *>(sb + a.off_q)[i];
        float A, g, qi = 0.f, s = 0.f, rh = 0.f;
        if (b == kPivotBits) {
            A = al;
            g = beta * k;
        } else {
            A = al * s_r[i];
            g = __fdiv_rn(beta * k, A);
            qi = __frcp_rn((float)qmax_of(b));
            s = rec->s[i];
            rh = rec->rho[i];
        }
        sm.rk2[i] = f2(A * k, A * k);
        sm.rl2[i] = f2(A * q, A * q);
        sm.rg2[i] = f2(g, g);
        sm.ra2[i] = f2(al, al);
        sm.rq2[i] = f2(qi, qi);
        sm.ra[i] = A;
        sm.rs[i] = s;
        sm.rrho[i] = rh;
        sm.rb[i] = b;
        float kq = k * q;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
        if (l == 0) sm.kq[w] = kq;
    } else {
        const int j = tid - kDK;
        sm.cc[j] = s_c[j];
        sm.cv[j] = reinterpret_cast<const float *>(sb + a.off_v)[j];
        if (j < kTiles) sm.tile_off[j] = rec->tile_off[j];
        if (j == kTiles) {
            sm.head_b = rec->head_b;
            sm.head_kind = rec->head_kind;
            sm.head_off = rec->head_off;
            sm.beta_item = beta;
        }
    }
}

// Phases after phase 0 of a staged item: reconstruct + project, release the
// slot (stage the next item into it), Delta update, readout, fit, store.
template <int B, bool KDA, bool MULTI>
__device__ __forceinline__ void run_item(ItemSmem &sm, const StepArgs &a, int item, const uint8_t *sb, int slot,
                                         uint8_t *ring)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int r0 = kRowsPerWarp * w;
    constexpr bool ROWWISE = (B == 0);
    X2 X;
    // ---- phase A: codes -> floats, key and query projections ---------------
    decode_stream<B>(sm, reinterpret_cast<const uint32_t *>(sb + sm.tile_off[w]) + l, kGroups, X);
    {
        const float4 c4 = ld4(&sm.cc[4 * l]);
        float2 V0 = f2(0.f, 0.f), V1 = V0, U0 = V0, U1 = V0;
        float2 ic0 = V0, ic1 = V0;
        if (ROWWISE) {
            ic0 = f2(rcp_approx(c4.x), rcp_approx(c4.y));
            ic1 = f2(rcp_approx(c4.z), rcp_approx(c4.w));
        }
#pragma unroll
        for (int r2 = 0; r2 < kRowsPerWarp; r2 += 2) {
            float2 kp[2], lp[2];
            ld_pairs(&sm.rk2[r0 + r2], kp);
            ld_pairs(&sm.rl2[r0 + r2], lp);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int rr = r2 + u, i = r0 + rr;
                if (ROWWISE && sm.rb[i] == kPivotBits) {
                    // a pivot value enters the projections in units of c_j; S' = alpha h
                    const float2 hs0 = __fmul2_rn(X[rr][0], ic0), hs1 = __fmul2_rn(X[rr][1], ic1);
                    V0 = __ffma2_rn(kp[u], hs0, V0);
                    V1 = __ffma2_rn(kp[u], hs1, V1);
                    U0 = __ffma2_rn(lp[u], hs0, U0);
                    U1 = __ffma2_rn(lp[u], hs1, U1);
                    const float2 aa = ld2(&sm.ra2[i]);
                    X[rr][0] = __fmul2_rn(aa, X[rr][0]);
                    X[rr][1] = __fmul2_rn(aa, X[rr][1]);
                } else {
                    V0 = __ffma2_rn(kp[u], X[rr][0], V0);
                    V1 = __ffma2_rn(kp[u], X[rr][1], V1);
                    U0 = __ffma2_rn(lp[u], X[rr][0], U0);
                    U1 = __ffma2_rn(lp[u], X[rr][1], U1);
                }
            }
        }
        stash(sm, 0, V0, V1);
        stash(sm, 1, U0, U1);
    }
    __syncthreads();
    // the slot has been read by every thread: stage the next item into it
    if (tid == 0 && sm.prod_n < a.n_items) produce<KDA>(sm, a, ring + slot * a.slot_bytes, &sm.bar[slot]);
    {
        // two threads per column, each over four warps' partials
        const int j = tid >> 1, half = tid & 1;
        float vs = sum_partials4(sm, 0, j, half), us = sum_partials4(sm, 1, j, half);
        vs += __shfl_xor_sync(0xffffffffu, vs, 1);
        us += __shfl_xor_sync(0xffffffffu, us, 1);
        const float c = sm.cc[j];
        if (half == 0) {
            const float d = sm.cv[j] - c * vs;
            sm.cd[j] = d;
            sm.cdt[j] = div_approx(d, c);
        } else {
            sm.cu[j] = c * us;
        }
    }
    __syncthreads();
    if (tid < kDV) {
        const float kq = (sm.kq[0] + sm.kq[1]) + (sm.kq[2] + sm.kq[3]);
        a.out[(long long)item * kDV + tid] = fmaf(sm.beta_item * kq, sm.cd[tid], sm.cu[tid]);
    }
    // ---- phase B: Delta update in old-scale units; P = S / a ----------------
    {
        const float4 c4 = ld4(&sm.cc[4 * l]);
        const float2 c0 = f2(c4.x, c4.y), c1 = f2(c4.z, c4.w);
        const float4 t4 = ld4(&sm.cdt[4 * l]);
        const float2 dt0 = f2(t4.x, t4.y), dt1 = f2(t4.z, t4.w);
        float2 dd0 = dt0, dd1 = dt1;
        if (ROWWISE) {
            const float4 d4 = ld4(&sm.cd[4 * l]);
            dd0 = f2(d4.x, d4.y);
            dd1 = f2(d4.z, d4.w);
        }
#pragma unroll
        for (int r2 = 0; r2 < kRowsPerWarp; r2 += 2) {
            float2 gp[2];
            ld_pairs(&sm.rg2[r0 + r2], gp);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int rr = r2 + u, i = r0 + rr;
                if (ROWWISE && sm.rb[i] == kPivotBits) {
                    X[rr][0] = __ffma2_rn(gp[u], dd0, X[rr][0]);
                    X[rr][1] = __ffma2_rn(gp[u], dd1, X[rr][1]);
                } else {
                    X[rr][0] = __fmul2_rn(c0, __ffma2_rn(gp[u], dt0, X[rr][0]));
                    X[rr][1] = __fmul2_rn(c1, __ffma2_rn(gp[u], dt1, X[rr][1]));
                }
            }
        }
    }
    const int rq = item / a.heads;
    uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + sm.head_off;
    fit_and_store<B, ROWWISE, MULTI>(sm, X, item_g, a.ls_iters);
    // the row-wise store reads the row widths, which the next item's phase 0
    // rewrites; the fixed-width store reads no shared state phase 0 writes
    if (ROWWISE) __syncthreads();
}

template <bool KDA, bool MULTI>
__global__ void __launch_bounds__(kThreads, 2) k_decode(StepArgs a)
{
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ ItemSmem sm;
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    if (tid == 0) {
        for (int s = 0; s < a.nslots; s++) mbar_init(&sm.bar[s], 2);
        fence_barrier_init();
    }
    __syncthreads();

    const int npiv = a.n_pivot_items;
    // first staged position of this CTA: the smallest n >= npiv with n = blockIdx.x (mod G)
    int n_first = blockIdx.x;
    if (n_first < npiv) n_first += ((npiv - n_first + G - 1) / G) * G;
    if (tid == 0) {
        sm.prod_n = n_first;
        sm.prod_issued = 0;
        prefetch_stage_rec(sm, a);
        for (int s = 0; s < a.nslots && sm.prod_n < a.n_items; s++)
            produce<KDA>(sm, a, ring + s * a.slot_bytes, &sm.bar[s]);
    }
    uint32_t n_cons = 0;
    int next_item = (blockIdx.x < a.n_items) ? a.t.order[blockIdx.x] : 0;
    for (int n = blockIdx.x; n < a.n_items; n += G) {
        const int item = next_item;
        if (n + G < a.n_items) next_item = a.t.order[n + G];
        if (n < npiv) {
            pivot_item(sm, a, item);
            continue;
        }
        const int slot = (int)(n_cons % (uint32_t)a.nslots);
        const uint32_t parity = (n_cons / (uint32_t)a.nslots) & 1u;
        n_cons++;
        const uint8_t *sb = ring + slot * a.slot_bytes;
        const bool ok = mbar_wait_bounded(&sm.bar[slot], parity, kWaitLimit);
        if (ok) phase0<KDA>(sm, a, sb);
        if (!__syncthreads_and(ok)) {
            // a staged copy never completed: record it, drain what is in flight, stop
            if (tid == 0) {
                atomicExch(a.t.status, kStatusWaitTimeout);
                for (uint32_t m = n_cons - 1; m < sm.prod_issued; m++)
                    mbar_wait_bounded(&sm.bar[m % (uint32_t)a.nslots], (m / (uint32_t)a.nslots) & 1u, kWaitLimit);
            }
            __syncthreads();
            return;
        }
        if (KDA) {
            run_item<0, KDA, MULTI>(sm, a, item, sb, slot, ring);
        } else {
            switch (sm.head_b) {
                case 2: run_item<2, KDA, MULTI>(sm, a, item, sb, slot, ring); break;
                case 3: run_item<3, KDA, MULTI>(sm, a, item, sb, slot, ring); break;
                case 4: run_item<4, KDA, MULTI>(sm, a, item, sb, slot, ring); break;
                case 5: run_item<5, KDA, MULTI>(sm, a, item, sb, slot, ring); break;
                case 6: run_item<6, KDA, MULTI>(sm, a, item, sb, slot, ring); break;
                case 7: run_item<7, KDA, MULTI>(sm, a, item, sb, slot, ring); break;
                case 8: run_item<8, KDA, MULTI>(sm, a, item, sb, slot, ring); break;
                default:  // unreachable: Gated-DeltaNet heads have one width, validated on the host
                    if (tid == 0) atomicExch(a.t.status, kStatusBadHead);
                    __syncthreads();
                    break;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Pack (fit + quantise full-precision states) and unpack (dequantise): one CTA
// per item, the same thread mapping and the same fit as the decode step.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_head(ItemSmem &sm, const StepArgs &a, int h)
{
    const int tid = threadIdx.x;
    const HeadRec *rec = a.t.rowrec + h;
    if (tid < kDK) {
        const int i = tid, b = rec->bits[i];
        const float qi = (b == kPivotBits) ? 0.f : __frcp_rn((float)qmax_of(b));
        sm.rb[i] = b;
        sm.ra[i] = 1.f;
        sm.rs[i] = rec->s[i];
        sm.rrho[i] = rec->rho[i];
        sm.rq2[i] = f2(qi, qi);
    } else {
        const int j = tid - kDK;
        if (j < kTiles) sm.tile_off[j] = rec->tile_off[j];
        if (j == kTiles) {
            sm.head_b = rec->head_b;
            sm.head_kind = rec->head_kind;
            sm.head_off = rec->head_off;
        }
    }
}

template <int B, bool ROWWISE>
__device__ __forceinline__ void pack_body(ItemSmem &sm, const StepArgs &a, int item, uint8_t *item_g)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    X2 X;
    const float *src = a.S_in + (long long)item * kDK * kDV;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const float4 x = ld4(src + (kRowsPerWarp * w + rr) * kDV + 4 * l);
        X[rr][0] = f2(x.x, x.y);
        X[rr][1] = f2(x.z, x.w);
    }
    fit_and_store<B, ROWWISE, true>(sm, X, item_g, a.ls_iters, sm.head_kind != kHeadAllPivot);
}

__global__ void __launch_bounds__(kThreads) k_pack(StepArgs a)
{
    __shared__ ItemSmem sm;
    const int item = blockIdx.x;
    const int rq = item / a.heads, h = item - rq * a.heads;
    load_head(sm, a, h);
    __syncthreads();
    uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + sm.head_off;
    switch (sm.head_kind == kHeadQuant ? sm.head_b : 0) {
        case 2: pack_body<2, false>(sm, a, item, item_g); break;
        case 3: pack_body<3, false>(sm, a, item, item_g); break;
        case 4: pack_body<4, false>(sm, a, item, item_g); break;
        case 5: pack_body<5, false>(sm, a, item, item_g); break;
        case 6: pack_body<6, false>(sm, a, item, item_g); break;
        case 7: pack_body<7, false>(sm, a, item, item_g); break;
        case 8: pack_body<8, false>(sm, a, item, item_g); break;
        default: pack_body<0, true>(sm, a, item, item_g); break;
    }
}

template <int B>
__device__ __forceinline__ void unpack_body(ItemSmem &sm, const StepArgs &a, int item, const uint8_t *item_g)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    X2 X;
    decode_stream<B>(sm, reinterpret_cast<const uint32_t *>(item_g + sm.tile_off[w]) + l, kGroups, X);
    const float *r = reinterpret_cast<const float *>(item_g);
    const float4 c4 = ld4(r + kDK + 4 * l);
    float *dst = a.S_out + (long long)item * kDK * kDV;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const int i = kRowsPerWarp * w + rr;
        float4 y;
        if (B == 0 && sm.rb[i] == kPivotBits) {
            y = make_float4(X[rr][0].x, X[rr][0].y, X[rr][1].x, X[rr][1].y);
        } else {
            const float ri = r[i];
            y = make_float4(__fmul_rn(__fmul_rn(ri, c4.x), X[rr][0].x), __fmul_rn(__fmul_rn(ri, c4.y), X[rr][0].y),
                            __fmul_rn(__fmul_rn(ri, c4.z), X[rr][1].x), __fmul_rn(__fmul_rn(ri, c4.w), X[rr][1].y));
        }
        *reinterpret_cast<float4 *>(dst + i * kDV + 4 * l) = y;
    }
}

__global__ void __launch_bounds__(kThreads) k_unpack(StepArgs a)
{
    __shared__ ItemSmem sm;
    const int item = blockIdx.x;
    const int rq = item / a.heads, h = item - rq * a.heads;
    load_head(sm, a, h);
    __syncthreads();
    const uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + sm.head_off;
    switch (sm.head_kind == kHeadQuant ? sm.head_b : 0) {
        case 2: unpack_body<2>(sm, a, item, item_g); break;
        case 3: unpack_body<3>(sm, a, item, item_g); break;
        case 4: unpack_body<4>(sm, a, item, item_g); break;
        case 5: unpack_body<5>(sm, a, item, item_g); break;
        case 6: unpack_body<6>(sm, a, item, item_g); break;
        case 7: unpack_body<7>(sm, a, item, item_g); break;
        case 8: unpack_body<8>(sm, a, item, item_g); break;
        default: unpack_body<0>(sm, a, item, item_g); break;
    }
}

// Unquantised fp32 state: the same update and readout, state read and written
// in full precision (the baseline the packed state is compared with).
__global__ void __launch_bounds__(kThreads) k_fp32_step(float *Sg, const float *q, const float *k,
                                                        const float *v, const float *alpha,
                                                        const float *beta, float *out, int kda)
{
    __shared__ float sk[kDK], sq[kDK], sa[kDK], sv[kDV], scol[kDV];
    __shared__ float red[8][kDV];
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const long long item = blockIdx.x;
    const long long vec = item * kDK;
    if (tid < kDK) {
        sk[tid] = k[vec + tid];
        sq[tid] = q[vec + tid];
        sa[tid] = kda ? alpha[vec + tid] : alpha[item];
    } else {
        sv[tid - kDK] = v[vec + tid - kDK];
    }
    __syncthreads();
    float *Sp = Sg + item * kDK * kDV;
    float S[kRowsPerWarp][4];
    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ii = 0; ii < kRowsPerWarp; ii++) {
        const int i = kRowsPerWarp * w + ii;
        const float4 x = *reinterpret_cast<const float4 *>(Sp + i * kDV + 4 * l);
        S[ii][0] = sa[i] * x.x; S[ii][1] = sa[i] * x.y; S[ii][2] = sa[i] * x.z; S[ii][3] = sa[i] * x.w;
#pragma unroll
        for (int kk = 0; kk < 4; kk++) part[kk] = fmaf(S[ii][kk], sk[i], part[kk]);
    }
    *reinterpret_cast<float4 *>(&red[w][4 * l]) = make_float4(part[0], part[1], part[2], part[3]);
    __syncthreads();
    if (tid < kDV) {
        float acc = 0.f;
#pragma unroll
        for (int ww = 0; ww < 8; ww++) acc += red[ww][tid];
        scol[tid] = sv[tid] - acc;
    }
    __syncthreads();
    float d[4];
#pragma unroll
    for (int kk = 0; kk < 4; kk++) { d[kk] = scol[4 * l + kk]; part[kk] = 0.f; }
    const float bt = beta[item];
#pragma unroll
    for (int ii = 0; ii < kRowsPerWarp; ii++) {
        const int i = kRowsPerWarp * w + ii;
        const float g = bt * sk[i];
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {
            S[ii][kk] = fmaf(g, d[kk], S[ii][kk]);
            part[kk] = fmaf(S[ii][kk], sq[i], part[kk]);
        }
        *reinterpret_cast<float4 *>(Sp + i * kDV + 4 * l) = make_float4(S[ii][0], S[ii][1], S[ii][2], S[ii][3]);
    }
    __syncthreads();
    *reinterpret_cast<float4 *>(&red[w][4 * l]) = make_float4(part[0], part[1], part[2], part[3]);
    __syncthreads();
    if (tid < kDV) {
        float acc = 0.f;
#pragma unroll
        for (int ww = 0; ww < 8; ww++) acc += red[ww][tid];
        out[item * kDV + tid] = acc;
    }
}

int g_sms = 0;

int sm_count()
{
    if (g_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_sms <= 0) g_sms = 1;
    }
    return g_sms;
}

template <bool KDA, bool MULTI>
cudaError_t launch_decode_t(const StepArgs &a, cudaStream_t s)
{
    const int dyn = a.nslots * a.slot_bytes;
    cudaError_t e = cudaFuncSetAttribute(k_decode<KDA, MULTI>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<KDA, MULTI>, kThreads, dyn);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long want = (long long)per_sm * sm_count();
    const int grid = (int)(a.n_items < want ? a.n_items : want);
    k_decode<KDA, MULTI><<<grid, kThreads, dyn, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_step(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    if (a.ls_iters <= 1) return a.kda ? launch_decode_t<true, false>(a, s) : launch_decode_t<false, false>(a, s);
    return a.kda ? launch_decode_t<true, true>(a, s) : launch_decode_t<false, true>(a, s);
}

int decode_ctas_per_sm(int nslots, int slot_bytes)
{
    const int dyn = nslots * slot_bytes;
    int per_sm = 0;
    if (cudaFuncSetAttribute(k_decode<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<false, false>, kThreads, dyn) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return per_sm;
}

cudaError_t launch_pack(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    k_pack<<<a.n_items, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    k_unpack<<<a.n_items, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_fp32_step(float *S, const float *q, const float *k, const float *v,
                             const float *alpha, const float *beta, float *out, int n_items,
                             int kda, cudaStream_t s)
{
    if (n_items == 0) return cudaSuccess;
    k_fp32_step<<<n_items, kThreads, 0, s>>>(S, q, k, v, alpha, beta, out, kda);
    return cudaGetLastError();
}

}  // namespace stepq
