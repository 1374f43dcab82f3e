// Kernels of the packed-state gated Delta-rule decode step (sm_100a).
//
// Thread mapping (every kernel): a CTA of 256 threads owns one (request,
// head) item at a time; warp w owns key rows 16w .. 16w+15 (= packed tile w),
// lane l owns value columns 4l .. 4l+3 (= column group l), so a thread holds
// 64 state elements in registers and reads / writes exactly one column-group
// stream of one tile: the pool layout is built around this mapping.
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
    float rk[kDK], rl[kDK], rg[kDK], ra[kDK];  // update factors per row
    float rs[kDK], rrho[kDK];                  // s_i, rho_i
    float rh[kDK], rw[kDK], rqi[kDK];          // fit factors per row
    int rb[kDK];                               // row widths
    float cc[kDV], cv[kDV], cd[kDV], cdt[kDV], cu[kDV];
    float cc0[kDV], ci0[kDV], cnew[kDV], ci[kDV], crat[kDV];
    float red[2][8][kDV];
    float rowt[8][16][36];                     // per-warp transposition for row sums
    float kq[4];
    float alpha_item, beta_item;
    uint32_t tile_off[kTiles];
    int head_b, head_kind;
    long long head_off;
    uint64_t bar[kMaxSlots];
};


// ---------------------------------------------------------------------------
// Column sums over the 8 warps of per-thread partials (two vectors at once).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void stash_partials(ItemSmem &sm, int vec, const float (&x)[4])
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    *reinterpret_cast<float4 *>(&sm.red[vec][w][4 * l]) = make_float4(x[0], x[1], x[2], x[3]);
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

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

// ---------------------------------------------------------------------------
// Decode the thread's column-group stream of its tile into X (code values as
// floats; pivot rows: binary16 values times mult_piv).  Fixed width B > 0 keeps
// the stream in registers; B == 0 reads widths per row from sm.rb.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void decode_stream(const ItemSmem &sm, const uint32_t *words, int stride,
                                              float (&X)[kRowsPerWarp][4])
{
    const int w = threadIdx.x >> 5;
    if constexpr (B > 0) {
        uint32_t wd[2 * B];
#pragma unroll
        for (int m = 0; m < 2 * B; m++) wd[m] = words[m * stride];
        const float mz = kMagic + (float)(1 << (B - 1));
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++)
#pragma unroll
            for (int kk = 0; kk < 4; kk++) X[rr][kk] = code_to_float(field_at<B>(wd, 4 * rr + kk), mz);
    } else {
        BitReader br;
        br.init(words, stride);
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++) {
            const int b = sm.rb[kRowsPerWarp * w + rr];
            if (b == kPivotBits) {
#pragma unroll
                for (int half = 0; half < 2; half++) {
                    const uint32_t hv = br.take(32);
                    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hv));
                    X[rr][2 * half] = f.x;
                    X[rr][2 * half + 1] = f.y;
                }
            } else {
                const uint32_t f = br.take(4 * b);
                const uint32_t mask = (1u << b) - 1u;
                const float mz = kMagic + (float)(1 << (b - 1));
#pragma unroll
                for (int kk = 0; kk < 4; kk++) X[rr][kk] = code_to_float((f >> (kk * b)) & mask, mz);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// The fit (row scales, column scales, least squares), requantisation and the
// packed store.  On entry X holds P_ij = S_ij / a_i on quantised rows and S_ij
// on pivot rows; sm.ra, rs, rrho, rb, rqi and sm.head_b are set.  Writes r', c
// and the streams of the item at item_g.  Contains __syncthreads.
// ---------------------------------------------------------------------------
template <int B, bool ROWWISE>
__device__ __forceinline__ void fit_and_store(ItemSmem &sm, float (&X)[kRowsPerWarp][4], uint8_t *item_g,
                                              int ls_iters)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    // ---- row magnitudes: sum over the 128 columns of P^2 -------------------
    {
        float *t = &sm.rowt[w][0][0];
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++) {
            float ss = X[rr][0] * X[rr][0];
            ss = fmaf(X[rr][1], X[rr][1], ss);
            ss = fmaf(X[rr][2], X[rr][2], ss);
            ss = fmaf(X[rr][3], X[rr][3], ss);
            t[rr * 36 + l] = ss;
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
            const int i = kRowsPerWarp * w + rr;
            const int b = sm.rb[i];
            float rnew = 0.f, h = 0.f, wt = 0.f;
            if (b != kPivotBits) {
                const float a = sm.ra[i];
                float m = a * sqrtf(ss * (1.0f / kDV));
                if (m == 0.f) m = 1.f;
                rnew = __fdiv_rn(m * sm.rs[i], (float)qmax_of(b));
                h = __fdiv_rn(a, rnew);
                wt = (sm.rrho[i] * rnew) * rnew;
            }
            sm.rh[i] = h;
            sm.rw[i] = wt;
            reinterpret_cast<float *>(item_g)[i] = rnew;
        }
        __syncwarp();
    }
    // ---- p = P h; column maxima ------------------------------------------
    {
        float mx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r4 = 0; r4 < kRowsPerWarp; r4 += 4) {
            const float4 h4 = ld4(&sm.rh[kRowsPerWarp * w + r4]);
            const float4 q4 = ld4(&sm.rqi[kRowsPerWarp * w + r4]);
            const float hv[4] = {h4.x, h4.y, h4.z, h4.w};
            const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int rr = r4 + u;
                if (ROWWISE && sm.rb[kRowsPerWarp * w + rr] == kPivotBits) continue;
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    const float p = X[rr][kk] * hv[u];
                    X[rr][kk] = p;
                    mx[kk] = fmaxf(mx[kk], ROWWISE ? fabsf(p) * qv[u] : fabsf(p));
                }
            }
        }
        stash_partials(sm, 0, mx);
    }
    __syncthreads();
    if (tid < kDV) {
        const int j = tid;
        float m = max_partials(sm, 0, j);
        if (!ROWWISE) m = __fdiv_rn(m, (float)qmax_of(sm.head_b));
        const float c0 = (m > 0.f) ? m : 1.f;
        const float ic0 = __frcp_rn(c0);
        sm.cc0[j] = c0;
        sm.ci0[j] = ic0;
        sm.cnew[j] = c0;
        sm.ci[j] = ic0;
        sm.crat[j] = 1.f;
    }
    __syncthreads();
    // ---- impact-weighted least squares for the column scales ---------------
    for (int it = 0; it < ls_iters; it++) {
        float ic[4];
        {
            const float4 v = ld4(&sm.ci[4 * l]);
            ic[0] = v.x; ic[1] = v.y; ic[2] = v.z; ic[3] = v.w;
        }
        float N[4] = {0.f, 0.f, 0.f, 0.f}, D[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r4 = 0; r4 < kRowsPerWarp; r4 += 4) {
            const float4 w4 = ld4(&sm.rw[kRowsPerWarp * w + r4]);
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int rr = r4 + u;
                if (ROWWISE && sm.rb[kRowsPerWarp * w + rr] == kPivotBits) continue;
                const float Q = (float)qmax_of(ROWWISE ? sm.rb[kRowsPerWarp * w + rr] : B);
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    float n = __fmaf_rn(X[rr][kk], ic[kk], kRoundMagic) - kRoundMagic;
                    if (it > 0 || ROWWISE) n = fminf(fmaxf(n, -Q), Q);  // later rounds may clip
                    const float wn = wv[u] * n;
                    N[kk] = fmaf(wn, X[rr][kk], N[kk]);
                    D[kk] = fmaf(wn, n, D[kk]);
                }
            }
        }
        stash_partials(sm, 0, N);
        stash_partials(sm, 1, D);
        __syncthreads();
        if (tid < kDV) {
            const int j = tid;
            const float nn = sum_partials(sm, 0, j), dd = sum_partials(sm, 1, j);
            const float c = (dd > 0.f) ? __fdiv_rn(nn, dd) : sm.cnew[j];
            const float icn = __frcp_rn(c);
            sm.cnew[j] = c;
            sm.ci[j] = icn;
            sm.crat[j] = sm.cc0[j] * icn;
        }
        __syncthreads();
    }
    // ---- requantise, pack, store -------------------------------------------
    float ic[4], rat = 0.f;
    {
        const float4 v = ld4(&sm.ci[4 * l]);
        ic[0] = v.x; ic[1] = v.y; ic[2] = v.z; ic[3] = v.w;
        const float4 r = ld4(&sm.crat[4 * l]);
        rat = fmaxf(fmaxf(r.x, r.y), fmaxf(r.z, r.w));
    }
    // the largest |p / c| of a column is Q c0 / c: clip only where it can pass Q + 1/2
    rat = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(rat)));
    uint32_t *words = reinterpret_cast<uint32_t *>(item_g + sm.tile_off[w]) + l;
    if constexpr (B > 0) {
        constexpr int Qb = (1 << (B - 1)) - 1;
        const bool clip = (float)Qb * (rat - 1.f) >= 0.49f;
        const float mz = kMagic + (float)(1 << (B - 1));
        constexpr uint32_t mask = (1u << B) - 1u;
        uint32_t ow[2 * B];
#pragma unroll
        for (int m = 0; m < 2 * B; m++) ow[m] = 0u;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++)
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                float mm;
                if (!clip) {
                    mm = __fmaf_rn(X[rr][kk], ic[kk], mz);
                } else {
                    const float t = fminf(fmaxf(X[rr][kk] * ic[kk], -(float)Qb), (float)Qb);
                    mm = t + mz;
                }
                field_put<B>(ow, 4 * rr + kk, __float_as_uint(mm) & mask);
            }
#pragma unroll
        for (int m = 0; m < 2 * B; m++) words[m * kGroups] = ow[m];
    } else {
        BitWriter bw;
        bw.init(words, kGroups);
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; rr++) {
            const int b = sm.rb[kRowsPerWarp * w + rr];
            if (b == kPivotBits) {
                const __half2 h0 = __floats2half2_rn(X[rr][0], X[rr][1]);
                const __half2 h1 = __floats2half2_rn(X[rr][2], X[rr][3]);
                bw.put(*reinterpret_cast<const uint32_t *>(&h0), 32);
                bw.put(*reinterpret_cast<const uint32_t *>(&h1), 32);
            } else {
                const int Qb = qmax_of(b);
                const bool clip = (float)Qb * (rat - 1.f) >= 0.49f;
                const float mz = kMagic + (float)(1 << (b - 1));
                const uint32_t mask = (1u << b) - 1u;
                uint32_t f = 0;
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    float mm;
                    if (!clip) {
                        mm = __fmaf_rn(X[rr][kk], ic[kk], mz);
                    } else {
                        const float t = fminf(fmaxf(X[rr][kk] * ic[kk], -(float)Qb), (float)Qb);
                        mm = t + mz;
                    }
                    f |= (__float_as_uint(mm) & mask) << (kk * b);
                }
                bw.put(f, 4 * b);
            }
        }
        bw.flush();
    }
    if (tid < kDV) reinterpret_cast<float *>(item_g)[kDK + tid] = (sm.head_kind == kHeadAllPivot) ? 0.f : sm.cnew[tid];
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
        sm.rk[i] = al * k;
        sm.rl[i] = al * q;
        sm.rg[i] = beta * k;
        sm.ra[i] = al;
        float kq = k * q;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
        if (l == 0) sm.kq[w] = kq;
    } else {
        sm.cv[tid - kDK] = a.v[vec + tid - kDK];
    }
    __syncthreads();
    uint32_t *words = reinterpret_cast<uint32_t *>(item_g + rec->tile_off[w]) + l;
    float X[kRowsPerWarp][4];
    float V[4] = {0.f, 0.f, 0.f, 0.f}, U[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const int i = kRowsPerWarp * w + rr;
        const uint32_t w0 = words[(2 * rr) * kGroups], w1 = words[(2 * rr + 1) * kGroups];
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&w0));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&w1));
        const float hv[4] = {f0.x, f0.y, f1.x, f1.y};
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {
            X[rr][kk] = sm.ra[i] * hv[kk];
            V[kk] = fmaf(sm.rk[i], hv[kk], V[kk]);
            U[kk] = fmaf(sm.rl[i], hv[kk], U[kk]);
        }
    }
    stash_partials(sm, 0, V);
    stash_partials(sm, 1, U);
    __syncthreads();
    if (tid < kDV) {
        const float d = sm.cv[tid] - sum_partials(sm, 0, tid);
        sm.cd[tid] = d;
    } else {
        sm.cu[tid - kDK] = sum_partials(sm, 1, tid - kDK);
    }
    __syncthreads();
    if (tid < kDV) {
        const float kq = (sm.kq[0] + sm.kq[1]) + (sm.kq[2] + sm.kq[3]);
        a.out[(long long)item * kDV + tid] = fmaf(beta * kq, sm.cd[tid], sm.cu[tid]);
    }
    const float4 d4 = ld4(&sm.cd[4 * l]);
    const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const int i = kRowsPerWarp * w + rr;
        const float g = sm.rg[i];
        const __half2 h0 = __floats2half2_rn(fmaf(g, dd[0], X[rr][0]), fmaf(g, dd[1], X[rr][1]));
        const __half2 h1 = __floats2half2_rn(fmaf(g, dd[2], X[rr][2]), fmaf(g, dd[3], X[rr][3]));
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

// Producer state, held by thread 0: the next position to stage and its record,
// loaded one issue ahead so that no global load sits on the critical path.
struct Producer {
    int n;          // next position to stage
    int4 rec;       // its staging record
    uint32_t issued;
    __device__ __forceinline__ void load(const StepArgs &a)
    {
        if (n < a.n_items) rec = a.t.stage[n];
    }
};

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
        if (b == kPivotBits) {
            sm.rk[i] = al * k;
            sm.rl[i] = al * q;
            sm.rg[i] = beta * k;
            sm.ra[i] = al;
            sm.rs[i] = 0.f;
            sm.rrho[i] = 0.f;
            sm.rqi[i] = 0.f;
        } else {
            const float A = al * s_r[i];
            sm.rk[i] = A * k;
            sm.rl[i] = A * q;
            sm.rg[i] = __fdiv_rn(beta * k, A);
            sm.ra[i] = A;
            sm.rs[i] = rec->s[i];
            sm.rrho[i] = rec->rho[i];
            sm.rqi[i] = __frcp_rn((float)qmax_of(b));
        }
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
template <int B, bool KDA>
__device__ __forceinline__ void run_item(ItemSmem &sm, const StepArgs &a, int item, const uint8_t *sb, int slot,
                                         Producer &prod, uint8_t *ring)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    constexpr bool ROWWISE = (B == 0);
    float X[kRowsPerWarp][4];
    // ---- phase A: codes -> floats, key and query projections ---------------
    decode_stream<B>(sm, reinterpret_cast<const uint32_t *>(sb + sm.tile_off[w]) + l, kGroups, X);
    float cj[4], icj[4];
    {
        const float4 c4 = ld4(&sm.cc[4 * l]);
        cj[0] = c4.x; cj[1] = c4.y; cj[2] = c4.z; cj[3] = c4.w;
#pragma unroll
        for (int kk = 0; kk < 4; kk++) icj[kk] = ROWWISE ? __frcp_rn(cj[kk]) : 0.f;
    }
    {
        float V[4] = {0.f, 0.f, 0.f, 0.f}, U[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r4 = 0; r4 < kRowsPerWarp; r4 += 4) {
            const float4 k4 = ld4(&sm.rk[kRowsPerWarp * w + r4]);
            const float4 l4 = ld4(&sm.rl[kRowsPerWarp * w + r4]);
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int rr = r4 + u, i = kRowsPerWarp * w + rr;
                if (ROWWISE && sm.rb[i] == kPivotBits) {
                    const float al = sm.ra[i];
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        const float hs = X[rr][kk] * icj[kk];  // pivot value in units of c_j
                        V[kk] = fmaf(kv[u], hs, V[kk]);
                        U[kk] = fmaf(lv[u], hs, U[kk]);
                        X[rr][kk] = al * X[rr][kk];           // S' = alpha h
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        V[kk] = fmaf(kv[u], X[rr][kk], V[kk]);
                        U[kk] = fmaf(lv[u], X[rr][kk], U[kk]);
                    }
                }
            }
        }
        stash_partials(sm, 0, V);
        stash_partials(sm, 1, U);
    }
    __syncthreads();
    // the slot has been read by every thread: stage the next item into it
    if (tid == 0 && prod.n < a.n_items) {
        stage_item<KDA>(a, prod.rec, ring + slot * a.slot_bytes, &sm.bar[slot]);
        prod.n += gridDim.x;
        prod.issued++;
        prod.load(a);
    }
    if (tid < kDV) {
        const int j = tid;
        const float c = sm.cc[j];
        const float d = sm.cv[j] - c * sum_partials(sm, 0, j);
        sm.cd[j] = d;
        sm.cdt[j] = __fdiv_rn(d, c);
    } else {
        const int j = tid - kDK;
        sm.cu[j] = sm.cc[j] * sum_partials(sm, 1, j);
    }
    __syncthreads();
    if (tid < kDV) {
        const float kq = (sm.kq[0] + sm.kq[1]) + (sm.kq[2] + sm.kq[3]);
        a.out[(long long)item * kDV + tid] = fmaf(sm.beta_item * kq, sm.cd[tid], sm.cu[tid]);
    }
    // ---- phase B: Delta update in old-scale units; P = S / a ----------------
    {
        const float4 t4 = ld4(&sm.cdt[4 * l]);
        const float4 d4 = ld4(&sm.cd[4 * l]);
        const float dt[4] = {t4.x, t4.y, t4.z, t4.w};
        const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int r4 = 0; r4 < kRowsPerWarp; r4 += 4) {
            const float4 g4 = ld4(&sm.rg[kRowsPerWarp * w + r4]);
            const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int rr = r4 + u, i = kRowsPerWarp * w + rr;
                if (ROWWISE && sm.rb[i] == kPivotBits) {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) X[rr][kk] = fmaf(gv[u], dd[kk], X[rr][kk]);
                } else {
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) X[rr][kk] = cj[kk] * fmaf(gv[u], dt[kk], X[rr][kk]);
                }
            }
        }
    }
    const int rq = item / a.heads;
    uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + sm.head_off;
    fit_and_store<B, ROWWISE>(sm, X, item_g, a.ls_iters);
    __syncthreads();
}

template <bool KDA>
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
    Producer prod;  // used by thread 0 only
    prod.n = n_first;
    prod.issued = 0;
    prod.rec = make_int4(0, 0, 0, 0);
    if (tid == 0) {
        prod.load(a);
        for (int s = 0; s < a.nslots && prod.n < a.n_items; s++) {
            stage_item<KDA>(a, prod.rec, ring + s * a.slot_bytes, &sm.bar[s]);
            prod.n += G;
            prod.issued++;
            prod.load(a);
        }
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
                for (uint32_t m = n_cons - 1; m < prod.issued; m++)
                    mbar_wait_bounded(&sm.bar[m % (uint32_t)a.nslots], (m / (uint32_t)a.nslots) & 1u, kWaitLimit);
            }
            __syncthreads();
            return;
        }
        const int hb = sm.head_b;
        // dispatch on the head's row width
#define STEPQ_ITEM_CASE(BB)                                                        \
    case BB:                                                                       \
        run_item<BB, KDA>(sm, a, item, sb, slot, prod, ring);         \
        break;
        if (KDA) {
            run_item<0, KDA>(sm, a, item, sb, slot, prod, ring);
        } else {
            switch (hb) {
                STEPQ_ITEM_CASE(2)
                STEPQ_ITEM_CASE(3)
                STEPQ_ITEM_CASE(4)
                STEPQ_ITEM_CASE(5)
                STEPQ_ITEM_CASE(6)
                STEPQ_ITEM_CASE(7)
                STEPQ_ITEM_CASE(8)
                default: run_item<0, KDA>(sm, a, item, sb, slot, prod, ring); break;
            }
        }
#undef STEPQ_ITEM_CASE
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
        sm.rb[i] = b;
        sm.ra[i] = 1.f;
        sm.rs[i] = rec->s[i];
        sm.rrho[i] = rec->rho[i];
        sm.rqi[i] = (b == kPivotBits) ? 0.f : __frcp_rn((float)qmax_of(b));
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
    float X[kRowsPerWarp][4];
    const float *src = a.S_in + (long long)item * kDK * kDV;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const float4 x = ld4(src + (kRowsPerWarp * w + rr) * kDV + 4 * l);
        X[rr][0] = x.x; X[rr][1] = x.y; X[rr][2] = x.z; X[rr][3] = x.w;
    }
    fit_and_store<B, ROWWISE>(sm, X, item_g, a.ls_iters);
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
    float X[kRowsPerWarp][4];
    decode_stream<B>(sm, reinterpret_cast<const uint32_t *>(item_g + sm.tile_off[w]) + l, kGroups, X);
    const float *r = reinterpret_cast<const float *>(item_g);
    const float4 c4 = ld4(r + kDK + 4 * l);
    const float cj[4] = {c4.x, c4.y, c4.z, c4.w};
    float *dst = a.S_out + (long long)item * kDK * kDV;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; rr++) {
        const int i = kRowsPerWarp * w + rr;
        float y[4];
        if (B == 0 && sm.rb[i] == kPivotBits) {
#pragma unroll
            for (int kk = 0; kk < 4; kk++) y[kk] = X[rr][kk];
        } else {
            const float ri = r[i];
#pragma unroll
            for (int kk = 0; kk < 4; kk++) y[kk] = __fmul_rn(__fmul_rn(ri, cj[kk]), X[rr][kk]);
        }
        *reinterpret_cast<float4 *>(dst + i * kDV + 4 * l) = make_float4(y[0], y[1], y[2], y[3]);
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

template <bool KDA>
cudaError_t launch_decode_t(const StepArgs &a, cudaStream_t s)
{
    const int dyn = a.nslots * a.slot_bytes;
    cudaError_t e = cudaFuncSetAttribute(k_decode<KDA>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<KDA>, kThreads, dyn);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long want = (long long)per_sm * sm_count();
    const int grid = (int)(a.n_items < want ? a.n_items : want);
    k_decode<KDA><<<grid, kThreads, dyn, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_step(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    return a.kda ? launch_decode_t<true>(a, s) : launch_decode_t<false>(a, s);
}

int decode_ctas_per_sm(int nslots, int slot_bytes)
{
    const int dyn = nslots * slot_bytes;
    int per_sm = 0;
    if (cudaFuncSetAttribute(k_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<false>, kThreads, dyn) != cudaSuccess) {
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
