// Kernels of the packed-state gated Delta-rule decode step (sm_100a).
//
// One CTA of 256 threads owns one (request, head) item at a time.  Warp w owns
// key rows 16w .. 16w+15, lane l owns value columns 4l .. 4l+3, so each thread
// holds 64 state elements in registers for the whole step: the state is read
// from HBM once (packed) and written once (packed).  Reductions over key rows
// (v_old, readout, column max, least-squares sums) go through shared memory
// across the 8 warps; reductions over value columns (row magnitude) are warp
// shuffles.
//
// Method (ai.info summary of STEPQuant, "Key Contributions" and "Methodology in
// Plain English"; ai-papers.net, "STEPQuantの仕組み"; ai-trend.me, "핵심 용어"):
//   reconstruct  S_ij = (r_i c_j) code_ij  (pivot rows: binary16 values)
//   gate         S'   = diag(alpha) S
//   update       S    = S' + (beta k)(v - S'^T k)^T
//   readout      o    = S^T q
//   refit        r_i  = (rms_i * rho_i^-1/2) / Q_i ; p = S / r ;
//                c_j  = max_i |p_ij| / Q_i, then least squares for fixed codes
//   requantise   code = clamp(rne(p / c)), pack, store.
// Element-wise operations use explicitly rounded intrinsics so that they are
// not contracted; only the order of the sums differs from a sequential sum.
#include <cuda_fp16.h>

#include "stepq_internal.cuh"

namespace stepq {
namespace {

enum Mode { kDecode = 0, kPack = 1, kUnpack = 2 };

struct ItemSmem {
    float k[kDK], q[kDK], alpha[kDK], r[kDK], s[kDK], rho[kDK];
    float c[kDV], v[kDV], col[kDV];
    float red[8][kDV];
    float red2[8][kDV];
    uint32_t off[kDK];
    int bits[kDK];
    uint32_t rowbuf[8][32];
};

__device__ __forceinline__ int qmax_of(int b) { return (1 << (b - 1)) - 1; }

// The 4*b-bit field of lane l in a packed row of 128 b-bit codes.
__device__ __forceinline__ uint32_t load_field(const uint8_t *row, int b, int lane)
{
    const uint32_t *w = reinterpret_cast<const uint32_t *>(row);
    const int bit = 4 * b * lane;
    const int w0 = bit >> 5, sh = bit & 31;
    const uint32_t x0 = w[w0];
    const uint32_t x1 = (sh + 4 * b > 32) ? w[w0 + 1] : 0u;
    return __funnelshift_r(x0, x1, sh);
}

// Sum of the per-thread column partials over the 8 warps, into dst[0..127].
__device__ __forceinline__ void column_sum(ItemSmem &sm, const float (&part)[4], float *dst)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    *reinterpret_cast<float4 *>(&sm.red[w][4 * l]) = make_float4(part[0], part[1], part[2], part[3]);
    __syncthreads();
    if (threadIdx.x < kDV) {
        float acc = 0.f;
#pragma unroll
        for (int ww = 0; ww < 8; ww++) acc = __fadd_rn(acc, sm.red[ww][threadIdx.x]);
        dst[threadIdx.x] = acc;
    }
    __syncthreads();
}

template <int MODE>
__global__ void __launch_bounds__(kThreads) k_item(StepArgs a)
{
    __shared__ ItemSmem sm;
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const int item = (MODE == kDecode) ? a.t.order[blockIdx.x] : (int)blockIdx.x;
    const int rq = item / a.heads, h = item - rq * a.heads;
    uint8_t *it = a.pool + (long long)rq * a.req_bytes + a.t.head_off[h];
    const int nq = a.t.head_nq[h];
    const long long vec = (long long)item * kDK;

    if (tid < kDK) {
        const int i = tid;
        sm.bits[i] = a.t.row_bits[h * kDK + i];
        sm.off[i] = a.t.row_off[h * kDK + i];
        sm.s[i] = a.t.row_s[h * kDK + i];
        sm.rho[i] = a.t.row_rho[h * kDK + i];
        if (MODE != kPack) sm.r[i] = reinterpret_cast<const float *>(it)[i];
        if (MODE == kDecode) {
            sm.k[i] = a.k[vec + i];
            sm.q[i] = a.q[vec + i];
            sm.alpha[i] = a.kda ? a.alpha[vec + i] : a.alpha[item];
        }
    } else {
        const int j = tid - kDK;
        if (MODE != kPack) sm.c[j] = reinterpret_cast<const float *>(it)[kDK + j];
        if (MODE == kDecode) sm.v[j] = a.v[vec + j];
    }
    __syncthreads();

    float S[kRowsPerWarp][4];

    // ---- reconstruct ------------------------------------------------------
    if (MODE == kPack) {
        const float *src = a.S_in + (long long)item * kDK * kDV;
#pragma unroll
        for (int ii = 0; ii < kRowsPerWarp; ii++) {
            const int i = kRowsPerWarp * w + ii;
            const float4 x = *reinterpret_cast<const float4 *>(src + i * kDV + 4 * l);
            S[ii][0] = x.x; S[ii][1] = x.y; S[ii][2] = x.z; S[ii][3] = x.w;
        }
    } else {
#pragma unroll
        for (int ii = 0; ii < kRowsPerWarp; ii++) {
            const int i = kRowsPerWarp * w + ii;
            const int bi = sm.bits[i];
            const uint8_t *row = it + sm.off[i];
            if (bi == kPivotBits) {
                const uint2 hv = *reinterpret_cast<const uint2 *>(row + 8 * l);
                const float2 f0 = __half22float2(*reinterpret_cast<const __half2 *>(&hv.x));
                const float2 f1 = __half22float2(*reinterpret_cast<const __half2 *>(&hv.y));
                S[ii][0] = f0.x; S[ii][1] = f0.y; S[ii][2] = f1.x; S[ii][3] = f1.y;
            } else {
                const uint32_t f = load_field(row, bi, l);
                const uint32_t mask = (1u << bi) - 1u;
                const int zero = 1 << (bi - 1);
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    const int code = (int)((f >> (kk * bi)) & mask) - zero;
                    S[ii][kk] = __fmul_rn(__fmul_rn(sm.r[i], sm.c[4 * l + kk]), (float)code);
                }
            }
        }
    }

    if (MODE == kUnpack) {
        float *dst = a.S_out + (long long)item * kDK * kDV;
#pragma unroll
        for (int ii = 0; ii < kRowsPerWarp; ii++) {
            const int i = kRowsPerWarp * w + ii;
            *reinterpret_cast<float4 *>(dst + i * kDV + 4 * l) = make_float4(S[ii][0], S[ii][1], S[ii][2], S[ii][3]);
        }
        return;
    }

    if (MODE == kDecode) {
        // ---- gate, key projection -----------------------------------------
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ii = 0; ii < kRowsPerWarp; ii++) {
            const int i = kRowsPerWarp * w + ii;
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                S[ii][kk] = __fmul_rn(sm.alpha[i], S[ii][kk]);
                part[kk] = __fmaf_rn(S[ii][kk], sm.k[i], part[kk]);
            }
        }
        column_sum(sm, part, sm.col);  // v_old
        // ---- Delta update, readout ------------------------------------------
        float d[4];
#pragma unroll
        for (int kk = 0; kk < 4; kk++) d[kk] = __fsub_rn(sm.v[4 * l + kk], sm.col[4 * l + kk]);
        const float beta = a.beta[item];
#pragma unroll
        for (int kk = 0; kk < 4; kk++) part[kk] = 0.f;
#pragma unroll
        for (int ii = 0; ii < kRowsPerWarp; ii++) {
            const int i = kRowsPerWarp * w + ii;
            const float g = __fmul_rn(beta, sm.k[i]);
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                S[ii][kk] = __fadd_rn(S[ii][kk], __fmul_rn(g, d[kk]));
                part[kk] = __fmaf_rn(S[ii][kk], sm.q[i], part[kk]);
            }
        }
        column_sum(sm, part, sm.col);  // o
        if (tid < kDV) a.out[(long long)item * kDV + tid] = sm.col[tid];
    }

    // ---- refit row scales -------------------------------------------------
    float rloc[kRowsPerWarp];
#pragma unroll
    for (int ii = 0; ii < kRowsPerWarp; ii++) {
        const int i = kRowsPerWarp * w + ii;
        float ss = __fmul_rn(S[ii][0], S[ii][0]);
        ss = __fmaf_rn(S[ii][1], S[ii][1], ss);
        ss = __fmaf_rn(S[ii][2], S[ii][2], ss);
        ss = __fmaf_rn(S[ii][3], S[ii][3], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        const int bi = sm.bits[i];
        float m = __fsqrt_rn(__fmul_rn(ss, 1.0f / kDV));
        if (m == 0.f) m = 1.f;
        rloc[ii] = (bi == kPivotBits) ? 0.f : __fdiv_rn(__fmul_rn(m, sm.s[i]), (float)qmax_of(bi));
    }
    // p_ij = S_ij / r_i on quantised rows (kept in S for the rest of the fit);
    // pivot rows keep S.
    float P[kRowsPerWarp][4];
#pragma unroll
    for (int ii = 0; ii < kRowsPerWarp; ii++) {
        const int i = kRowsPerWarp * w + ii;
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
            P[ii][kk] = (sm.bits[i] == kPivotBits) ? 0.f : __fdiv_rn(S[ii][kk], rloc[ii]);
    }

    float cj[4] = {0.f, 0.f, 0.f, 0.f};
    if (nq > 0) {
        // ---- column scales: start at the column maximum ----------------------
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ii = 0; ii < kRowsPerWarp; ii++) {
            const int i = kRowsPerWarp * w + ii;
            const int bi = sm.bits[i];
            if (bi == kPivotBits) continue;
            const float qf = (float)qmax_of(bi);
#pragma unroll
            for (int kk = 0; kk < 4; kk++) part[kk] = fmaxf(part[kk], __fdiv_rn(fabsf(P[ii][kk]), qf));
        }
        *reinterpret_cast<float4 *>(&sm.red[w][4 * l]) = make_float4(part[0], part[1], part[2], part[3]);
        __syncthreads();
        if (tid < kDV) {
            float mx = 0.f;
#pragma unroll
            for (int ww = 0; ww < 8; ww++) mx = fmaxf(mx, sm.red[ww][tid]);
            sm.col[tid] = (mx > 0.f) ? mx : 1.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 4; kk++) cj[kk] = sm.col[4 * l + kk];

        // ---- impact-weighted least squares, fixed number of rounds -----------
        for (int itn = 0; itn < a.ls_iters; itn++) {
            float N[4] = {0.f, 0.f, 0.f, 0.f}, D[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ii = 0; ii < kRowsPerWarp; ii++) {
                const int i = kRowsPerWarp * w + ii;
                const int bi = sm.bits[i];
                if (bi == kPivotBits) continue;
                const float qf = (float)qmax_of(bi);
                const float wi = __fmul_rn(__fmul_rn(sm.rho[i], rloc[ii]), rloc[ii]);
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    float n = rintf(__fdiv_rn(P[ii][kk], cj[kk]));
                    n = fminf(fmaxf(n, -qf), qf);
                    const float wn = __fmul_rn(wi, n);
                    N[kk] = __fmaf_rn(wn, P[ii][kk], N[kk]);
                    D[kk] = __fmaf_rn(wn, n, D[kk]);
                }
            }
            *reinterpret_cast<float4 *>(&sm.red[w][4 * l]) = make_float4(N[0], N[1], N[2], N[3]);
            *reinterpret_cast<float4 *>(&sm.red2[w][4 * l]) = make_float4(D[0], D[1], D[2], D[3]);
            __syncthreads();
            if (tid < kDV) {
                float nn = 0.f, dd = 0.f;
#pragma unroll
                for (int ww = 0; ww < 8; ww++) {
                    nn = __fadd_rn(nn, sm.red[ww][tid]);
                    dd = __fadd_rn(dd, sm.red2[ww][tid]);
                }
                if (dd > 0.f) sm.col[tid] = __fdiv_rn(nn, dd);
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < 4; kk++) cj[kk] = sm.col[4 * l + kk];
        }
    }

    // ---- requantise, pack, store ------------------------------------------
    uint32_t *buf = sm.rowbuf[w];
#pragma unroll
    for (int ii = 0; ii < kRowsPerWarp; ii++) {
        const int i = kRowsPerWarp * w + ii;
        const int bi = sm.bits[i];
        uint8_t *row = it + sm.off[i];
        if (bi == kPivotBits) {
            const __half2 h0 = __floats2half2_rn(S[ii][0], S[ii][1]);
            const __half2 h1 = __floats2half2_rn(S[ii][2], S[ii][3]);
            uint2 hv;
            hv.x = *reinterpret_cast<const uint32_t *>(&h0);
            hv.y = *reinterpret_cast<const uint32_t *>(&h1);
            *reinterpret_cast<uint2 *>(row + 8 * l) = hv;
        } else {
            const float qf = (float)qmax_of(bi);
            const uint32_t zero = 1u << (bi - 1);
            uint32_t field = 0;
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                float n = rintf(__fdiv_rn(P[ii][kk], cj[kk]));
                n = fminf(fmaxf(n, -qf), qf);
                field |= ((uint32_t)((int)n + (int)zero)) << (kk * bi);
            }
            const int nwords = 4 * bi;
            if (l < nwords) buf[l] = 0u;
            __syncwarp();
            const int bit = 4 * bi * l, w0 = bit >> 5, sh = bit & 31;
            atomicOr(&buf[w0], field << sh);
            if (sh + 4 * bi > 32) atomicOr(&buf[w0 + 1], field >> (32 - sh));
            __syncwarp();
            if (l < nwords) reinterpret_cast<uint32_t *>(row)[l] = buf[l];
            __syncwarp();
        }
        if (l == 0) reinterpret_cast<float *>(it)[i] = rloc[ii];
    }
    if (tid < kDV) reinterpret_cast<float *>(it)[kDK + tid] = (nq > 0) ? sm.col[tid] : 0.f;
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

}  // namespace

cudaError_t launch_decode_step(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    k_item<kDecode><<<a.n_items, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_pack(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    k_item<kPack><<<a.n_items, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    k_item<kUnpack><<<a.n_items, kThreads, 0, s>>>(a);
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
