// Internal declarations shared by the host library and the kernels of the
// packed-state gated Delta-rule decode step.  Not part of the C ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace stepq {

constexpr int kDK = 128;          // key dimension (rows of a state)
constexpr int kDV = 128;          // value dimension (columns of a state)
constexpr int kThreads = 256;     // threads per item: 8 warps x 16 rows, lane = 4 columns
constexpr int kRowsPerWarp = 16;
constexpr int kPivotBits = 16;
constexpr int kHeaderBytes = 4 * kDK + 4 * kDV;  // r[dk] | c[dv]

// Per-head tables derived on the host at pool creation, resident in the tail
// of the caller's pool buffer.
struct Tables {
    const uint32_t *row_off;   // [H*dk] byte offset of row i inside its item
    const uint8_t *row_bits;   // [H*dk] width of row i (16 = pivot)
    const float *row_s;        // [H*dk] fp32(rho^-1/2), rounded once from fp64
    const float *row_rho;      // [H*dk] impact weight
    const long long *head_off; // [H] byte offset of head h's item inside a request
    const int *head_nq;        // [H] number of quantised (non-pivot) rows
    const int *order;          // [B*H] item processing order (heaviest first)
};

struct StepArgs {
    uint8_t *pool;
    Tables t;
    long long req_bytes;  // bytes of one request's items
    int heads;
    int n_items;
    int ls_iters;
    int kda;
    const float *q, *k, *v, *alpha, *beta;
    float *out;
    const float *S_in;  // pack
    float *S_out;       // unpack
};

cudaError_t launch_decode_step(const StepArgs &a, cudaStream_t s);
cudaError_t launch_pack(const StepArgs &a, cudaStream_t s);
cudaError_t launch_unpack(const StepArgs &a, cudaStream_t s);
cudaError_t launch_fp32_step(float *S, const float *q, const float *k, const float *v,
                             const float *alpha, const float *beta, float *out, int n_items,
                             int kda, cudaStream_t s);

}  // namespace stepq
