// Kernels of the packed-state gated Delta-rule decode step (sm_100a).
//
// Thread mapping (every kernel): a CTA of 256 threads owns one (request, head)
// item at a time.  Warp w owns value columns 16w .. 16w+15 over all 128 key
// rows (= packed slab w); lane l = rg + 8 cg owns key rows 16rg .. 16rg+15 and
// value columns 16w + 4cg .. +3 (= stream l of slab w).  A thread therefore
// holds 64 state values in registers and reads / writes exactly one stream of
// the pool, and the 32 lanes of a warp touch whole 128-byte lines.  The values are
// kept as float2 pairs (columns 4g, 4g+1 and 4g+2, 4g+3) so that every
// floating-point operation on the state is one packed f32x2 instruction;
// per-row factors are stored duplicated, (x, x), so broadcasting them is free.
//
// Every column sum of the step (key projection, readout, column maxima,
// least-squares sums) runs over the 8 lanes of one warp that share cg, by
// shuffles; only the row magnitudes cross warps, through shared memory, so an
// item costs two CTA barriers.
//
// Method (ai.info summary of STEPQuant, "Key Contributions" and "Methodology in
// Plain English"; ai-papers.net, "STEPQuantの仕組み"; ai-trend.me, "핵심 용어"):
//   reconstruct  S_ij = r_i c_j code_ij   (pivot rows: binary16 values)
//   gate         S'   = diag(alpha) S
//   update       S    = S' + (beta k)(v - S'^T k)^T
//   readout      o    = S^T q
//   refit        r_i  = rms_i s_i / Q_i, s_i = max(rho_i, rho_max / 4)^-1/2 (no row
//                coarsened by more than a factor 2 against the highest-impact row);
//                p = S / r ;
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
constexpr unsigned kFull = 0xffffffffu;
constexpr int kProducerWarp = 7;                // the warp that issues the staging copies

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

// Row i's place in the arrays of duplicated row factors: float4 number
// pslot(i) holds rows i & ~1 and i | 1 as (f, f, f', f'), ordered so that the
// 8 row groups of a warp read 8 consecutive float4.
__device__ __forceinline__ int pslot(int i) { return ((i & 15) >> 1) * 8 + (i >> 4); }
// Row i's place in per-row scalar arrays read by row group.
__device__ __forceinline__ int sslot(int i) { return (i & 15) * 8 + (i >> 4); }

// Row-wise widths (KDA): the row handled by thread t (0..127) where one thread
// per row writes the duplicated-pair factors.  A half-warp covers the 8 row
// groups x 2 rows of one pair position, so its 16 float2 writes fill 16
// consecutive slots (no bank conflict, where consecutive rows per thread give
// an 8-way conflict), and the row-partial reads stay conflict-free under
// rowp_chunk's swizzle.  (The fixed-width kernels keep row = thread: there
// the remap's extra registers cost more than the conflicts.)
__device__ __forceinline__ int frow(int t)
{
    const int l = t & 31, m = 2 * (t >> 5) + (l >> 4);
    return 16 * (l & 7) + 2 * m + ((l >> 3) & 1);
}

__device__ __forceinline__ void put_pair(float4 *arr, int i, float v)
{
    reinterpret_cast<float2 *>(arr + pslot(i))[i & 1] = make_float2(v, v);
}

// The duplicated factors of rows 16 rg + 2p and 16 rg + 2p + 1.
__device__ __forceinline__ void ld_pairs(const float4 *arr, int p, int rg, float2 (&out)[2])
{
    const float4 v = arr[p * 8 + rg];
    out[0] = make_float2(v.x, v.y);
    out[1] = make_float2(v.z, v.w);
}

// Call-free reciprocal, quotient and square root (within 2 ulp of the correctly
// rounded results) for the per-row and per-column factors computed while a
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

__device__ __forceinline__ float2 shfl2(float2 v, int m)
{
    return f2(__shfl_xor_sync(kFull, v.x, m), __shfl_xor_sync(kFull, v.y, m));
}

// Row position p of a row-wise head: where its fields sit in every stream and
// the constants of their decode and pack, all derived from the field width F
// and the bit offset O of the position (built once per item by 16 threads).
struct alignas(16) PosRec {
    int w0, w1, sh, f2;          // word offsets (x 32 streams) of words O/32 and O/32 + 1 (last word
                                 // at most), O % 32, 2F
    uint32_t m0, m1, e1, done;   // masks of fields 0 and 1, exponent bits of 2^(23 - F), whether
                                 // the position ends a word
    float s0, s1, mz, qf;        // -(2^23 + 2^(F-1)), -(2^(23-F) + 2^(F-1)), 2^23 + 2^(F-1), 2^(F-1) - 1
    uint32_t M1, M2, M3, share;  // 2^F, 2^2F, 2^3F; the share of 0x4B000000 in sum_e y_e 2^(e F)
};

// Per-item factors, double-buffered by item parity: the factors of the next
// item are written while the current item's fit still reads its own.
struct alignas(16) RowFactors {
    float4 k2[64], l2[64], g2[64];  // a k, a q, gamma (see pslot)
    float4 a2[64], q2[64];          // alpha, 1/Q (0 on pivot rows); row-wise widths only
    float4 h2[64], w2[64];          // fit: h = a / r', w = rho r'^2
    float kqp[4];
    float ra[kDK];                  // a_i = alpha_i r_i (alpha_i on pivot rows), by row-factor thread
    int rb[kDK];                    // widths, by sslot (row-wise widths only)
    float qf[kDK];                  // Q_i as a float (0 on pivot rows), by sslot (row-wise widths only)
    int2 qlh[kDK];                  // bit patterns of 2^23 + 2^(F-1) -+ Q_i (F: the row's position width), by sslot
    float beta;
    int item, head_b;               // the item; its head's common width (0: row-wise)
    int n16;                        // its head's leading positions of 16-bit fields
    int tail_w;                     // row-wise: word offset of the last, partial word (-1: none)
    PosRec pos[kRowsPerGroup];      // row-wise: the head's row positions
};

// Thread p < 16: position p of the head's table (row-wise widths).
__device__ __forceinline__ void make_pos(RowFactors &rf, const HeadRec *rec, int p)
{
    const int O = rec->pos_off[p];
    const int F = rec->pos_bits[p], W = rec->slab_words, m = O >> 5, sh = O & 31;
    PosRec r;
    r.w0 = m * kStreams;
    r.w1 = min(m + 1, W - 1) * kStreams;
    r.sh = sh;
    r.f2 = 2 * F;
    r.m0 = (1u << F) - 1u;
    r.m1 = r.m0 << F;
    r.e1 = (150u - (uint32_t)F) << 23;
    r.done = (sh + 4 * F >= 32) ? 1u : 0u;
    const float z = (float)(1 << (F - 1));
    r.s0 = -(kMagic + z);
    r.s1 = -(__uint_as_float(r.e1) + z);
    r.mz = kMagic + z;
    r.qf = z - 1.f;
    r.M1 = 1u << F;
    r.M2 = r.M1 << F;
    r.M3 = r.M2 << F;
    r.share = kMagicBits * (1u + r.M1 + r.M2 + r.M3);
    rf.pos[p] = r;
    if (p == kRowsPerGroup - 1) {
        const int end = O + 4 * F;
        rf.tail_w = (end & 31) ? (end >> 5) * kStreams : -1;
    }
}

struct alignas(16) ItemSmem {
    struct {
        RowFactors rf[2];
    } u;
    // per value column; warp w touches only its own 16 columns
    float cd[kDV], cdt[kDV], cc0[kDV], cnew[kDV], ci[kDV], crat[kDV];
    // row partials of P^2: [warp][column subgroup][128 rows] in 16-byte
    // chunks swizzled by row group (rowp_chunk)
    float rowp[8 * 4 * kDK];
    uint64_t bar[kMaxSlots];
    int4 recs[2][32];       // producer: staging records, 32 stagings per chunk
};

using X2 = float2[kRowsPerGroup][2];  // the thread's 16 x 4 block as float2 pairs

// Word offset, inside a 128-float row-partial block, of the chunk holding rows
// 16 rg + 4 q .. +3 (conflict-free for both the writes and the row reads).
__device__ __forceinline__ int rowp_chunk(int rg, int q) { return 16 * rg + 4 * (q ^ ((rg >> 1) & 3)); }

// ---------------------------------------------------------------------------
// Field extraction without shifting: a b-bit field at bit sh of a word, kept in
// place and given the exponent 150 - sh, is the float 2^(23 - sh) + u exactly
// (its mantissa bits sh .. sh+b-1 weigh 1 .. 2^(b-1)); subtracting 2^(23 - sh)
// + z leaves the code.  Fields that end above bit 23 are taken from the word's
// upper half (shifted down by 16 once per word); fields that straddle two
// words are funnel-shifted to bit 0.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ constexpr int field_mode(int pos)
{
    return ((pos & 31) + B <= 23) ? 0 : (((pos & 31) + B <= 32) ? 1 : 2);
}

template <int B>
__device__ __forceinline__ void field_raw(const uint32_t *wd, const uint32_t *hw, int pos, int mode, uint32_t &bits,
                                          float &sub)
{
    constexpr uint32_t mask = (1u << B) - 1u;
    const int lo = pos >> 5, sh = pos & 31;
    const float z = (float)(1 << (B - 1));
    if (mode == 0) {
        bits = (wd[lo] & (mask << sh)) | ((150u - (uint32_t)sh) << 23);
        sub = (float)(1 << (23 - sh)) + z;
    } else if (mode == 1) {
        bits = (hw[lo] & (mask << (sh - 16))) | ((150u - (uint32_t)(sh - 16)) << 23);
        sub = (float)(1 << (23 - (sh - 16))) + z;
    } else {
        bits = (__funnelshift_r(wd[lo], wd[lo + 1], sh) & mask) | (150u << 23);
        sub = kMagic + z;
    }
}

// Fields c and c+1 as a float2 of codes.
template <int B>
__device__ __forceinline__ float2 decode_pair(const uint32_t *wd, const uint32_t *hw, int c)
{
    const int p0 = c * B, p1 = p0 + B;
    int m0 = field_mode<B>(p0);
    const int m1 = field_mode<B>(p1);
    // a field that fits either way joins its partner in the upper half
    if (m0 == 0 && m1 == 1 && (p0 >> 5) == (p1 >> 5) && (p0 & 31) >= 16) m0 = 1;
    uint32_t b0, b1;
    float s0, s1;
    field_raw<B>(wd, hw, p0, m0, b0, s0);
    field_raw<B>(wd, hw, p1, m1, b1, s1);
    return __fadd2_rn(f2(__uint_as_float(b0), __uint_as_float(b1)), f2(-s0, -s1));
}

// ---------------------------------------------------------------------------
// Decode the thread's stream (word m at words[32 m]) of a head of one width B
// into X (code values as floats), the stream kept in registers.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void decode_stream(const uint32_t *words, X2 &X)
{
    static_assert(B > 0, "fixed widths only");
    {
        uint32_t wd[2 * B + 1], hw[2 * B];
#pragma unroll
        for (int m = 0; m < 2 * B; m++) wd[m] = words[m * kStreams];
        wd[2 * B] = 0u;
#pragma unroll
        for (int m = 0; m < 2 * B; m++) hw[m] = wd[m] >> 16;
#pragma unroll
        for (int rr = 0; rr < kRowsPerGroup; rr++)
#pragma unroll
            for (int hh = 0; hh < 2; hh++) X[rr][hh] = decode_pair<B>(wd, hw, 4 * rr + 2 * hh);
    }
}

// ---------------------------------------------------------------------------
// Decode for row-wise widths.  The 4 fields of row position rr lie at the same
// bit offset O in every stream of the head, F = pos_bits[rr] bits each, so the
// lanes of a warp decode in lockstep at warp-uniform offsets: the 32 bits from
// O on (a funnel shift of two words), fields 0 and 1 in place and fields 2
// and 3 from the bits shifted down by 2F, each as 2^(23 - e F) + u by the
// exponent trick.  Positions of 16-bit fields (rows at a pivot row's
// position) lead, word aligned; a pivot row's field is its binary16 value.
// Only positions rr < NP are checked for them (NP = 1 when the head has at
// most one such position).  rf.pos is the head's position table.
// ---------------------------------------------------------------------------
template <int NP>
__device__ __forceinline__ void decode_rowwise(const RowFactors &rf, int rg, const uint32_t *words, X2 &X)
{
    const int n16 = rf.n16;
#pragma unroll
    for (int rr = 0; rr < kRowsPerGroup; rr++) {
        const uint4 A = *reinterpret_cast<const uint4 *>(&rf.pos[rr].w0);
        if (rr < NP && rr < n16) {
            const uint32_t w0 = words[A.x], w1 = words[A.y];
            if (rf.rb[8 * rr + rg] == kPivotBits) {
                X[rr][0] = __half22float2(*reinterpret_cast<const __half2 *>(&w0));
                X[rr][1] = __half22float2(*reinterpret_cast<const __half2 *>(&w1));
            } else {
                const float2 sub = f2(-(kMagic + 32768.f), -(kMagic + 32768.f));
                X[rr][0] = __fadd2_rn(
                    f2(__uint_as_float((w0 & 0xFFFFu) | kMagicBits), __uint_as_float((w0 >> 16) | kMagicBits)), sub);
                X[rr][1] = __fadd2_rn(
                    f2(__uint_as_float((w1 & 0xFFFFu) | kMagicBits), __uint_as_float((w1 >> 16) | kMagicBits)), sub);
            }
        } else {
            const uint4 M = *reinterpret_cast<const uint4 *>(&rf.pos[rr].m0);
            const float2 sub = *reinterpret_cast<const float2 *>(&rf.pos[rr].s0);
            const uint32_t f = __funnelshift_r(words[A.x], words[A.y], A.z);
            const uint32_t fh = f >> A.w;
            X[rr][0] = __fadd2_rn(f2(__uint_as_float((f & M.x) | kMagicBits), __uint_as_float((f & M.y) | M.z)), sub);
            X[rr][1] = __fadd2_rn(f2(__uint_as_float((fh & M.x) | kMagicBits), __uint_as_float((fh & M.y) | M.z)), sub);
        }
    }
}

// Sum over the 8 lanes sharing cg of two 4-column vectors (A0|A1 and B0|B1,
// float2 each), scattered: on return lane rg holds the full sum of vector
// (rg & 4 ? B : A) at column rg & 3 of the thread's four.
__device__ __forceinline__ float reduce_scatter_2x4(float2 A0, float2 A1, float2 B0, float2 B1, int rg)
{
    const bool hiA = rg & 4, hiB = rg & 2, hiC = rg & 1;
    float2 k0 = hiA ? B0 : A0, k1 = hiA ? B1 : A1;
    const float2 s0 = hiA ? A0 : B0, s1 = hiA ? A1 : B1;
    k0 = __fadd2_rn(k0, shfl2(s0, 4));
    k1 = __fadd2_rn(k1, shfl2(s1, 4));
    float2 kk = hiB ? k1 : k0;
    const float2 ss = hiB ? k0 : k1;
    kk = __fadd2_rn(kk, shfl2(ss, 2));
    const float v = hiC ? kk.y : kk.x;
    const float sv = hiC ? kk.x : kk.y;
    return v + __shfl_xor_sync(kFull, sv, 1);
}

// ---------------------------------------------------------------------------
// One least-squares round: with n = rne(p / c) (clipped to the row's range
// when CLIP), N_j = sum w_i n_ij p_ij and D_j = sum w_i n_ij^2 over the
// warp's rows; then c_j = N_j / D_j (kept when D_j = 0), its reciprocal and
// c0_j / c_j for the warp's 16 columns.
// ---------------------------------------------------------------------------
template <int B, bool ROWWISE, bool CLIP, int NP>
__device__ __forceinline__ void ls_round(ItemSmem &sm, const RowFactors &rf, const X2 &X)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    const float2 rm2 = f2(kRoundMagic, kRoundMagic), nrm2 = f2(-kRoundMagic, -kRoundMagic);
    const float4 i4 = ld4(&sm.ci[col0]);
    const float2 ic0 = f2(i4.x, i4.y), ic1 = f2(i4.z, i4.w);
    float2 N0 = f2(0.f, 0.f), N1 = N0, D0 = N0, D1 = N0;
#pragma unroll
    for (int p = 0; p < kRowsPerGroup / 2; p++) {
        float2 wp[2];
        ld_pairs(rf.w2, p, rg, wp);
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const int rr = 2 * p + u;
            if (ROWWISE && rr < NP && rr < rf.n16 && rf.rb[8 * rr + rg] == kPivotBits) continue;
            // round to the nearest integer, ties to even: x + 1.5 * 2^23 - 1.5 * 2^23;
            // clipping acts on the biased value
            float2 m0 = __ffma2_rn(X[rr][0], ic0, rm2);
            float2 m1 = __ffma2_rn(X[rr][1], ic1, rm2);
            if (CLIP) {
                const float Q = ROWWISE ? rf.qf[8 * rr + rg] : (float)qmax_of(B);
                const float lo = kRoundMagic - Q, hi = kRoundMagic + Q;
                m0 = f2(fminf(fmaxf(m0.x, lo), hi), fminf(fmaxf(m0.y, lo), hi));
                m1 = f2(fminf(fmaxf(m1.x, lo), hi), fminf(fmaxf(m1.y, lo), hi));
            }
            const float2 n0 = __fadd2_rn(m0, nrm2), n1 = __fadd2_rn(m1, nrm2);
            const float2 wn0 = __fmul2_rn(wp[u], n0), wn1 = __fmul2_rn(wp[u], n1);
            N0 = __ffma2_rn(wn0, X[rr][0], N0);
            N1 = __ffma2_rn(wn1, X[rr][1], N1);
            D0 = __ffma2_rn(wn0, n0, D0);
            D1 = __ffma2_rn(wn1, n1, D1);
        }
    }
    // lane rg: N (rg < 4) or D (rg >= 4) of column col0 + (rg & 3)
    const float part = reduce_scatter_2x4(N0, N1, D0, D1, rg);
    const float other = __shfl_xor_sync(kFull, part, 4);
    if (rg < 4) {
        const int j = col0 + rg;
        const float c = (other > 0.f) ? div_approx(part, other) : sm.cnew[j];
        const float icn = rcp_approx(c);
        sm.cnew[j] = c;
        sm.ci[j] = icn;
        sm.crat[j] = sm.cc0[j] * icn;
    }
    __syncwarp();
}

// Final codes of a fixed-width stream and their store: u = z + clip(rne(p / c))
// taken from the low mantissa bits of p / c + 2^23 + z; each 32-bit word is
// stored as soon as its last code is placed.
// Word m of a fixed-width stream is the sum over its fields of y << sh, y =
// 0x4B000000 | u the float bits of 2^23 + u (fields that straddle into the next
// word enter as u alone), minus the words' share of 0x4B000000 << sh, a
// constant: the sum has no carries between fields.
template <int B>
__device__ __forceinline__ constexpr uint32_t magic_share(int m)
{
    uint32_t acc = 0u;
    for (int c = 0; c < 64; c++) {
        const int pos = c * B;
        if ((pos >> 5) == m && (pos & 31) + B <= 32) acc += kMagicBits << (pos & 31);
    }
    return acc;
}

template <int B, bool CLIP>
__device__ __forceinline__ void pack_fixed(const X2 &X, float2 ic0, float2 ic1, uint32_t *words)
{
    constexpr int Qb = (1 << (B - 1)) - 1;
    const float mz = kMagic + (float)(1 << (B - 1));
    const float2 mz2 = f2(mz, mz);
    uint32_t ow[2 * B + 1];
#pragma unroll
    for (int m = 0; m <= 2 * B; m++) ow[m] = 0u - magic_share<B>(m);
#pragma unroll
    for (int rr = 0; rr < kRowsPerGroup; rr++)
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
            // p / c + 2^23 + z rounded once; clipping clamps its bit pattern to those
            // of 2^23 + z -+ Q (the float order is the integer order of the bits,
            // negative values included as signed integers)
            const float2 mm = __ffma2_rn(X[rr][hh], hh ? ic1 : ic0, mz2);
            constexpr int kLo = (int)kMagicBits + (1 << (B - 1)) - Qb, kHi = (int)kMagicBits + (1 << (B - 1)) + Qb;
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int c = 4 * rr + 2 * hh + e;
                uint32_t y = __float_as_uint(e ? mm.y : mm.x);
                if (CLIP) y = (uint32_t)min(max((int)y, kLo), kHi);
                const int pos = c * B, lo = pos >> 5, sh = pos & 31;
                if (sh + B <= 32) {
                    ow[lo] += y << sh;
                } else {
                    const uint32_t u = y & ((1u << B) - 1u);
                    ow[lo] += u << sh;
                    ow[lo + 1] += u >> (32 - sh);
                }
#pragma unroll
                for (int m = (c * B) / 32; m < ((c + 1) * B) / 32; m++) words[m * kStreams] = ow[m];
            }
        }
}

// Final codes and store for row-wise widths: the fields of row position rr go
// to the head's common bit offset O in F = pos_bits[rr] bits (offset-binary
// about 2^(F - 1)), the code clipped to the row's own range +-Q_i.  The four
// fields of a position form one value f = sum_e y_e 2^(e F) minus the share of
// the constant 0x4B000000 in it (y_e the float bits of 2^23 + u_e); f joins
// the pending word at bit O % 32, and a word is stored as soon as it is
// complete.  Clipping is decided per position with the widest range there,
// which bounds every row's.  Leading positions of 16-bit fields store a pivot
// row's binary16 values or the 16-bit codes of the rows beside it.
template <int NP>
__device__ __forceinline__ void pack_rowwise(const X2 &X, float2 ic0, float2 ic1, const RowFactors &rf, float rat,
                                             int rg, uint32_t *words)
{
    const int n16 = rf.n16;
    uint32_t acc = 0u;  // the bits of the current word below the position's offset
#pragma unroll
    for (int rr = 0; rr < kRowsPerGroup; rr++) {
        const uint4 A = *reinterpret_cast<const uint4 *>(&rf.pos[rr].w0);
        if (rr < NP && rr < n16) {
            uint32_t o0, o1;
            if (rf.rb[8 * rr + rg] == kPivotBits) {
                const __half2 h0 = __floats2half2_rn(X[rr][0].x, X[rr][0].y);
                const __half2 h1 = __floats2half2_rn(X[rr][1].x, X[rr][1].y);
                o0 = *reinterpret_cast<const uint32_t *>(&h0);
                o1 = *reinterpret_cast<const uint32_t *>(&h1);
            } else {
                const float Q = rf.qf[8 * rr + rg];
                const float2 mz2 = f2(kMagic + 32768.f, kMagic + 32768.f);
                float2 t0 = __fmul2_rn(X[rr][0], ic0), t1 = __fmul2_rn(X[rr][1], ic1);
                t0 = f2(fminf(fmaxf(t0.x, -Q), Q), fminf(fmaxf(t0.y, -Q), Q));
                t1 = f2(fminf(fmaxf(t1.x, -Q), Q), fminf(fmaxf(t1.y, -Q), Q));
                const float2 y0 = __fadd2_rn(t0, mz2), y1 = __fadd2_rn(t1, mz2);
                o0 = (__float_as_uint(y0.x) & 0xFFFFu) | (__float_as_uint(y0.y) << 16);
                o1 = (__float_as_uint(y1.x) & 0xFFFFu) | (__float_as_uint(y1.y) << 16);
            }
            words[A.x] = o0;
            words[A.y] = o1;
        } else {
            const float2 zq = *reinterpret_cast<const float2 *>(&rf.pos[rr].mz);  // (2^23 + z, Q_F)
            const uint4 M = *reinterpret_cast<const uint4 *>(&rf.pos[rr].M1);
            const float2 mz2 = f2(zq.x, zq.x);
            const float2 y0 = __ffma2_rn(X[rr][0], ic0, mz2), y1 = __ffma2_rn(X[rr][1], ic1, mz2);
            uint32_t u0 = __float_as_uint(y0.x), u1 = __float_as_uint(y0.y);
            uint32_t u2 = __float_as_uint(y1.x), u3 = __float_as_uint(y1.y);
            if (zq.y * (rat - 1.f) >= 0.49f) {  // clip to the row's own range, on the bit patterns
                const int2 b = rf.qlh[8 * rr + rg];
                u0 = (uint32_t)min(max((int)u0, b.x), b.y);
                u1 = (uint32_t)min(max((int)u1, b.x), b.y);
                u2 = (uint32_t)min(max((int)u2, b.x), b.y);
                u3 = (uint32_t)min(max((int)u3, b.x), b.y);
            }
            uint32_t f = u0 - M.w;
            f += u1 * M.x;
            f += u2 * M.y;
            f += u3 * M.z;
            acc |= f << A.z;
            if (rf.pos[rr].done) {
                words[A.x] = acc;
                acc = __funnelshift_l(f, 0u, A.z);  // the bits of f beyond the word (none when O % 32 = 0)
            }
        }
    }
    if (rf.tail_w >= 0) words[rf.tail_w] = acc;
}

// The calibration's per-row error of a fixed width B: the codes the pack would
// store (same clip decision), e = p - c code per element, the thread's row
// partials of e^2 through the row-partial buffer, then row i (thread i):
// r'_i^2 times the sum of its 32 partials.  r' is read back from the r[]
// the fit wrote (by the same thread).
template <int B>
__device__ __forceinline__ void row_errors(ItemSmem &sm, const X2 &X, float2 ic0, float2 ic1, float rat,
                                           const float *r_out, float *err_out)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    constexpr int Qb = (1 << (B - 1)) - 1;
    const bool clip = (float)Qb * (rat - 1.f) >= 0.49f;
    const float4 c4 = ld4(&sm.cnew[col0]);
    const float2 nc0 = f2(-c4.x, -c4.y), nc1 = f2(-c4.z, -c4.w);
    const float2 rm2 = f2(kRoundMagic, kRoundMagic), nrm2 = f2(-kRoundMagic, -kRoundMagic);
    float *T = &sm.rowp[(4 * w + cg) * kDK];
#pragma unroll
    for (int q = 0; q < 4; q++) {
        float s[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int rr = 4 * q + e;
            float2 n0, n1;
            if (!clip) {
                n0 = __fadd2_rn(__ffma2_rn(X[rr][0], ic0, rm2), nrm2);
                n1 = __fadd2_rn(__ffma2_rn(X[rr][1], ic1, rm2), nrm2);
            } else {
                float2 t0 = __fmul2_rn(X[rr][0], ic0), t1 = __fmul2_rn(X[rr][1], ic1);
                t0 = f2(fminf(fmaxf(t0.x, -(float)Qb), (float)Qb), fminf(fmaxf(t0.y, -(float)Qb), (float)Qb));
                t1 = f2(fminf(fmaxf(t1.x, -(float)Qb), (float)Qb), fminf(fmaxf(t1.y, -(float)Qb), (float)Qb));
                n0 = __fadd2_rn(__fadd2_rn(t0, rm2), nrm2);
                n1 = __fadd2_rn(__fadd2_rn(t1, rm2), nrm2);
            }
            const float2 e0 = __ffma2_rn(nc0, n0, X[rr][0]), e1 = __ffma2_rn(nc1, n1, X[rr][1]);
            float2 s2 = __fmul2_rn(e0, e0);
            s2 = __ffma2_rn(e1, e1, s2);
            s[e] = s2.x + s2.y;
        }
        *reinterpret_cast<float4 *>(T + rowp_chunk(rg, q)) = make_float4(s[0], s[1], s[2], s[3]);
    }
    __syncthreads();
    if (tid < kDK) {
        const int i = tid, irg = i >> 4, irr = i & 15;
        const float *src = &sm.rowp[rowp_chunk(irg, irr >> 2) + (irr & 3)];
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int bk = 0; bk < 32; bk += 4) {
            s0 += src[(bk + 0) * kDK];
            s1 += src[(bk + 1) * kDK];
            s2 += src[(bk + 2) * kDK];
            s3 += src[(bk + 3) * kDK];
        }
        const float rp = r_out[i];
        err_out[i] = (rp * rp) * ((s0 + s1) + (s2 + s3));
    }
}

// Nothing to do between the two barriers of the fit (pack kernel).
struct NoMid {
    __device__ __forceinline__ bool operator()() const { return true; }
    __device__ __forceinline__ bool rowside(int) const { return true; }
};

enum FitResult { kFitDone = 0, kFitAbortNow = 1, kFitAbortAfter = 2 };

// ---------------------------------------------------------------------------
// The fit (row scales, column scales, least squares), requantisation and the
// packed store.  On entry X holds P_ij = S_ij / a_i on quantised rows and S_ij
// on pivot rows; rf.ra, rb (and q2 for row-wise widths) are set, rec is the
// head's record (fit constants).  Writes r', c and the item's streams at
// item_g (W words per stream).
//
// Barrier 1 publishes the row partials of P^2; threads 0..127 then derive row
// i's scale and fit factors and run mid.rowside(i), while mid() runs on
// threads 128..255 (the fused step prepares the next item there); barrier 2
// publishes both, and everything after it is warp-local.  If ok_in is false on any thread the
// item is abandoned at barrier 1 with nothing stored (kFitAbortNow); if `mid`
// fails on any thread the item is completed and kFitAbortAfter returned.
// ---------------------------------------------------------------------------
// ERR (fixed widths; calibration): instead of packing, the squared
// reconstruction error of every row, r'^2 sum_j (p_ij - c_j code_ij)^2 with the
// codes the pack would store, goes to err_out[row] (item_g receives r' and c).
// MODE (ablations): kScaleDual is the method; kScaleRow keeps c = 1 and sets
// r_i = max_j |S_ij| / Q_i (0 -> 1 / Q_i); kScaleCol sets r_i = 1 / Q_i and
// c_j = max_i |S_ij| (0 -> 1); kScaleHead as kScaleCol with every c_j the
// largest of them.  The variants use no impact weights and no least squares.
template <int B, bool ROWWISE, bool MULTI, int NP, class Mid, bool ERR = false, int MODE = kScaleDual>
__device__ __forceinline__ FitResult fit_and_store(ItemSmem &sm, RowFactors &rf, const HeadRec *rec, X2 &X,
                                                   uint8_t *item_g, int W, int ls_iters, bool store_c,
                                                   bool ok_in, const Mid &mid, float *err_out = nullptr)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    // ---- row partials of P^2 over the thread's 4 columns -------------------
    {
        float *T = &sm.rowp[(4 * w + cg) * kDK];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            float s[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int rr = 4 * q + e;
                if constexpr (MODE == kScaleRow) {  // row maxima of |P|
                    s[e] = max_abs3(fabsf(X[rr][0].x), X[rr][0].y, X[rr][1].x);
                    s[e] = max_abs3(s[e], X[rr][1].y, 0.f);
                } else {
                    float2 s2 = __fmul2_rn(X[rr][0], X[rr][0]);
                    s2 = __ffma2_rn(X[rr][1], X[rr][1], s2);
                    s[e] = s2.x + s2.y;
                }
            }
            *reinterpret_cast<float4 *>(T + rowp_chunk(rg, q)) = make_float4(s[0], s[1], s[2], s[3]);
        }
    }
    if (__syncthreads_or(!ok_in)) return kFitAbortNow;
    bool ok_mid = true;
    if (tid < kDK) {
        // ---- row i: RMS over the 128 columns, new row scale, fit factors -----
        const int i = ROWWISE ? frow(tid) : tid, irg = i >> 4, irr = i & 15;
        const float *src = &sm.rowp[rowp_chunk(irg, irr >> 2) + (irr & 3)];
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int bk = 0; bk < 32; bk += 4) {
            if constexpr (MODE == kScaleRow) {
                s0 = fmaxf(s0, src[(bk + 0) * kDK]);
                s1 = fmaxf(s1, src[(bk + 1) * kDK]);
                s2 = fmaxf(s2, src[(bk + 2) * kDK]);
                s3 = fmaxf(s3, src[(bk + 3) * kDK]);
            } else {
                s0 += src[(bk + 0) * kDK];
                s1 += src[(bk + 1) * kDK];
                s2 += src[(bk + 2) * kDK];
                s3 += src[(bk + 3) * kDK];
            }
        }
        const int b = ROWWISE ? rec->bits[i] : B;
        float rnew = 0.f, h = 1.f, wt = 0.f;  // pivot rows: p = S, not part of any fit
        if (!ROWWISE || b != kPivotBits) {
            const float a = rf.ra[tid];
            if constexpr (MODE == kScaleDual) {
                const float ss = (s0 + s1) + (s2 + s3);
                float m = a * sqrt_approx(ss * (1.0f / kDV));
                if (m == 0.f) m = 1.f;
                rnew = (m * rec->s[i]) * rec->rq[i];
                wt = (rec->rho[i] * rnew) * rnew;
            } else if constexpr (MODE == kScaleRow) {
                float m = a * fmaxf(fmaxf(s0, s1), fmaxf(s2, s3));
                if (m == 0.f) m = 1.f;
                rnew = m * rec->rq[i];
            } else {
                rnew = rec->rq[i];
            }
            h = div_approx(a, rnew);
        }
        put_pair(rf.h2, i, h);
        put_pair(rf.w2, i, wt);
        reinterpret_cast<float *>(item_g)[i] = rnew;
        ok_mid = mid.rowside(i);
    } else {
        ok_mid = mid();
    }
    const bool abort_after = __syncthreads_or(!ok_mid);
    // ---- p = P h; column maxima (of |p| / Q_i for row-wise widths) ----------
    {
        float mx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < kRowsPerGroup / 2; p++) {
            float2 hh[2], qq[2], pv[2][2];
            ld_pairs(rf.h2, p, rg, hh);
            if (ROWWISE) ld_pairs(rf.q2, p, rg, qq);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int rr = 2 * p + u;
                X[rr][0] = __fmul2_rn(X[rr][0], hh[u]);
                X[rr][1] = __fmul2_rn(X[rr][1], hh[u]);
                pv[u][0] = X[rr][0];
                pv[u][1] = X[rr][1];
                if (ROWWISE) {  // pivot rows have q = 0 and do not count
                    pv[u][0] = __fmul2_rn(pv[u][0], qq[u]);
                    pv[u][1] = __fmul2_rn(pv[u][1], qq[u]);
                }
            }
            mx[0] = max_abs3(mx[0], pv[0][0].x, pv[1][0].x);
            mx[1] = max_abs3(mx[1], pv[0][0].y, pv[1][0].y);
            mx[2] = max_abs3(mx[2], pv[0][1].x, pv[1][1].x);
            mx[3] = max_abs3(mx[3], pv[0][1].y, pv[1][1].y);
        }
        // maximum over the 8 lanes sharing cg: lanes rg and rg ^ 1 end with
        // column col0 + 2 (rg >> 2 & 1) + (rg >> 1 & 1)
        const bool hiA = rg & 4, hiB = rg & 2;
        float k0 = hiA ? mx[2] : mx[0], k1 = hiA ? mx[3] : mx[1];
        const float t0 = hiA ? mx[0] : mx[2], t1 = hiA ? mx[1] : mx[3];
        k0 = fmaxf(k0, __shfl_xor_sync(kFull, t0, 4));
        k1 = fmaxf(k1, __shfl_xor_sync(kFull, t1, 4));
        float m = hiB ? k1 : k0;
        m = fmaxf(m, __shfl_xor_sync(kFull, hiB ? k0 : k1, 2));
        m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
        if constexpr (!ROWWISE) m = m * (1.0f / (float)((1 << (B - 1)) - 1));  // every row has width B
        if constexpr (MODE == kScaleRow) m = 1.f;
        if constexpr (MODE == kScaleHead) {  // the largest over all 128 columns
            if ((rg & 1) == 0) sm.cnew[col0 + 2 * hiA + hiB] = m;
            __syncthreads();
            float top = fmaxf(fmaxf(sm.cnew[l], sm.cnew[l + 32]), fmaxf(sm.cnew[l + 64], sm.cnew[l + 96]));
            top = __uint_as_float(__reduce_max_sync(kFull, __float_as_uint(top)));  // non-negative floats
            __syncthreads();
            m = top;
        }
        if ((rg & 1) == 0) {
            const int j = col0 + 2 * hiA + hiB;
            const float c0 = (m > 0.f) ? m : 1.f;
            sm.cc0[j] = c0;
            sm.cnew[j] = c0;
            sm.ci[j] = rcp_approx(c0);
            sm.crat[j] = 1.f;
        }
        __syncwarp();
    }
    // ---- impact-weighted least squares for the column scales ---------------
    // |p / c0| <= Q, so the first round needs no clipping; later rounds clip to
    // the row's range.  More than one round is a separate instantiation (MULTI)
    // so that the one-round code holds a single round body.
    if constexpr (MODE != kScaleDual) {
        // the variants keep the maxima
    } else if (!MULTI) {
        if (ls_iters > 0) ls_round<B, ROWWISE, false, NP>(sm, rf, X);
    } else {
        for (int it = 0; it < ls_iters; it++) {
            if (it == 0)
                ls_round<B, ROWWISE, false, NP>(sm, rf, X);
            else
                ls_round<B, ROWWISE, true, NP>(sm, rf, X);
        }
    }
    // the column scales are final: store them before the codes
    if (l < 16) reinterpret_cast<float *>(item_g)[kDK + 16 * w + l] = store_c ? sm.cnew[16 * w + l] : 0.f;
    // ---- requantise, pack, store -------------------------------------------
    const float4 i4 = ld4(&sm.ci[col0]);
    const float2 ic0 = f2(i4.x, i4.y), ic1 = f2(i4.z, i4.w);
    float rat;
    {
        const float4 r = ld4(&sm.crat[col0]);
        rat = fmaxf(fmaxf(r.x, r.y), fmaxf(r.z, r.w));
    }
    // the largest |p / c| of a column is at most Q c0 / c: clip only where that
    // can reach Q + 1/2 (decided per warp)
    rat = __uint_as_float(__reduce_max_sync(kFull, __float_as_uint(rat)));
    if constexpr (ERR) {
        static_assert(B > 0 && !ROWWISE, "the error mode fits one width");
        row_errors<B>(sm, X, ic0, ic1, rat, reinterpret_cast<const float *>(item_g), err_out);
        return kFitDone;
    }
    uint32_t *words = reinterpret_cast<uint32_t *>(item_g + kHeaderBytes) + (kStreams * W) * w + l;
    if constexpr (B > 0) {
        constexpr int Qb = (1 << (B - 1)) - 1;
        if ((float)Qb * (rat - 1.f) >= 0.49f)
            pack_fixed<B, true>(X, ic0, ic1, words);
        else
            pack_fixed<B, false>(X, ic0, ic1, words);
    } else {
        pack_rowwise<NP>(X, ic0, ic1, rf, rat, rg, words);
    }
    return abort_after ? kFitAbortAfter : kFitDone;
}

#ifndef STEPQ_CHECK
#define STEPQ_CHECK 0
#endif

#if STEPQ_CHECK
// Checking build: every head record against the head tables and the layout
// (threads n < heads), every staging record n < n_pos against the order table,
// the head tables and the packed states' extent.  Any mismatch sets the status
// word; the kernels that read the tables then return without touching memory.
__global__ void __launch_bounds__(256) k_check_tables(StepArgs a, int n_pos)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    bool bad = false;
    if (n < a.heads) {
        const HeadRec &R = a.t.rowrec[n];
        const long long off = a.t.head_off[n];
        const int hb = a.t.head_bytes[n], W = R.slab_words;
        bad |= R.head_off != off || R.head_bytes != hb || off < 0 || off + hb > a.req_bytes;
        bad |= hb != kHeaderBytes + 4 * W * kStreams * kSlabs;
        if (R.head_kind == kHeadAllPivot) {
            bad |= W != 2 * kRowsPerGroup;
        } else {
            int sum_f = 0;
            for (int p = 0; p < kRowsPerGroup; p++) {
                bad |= R.pos_off[p] != 4 * sum_f;
                sum_f += R.pos_bits[p];
            }
            bad |= (R.head_b > 0) ? (W != 2 * R.head_b) : (W != (4 * sum_f + 31) / 32);
        }
    }
    if (n < n_pos) {
        const int4 st = a.t.stage[n];
        const int item = st.x, h = (int)((uint32_t)st.y >> 16), bytes = st.y & 0xFFFF;
        const long long off = (long long)(uint32_t)st.z << 10;
        bad |= item < 0 || (long long)item >= (long long)a.batch * a.heads || h >= a.heads || h != item % a.heads ||
               st.w != item / a.heads;
        if (!bad) {
            bad |= a.t.order[n] != item || bytes != a.t.head_bytes[h];
            bad |= off != (long long)st.w * a.req_bytes + a.t.head_off[h] || off + bytes > a.state_bytes;
            bad |= (n < a.n_pivot_items) != (a.t.rowrec[h].head_kind == kHeadAllPivot);
        }
    }
    if (bad) atomicExch(a.t.status, kStatusBadTable);
}

// CTA-uniform: whether the status word is set (the kernel then returns).
__device__ __forceinline__ bool tables_rejected(const StepArgs &a)
{
    return __syncthreads_or(threadIdx.x == 0 && *reinterpret_cast<volatile int *>(a.t.status) != 0);
}
#define STEPQ_RETURN_IF_REJECTED(a) \
    if (tables_rejected(a)) return
#else
#define STEPQ_RETURN_IF_REJECTED(a) \
    do {                            \
    } while (0)
#endif

// ---------------------------------------------------------------------------
// The fused decode step: persistent CTAs walk the item order.  Items of heads
// whose rows are all FP16 pivots come first in the order and are processed
// straight from global memory; every other item is staged into a ring of
// shared-memory slots by bulk copies (one mbarrier per slot) several items
// ahead of the compute.
// ---------------------------------------------------------------------------

// An item of an all-pivot head, straight from global memory: binary16 state,
// update and readout, no fit.  Every row of the item is a pivot row, so each
// stream holds 16 rows x 4 binary16 values (two words per row), and each
// thread derives its own rows' factors; no barrier.
__device__ void pivot_item(const StepArgs &a, int pos)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    const int4 st = a.t.stage[pos];  // {item, bytes | head << 16, state offset / 1024, request}
    const int item = st.x;
    uint8_t *item_g = a.pool + ((long long)(uint32_t)st.z << 10);
    const long long vec = (long long)item * kDK + kRowsPerGroup * rg;
    const float beta = a.beta[item];
    uint32_t *words = reinterpret_cast<uint32_t *>(item_g + kHeaderBytes) + (kStreams * 2 * kRowsPerGroup) * w + l;
    X2 X;
    float2 V0 = f2(0.f, 0.f), V1 = V0, U0 = V0, U1 = V0;
    float kq = 0.f;
#pragma unroll
    for (int q4 = 0; q4 < kRowsPerGroup / 4; q4++) {
        const float4 k4 = ld4(a.k + vec + 4 * q4), qv4 = ld4(a.q + vec + 4 * q4);
        const float4 al4 = a.kda ? ld4(a.alpha + vec + 4 * q4) : make_float4(a.alpha[item], a.alpha[item],
                                                                             a.alpha[item], a.alpha[item]);
        const float kk[4] = {k4.x, k4.y, k4.z, k4.w}, qq[4] = {qv4.x, qv4.y, qv4.z, qv4.w};
        const float aa[4] = {al4.x, al4.y, al4.z, al4.w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int rr = 4 * q4 + e;
            const uint32_t w0 = words[(2 * rr) * kStreams], w1 = words[(2 * rr + 1) * kStreams];
            const float2 h0 = __half22float2(*reinterpret_cast<const __half2 *>(&w0));
            const float2 h1 = __half22float2(*reinterpret_cast<const __half2 *>(&w1));
            const float2 a2 = f2(aa[e], aa[e]);
            const float2 kp = f2(aa[e] * kk[e], aa[e] * kk[e]), lp = f2(aa[e] * qq[e], aa[e] * qq[e]);
            X[rr][0] = __fmul2_rn(a2, h0);
            X[rr][1] = __fmul2_rn(a2, h1);
            V0 = __ffma2_rn(kp, h0, V0);
            V1 = __ffma2_rn(kp, h1, V1);
            U0 = __ffma2_rn(lp, h0, U0);
            U1 = __ffma2_rn(lp, h1, U1);
            kq = fmaf(kk[e], qq[e], kq);
        }
    }
    // k.q over all rows: the 8 row groups are the lanes sharing cg
    kq += __shfl_xor_sync(kFull, kq, 1);
    kq += __shfl_xor_sync(kFull, kq, 2);
    kq += __shfl_xor_sync(kFull, kq, 4);
    // lane rg: v_old (rg < 4) or the query projection (rg >= 4) of column col0 + (rg & 3)
    const float part = reduce_scatter_2x4(V0, V1, U0, U1, rg);
    const int j = col0 + (rg & 3);
    const float d = a.v[(long long)item * kDV + j] - part;
    const float d_col = __shfl_xor_sync(kFull, d, 4);
    if (rg >= 4) a.out[(long long)item * kDV + j] = fmaf(beta * kq, d_col, part);
    // d of the thread's four columns: lanes cg*8 + 0..3 hold them
    float dd[4];
#pragma unroll
    for (int e = 0; e < 4; e++) dd[e] = __shfl_sync(kFull, d, 8 * cg + e);
    const float2 d0 = f2(dd[0], dd[1]), d1 = f2(dd[2], dd[3]);
#pragma unroll
    for (int q4 = 0; q4 < kRowsPerGroup / 4; q4++) {
        const float4 k4 = ld4(a.k + vec + 4 * q4);
        const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int rr = 4 * q4 + e;
            const float2 gg = f2(beta * kk[e], beta * kk[e]);
            const float2 s0 = __ffma2_rn(gg, d0, X[rr][0]), s1 = __ffma2_rn(gg, d1, X[rr][1]);
            const __half2 h0 = __floats2half2_rn(s0.x, s0.y);
            const __half2 h1 = __floats2half2_rn(s1.x, s1.y);
            words[(2 * rr) * kStreams] = *reinterpret_cast<const uint32_t *>(&h0);
            words[(2 * rr + 1) * kStreams] = *reinterpret_cast<const uint32_t *>(&h1);
        }
    }
}

// Stage one item into slot buffer sb, on every lane of the producer warp: the
// packed item and the head record by bulk copies (lane 0), q, k, v (and the
// KDA gates) as 16-byte asynchronous copies, one per lane and vector, and the
// per-item scalars (lane 0).  All of it completes on the slot's barrier, which
// counts lane 0's expect-tx arrival and one arrival per lane for its copies.
template <bool KDA>
__device__ __forceinline__ void stage_item(const StepArgs &a, int4 st, uint8_t *sb, uint64_t *bar)
{
    const int lane = threadIdx.x & 31;
    const int item = st.x, h = (int)((uint32_t)st.y >> 16);
    const long long vec = (long long)item * kDK;
    if (lane == 0) {
        const uint32_t bytes = (uint32_t)st.y & 0xFFFFu;
        const uint8_t *src = a.pool + ((long long)(uint32_t)st.z << 10);
        mbar_arrive_expect_tx(bar, bytes + (uint32_t)sizeof(HeadRec));
        bulk_g2s(sb, src, bytes, bar);
        bulk_g2s(sb + a.off_rec, a.t.rowrec + h, sizeof(HeadRec), bar);
        const uint32_t dab = smem_addr(sb + a.off_ab);
        if (!KDA) asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dab), "l"(a.alpha + item) : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dab + 4), "l"(a.beta + item) : "memory");
    }
    const uint32_t o = 16u * lane;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(sb + a.off_q) + o), "l"(a.q + vec + 4 * lane)
                 : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(sb + a.off_k) + o), "l"(a.k + vec + 4 * lane)
                 : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(sb + a.off_v) + o),
                 "l"(a.v + (long long)item * kDV + 4 * lane)
                 : "memory");
    if (KDA)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(sb + a.off_alpha) + o),
                     "l"(a.alpha + vec + 4 * lane)
                     : "memory");
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Arrivals that complete one staging: lane 0's expect-tx arrival and the 32
// lanes' asynchronous-copy arrivals.
constexpr uint32_t kStageArrivals = 1 + 32;

// Staging records: staging number k of the CTA stages position n_first + k G
// (if it exists) from recs[k / 32 % 2][k % 32].  The producer warp fetches
// them 32 at a time (one 16-byte async copy per lane) a chunk ahead of use.
__device__ __forceinline__ void fetch_rec_chunk(ItemSmem &sm, const StepArgs &a, int n_first, uint32_t chunk)
{
    const int lane = threadIdx.x & 31;
    const long long n = (long long)n_first + (long long)(32 * chunk + lane) * gridDim.x;
    if (n < a.n_items)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(&sm.recs[chunk & 1][lane])),
                     "l"(a.t.stage + n)
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Issue staging k into slot buffer sb (the whole producer warp; the caller
// checks that the position exists).  At the start of every chunk of 32
// stagings the warp waits for that chunk's records and fetches the next
// chunk's.
template <bool KDA>
__device__ __forceinline__ void produce(ItemSmem &sm, const StepArgs &a, int n_first, uint32_t k, uint8_t *sb,
                                        uint64_t *bar)
{
    if ((k & 31u) == 0) {
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        fetch_rec_chunk(sm, a, n_first, (k >> 5) + 1);
    }
    stage_item<KDA>(a, sm.recs[(k >> 5) & 1][k & 31], sb, bar);
}

// Phase 0 of a staged item (threads 128..255, row i = tid - 128): per-row
// factors from the slot into rf.  Runs while the previous item's state is live
// in registers, hence the call-free quotient.
template <bool KDA>
__device__ __forceinline__ void phase0(RowFactors &rf, const StepArgs &a, const uint8_t *sb, int item)
{
    const int t = threadIdx.x - kDK, i = KDA ? frow(t) : t;  // storage row
    const HeadRec *rec = reinterpret_cast<const HeadRec *>(sb + a.off_rec);
    const float beta = *reinterpret_cast<const float *>(sb + a.off_ab + 4);
    const int b = rec->bits[i], key = rec->key_row[i];
    const float al = KDA ? reinterpret_cast<const float *>(sb + a.off_alpha)[key]
                         : *reinterpret_cast<const float *>(sb + a.off_ab);
    const float k = reinterpret_cast<const float *>(sb + a.off_k)[key];
    const float q = reinterpret_cast<const float *>(sb + a.off_q)[key];
    const float r = reinterpret_cast<const float *>(sb)[i];
    float A, g;
    if (b == kPivotBits) {
        A = al;
        g = beta * k;
    } else {
        A = al * r;
        g = div_approx(beta * k, A);
    }
    put_pair(rf.k2, i, A * k);
    put_pair(rf.l2, i, A * q);
    put_pair(rf.g2, i, g);
    if (KDA) {
        put_pair(rf.a2, i, al);
        put_pair(rf.q2, i, rec->rq[i]);
    }
    rf.ra[t] = A;  // by thread: read back by row-factor thread t, which handles the same row
    if (KDA) {
        rf.rb[sslot(i)] = b;
        const int Q = (b == kPivotBits) ? 0 : qmax_of(b);
        rf.qf[sslot(i)] = (float)Q;
        const int zb = (int)kMagicBits + (1 << (rec->pos_bits[i & 15] - 1));
        rf.qlh[sslot(i)] = make_int2(zb - Q, zb + Q);
        if (i < kRowsPerGroup) make_pos(rf, rec, i);
    }
    if (i == 0) {
        rf.beta = beta;
        rf.item = item;
        rf.head_b = rec->head_b;
        if (KDA) rf.n16 = rec->n16;

    }
}

// Work between the fit's two barriers of staged item n for the CTA's next
// staged item, written to the other factor buffer: phase 0 on threads
// 128..255 (operator()), its k.q on threads 0..127 after their row factors
// (rowside).  Both return false if that item's copy never landed.
template <bool KDA>
struct StageNext {
    ItemSmem &sm;
    const StepArgs &a;
    uint8_t *ring;
    int next_pos;      // position of the next staged item (>= n_items: none)
    int next_slot;     // its slot and the barrier phase parity it completes
    uint32_t next_parity;
    RowFactors &rf_next;
    __device__ __forceinline__ bool operator()() const
    {
        if (next_pos >= a.n_items) return true;
        if (!mbar_wait_bounded(&sm.bar[next_slot], next_parity, kWaitLimit)) return false;
        phase0<KDA>(rf_next, a, ring + next_slot * a.slot_bytes, a.t.order[next_pos]);
        return true;
    }
    // on threads 0..127, after their row factors: row i's k.q of the next
    // item, summed per 32 rows (the readout's scalar)
    __device__ __forceinline__ bool rowside(int i) const
    {
        if (next_pos >= a.n_items) return true;
        if (!mbar_wait_bounded(&sm.bar[next_slot], next_parity, kWaitLimit)) return false;
        const uint8_t *sb = ring + next_slot * a.slot_bytes;
        float kq = reinterpret_cast<const float *>(sb + a.off_k)[i] * reinterpret_cast<const float *>(sb + a.off_q)[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(kFull, kq, o);
        if ((threadIdx.x & 31) == 0) rf_next.kqp[threadIdx.x >> 5] = kq;  // any split of the rows
        return true;
    }
};

// A staged item: reconstruct + project (phase A), read out, Delta update
// (phase B), then the fit, during which the next item is prepared.  The slot
// sb stays untouched until the fit's second barrier.
template <int B, bool KDA, bool MULTI, int NP, int MODE>
__device__ __forceinline__ FitResult run_item(ItemSmem &sm, const StepArgs &a, RowFactors &rf, const uint8_t *sb,
                                              bool ok_slot, const StageNext<KDA> &next)
{
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    constexpr bool ROWWISE = (B == 0);
    const int item = rf.item;
    const HeadRec *rec = reinterpret_cast<const HeadRec *>(sb + a.off_rec);
    const int W = (B > 0) ? 2 * B : rec->slab_words;
    X2 X;
    // ---- phase A: codes -> floats, key and query projections, readout -------
    {
        const uint32_t *words = reinterpret_cast<const uint32_t *>(sb + kHeaderBytes) + (kStreams * W) * w + l;
        if constexpr (B > 0)
            decode_stream<B>(words, X);
        else
            decode_rowwise<NP>(rf, rg, words, X);
    }
    const float *s_c = reinterpret_cast<const float *>(sb) + kDK;
    const float4 c4 = ld4(s_c + col0);
    {
        float2 V0 = f2(0.f, 0.f), V1 = V0, U0 = V0, U1 = V0;
        float2 ic0 = V0, ic1 = V0;
        if (ROWWISE) {
            ic0 = f2(rcp_approx(c4.x), rcp_approx(c4.y));
            ic1 = f2(rcp_approx(c4.z), rcp_approx(c4.w));
        }
#pragma unroll
        for (int p = 0; p < kRowsPerGroup / 2; p++) {
            float2 kp[2], lp[2];
            ld_pairs(rf.k2, p, rg, kp);
            ld_pairs(rf.l2, p, rg, lp);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int rr = 2 * p + u;
                if (ROWWISE && rr < NP && rr < rf.n16 && rf.rb[8 * rr + rg] == kPivotBits) {
                    // a pivot value enters the projections in units of c_j; S' = alpha h
                    const float2 hs0 = __fmul2_rn(X[rr][0], ic0), hs1 = __fmul2_rn(X[rr][1], ic1);
                    V0 = __ffma2_rn(kp[u], hs0, V0);
                    V1 = __ffma2_rn(kp[u], hs1, V1);
                    U0 = __ffma2_rn(lp[u], hs0, U0);
                    U1 = __ffma2_rn(lp[u], hs1, U1);
                    float2 aa[2];
                    ld_pairs(rf.a2, p, rg, aa);
                    X[rr][0] = __fmul2_rn(aa[u], X[rr][0]);
                    X[rr][1] = __fmul2_rn(aa[u], X[rr][1]);
                } else {
                    V0 = __ffma2_rn(kp[u], X[rr][0], V0);
                    V1 = __ffma2_rn(kp[u], X[rr][1], V1);
                    U0 = __ffma2_rn(lp[u], X[rr][0], U0);
                    U1 = __ffma2_rn(lp[u], X[rr][1], U1);
                }
            }
        }
        // lane rg: the key projection (rg < 4) or the query projection (rg >= 4)
        // of column j, in units of c_j
        const float part = reduce_scatter_2x4(V0, V1, U0, U1, rg);
        const int j = col0 + (rg & 3);
        const float c = s_c[j];
        const float d = reinterpret_cast<const float *>(sb + a.off_v)[j] - c * part;
        if (rg < 4) {
            sm.cdt[j] = div_approx(d, c);
            if (ROWWISE) sm.cd[j] = d;
        }
        const float d_col = __shfl_xor_sync(kFull, d, 4);
        if (rg >= 4) {
            const float kq = (rf.kqp[0] + rf.kqp[1]) + (rf.kqp[2] + rf.kqp[3]);
            a.out[(long long)item * kDV + j] = fmaf(rf.beta * kq, d_col, c * part);
        }
        __syncwarp();
    }
    // ---- phase B: Delta update in old-scale units; P = S / a ----------------
    {
        const float2 c0 = f2(c4.x, c4.y), c1 = f2(c4.z, c4.w);
        const float4 t4 = ld4(&sm.cdt[col0]);
        const float2 dt0 = f2(t4.x, t4.y), dt1 = f2(t4.z, t4.w);
        float2 dd0 = dt0, dd1 = dt1;
        if (ROWWISE) {
            const float4 d4 = ld4(&sm.cd[col0]);
            dd0 = f2(d4.x, d4.y);
            dd1 = f2(d4.z, d4.w);
        }
#pragma unroll
        for (int p = 0; p < kRowsPerGroup / 2; p++) {
            float2 gp[2];
            ld_pairs(rf.g2, p, rg, gp);
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int rr = 2 * p + u;
                if (ROWWISE && rr < NP && rr < rf.n16 && rf.rb[8 * rr + rg] == kPivotBits) {
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
    uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + rec->head_off;
    return fit_and_store<B, ROWWISE, MULTI, NP, StageNext<KDA>, false, MODE>(sm, rf, rec, X, item_g, W, a.ls_iters,
                                                                           true, ok_slot, next);
}

// After a failed wait: record it, let every copy that may still be in flight
// (stagings first_pending .. issued - 1) land, then the CTA returns.
__device__ __forceinline__ void abort_drain(ItemSmem &sm, const StepArgs &a, uint32_t first_pending, uint32_t issued,
                                            int code)
{
    if ((threadIdx.x >> 5) == kProducerWarp) {
        asm volatile("cp.async.wait_all;" ::: "memory");
        if ((threadIdx.x & 31) == 0) {
            atomicExch(a.t.status, code);
            for (uint32_t m = first_pending; m < issued; m++)
                mbar_wait_bounded(&sm.bar[m % (uint32_t)a.nslots], (m / (uint32_t)a.nslots) & 1u, kWaitLimit);
        }
    }
    __syncthreads();
}

// Self-test of the bounded wait (one CTA, thread 0): a barrier that needs one
// arrival, which thread 0 makes first when `arrive` is set; otherwise nothing
// arrives and the wait gives up after `limit` cycles, as a wait for a staged
// copy that never lands does in the decode kernel.  result[0]: 0 or
// kStatusWaitTimeout; result[1]: cycles spent in the wait (saturated).
__global__ void k_wait_selftest(int *result, long long limit, int arrive)
{
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    if (arrive) mbar_arrive(&bar);
    const long long t0 = clock64();
    const bool ok = mbar_wait_bounded(&bar, 0u, limit);
    const long long dt = clock64() - t0;
    result[0] = ok ? 0 : kStatusWaitTimeout;
    result[1] = (int)min(dt, 2147483647LL);
}

// NP (row-wise widths): the leading positions checked for 16-bit fields; 1
// when no head of the pool has more than one, else all 16.
template <bool KDA, bool MULTI, int NP, int MODE>
__global__ void __launch_bounds__(kThreads, 2) k_decode(StepArgs a)
{
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ ItemSmem sm;
    STEPQ_RETURN_IF_REJECTED(a);
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    if (tid == 0) {
        for (int s = 0; s < a.nslots; s++) mbar_init(&sm.bar[s], kStageArrivals);
        fence_barrier_init();
    }
    __syncthreads();

    const int npiv = a.n_pivot_items;
    // first staged position of this CTA: the smallest n >= npiv with n = blockIdx.x (mod G)
    int n_first = blockIdx.x;
    if (n_first < npiv) n_first += ((npiv - n_first + G - 1) / G) * G;
    // stagings of this CTA: positions n_first, n_first + G, ...
    const uint32_t n_stage = (n_first < a.n_items) ? (uint32_t)((a.n_items - n_first + G - 1) / G) : 0u;
    const uint32_t in_flight0 = (n_stage < (uint32_t)a.nslots) ? n_stage : (uint32_t)a.nslots;
    if ((tid >> 5) == kProducerWarp) {
        fetch_rec_chunk(sm, a, n_first, 0);
        for (uint32_t k = 0; k < in_flight0; k++) produce<KDA>(sm, a, n_first, k, ring + k * a.slot_bytes, &sm.bar[k]);
    }
    for (int n = blockIdx.x; n < npiv && n < a.n_items; n += G) pivot_item(a, n);
    if (n_stage == 0) {  // nothing was staged
        if ((tid >> 5) == kProducerWarp) asm volatile("cp.async.wait_all;" ::: "memory");
        return;
    }

    // phase 0 of the first staged item
    {
        const StageNext<KDA> first{sm, a, ring, n_first, 0, 0u, sm.u.rf[0]};
        const bool ok = (tid >= kDK) ? first() : first.rowside(tid);
        if (!__syncthreads_and(ok)) {
            abort_drain(sm, a, 0u, in_flight0, kStatusWaitTimeout);
            return;
        }
    }
    uint32_t n_cons = 0;  // consumption count of the item; its slot and barrier parity below
    int par = 0, slot = 0;
    const uint32_t nsl = (uint32_t)a.nslots;
    uint32_t parity = 0;
    for (int n = n_first; n < a.n_items; n += G, par ^= 1) {
        RowFactors &rf = sm.u.rf[par];
        const uint8_t *sb = ring + slot * a.slot_bytes;
        const bool ok = mbar_wait_bounded(&sm.bar[slot], parity, kWaitLimit);
        const int slot_next = (slot + 1 == a.nslots) ? 0 : slot + 1;
        const uint32_t parity_next = (slot_next == 0) ? (parity ^ 1u) : parity;
        const StageNext<KDA> next{sm, a, ring, n + G, slot_next, parity_next, sm.u.rf[par ^ 1]};
        FitResult res = kFitDone;
        if (KDA) {
            res = run_item<0, KDA, MULTI, NP, MODE>(sm, a, rf, sb, ok, next);
        } else {
            switch (rf.head_b) {
                case 2: res = run_item<2, KDA, MULTI, 0, MODE>(sm, a, rf, sb, ok, next); break;
                case 3: res = run_item<3, KDA, MULTI, 0, MODE>(sm, a, rf, sb, ok, next); break;
                case 4: res = run_item<4, KDA, MULTI, 0, MODE>(sm, a, rf, sb, ok, next); break;
                case 5: res = run_item<5, KDA, MULTI, 0, MODE>(sm, a, rf, sb, ok, next); break;
                case 6: res = run_item<6, KDA, MULTI, 0, MODE>(sm, a, rf, sb, ok, next); break;
                case 7: res = run_item<7, KDA, MULTI, 0, MODE>(sm, a, rf, sb, ok, next); break;
                case 8: res = run_item<8, KDA, MULTI, 0, MODE>(sm, a, rf, sb, ok, next); break;
                default:  // unreachable: Gated-DeltaNet heads have one width, validated on the host
                    abort_drain(sm, a, n_cons, min(n_cons + nsl, n_stage), kStatusBadHead);
                    return;
            }
        }
        if (res == kFitAbortNow) {
            abort_drain(sm, a, n_cons, min(n_cons + nsl, n_stage), kStatusWaitTimeout);
            return;
        }
        if (res == kFitAbortAfter) {
            abort_drain(sm, a, n_cons + 1, min(n_cons + nsl, n_stage), kStatusWaitTimeout);
            return;
        }
        // every warp is past the item's second barrier, so the slot is free:
        // stage the position n_cons + nslots stagings on into it
        if ((tid >> 5) == kProducerWarp && n_cons + nsl < n_stage)
            produce<KDA>(sm, a, n_first, n_cons + nsl, ring + slot * a.slot_bytes, &sm.bar[slot]);
        n_cons++;
        slot = slot_next;
        parity = parity_next;
    }
    if ((tid >> 5) == kProducerWarp) asm volatile("cp.async.wait_all;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Pack (fit + quantise full-precision states) and unpack (dequantise): one CTA
// per item, the same thread mapping and the same fit as the decode step.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_head(RowFactors &rf, const HeadRec *rec)
{
    const int tid = threadIdx.x;
    if (tid < kDK) {
        const int i = tid;
        rf.ra[i] = 1.f;
        rf.rb[sslot(i)] = rec->bits[i];
        const int Q = (rec->bits[i] == kPivotBits) ? 0 : qmax_of(rec->bits[i]);
        rf.qf[sslot(i)] = (float)Q;
        const int zb = (int)kMagicBits + (1 << (rec->pos_bits[i & 15] - 1));
        rf.qlh[sslot(i)] = make_int2(zb - Q, zb + Q);
        put_pair(rf.q2, i, rec->rq[i]);
        if (i == 0) rf.n16 = rec->n16;
        if (i < kRowsPerGroup) make_pos(rf, rec, i);
    }
}

template <int B, bool ROWWISE, int MODE>
__device__ __forceinline__ void pack_body(ItemSmem &sm, RowFactors &rf, const HeadRec *rec, const StepArgs &a,
                                          int item, uint8_t *item_g)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    X2 X;
    const float *src = a.S_in + (long long)item * kDK * kDV;
#pragma unroll
    for (int rr = 0; rr < kRowsPerGroup; rr++) {
        const float4 x = ld4(src + rec->key_row[kRowsPerGroup * rg + rr] * kDV + col0);
        X[rr][0] = f2(x.x, x.y);
        X[rr][1] = f2(x.z, x.w);
    }
    fit_and_store<B, ROWWISE, true, kRowsPerGroup, NoMid, false, MODE>(sm, rf, rec, X, item_g,
                                                                       (B > 0) ? 2 * B : rec->slab_words, a.ls_iters,
                                                                       rec->head_kind != kHeadAllPivot, true, NoMid{});
}

template <int MODE>
__global__ void __launch_bounds__(kThreads) k_pack(StepArgs a)
{
    __shared__ ItemSmem sm;
    STEPQ_RETURN_IF_REJECTED(a);
    RowFactors &rf = sm.u.rf[0];
    const int item = blockIdx.x;
    const int rq = item / a.heads, h = item - rq * a.heads;
    const HeadRec *rec = a.t.rowrec + h;
    load_head(rf, rec);
    __syncthreads();
    uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + rec->head_off;
    switch (rec->head_kind == kHeadQuant ? rec->head_b : 0) {
        case 2: pack_body<2, false, MODE>(sm, rf, rec, a, item, item_g); break;
        case 3: pack_body<3, false, MODE>(sm, rf, rec, a, item, item_g); break;
        case 4: pack_body<4, false, MODE>(sm, rf, rec, a, item, item_g); break;
        case 5: pack_body<5, false, MODE>(sm, rf, rec, a, item, item_g); break;
        case 6: pack_body<6, false, MODE>(sm, rf, rec, a, item, item_g); break;
        case 7: pack_body<7, false, MODE>(sm, rf, rec, a, item, item_g); break;
        case 8: pack_body<8, false, MODE>(sm, rf, rec, a, item, item_g); break;
        default: pack_body<0, true, MODE>(sm, rf, rec, a, item, item_g); break;
    }
}

template <int B>
__device__ __forceinline__ void unpack_body(const RowFactors &rf, const HeadRec *rec, const StepArgs &a, int item,
                                            const uint8_t *item_g)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    X2 X;
    const int W = (B > 0) ? 2 * B : rec->slab_words;
    {
        const uint32_t *words = reinterpret_cast<const uint32_t *>(item_g + kHeaderBytes) + (kStreams * W) * w + l;
        if constexpr (B > 0)
            decode_stream<B>(words, X);
        else
            decode_rowwise<kRowsPerGroup>(rf, rg, words, X);
    }
    const float *r = reinterpret_cast<const float *>(item_g);
    const float4 c4 = ld4(r + kDK + col0);
    float *dst = a.S_out + (long long)item * kDK * kDV;
#pragma unroll
    for (int rr = 0; rr < kRowsPerGroup; rr++) {
        const int i = kRowsPerGroup * rg + rr;
        float4 y;
        if (B == 0 && rf.rb[8 * rr + rg] == kPivotBits) {
            y = make_float4(X[rr][0].x, X[rr][0].y, X[rr][1].x, X[rr][1].y);
        } else {
            const float ri = r[i];
            y = make_float4(__fmul_rn(__fmul_rn(ri, c4.x), X[rr][0].x), __fmul_rn(__fmul_rn(ri, c4.y), X[rr][0].y),
                            __fmul_rn(__fmul_rn(ri, c4.z), X[rr][1].x), __fmul_rn(__fmul_rn(ri, c4.w), X[rr][1].y));
        }
        *reinterpret_cast<float4 *>(dst + rec->key_row[i] * kDV + col0) = y;
    }
}

__global__ void __launch_bounds__(kThreads) k_unpack(StepArgs a)
{
    __shared__ RowFactors rf;
    STEPQ_RETURN_IF_REJECTED(a);
    const int item = blockIdx.x;
    const int rq = item / a.heads, h = item - rq * a.heads;
    const HeadRec *rec = a.t.rowrec + h;
    load_head(rf, rec);
    __syncthreads();
    const uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + rec->head_off;
    switch (rec->head_kind == kHeadQuant ? rec->head_b : 0) {
        case 2: unpack_body<2>(rf, rec, a, item, item_g); break;
        case 3: unpack_body<3>(rf, rec, a, item, item_g); break;
        case 4: unpack_body<4>(rf, rec, a, item, item_g); break;
        case 5: unpack_body<5>(rf, rec, a, item, item_g); break;
        case 6: unpack_body<6>(rf, rec, a, item, item_g); break;
        case 7: unpack_body<7>(rf, rec, a, item, item_g); break;
        case 8: unpack_body<8>(rf, rec, a, item, item_g); break;
        default: unpack_body<0>(rf, rec, a, item, item_g); break;
    }
}

// ---------------------------------------------------------------------------
// The pages' own pipeline, kept for comparison with the fused step: a kernel
// that reconstructs the state, applies the gated Delta update and reads out
// (writing the updated unquantised state to a work buffer), followed by the
// fit and packed writeback (k_pack on that buffer) on a second stream.  One
// CTA per item, the decode mapping; the state is formed in absolute units in
// the order of the recurrence: S' = alpha S, v_old = S'^T k,
// S = S' + beta k (v - v_old)^T, o = S^T q.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void split_update_body(const RowFactors &rf, const HeadRec *rec, const StepArgs &a,
                                                  int item, const uint8_t *item_g, float *S_work)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, rg = l & 7, cg = l >> 3;
    const int col0 = 16 * w + 4 * cg;
    const int W = (B > 0) ? 2 * B : rec->slab_words;
    X2 X;
    {
        const uint32_t *words = reinterpret_cast<const uint32_t *>(item_g + kHeaderBytes) + (kStreams * W) * w + l;
        if constexpr (B > 0)
            decode_stream<B>(words, X);
        else
            decode_rowwise<kRowsPerGroup>(rf, rg, words, X);
    }
    const float *r = reinterpret_cast<const float *>(item_g);
    const float4 c4 = ld4(r + kDK + col0);
    const long long vec = (long long)item * kDK;
    float2 V0 = f2(0.f, 0.f), V1 = V0;
    float kk[kRowsPerGroup], qq[kRowsPerGroup];
#pragma unroll
    for (int q4 = 0; q4 < kRowsPerGroup / 4; q4++) {
        float ka[4], qa[4], aa[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {  // the inputs of the key rows this thread's storage rows hold
            const int key = rec->key_row[kRowsPerGroup * rg + 4 * q4 + e];
            ka[e] = a.k[vec + key];
            qa[e] = a.q[vec + key];
            aa[e] = a.kda ? a.alpha[vec + key] : a.alpha[item];
        }
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int rr = 4 * q4 + e, i = kRowsPerGroup * rg + rr;
            kk[rr] = ka[e];
            qq[rr] = qa[e];
            float2 s0, s1;
            if (B == 0 && rf.rb[8 * rr + rg] == kPivotBits) {
                s0 = X[rr][0];
                s1 = X[rr][1];
            } else {
                const float ri = r[i];
                s0 = f2(__fmul_rn(__fmul_rn(ri, c4.x), X[rr][0].x), __fmul_rn(__fmul_rn(ri, c4.y), X[rr][0].y));
                s1 = f2(__fmul_rn(__fmul_rn(ri, c4.z), X[rr][1].x), __fmul_rn(__fmul_rn(ri, c4.w), X[rr][1].y));
            }
            const float2 a2 = f2(aa[e], aa[e]);
            X[rr][0] = __fmul2_rn(a2, s0);
            X[rr][1] = __fmul2_rn(a2, s1);
            const float2 k2 = f2(ka[e], ka[e]);
            V0 = __ffma2_rn(k2, X[rr][0], V0);
            V1 = __ffma2_rn(k2, X[rr][1], V1);
        }
    }
    // v_old over the 8 row groups (butterfly), then d for the thread's columns
    V0 = __fadd2_rn(V0, shfl2(V0, 1)); V1 = __fadd2_rn(V1, shfl2(V1, 1));
    V0 = __fadd2_rn(V0, shfl2(V0, 2)); V1 = __fadd2_rn(V1, shfl2(V1, 2));
    V0 = __fadd2_rn(V0, shfl2(V0, 4)); V1 = __fadd2_rn(V1, shfl2(V1, 4));
    const float4 v4 = ld4(a.v + (long long)item * kDV + col0);
    const float2 d0 = f2(v4.x - V0.x, v4.y - V0.y), d1 = f2(v4.z - V1.x, v4.w - V1.y);
    const float beta = a.beta[item];
    float2 U0 = f2(0.f, 0.f), U1 = U0;
    float *dst = S_work + (long long)item * kDK * kDV;
#pragma unroll
    for (int rr = 0; rr < kRowsPerGroup; rr++) {
        const float g = beta * kk[rr];
        const float2 g2 = f2(g, g), q2 = f2(qq[rr], qq[rr]);
        X[rr][0] = __ffma2_rn(g2, d0, X[rr][0]);
        X[rr][1] = __ffma2_rn(g2, d1, X[rr][1]);
        U0 = __ffma2_rn(q2, X[rr][0], U0);
        U1 = __ffma2_rn(q2, X[rr][1], U1);
        *reinterpret_cast<float4 *>(dst + rec->key_row[kRowsPerGroup * rg + rr] * kDV + col0) =
            make_float4(X[rr][0].x, X[rr][0].y, X[rr][1].x, X[rr][1].y);
    }
    U0 = __fadd2_rn(U0, shfl2(U0, 1)); U1 = __fadd2_rn(U1, shfl2(U1, 1));
    U0 = __fadd2_rn(U0, shfl2(U0, 2)); U1 = __fadd2_rn(U1, shfl2(U1, 2));
    U0 = __fadd2_rn(U0, shfl2(U0, 4)); U1 = __fadd2_rn(U1, shfl2(U1, 4));
    if (rg == 0)
        *reinterpret_cast<float4 *>(a.out + (long long)item * kDV + col0) = make_float4(U0.x, U0.y, U1.x, U1.y);
}

__global__ void __launch_bounds__(kThreads) k_split_update(StepArgs a)
{
    __shared__ RowFactors rf;
    STEPQ_RETURN_IF_REJECTED(a);
    const int item = blockIdx.x;
    const int rq = item / a.heads, h = item - rq * a.heads;
    const HeadRec *rec = a.t.rowrec + h;
    load_head(rf, rec);
    __syncthreads();
    const uint8_t *item_g = a.pool + (long long)rq * a.req_bytes + rec->head_off;
    float *S_work = const_cast<float *>(a.S_in);
    switch (rec->head_kind == kHeadQuant ? rec->head_b : 0) {
        case 2: split_update_body<2>(rf, rec, a, item, item_g, S_work); break;
        case 3: split_update_body<3>(rf, rec, a, item, item_g, S_work); break;
        case 4: split_update_body<4>(rf, rec, a, item, item_g, S_work); break;
        case 5: split_update_body<5>(rf, rec, a, item, item_g, S_work); break;
        case 6: split_update_body<6>(rf, rec, a, item, item_g, S_work); break;
        case 7: split_update_body<7>(rf, rec, a, item, item_g, S_work); break;
        case 8: split_update_body<8>(rf, rec, a, item, item_g, S_work); break;
        default: split_update_body<0>(rf, rec, a, item, item_g, S_work); break;
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
    float S[kRowsPerGroup][4];
    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ii = 0; ii < kRowsPerGroup; ii++) {
        const int i = kRowsPerGroup * w + ii;
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
    for (int ii = 0; ii < kRowsPerGroup; ii++) {
        const int i = kRowsPerGroup * w + ii;
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

template <bool KDA, bool MULTI, int NP, int MODE>
cudaError_t launch_decode_t(const StepArgs &a, cudaStream_t s)
{
    const int dyn = a.nslots * a.slot_bytes;
    cudaError_t e =
        cudaFuncSetAttribute(k_decode<KDA, MULTI, NP, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<KDA, MULTI, NP, MODE>, kThreads, dyn);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const long long want = (long long)per_sm * sm_count();
    const int grid = (int)(a.n_items < want ? a.n_items : want);
    k_decode<KDA, MULTI, NP, MODE><<<grid, kThreads, dyn, s>>>(a);
    return cudaGetLastError();
}

template <bool MULTI, int MODE>
cudaError_t launch_decode_m(const StepArgs &a, cudaStream_t s)
{
    if (!a.kda) return launch_decode_t<false, MULTI, 0, MODE>(a, s);
    return (a.max_n16 <= 1) ? launch_decode_t<true, MULTI, 1, MODE>(a, s)
                            : launch_decode_t<true, MULTI, kRowsPerGroup, MODE>(a, s);
}

// ---------------------------------------------------------------------------
// Calibration.  k_calib_accumulate: one step's sums of q^2 per (head, key row)
// and of log alpha per unit, over the batch in request order (fp64; one CTA
// per head, thread i = key row).  k_calib_error: one CTA per (request, head)
// state; for every candidate width the state is fitted and quantised with all
// rows at that width, as the pack kernel would, and each row's squared
// reconstruction error is written.  k_calib_reduce: the errors of a sampled
// state added into the running fp64 sums, request by request.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kDK) k_calib_accumulate(CalibArgs c)
{
    const int h = blockIdx.x, i = threadIdx.x, H = c.heads;
    double s = 0.0;
    for (int b = 0; b < c.batch; b++) {
        const double x = (double)c.q[((long long)b * H + h) * kDK + i];
        s += x * x;
    }
    c.acc_q2[h * kDK + i] += s;
    if (c.kda) {
        double t = 0.0;
        for (int b = 0; b < c.batch; b++) t += log((double)c.alpha[((long long)b * H + h) * kDK + i]);
        c.acc_loga[h * kDK + i] += t;
    } else if (i == 0) {
        double t = 0.0;
        for (int b = 0; b < c.batch; b++) t += log((double)c.alpha[(long long)b * H + h]);
        c.acc_loga[h] += t;
    }
}

// One candidate width of the calibration's per-row errors; the thread's 64
// state values come from its own block of the shared-memory copy (`own`,
// value rr at own[rr * kThreads]: a warp's lanes read consecutive 16-byte
// chunks).
template <int B, bool MULTI>
__device__ __forceinline__ void calib_width(ItemSmem &sm, RowFactors &rf, const HeadRec *rec, const CalibArgs &c,
                                            int item, int x, const float4 *own)
{
    X2 X;
#pragma unroll
    for (int rr = 0; rr < kRowsPerGroup; rr++) {
        const float4 v = own[rr * kThreads];
        X[rr][0] = f2(v.x, v.y);
        X[rr][1] = f2(v.z, v.w);
    }
    const long long o = (long long)item * c.n_widths + x;
    fit_and_store<B, false, MULTI, 0, NoMid, true>(sm, rf, rec, X,
                                                  reinterpret_cast<uint8_t *>(c.rc + o * (kDK + kDV)), 2 * B,
                                                  c.ls_iters, true, true, NoMid{}, c.err + o * kDK);
}

// The state is copied once per CTA into shared memory (each thread its own 16
// rows x 4 columns, 256 bytes, by asynchronous copies; 64 KiB of dynamic
// shared memory per CTA), so that the candidate widths after the first reload
// it from there instead of from L2.
template <bool MULTI>
__global__ void __launch_bounds__(kThreads) k_calib_error(CalibArgs c)
{
    extern __shared__ __align__(16) float4 state_copy[];
    __shared__ ItemSmem sm;
    __shared__ HeadRec rec;
    RowFactors &rf = sm.u.rf[0];
    const int item = blockIdx.x, h = item % c.heads, tid = threadIdx.x;
    float4 *own = state_copy + tid;
    {
        const int w = tid >> 5, l = tid & 31, rg = l & 7, cg = l >> 3;
        const float *src = c.S + (long long)item * kDK * kDV + (kRowsPerGroup * rg) * kDV + 16 * w + 4 * cg;
#pragma unroll
        for (int rr = 0; rr < kRowsPerGroup; rr++)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(own + rr * kThreads)),
                         "l"(src + rr * kDV)
                         : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    float s_i = 0.f, rho_i = 0.f;
    __shared__ float rho_wmax[kThreads / 32];
    if (tid < kDK) rho_i = c.rho[h * kDK + tid];
    {  // the head's largest impact weight (every row is quantised here); weights are positive floats
        const unsigned m = __reduce_max_sync(kFull, __float_as_uint(rho_i));
        if ((tid & 31) == 0) rho_wmax[tid >> 5] = __uint_as_float(m);
        __syncthreads();
    }
    if (tid < kDK) {
        float rmax = rho_wmax[0];
#pragma unroll
        for (int x = 1; x < kDK / 32; x++) rmax = fmaxf(rmax, rho_wmax[x]);
        // fp32(max(rho, rho_max / 4)^-1/2) from fp64, as the host tables
        s_i = (float)(1.0 / sqrt(fmax((double)rho_i, (double)rmax / 4.0)));
    }
    for (int x = 0; x < c.n_widths; x++) {
        const int b = c.widths[x];
        __syncthreads();  // the previous width's readers of rec, rf and the row partials are done
        if (tid < kDK) {
            const int i = tid;
            rec.s[i] = s_i;
            rec.rho[i] = rho_i;
            rec.rq[i] = (float)(1.0 / (double)qmax_of(b));
            rec.bits[i] = (uint8_t)b;
            rec.key_row[i] = (uint8_t)i;
            rf.ra[i] = 1.f;
        }
        if (tid == 0) {
            rec.head_b = b;
            rec.head_kind = kHeadQuant;
            rec.n16 = 0;
        }
        __syncthreads();
        if (x == 0) asm volatile("cp.async.wait_all;" ::: "memory");  // the thread's own copy has landed
        switch (b) {
            case 2: calib_width<2, MULTI>(sm, rf, &rec, c, item, x, own); break;
            case 3: calib_width<3, MULTI>(sm, rf, &rec, c, item, x, own); break;
            case 4: calib_width<4, MULTI>(sm, rf, &rec, c, item, x, own); break;
            case 5: calib_width<5, MULTI>(sm, rf, &rec, c, item, x, own); break;
            case 6: calib_width<6, MULTI>(sm, rf, &rec, c, item, x, own); break;
            case 7: calib_width<7, MULTI>(sm, rf, &rec, c, item, x, own); break;
            default: calib_width<8, MULTI>(sm, rf, &rec, c, item, x, own); break;  // widths are validated on the host
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // (no width: the copy lands before the CTA ends)
}

__global__ void __launch_bounds__(kDK) k_calib_reduce(CalibArgs c)
{
    const int h = blockIdx.x / c.n_widths, x = blockIdx.x % c.n_widths, i = threadIdx.x;
    double acc = c.err_sum[((long long)h * c.n_widths + x) * kDK + i];
    for (int b = 0; b < c.batch; b++)
        acc += (double)c.err[(((long long)b * c.heads + h) * c.n_widths + x) * kDK + i];
    c.err_sum[((long long)h * c.n_widths + x) * kDK + i] = acc;
}

}  // namespace

cudaError_t launch_calib_accumulate(const CalibArgs &c, cudaStream_t s)
{
    if (c.heads == 0 || c.batch == 0) return cudaSuccess;
    k_calib_accumulate<<<c.heads, kDK, 0, s>>>(c);
    return cudaGetLastError();
}

cudaError_t launch_calib_error(const CalibArgs &c, cudaStream_t s)
{
    const long long n = (long long)c.batch * c.heads;
    if (n == 0 || c.n_widths == 0) return cudaSuccess;
    constexpr int dyn = kThreads * kRowsPerGroup * (int)sizeof(float4);  // the state copy, 64 KiB
    cudaError_t e = cudaFuncSetAttribute(k_calib_error<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_calib_error<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return e;
    if (c.ls_iters <= 1)
        k_calib_error<false><<<(unsigned)n, kThreads, dyn, s>>>(c);
    else
        k_calib_error<true><<<(unsigned)n, kThreads, dyn, s>>>(c);
    return cudaGetLastError();
}

cudaError_t launch_calib_reduce(const CalibArgs &c, cudaStream_t s)
{
    if (c.heads == 0 || c.n_widths == 0) return cudaSuccess;
    k_calib_reduce<<<c.heads * c.n_widths, kDK, 0, s>>>(c);
    return cudaGetLastError();
}

// Checking build: validate the tables the next launch reads (n_pos staging
// records; the head records always).
static inline void check_tables(const StepArgs &a, int n_pos, cudaStream_t s)
{
#if STEPQ_CHECK
    const int n = n_pos > a.heads ? n_pos : a.heads;
    k_check_tables<<<(n + 255) / 256, 256, 0, s>>>(a, n_pos);
#else
    (void)a, (void)n_pos, (void)s;
#endif
}

cudaError_t launch_decode_step(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    check_tables(a, a.n_items, s);
    switch (a.scale_mode) {  // the variants fit without least squares: one instantiation each
        case kScaleRow: return launch_decode_m<false, kScaleRow>(a, s);
        case kScaleCol: return launch_decode_m<false, kScaleCol>(a, s);
        case kScaleHead: return launch_decode_m<false, kScaleHead>(a, s);
        default: break;
    }
    return (a.ls_iters <= 1) ? launch_decode_m<false, kScaleDual>(a, s) : launch_decode_m<true, kScaleDual>(a, s);
}

int decode_ctas_per_sm(int nslots, int slot_bytes)
{
    const int dyn = nslots * slot_bytes;
    int per_sm = 0;
    if (cudaFuncSetAttribute(k_decode<false, false, 0, kScaleDual>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<false, false, 0, kScaleDual>, kThreads, dyn) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return per_sm;
}

cudaError_t launch_pack(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    check_tables(a, 0, s);
    switch (a.scale_mode) {
        case kScaleRow: k_pack<kScaleRow><<<a.n_items, kThreads, 0, s>>>(a); break;
        case kScaleCol: k_pack<kScaleCol><<<a.n_items, kThreads, 0, s>>>(a); break;
        case kScaleHead: k_pack<kScaleHead><<<a.n_items, kThreads, 0, s>>>(a); break;
        default: k_pack<kScaleDual><<<a.n_items, kThreads, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_split_update(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    check_tables(a, 0, s);
    k_split_update<<<a.n_items, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const StepArgs &a, cudaStream_t s)
{
    if (a.n_items == 0) return cudaSuccess;
    check_tables(a, 0, s);
    k_unpack<<<a.n_items, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int *result, long long limit, int arrive, cudaStream_t s)
{
    k_wait_selftest<<<1, 32, 0, s>>>(result, limit, arrive);
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
