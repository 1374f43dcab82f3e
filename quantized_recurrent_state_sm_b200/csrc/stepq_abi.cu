// Host side of the C ABI declared in include/stepq.h: argument validation, the
// per-head tables derived at pool creation (stored in the tail of the caller's
// pool buffer), and kernel launches.  No device allocation anywhere.
#include <algorithm>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <numeric>
#include <set>
#include <string>
#include <vector>

#include "stepq.h"
#include "stepq_internal.cuh"

using stepq::kDK;
using stepq::kDV;

struct stepq_pool {
    stepq_desc desc;  // table pointers cleared; the tables are copied below
    std::vector<uint8_t> bits;
    std::vector<float> rho;
    uint8_t *dev = nullptr;
    size_t bytes = 0, state_bytes = 0;
    long long req_bytes = 0;
    cudaStream_t stream = nullptr;
    stepq::Tables t{};
};

namespace {

thread_local std::string g_err;
std::mutex g_live_mu;
std::set<const stepq_pool *> g_live;

stepq_status fail(stepq_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
stepq_status fail(stepq_status s, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
    size_t state = 0;
    size_t off_row_off = 0, off_row_bits = 0, off_row_s = 0, off_row_rho = 0;
    size_t off_head_off = 0, off_head_nq = 0, off_order = 0, total = 0;
    long long req_bytes = 0;
    std::vector<long long> item_bytes;  // per head
};

// Checks a descriptor; fills the layout when valid.
stepq_status check_desc(const stepq_desc *d, bool need_tables, Layout *L)
{
    if (!d) return fail(STEPQ_ERR_INVALID_ARG, "descriptor is NULL");
    if (d->variant != STEPQ_GDN && d->variant != STEPQ_KDA)
        return fail(STEPQ_ERR_INVALID_ARG, "variant %d is neither STEPQ_GDN nor STEPQ_KDA", d->variant);
    if (d->batch < 0) return fail(STEPQ_ERR_INVALID_ARG, "batch %d < 0", d->batch);
    if (d->heads < 1) return fail(STEPQ_ERR_INVALID_ARG, "heads %d < 1", d->heads);
    if (d->dk < 1 || d->dv < 1) return fail(STEPQ_ERR_INVALID_ARG, "dk, dv must be positive");
    if (d->dk != kDK || d->dv != kDV)
        return fail(STEPQ_ERR_UNSUPPORTED, "only dk = dv = 128 is implemented (got %d x %d)", d->dk, d->dv);
    if ((long long)d->batch * d->heads > STEPQ_MAX_ITEMS)
        return fail(STEPQ_ERR_INVALID_ARG, "batch * heads exceeds %d", STEPQ_MAX_ITEMS);
    if (!need_tables) return STEPQ_OK;
    if (d->ls_iters < 0 || d->ls_iters > 8)
        return fail(STEPQ_ERR_INVALID_ARG, "ls_iters %d outside 0..8", d->ls_iters);
    if (!d->bits || !d->rho) return fail(STEPQ_ERR_INVALID_ARG, "bits and rho tables are required");
    const int H = d->heads;
    for (int h = 0; h < H; h++) {
        for (int i = 0; i < kDK; i++) {
            const int b = d->bits[h * kDK + i];
            if (!((b >= 2 && b <= 8) || b == STEPQ_PIVOT_BITS))
                return fail(STEPQ_ERR_INVALID_ARG, "bits[%d][%d] = %d is not in 2..8 or 16", h, i, b);
            if (d->variant == STEPQ_GDN && b != d->bits[h * kDK])
                return fail(STEPQ_ERR_INVALID_ARG, "Gated-DeltaNet needs one width per head (head %d)", h);
            const float r = d->rho[h * kDK + i];
            if (b != STEPQ_PIVOT_BITS && !(std::isfinite(r) && r > 0.f))
                return fail(STEPQ_ERR_INVALID_ARG, "rho[%d][%d] must be finite and > 0", h, i);
        }
    }
    if (L) {
        L->item_bytes.assign(H, 0);
        long long req = 0;
        for (int h = 0; h < H; h++) {
            long long n = stepq::kHeaderBytes;
            for (int i = 0; i < kDK; i++) n += (long long)kDV * d->bits[h * kDK + i] / 8;
            L->item_bytes[h] = n;
            req += n;
        }
        L->req_bytes = req;
        L->state = (size_t)req * (size_t)d->batch;
        size_t o = align_up(L->state, 256);
        const size_t HD = (size_t)H * kDK;
        L->off_row_off = o;  o = align_up(o + 4 * HD, 16);
        L->off_row_bits = o; o = align_up(o + HD, 16);
        L->off_row_s = o;    o = align_up(o + 4 * HD, 16);
        L->off_row_rho = o;  o = align_up(o + 4 * HD, 16);
        L->off_head_off = o; o = align_up(o + 8 * (size_t)H, 16);
        L->off_head_nq = o;  o = align_up(o + 4 * (size_t)H, 16);
        L->off_order = o;    o = align_up(o + 4 * (size_t)H * d->batch, 16);
        L->total = o;
    }
    return STEPQ_OK;
}

stepq_status check_pool(const stepq_pool *p)
{
    if (!p) return fail(STEPQ_ERR_INVALID_ARG, "pool is NULL");
    std::lock_guard<std::mutex> g(g_live_mu);
    if (!g_live.count(p)) return fail(STEPQ_ERR_STATE, "pool handle is not live (destroyed or never created)");
    return STEPQ_OK;
}

// A device tensor argument: non-null, aligned, and memory the GPU can address.
stepq_status check_dev(const void *ptr, const char *name, size_t align)
{
    if (!ptr) return fail(STEPQ_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned(ptr, align)) return fail(STEPQ_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
    cudaPointerAttributes at{};
    cudaError_t e = cudaPointerGetAttributes(&at, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(STEPQ_ERR_INVALID_ARG, "%s: cannot query pointer (%s)", name, cudaGetErrorString(e));
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return fail(STEPQ_ERR_INVALID_ARG, "%s is not device memory", name);
    return STEPQ_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

stepq_status cuda_fail(cudaError_t e, const char *what)
{
    cudaGetLastError();
    return fail(STEPQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

stepq::StepArgs base_args(const stepq_pool *p)
{
    stepq::StepArgs a{};
    a.pool = p->dev;
    a.t = p->t;
    a.req_bytes = p->req_bytes;
    a.heads = p->desc.heads;
    a.n_items = p->desc.batch * p->desc.heads;
    a.ls_iters = p->desc.ls_iters;
    a.kda = p->desc.variant == STEPQ_KDA;
    return a;
}

}  // namespace

extern "C" {

size_t stepq_pool_bytes(const stepq_desc *desc)
{
    Layout L;
    return check_desc(desc, true, &L) == STEPQ_OK ? L.total : 0;
}

size_t stepq_state_bytes(const stepq_desc *desc)
{
    Layout L;
    return check_desc(desc, true, &L) == STEPQ_OK ? L.state : 0;
}

stepq_status stepq_pool_create(const stepq_desc *desc, void *dev_buf, size_t bytes, void *cuda_stream,
                               stepq_pool **out)
{
    if (!out) return fail(STEPQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    Layout L;
    stepq_status st = check_desc(desc, true, &L);
    if (st != STEPQ_OK) return st;
    if (bytes < L.total) return fail(STEPQ_ERR_INVALID_ARG, "buffer of %zu bytes < %zu required", bytes, L.total);
    if ((st = check_dev(dev_buf, "dev_buf", 16)) != STEPQ_OK) return st;

    const int H = desc->heads, B = desc->batch;
    const size_t HD = (size_t)H * kDK;
    std::vector<uint8_t> host(L.total - L.off_row_off, 0);
    auto at = [&](size_t off) { return host.data() + (off - L.off_row_off); };
    uint32_t *row_off = reinterpret_cast<uint32_t *>(at(L.off_row_off));
    uint8_t *row_bits = at(L.off_row_bits);
    float *row_s = reinterpret_cast<float *>(at(L.off_row_s));
    float *row_rho = reinterpret_cast<float *>(at(L.off_row_rho));
    long long *head_off = reinterpret_cast<long long *>(at(L.off_head_off));
    int *head_nq = reinterpret_cast<int *>(at(L.off_head_nq));
    int *order = reinterpret_cast<int *>(at(L.off_order));
    long long pre = 0;
    for (int h = 0; h < H; h++) {
        head_off[h] = pre;
        pre += L.item_bytes[h];
        uint32_t o = stepq::kHeaderBytes;
        int nq = 0;
        for (int i = 0; i < kDK; i++) {
            const int b = desc->bits[h * kDK + i];
            row_off[h * kDK + i] = o;
            o += (uint32_t)(kDV * b / 8);
            row_bits[h * kDK + i] = (uint8_t)b;
            const float r = desc->rho[h * kDK + i];
            if (b != STEPQ_PIVOT_BITS) {
                nq++;
                row_s[h * kDK + i] = (float)(1.0 / std::sqrt((double)r));
                row_rho[h * kDK + i] = r;
            } else {
                row_s[h * kDK + i] = 0.f;
                row_rho[h * kDK + i] = 0.f;
            }
        }
        head_nq[h] = nq;
    }
    // heaviest items (most packed bytes) are scheduled first
    std::vector<int> idx((size_t)B * H);
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(), [&](int x, int y) {
        return L.item_bytes[x % H] > L.item_bytes[y % H];
    });
    std::memcpy(order, idx.data(), idx.size() * sizeof(int));

    cudaStream_t s = reinterpret_cast<cudaStream_t>(cuda_stream);
    uint8_t *dev = static_cast<uint8_t *>(dev_buf);
    cudaError_t e = cudaMemcpyAsync(dev + L.off_row_off, host.data(), host.size(), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "table upload");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "table upload sync");

    stepq_pool *p = new stepq_pool();
    p->desc = *desc;
    p->bits.assign(desc->bits, desc->bits + HD);
    p->rho.assign(desc->rho, desc->rho + HD);
    p->desc.bits = nullptr;
    p->desc.rho = nullptr;
    p->dev = dev;
    p->bytes = bytes;
    p->state_bytes = L.state;
    p->req_bytes = L.req_bytes;
    p->stream = s;
    p->t.row_off = reinterpret_cast<const uint32_t *>(dev + L.off_row_off);
    p->t.row_bits = dev + L.off_row_bits;
    p->t.row_s = reinterpret_cast<const float *>(dev + L.off_row_s);
    p->t.row_rho = reinterpret_cast<const float *>(dev + L.off_row_rho);
    p->t.head_off = reinterpret_cast<const long long *>(dev + L.off_head_off);
    p->t.head_nq = reinterpret_cast<const int *>(dev + L.off_head_nq);
    p->t.order = reinterpret_cast<const int *>(dev + L.off_order);
    {
        std::lock_guard<std::mutex> g(g_live_mu);
        g_live.insert(p);
    }
    *out = p;
    g_err.clear();
    return STEPQ_OK;
}

stepq_status stepq_pool_destroy(stepq_pool *pool)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    {
        std::lock_guard<std::mutex> g(g_live_mu);
        g_live.erase(pool);
    }
    delete pool;
    return STEPQ_OK;
}

stepq_status stepq_pool_set_stream(stepq_pool *pool, void *cuda_stream)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    pool->stream = reinterpret_cast<cudaStream_t>(cuda_stream);
    return STEPQ_OK;
}

stepq_status stepq_pack(stepq_pool *pool, const float *S)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    const size_t n = (size_t)pool->desc.batch * pool->desc.heads;
    if (n == 0) return STEPQ_OK;
    if ((st = check_dev(S, "S", 16)) != STEPQ_OK) return st;
    if (overlaps(S, n * kDK * kDV * 4, pool->dev, pool->bytes))
        return fail(STEPQ_ERR_INVALID_ARG, "S overlaps the pool buffer");
    stepq::StepArgs a = base_args(pool);
    a.S_in = S;
    cudaError_t e = stepq::launch_pack(a, pool->stream);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_pack launch");
}

stepq_status stepq_unpack(stepq_pool *pool, float *S_out)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    const size_t n = (size_t)pool->desc.batch * pool->desc.heads;
    if (n == 0) return STEPQ_OK;
    if ((st = check_dev(S_out, "S_out", 16)) != STEPQ_OK) return st;
    if (overlaps(S_out, n * kDK * kDV * 4, pool->dev, pool->bytes))
        return fail(STEPQ_ERR_INVALID_ARG, "S_out overlaps the pool buffer");
    stepq::StepArgs a = base_args(pool);
    a.S_out = S_out;
    cudaError_t e = stepq::launch_unpack(a, pool->stream);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_unpack launch");
}

static stepq_status check_step_tensors(int variant, size_t n, const float *q, const float *k,
                                       const float *v, const float *alpha, const float *beta,
                                       const float *out)
{
    stepq_status st;
    if ((st = check_dev(q, "q", 16)) != STEPQ_OK) return st;
    if ((st = check_dev(k, "k", 16)) != STEPQ_OK) return st;
    if ((st = check_dev(v, "v", 16)) != STEPQ_OK) return st;
    if ((st = check_dev(alpha, "alpha", variant == STEPQ_KDA ? 16 : 4)) != STEPQ_OK) return st;
    if ((st = check_dev(beta, "beta", 4)) != STEPQ_OK) return st;
    if ((st = check_dev(out, "out", 16)) != STEPQ_OK) return st;
    const size_t nout = n * kDV * 4;
    const size_t na = (variant == STEPQ_KDA ? n * kDK : n) * 4;
    if (overlaps(out, nout, q, n * kDK * 4) || overlaps(out, nout, k, n * kDK * 4) ||
        overlaps(out, nout, v, n * kDV * 4) || overlaps(out, nout, alpha, na) ||
        overlaps(out, nout, beta, n * 4))
        return fail(STEPQ_ERR_INVALID_ARG, "out aliases an input");
    return STEPQ_OK;
}

stepq_status stepq_decode_step(stepq_pool *pool, const float *q, const float *k, const float *v,
                               const float *alpha, const float *beta, float *out)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    const size_t n = (size_t)pool->desc.batch * pool->desc.heads;
    if (n == 0) return STEPQ_OK;
    if ((st = check_step_tensors(pool->desc.variant, n, q, k, v, alpha, beta, out)) != STEPQ_OK) return st;
    if (overlaps(out, n * kDV * 4, pool->dev, pool->bytes))
        return fail(STEPQ_ERR_INVALID_ARG, "out overlaps the pool buffer");
    stepq::StepArgs a = base_args(pool);
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.out = out;
    cudaError_t e = stepq::launch_decode_step(a, pool->stream);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_decode_step launch");
}

stepq_status stepq_fp32_step(const stepq_desc *desc, float *S, const float *q, const float *k,
                             const float *v, const float *alpha, const float *beta, float *out,
                             void *cuda_stream)
{
    stepq_status st = check_desc(desc, false, nullptr);
    if (st != STEPQ_OK) return st;
    const size_t n = (size_t)desc->batch * desc->heads;
    if (n == 0) return STEPQ_OK;
    if ((st = check_dev(S, "S", 16)) != STEPQ_OK) return st;
    if ((st = check_step_tensors(desc->variant, n, q, k, v, alpha, beta, out)) != STEPQ_OK) return st;
    if (overlaps(out, n * kDV * 4, S, n * kDK * kDV * 4))
        return fail(STEPQ_ERR_INVALID_ARG, "out overlaps S");
    cudaError_t e = stepq::launch_fp32_step(S, q, k, v, alpha, beta, out, (int)n,
                                            desc->variant == STEPQ_KDA,
                                            reinterpret_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_fp32_step launch");
}

const char *stepq_status_string(stepq_status s)
{
    switch (s) {
    case STEPQ_OK: return "STEPQ_OK";
    case STEPQ_ERR_INVALID_ARG: return "STEPQ_ERR_INVALID_ARG";
    case STEPQ_ERR_UNSUPPORTED: return "STEPQ_ERR_UNSUPPORTED";
    case STEPQ_ERR_CUDA: return "STEPQ_ERR_CUDA";
    case STEPQ_ERR_STATE: return "STEPQ_ERR_STATE";
    }
    return "STEPQ_ERR_UNKNOWN";
}

const char *stepq_last_error(void) { return g_err.c_str(); }

}  // extern "C"
