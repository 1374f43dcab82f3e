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
#include <queue>
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
    int n_pivot_items = 0;
    int max_n16 = 0;  // the most leading 16-bit field positions of a staged head
    int scale_mode = STEPQ_SCALE_DUAL;
    int nslots = 0, slot_bytes = 0;
    int off_q = 0, off_k = 0, off_v = 0, off_alpha = 0, off_ab = 0, off_rec = 0;
    // the active request set: decode steps update requests active[0..n_active)
    int n_active = 0;
    std::vector<int> kind;               // per head: kHeadQuant / kHeadAllPivot / kHeadMixed
    std::vector<long long> item_bytes;   // per head
    std::vector<long long> head_off;     // per head
    std::vector<int> active_tables;      // host copy of the uploaded order and staging records
    size_t guard[7] = {};                // offsets of the guard regions (kGuardRegions)
    size_t total = 0;                    // bytes of the pool's regions, guards included
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

// key_of[s]: the key row stored as storage row s.  Key order when the head's
// rows share one width; otherwise the key rows sorted by width (widest first,
// ties by key index), the j-th stored as row 16 (j % 8) + j / 8, so that every
// row group holds rows of the same widths.
void storage_rows(const uint8_t *bits, int *key_of)
{
    bool uniform = true;
    for (int i = 1; i < kDK; i++) uniform &= bits[i] == bits[0];
    if (uniform) {
        for (int s = 0; s < kDK; s++) key_of[s] = s;
        return;
    }
    int j = 0;
    for (int b = STEPQ_PIVOT_BITS; b >= 1; b--)
        for (int i = 0; i < kDK; i++)
            if (bits[i] == b) {
                key_of[stepq::kRowsPerGroup * (j % stepq::kRowGroups) + j / stepq::kRowGroups] = i;
                j++;
            }
}

// F[p]: the field width of row position p (storage rows 16 g + p), the widest
// row at that position over the row groups.
void position_widths(const uint8_t *bits, const int *key_of, int *F)
{
    for (int p = 0; p < stepq::kRowsPerGroup; p++) {
        F[p] = 0;
        for (int g = 0; g < stepq::kRowGroups; g++)
            F[p] = std::max(F[p], (int)bits[key_of[g * stepq::kRowsPerGroup + p]]);
    }
}

// 32-bit words per stream (W): ceil(4 sum_p F[p] / 32).
int stream_words(const uint8_t *bits)
{
    int key_of[kDK], F[stepq::kRowsPerGroup];
    storage_rows(bits, key_of);
    position_widths(bits, key_of, F);
    int nbits = 0;
    for (int p = 0; p < stepq::kRowsPerGroup; p++) nbits += 4 * F[p];
    return (nbits + 31) / 32;
}

// The fit constants of head h in storage order (rec fields bits, s, rho, rq,
// key_row, head_b); returns the number of pivot rows.
int fill_rows(const stepq_desc *d, int h, stepq::HeadRec &R)
{
    const uint8_t *bits = d->bits + (size_t)h * kDK;
    int key_of[kDK];
    storage_rows(bits, key_of);
    // impact floor of the row-scale factor: a quarter of the largest weight
    // among the head's quantised rows, so that no row's step is coarsened by
    // more than a factor 2 against the head's highest-impact row
    double rho_max = 0.0;
    for (int i = 0; i < kDK; i++)
        if (bits[i] != STEPQ_PIVOT_BITS) rho_max = std::max(rho_max, (double)d->rho[(size_t)h * kDK + i]);
    const double rho_floor = rho_max / 4.0;
    int npiv = 0, same = 1;
    for (int s = 0; s < kDK; s++) {
        const int i = key_of[s], b = bits[i];
        R.key_row[s] = (uint8_t)i;
        R.bits[s] = (uint8_t)b;
        same &= (b == bits[0]);
        if (b == STEPQ_PIVOT_BITS) {
            npiv++;
            R.s[s] = 0.f;
            R.rho[s] = 0.f;
            R.rq[s] = 0.f;
        } else {
            R.s[s] = (float)(1.0 / std::sqrt(std::max((double)d->rho[(size_t)h * kDK + i], rho_floor)));
            R.rho[s] = d->rho[(size_t)h * kDK + i];
            R.rq[s] = (float)(1.0 / (double)((1 << (b - 1)) - 1));
        }
    }
    R.head_b = (same && bits[0] != STEPQ_PIVOT_BITS) ? bits[0] : 0;
    int F[stepq::kRowsPerGroup];
    position_widths(bits, key_of, F);
    R.n16 = 0;
    for (int p = 0; p < stepq::kRowsPerGroup; p++) {
        R.pos_bits[p] = (uint8_t)F[p];
        R.pos_off[p] = (uint16_t)(p == 0 ? 0 : R.pos_off[p - 1] + 4 * F[p - 1]);
        R.n16 += F[p] == STEPQ_PIVOT_BITS;
    }
    R.pad = 0;
    return npiv;
}

// Guard words: a 64-byte region after every region of a pool buffer, filled
// at creation with a fixed pattern and compared by stepq_pool_check_guards.
constexpr size_t kGuardBytes = 64;
constexpr int kGuardRegions = 7;
const char *const kGuardAfter[kGuardRegions] = {"packed states", "head records", "head offsets", "item sizes",
                                                "status word", "item order", "staging records"};

uint32_t guard_word(int g, int k)
{
    return 0x5A17C0DEu ^ (uint32_t)g * 0x9E3779B9u ^ (uint32_t)k * 0x85EBCA6Bu;
}

struct Layout {
    size_t state = 0;
    size_t off_rec = 0, off_head_off = 0, off_head_bytes = 0, off_order = 0, off_stage = 0, off_status = 0,
           total = 0;
    size_t guard[kGuardRegions] = {};
    long long req_bytes = 0;
    std::vector<long long> item_bytes;  // per head
    std::vector<int> slab_words;        // per head: 32-bit words per stream
};

// Checks a descriptor; fills the layout when valid.
stepq_status check_desc(const stepq_desc *d, bool need_tables, Layout *L)
{
    if (!d) return fail(STEPQ_ERR_INVALID_ARG, "descriptor is NULL");
    if (d->variant != STEPQ_GDN && d->variant != STEPQ_KDA)
        return fail(STEPQ_ERR_INVALID_ARG, "variant %d is neither STEPQ_GDN nor STEPQ_KDA", d->variant);
    if (d->batch < 0) return fail(STEPQ_ERR_INVALID_ARG, "batch %d < 0", d->batch);
    if (d->heads < 1) return fail(STEPQ_ERR_INVALID_ARG, "heads %d < 1", d->heads);
    if (d->heads > 65535) return fail(STEPQ_ERR_UNSUPPORTED, "heads %d > 65535", d->heads);
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
        // packed item: header, then 8 slabs of 16 value columns; a slab holds 32
        // streams (8 row groups x 4 column groups) of W words each, W = the
        // largest over the row groups of ceil(4 * sum of the group's widths / 32)
        L->item_bytes.assign(H, 0);
        L->slab_words.assign(H, 0);
        long long req = 0;
        for (int h = 0; h < H; h++) {
            const int W = stream_words(d->bits + (size_t)h * kDK);
            L->slab_words[h] = W;
            const long long n = stepq::kHeaderBytes + 4LL * W * stepq::kStreams * stepq::kSlabs;
            L->item_bytes[h] = n;
            req += n;
        }
        L->req_bytes = req;
        L->state = (size_t)req * (size_t)d->batch;
        // each region is followed by a guard region
        size_t o = align_up(L->state, 16);
        L->guard[0] = o;       o = align_up(o + kGuardBytes, 256);
        L->off_rec = o;        o = align_up(o + sizeof(stepq::HeadRec) * (size_t)H, 16);
        L->guard[1] = o;       o = align_up(o + kGuardBytes, 16);
        L->off_head_off = o;   o = align_up(o + 8 * (size_t)H, 16);
        L->guard[2] = o;       o = align_up(o + kGuardBytes, 16);
        L->off_head_bytes = o; o = align_up(o + 4 * (size_t)H, 16);
        L->guard[3] = o;       o = align_up(o + kGuardBytes, 16);
        L->off_status = o;     o = align_up(o + 16, 16);
        L->guard[4] = o;       o = align_up(o + kGuardBytes, 16);
        L->off_order = o;      o = align_up(o + 4 * (size_t)H * d->batch, 16);
        L->guard[5] = o;       o = align_up(o + kGuardBytes, 16);
        L->off_stage = o;      o = align_up(o + 16 * (size_t)H * d->batch, 16);
        L->guard[6] = o;       o = align_up(o + kGuardBytes, 16);
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
    a.nslots = p->nslots;
    a.slot_bytes = p->slot_bytes;
    a.off_q = p->off_q; a.off_k = p->off_k; a.off_v = p->off_v;
    a.off_alpha = p->off_alpha; a.off_ab = p->off_ab; a.off_rec = p->off_rec;
    a.n_pivot_items = p->n_pivot_items;
    a.max_n16 = p->max_n16;
    a.scale_mode = p->scale_mode;
    a.batch = p->desc.batch;
    a.state_bytes = (long long)p->state_bytes;
    return a;
}

// Item order and staging records of a decode step over the requests
// active[0 .. n_active) (all requests in order when active is NULL): position
// list of the items b * H + h of the listed requests b.  Items of all-pivot
// heads come first (processed from global memory), then the staged items,
// heaviest heads first, equal weights in list order.
void build_order_stage(int H, const int *active, int n_active, const std::vector<int> &kind,
                       const std::vector<long long> &item_bytes, const long long *head_off, long long req_bytes,
                       int *order, int *stage)
{
    std::vector<int> idx((size_t)n_active * H);
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(), [&](int x, int y) {
        const int hx = x % H, hy = y % H;
        const int px = kind[hx] == stepq::kHeadAllPivot, py = kind[hy] == stepq::kHeadAllPivot;
        if (px != py) return px > py;
        return item_bytes[hx] > item_bytes[hy];
    });
    for (size_t n = 0; n < idx.size(); n++) {
        const int x = idx[n], h = x % H, r = x / H;
        const int b = active ? active[r] : r;
        const unsigned long long off = (unsigned long long)b * (unsigned long long)req_bytes +
                                       (unsigned long long)head_off[h];
        order[n] = b * H + h;
        stage[4 * n + 0] = b * H + h;
        stage[4 * n + 1] = (int)item_bytes[h] | (h << 16);
        stage[4 * n + 2] = (int)(uint32_t)(off >> 10);  // items start at multiples of 1024 bytes
        stage[4 * n + 3] = b;
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// Decode step without a pool, allocating nothing.  The fused decode kernel
// needs scratch tables next to the packed states: per-head records, the item
// order, one staging record per item and a status word.  A pool keeps them in
// the tail of the caller's buffer; this variant keeps them in a fixed
// file-scope device array instead and builds them on every call into a fixed
// host image.  It serves callers that hold the packed states in memory they
// manage themselves and may not allocate at decode time: a serving runtime
// that gives all free HBM to its own caching allocator (a cudaMalloc there
// fails or synchronises the device), or one whose state buffer has no room
// for a pool's table tail.  No cudaMalloc, cudaFree, host heap or other
// allocating call is made on the success path.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = 256 * 1024;  // the largest table image this variant accepts
constexpr int kNoAllocMaxHeads = 64;
constexpr int kNoAllocMaxDevices = 64;

// Device scratch.  Only its status word must start at zero; every call uploads
// the whole table image, status word (zero) included, before its launch.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;                             // guards the two arrays below
unsigned char g_noalloc_host[kNoAllocScratchBytes];  // host image of the scratch
void *g_noalloc_dev[kNoAllocMaxDevices];             // scratch address per device (first call)

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

stepq_status stepq_pool_layout(const stepq_desc *desc, stepq_pool_regions *out)
{
    if (!out) return fail(STEPQ_ERR_INVALID_ARG, "out is NULL");
    Layout L;
    stepq_status st = check_desc(desc, true, &L);
    if (st != STEPQ_OK) return st;
    out->states = 0;
    out->state_bytes = L.state;
    out->head_records = L.off_rec;
    out->head_offsets = L.off_head_off;
    out->item_sizes = L.off_head_bytes;
    out->status_word = L.off_status;
    out->item_order = L.off_order;
    out->staging_records = L.off_stage;
    for (int g = 0; g < kGuardRegions; g++) out->guards[g] = L.guard[g];
    out->guard_bytes = kGuardBytes;
    out->total = L.total;
    return STEPQ_OK;
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
    std::vector<uint8_t> host(L.total - L.guard[0], 0);
    auto at = [&](size_t off) { return host.data() + (off - L.guard[0]); };
    for (int g = 0; g < kGuardRegions; g++) {
        uint32_t *gw = reinterpret_cast<uint32_t *>(at(L.guard[g]));
        for (int k = 0; k < (int)(kGuardBytes / 4); k++) gw[k] = guard_word(g, k);
    }
    stepq::HeadRec *rec = reinterpret_cast<stepq::HeadRec *>(at(L.off_rec));
    long long *head_off = reinterpret_cast<long long *>(at(L.off_head_off));
    int *head_bytes = reinterpret_cast<int *>(at(L.off_head_bytes));
    int *order = reinterpret_cast<int *>(at(L.off_order));
    long long pre = 0;
    long long max_staged = 0;
    int max_n16 = 0;
    std::vector<int> kind(H, stepq::kHeadQuant);
    for (int h = 0; h < H; h++) {
        stepq::HeadRec &R = rec[h];
        head_off[h] = pre;
        head_bytes[h] = (int)L.item_bytes[h];
        R.head_off = pre;
        R.head_bytes = (int)L.item_bytes[h];
        pre += L.item_bytes[h];
        const int npiv = fill_rows(desc, h, R);
        kind[h] = npiv == 0 ? stepq::kHeadQuant : (npiv == kDK ? stepq::kHeadAllPivot : stepq::kHeadMixed);
        R.head_kind = kind[h];
        R.slab_words = L.slab_words[h];
        if (kind[h] != stepq::kHeadAllPivot) {
            max_staged = std::max(max_staged, L.item_bytes[h]);
            max_n16 = std::max(max_n16, R.n16);
        }
    }
    build_order_stage(H, nullptr, B, kind, L.item_bytes, head_off, L.req_bytes, order,
                      reinterpret_cast<int *>(at(L.off_stage)));
    int n_pivot_items = 0;
    for (int h = 0; h < H; h++) n_pivot_items += (kind[h] == stepq::kHeadAllPivot) ? B : 0;

    // staging slot geometry of the fused decode kernel: the item as stored, then
    // the step inputs and the head record
    const int kda = desc->variant == STEPQ_KDA;
    int off = (int)align_up((size_t)max_staged, 16);
    const int off_q = off; off += 4 * kDK;
    const int off_k = off; off += 4 * kDK;
    const int off_v = off; off += 4 * kDV;
    const int off_alpha = off; off += kda ? 4 * kDK : 0;
    const int off_ab = off; off += 16;
    const int off_rec = off; off += (int)sizeof(stepq::HeadRec);
    const int slot_bytes = (int)align_up((size_t)off, 128);
    int nslots = 0;
    for (int ns = stepq::kMaxSlots; ns >= 2; ns--) {
        if (stepq::decode_ctas_per_sm(ns, slot_bytes) >= 2) { nslots = ns; break; }
    }
    if (nslots == 0) {
        for (int ns = stepq::kMaxSlots; ns >= 2; ns--)
            if (stepq::decode_ctas_per_sm(ns, slot_bytes) >= 1) { nslots = ns; break; }
    }
    if (nslots == 0 && max_staged > 0) return fail(STEPQ_ERR_CUDA, "no staging ring fits in shared memory");

    cudaStream_t s = reinterpret_cast<cudaStream_t>(cuda_stream);
    uint8_t *dev = static_cast<uint8_t *>(dev_buf);
    cudaError_t e = cudaMemcpyAsync(dev + L.guard[0], host.data(), host.size(), cudaMemcpyHostToDevice, s);
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
    for (int g = 0; g < kGuardRegions; g++) p->guard[g] = L.guard[g];
    p->total = L.total;
    p->req_bytes = L.req_bytes;
    p->stream = s;
    p->t.rowrec = reinterpret_cast<const stepq::HeadRec *>(dev + L.off_rec);
    p->t.head_off = reinterpret_cast<const long long *>(dev + L.off_head_off);
    p->t.head_bytes = reinterpret_cast<const int *>(dev + L.off_head_bytes);
    p->t.order = reinterpret_cast<const int *>(dev + L.off_order);
    p->t.stage = reinterpret_cast<const int4 *>(dev + L.off_stage);
    p->t.status = reinterpret_cast<int *>(dev + L.off_status);
    p->n_pivot_items = n_pivot_items;
    p->max_n16 = max_n16;
    p->nslots = nslots;
    p->slot_bytes = slot_bytes;
    p->off_q = off_q; p->off_k = off_k; p->off_v = off_v;
    p->off_alpha = off_alpha; p->off_ab = off_ab; p->off_rec = off_rec;
    p->n_active = B;
    p->kind = kind;
    p->item_bytes = L.item_bytes;
    p->head_off.assign(head_off, head_off + H);
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

stepq_status stepq_pool_set_scale_mode(stepq_pool *pool, int mode)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    if (mode < STEPQ_SCALE_DUAL || mode > STEPQ_SCALE_HEAD) return fail(STEPQ_ERR_INVALID_ARG, "scale mode %d", mode);
    pool->scale_mode = mode;
    return STEPQ_OK;
}

stepq_status stepq_pool_set_active(stepq_pool *pool, const int *active, int n_active)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    const int B = pool->desc.batch, H = pool->desc.heads;
    if (!active) n_active = B;
    if (n_active < 0 || n_active > B)
        return fail(STEPQ_ERR_INVALID_ARG, "n_active = %d is outside 0 .. batch = %d", n_active, B);
    if (active) {
        std::vector<char> seen((size_t)B, 0);
        for (int r = 0; r < n_active; r++) {
            const int b = active[r];
            if (b < 0 || b >= B) return fail(STEPQ_ERR_INVALID_ARG, "active[%d] = %d is not a request of the pool", r, b);
            if (seen[b]) return fail(STEPQ_ERR_INVALID_ARG, "request %d is listed twice", b);
            seen[b] = 1;
        }
    }
    const size_t n = (size_t)n_active * H;
    std::vector<int> &tb = pool->active_tables;
    tb.assign(5 * n, 0);
    build_order_stage(H, active, n_active, pool->kind, pool->item_bytes, pool->head_off.data(), pool->req_bytes,
                      tb.data(), tb.data() + n);
    if (n > 0) {
        cudaError_t e = cudaMemcpyAsync(const_cast<int *>(pool->t.order), tb.data(), 4 * n, cudaMemcpyHostToDevice,
                                        pool->stream);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(const_cast<int4 *>(pool->t.stage), tb.data() + n, 16 * n, cudaMemcpyHostToDevice,
                                pool->stream);
        if (e != cudaSuccess) return cuda_fail(e, "stepq_pool_set_active upload");
    }
    pool->n_active = n_active;
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
    const size_t n = (size_t)pool->desc.batch * pool->desc.heads;  // rows of the step tensors
    if (n == 0 || pool->n_active == 0) return STEPQ_OK;
    if ((st = check_step_tensors(pool->desc.variant, n, q, k, v, alpha, beta, out)) != STEPQ_OK) return st;
    if (overlaps(out, n * kDV * 4, pool->dev, pool->bytes))
        return fail(STEPQ_ERR_INVALID_ARG, "out overlaps the pool buffer");
    stepq::StepArgs a = base_args(pool);
    // the active requests' items: the tables hold n_active * heads positions
    a.n_items = pool->n_active * pool->desc.heads;
    a.n_pivot_items = 0;
    for (int h = 0; h < pool->desc.heads; h++)
        a.n_pivot_items += (pool->kind[h] == stepq::kHeadAllPivot) ? pool->n_active : 0;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.out = out;
    cudaError_t e = stepq::launch_decode_step(a, pool->stream);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_decode_step launch");
}

stepq_status stepq_decode_step_split(stepq_pool *pool, float *S_work, const float *q, const float *k,
                                     const float *v, const float *alpha, const float *beta, float *out,
                                     void *side_stream)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    if (pool->n_active != pool->desc.batch)
        return fail(STEPQ_ERR_UNSUPPORTED, "stepq_decode_step_split needs every request active");
    const size_t n = (size_t)pool->desc.batch * pool->desc.heads;
    if (n == 0) return STEPQ_OK;
    if ((st = check_step_tensors(pool->desc.variant, n, q, k, v, alpha, beta, out)) != STEPQ_OK) return st;
    if ((st = check_dev(S_work, "S_work", 16)) != STEPQ_OK) return st;
    const size_t nw = n * kDK * kDV * 4;
    if (overlaps(out, n * kDV * 4, pool->dev, pool->bytes))
        return fail(STEPQ_ERR_INVALID_ARG, "out overlaps the pool buffer");
    if (overlaps(S_work, nw, pool->dev, pool->bytes) || overlaps(S_work, nw, out, n * kDV * 4) ||
        overlaps(S_work, nw, q, n * kDK * 4) || overlaps(S_work, nw, k, n * kDK * 4) ||
        overlaps(S_work, nw, v, n * kDV * 4))
        return fail(STEPQ_ERR_INVALID_ARG, "S_work overlaps the pool or a step tensor");
    stepq::StepArgs a = base_args(pool);
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.out = out;
    a.S_in = S_work;
    cudaError_t e = stepq::launch_split_update(a, pool->stream);
    if (e != cudaSuccess) return cuda_fail(e, "stepq_decode_step_split update launch");
    cudaStream_t side = reinterpret_cast<cudaStream_t>(side_stream);
    if (side == nullptr || side == pool->stream) {
        e = stepq::launch_pack(a, pool->stream);
        return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_decode_step_split pack launch");
    }
    // fit + writeback on the side stream, ordered after the update and before
    // the pool stream's later work
    cudaEvent_t ev[2] = {nullptr, nullptr};
    for (int i = 0; i < 2; i++) {
        e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
        if (e != cudaSuccess) {
            if (ev[0]) cudaEventDestroy(ev[0]);
            return cuda_fail(e, "stepq_decode_step_split event");
        }
    }
    if ((e = cudaEventRecord(ev[0], pool->stream)) == cudaSuccess &&
        (e = cudaStreamWaitEvent(side, ev[0], 0)) == cudaSuccess &&
        (e = stepq::launch_pack(a, side)) == cudaSuccess && (e = cudaEventRecord(ev[1], side)) == cudaSuccess)
        e = cudaStreamWaitEvent(pool->stream, ev[1], 0);
    cudaEventDestroy(ev[0]);
    cudaEventDestroy(ev[1]);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_decode_step_split side stream");
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

stepq_status stepq_pool_check(stepq_pool *pool)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    cudaError_t e = cudaStreamSynchronize(pool->stream);
    if (e != cudaSuccess) return cuda_fail(e, "stepq_pool_check sync");
    int code = 0;
    e = cudaMemcpy(&code, pool->t.status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "stepq_pool_check read");
    if (code != 0) {
        const int zero = 0;
        cudaMemcpy(pool->t.status, &zero, sizeof(int), cudaMemcpyHostToDevice);
        if (code == stepq::kStatusBadTable)
            return fail(STEPQ_ERR_CUDA, "the checking build found a staging record or head record that does not "
                                        "match the pool's layout (device status %d); no item was updated", code);
        return fail(STEPQ_ERR_CUDA, "a kernel gave up waiting for a staged copy (device status %d); "
                                    "the affected items were not updated", code);
    }
    return STEPQ_OK;
}

stepq_status stepq_selftest_bounded_wait(int *result, long long limit_cycles, int arrive, void *cuda_stream)
{
    if (!result) return fail(STEPQ_ERR_INVALID_ARG, "stepq_selftest_bounded_wait: result is NULL");
    if (limit_cycles < 0 || limit_cycles > (1LL << 34))
        return fail(STEPQ_ERR_INVALID_ARG, "stepq_selftest_bounded_wait: limit_cycles %lld outside [0, 2^34]",
                    limit_cycles);
    cudaError_t e = stepq::launch_wait_selftest(result, limit_cycles, arrive ? 1 : 0,
                                                static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess) return cuda_fail(e, "stepq_selftest_bounded_wait launch");
    return STEPQ_OK;
}

stepq_status stepq_pool_check_guards(stepq_pool *pool)
{
    stepq_status st = check_pool(pool);
    if (st != STEPQ_OK) return st;
    cudaError_t e = cudaStreamSynchronize(pool->stream);
    if (e != cudaSuccess) return cuda_fail(e, "stepq_pool_check_guards: stream");
    uint32_t w[kGuardBytes / 4];
    for (int g = 0; g < kGuardRegions; g++) {
        e = cudaMemcpy(w, pool->dev + pool->guard[g], kGuardBytes, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "stepq_pool_check_guards: read back");
        for (int k = 0; k < (int)(kGuardBytes / 4); k++)
            if (w[k] != guard_word(g, k))
                return fail(STEPQ_ERR_STATE, "guard word %d after the %s changed: 0x%08x, expected 0x%08x", k,
                            kGuardAfter[g], w[k], guard_word(g, k));
    }
    g_err.clear();
    return STEPQ_OK;
}

// ---- calibration ----------------------------------------------------------

namespace {

constexpr double kRhoFloor = 1e-30;  // rho of a row whose query weight is always 0
constexpr double kGapFloor = 1e-12;  // floor of 1 - abar^2 (a unit that never decays)

stepq_status check_widths(int n_widths, const int *widths)
{
    if (n_widths < 1 || n_widths > stepq::kCalibMaxWidths)
        return fail(STEPQ_ERR_INVALID_ARG, "n_widths %d outside 1..%d", n_widths, stepq::kCalibMaxWidths);
    if (!widths) return fail(STEPQ_ERR_INVALID_ARG, "widths is NULL");
    for (int x = 0; x < n_widths; x++) {
        if (widths[x] < 2 || widths[x] > 8) return fail(STEPQ_ERR_INVALID_ARG, "width %d outside 2..8", widths[x]);
        if (x > 0 && widths[x] <= widths[x - 1]) return fail(STEPQ_ERR_INVALID_ARG, "widths not ascending");
    }
    return STEPQ_OK;
}

stepq_status check_calib_desc(const stepq_calib_desc *cd)
{
    if (!cd) return fail(STEPQ_ERR_INVALID_ARG, "calibration descriptor is NULL");
    if (cd->variant != STEPQ_GDN && cd->variant != STEPQ_KDA)
        return fail(STEPQ_ERR_INVALID_ARG, "variant %d", cd->variant);
    if (cd->dk != kDK || cd->dv != kDV) return fail(STEPQ_ERR_UNSUPPORTED, "dk = dv = 128 only");
    if (cd->batch < 1 || cd->heads < 1 || (long long)cd->batch * cd->heads > (1LL << 24))
        return fail(STEPQ_ERR_INVALID_ARG, "batch %d x heads %d", cd->batch, cd->heads);
    if (cd->steps < 1 || cd->sample_every < 1 || cd->sample_every > cd->steps)
        return fail(STEPQ_ERR_INVALID_ARG, "steps %d, sample_every %d: no state would be sampled", cd->steps,
                    cd->sample_every);
    if (cd->ls_iters < 0 || cd->ls_iters > 16) return fail(STEPQ_ERR_INVALID_ARG, "ls_iters %d", cd->ls_iters);
    if (!(cd->avg_bits > 0.0 && cd->avg_bits <= 16.0)) return fail(STEPQ_ERR_INVALID_ARG, "avg_bits");
    if (!(cd->pivot_frac >= 0.0 && cd->pivot_frac <= 1.0)) return fail(STEPQ_ERR_INVALID_ARG, "pivot_frac");
    return check_widths(cd->n_widths, cd->widths);
}

struct CalibLayout {
    size_t S, out, err, rc, acc_q2, acc_loga, err_sum, rho, total;
};

CalibLayout calib_layout(const stepq_calib_desc *cd)
{
    const size_t n = (size_t)cd->batch * cd->heads, H = (size_t)cd->heads, nW = (size_t)cd->n_widths;
    CalibLayout L;
    size_t o = 0;
    L.S = o;        o = align_up(o + n * kDK * kDV * 4, 256);
    L.out = o;      o = align_up(o + n * kDV * 4, 256);
    L.err = o;      o = align_up(o + n * nW * kDK * 4, 256);
    L.rc = o;       o = align_up(o + n * nW * (kDK + kDV) * 4, 256);
    L.acc_q2 = o;   o = align_up(o + H * kDK * 8, 256);
    L.acc_loga = o; o = align_up(o + H * kDK * 8, 256);
    L.err_sum = o;  o = align_up(o + H * nW * kDK * 8, 256);
    L.rho = o;      o = align_up(o + H * kDK * 4, 256);
    L.total = o;
    return L;
}

// Lifetime weight of a unit with mean log retention m.
double lifetime_weight(double m)
{
    const double a = std::exp(m);
    return 1.0 / std::max(1.0 - a * a, kGapFloor);
}

// The greedy allocation over n units (D: n x nc, by unit); false if the
// pivots and the narrowest width alone exceed the budget.
bool allocate_units(int n, const std::vector<double> &w, const std::vector<double> &D, int nc, const int *widths,
                    double avg_bits, int n_piv, std::vector<uint8_t> &out)
{
    std::vector<int> level(n, 0);  // index into widths; -1: pivot
    for (int p = 0; p < std::min(n_piv, n); p++) {
        int pick = -1;
        double top = 0.0;
        for (int u = 0; u < n; u++) {
            if (level[u] < 0) continue;
            const double risk = w[u] * D[(size_t)u * nc];
            if (pick < 0 || risk > top) {
                pick = u;
                top = risk;
            }
        }
        level[pick] = -1;
    }
    long long spent = 0;
    for (int u = 0; u < n; u++) spent += level[u] < 0 ? STEPQ_PIVOT_BITS : widths[0];
    long long left = std::llround(avg_bits * n) - spent;
    const bool feasible = left >= 0;
    // upgrades by gain, largest first, ties to the lower unit: a unit's gain
    // changes only when it is upgraded, and an upgrade that does not fit never
    // fits later (the budget only shrinks), so a heap gives the picks of a
    // scan over all units at every step
    struct Up {
        double gain;
        int u;
    };
    auto below = [](const Up &a, const Up &b) { return a.gain < b.gain || (a.gain == b.gain && a.u > b.u); };
    std::priority_queue<Up, std::vector<Up>, decltype(below)> heap(below);
    auto offer = [&](int u) {
        const int x = level[u];
        if (x < 0 || x + 1 >= nc) return;
        const int cost = widths[x + 1] - widths[x];
        const double gain = w[u] * (D[(size_t)u * nc + x] - D[(size_t)u * nc + x + 1]) / cost;
        if (gain > 0.0) heap.push({gain, u});
    };
    for (int u = 0; u < n; u++) offer(u);
    while (!heap.empty() && left > 0) {
        const int u = heap.top().u;
        heap.pop();
        const int cost = widths[level[u] + 1] - widths[level[u]];
        if (cost > left) continue;
        left -= cost;
        level[u]++;
        offer(u);
    }
    out.resize(n);
    for (int u = 0; u < n; u++) out[u] = (uint8_t)(level[u] < 0 ? STEPQ_PIVOT_BITS : widths[level[u]]);
    return feasible;
}

}  // namespace

stepq_status stepq_calib_rho(int heads, double n_samples, const double *acc_q2, float *rho)
{
    if (heads < 1 || !acc_q2 || !rho || !(n_samples > 0.0))
        return fail(STEPQ_ERR_INVALID_ARG, "stepq_calib_rho arguments");
    for (long long u = 0; u < (long long)heads * kDK; u++)
        rho[u] = (float)std::max(acc_q2[u] / n_samples, kRhoFloor);
    return STEPQ_OK;
}

stepq_status stepq_calib_bits(int variant, int heads, double n_samples, const double *acc_loga, const float *rho,
                              const double *err_sum, int n_widths, const int *widths, double avg_bits,
                              double pivot_frac, uint8_t *bits)
{
    if ((variant != STEPQ_GDN && variant != STEPQ_KDA) || heads < 1 || !acc_loga || !rho || !err_sum || !bits ||
        !(n_samples > 0.0) || !(avg_bits > 0.0) || !(pivot_frac >= 0.0 && pivot_frac <= 1.0))
        return fail(STEPQ_ERR_INVALID_ARG, "stepq_calib_bits arguments");
    stepq_status st = check_widths(n_widths, widths);
    if (st != STEPQ_OK) return st;
    const bool kda = variant == STEPQ_KDA;
    const int n = kda ? heads * kDK : heads;
    std::vector<double> w(n), D((size_t)n * n_widths);
    for (int u = 0; u < n; u++) w[u] = lifetime_weight(acc_loga[u] / n_samples);
    for (int h = 0; h < heads; h++)
        for (int x = 0; x < n_widths; x++) {
            const double *e = err_sum + ((size_t)h * n_widths + x) * kDK;
            if (kda) {
                for (int i = 0; i < kDK; i++) D[((size_t)h * kDK + i) * n_widths + x] = (double)rho[h * kDK + i] * e[i];
            } else {
                double acc = 0.0;
                for (int i = 0; i < kDK; i++) acc += (double)rho[h * kDK + i] * e[i];
                D[(size_t)h * n_widths + x] = acc;
            }
        }
    const int n_piv = pivot_frac > 0.0 ? (int)std::ceil(pivot_frac * n - 1e-9) : 0;
    std::vector<uint8_t> units;
    const bool ok = allocate_units(n, w, D, n_widths, widths, avg_bits, n_piv, units);
    for (int h = 0; h < heads; h++)
        for (int i = 0; i < kDK; i++) bits[h * kDK + i] = kda ? units[h * kDK + i] : units[h];
    if (!ok)
        return fail(STEPQ_ERR_INVALID_ARG, "bit budget %.4f x %d below the pivots and the narrowest width",
                    avg_bits, n);
    return STEPQ_OK;
}

stepq_status stepq_calib_accumulate(int variant, int batch, int heads, const float *q, const float *alpha,
                                    double *acc_q2, double *acc_loga, void *cuda_stream)
{
    if ((variant != STEPQ_GDN && variant != STEPQ_KDA) || batch < 0 || heads < 0)
        return fail(STEPQ_ERR_INVALID_ARG, "stepq_calib_accumulate shape");
    if (batch == 0 || heads == 0) return STEPQ_OK;
    stepq_status st;
    if ((st = check_dev(q, "q", 16)) != STEPQ_OK || (st = check_dev(alpha, "alpha", 4)) != STEPQ_OK ||
        (st = check_dev(acc_q2, "acc_q2", 8)) != STEPQ_OK || (st = check_dev(acc_loga, "acc_loga", 8)) != STEPQ_OK)
        return st;
    stepq::CalibArgs c{};
    c.batch = batch; c.heads = heads; c.kda = variant == STEPQ_KDA;
    c.q = q; c.alpha = alpha; c.acc_q2 = acc_q2; c.acc_loga = acc_loga;
    cudaError_t e = stepq::launch_calib_accumulate(c, reinterpret_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_calib_accumulate launch");
}

stepq_status stepq_calib_row_error(int batch, int heads, const float *S, const float *rho, int n_widths,
                                   const int *widths, int ls_iters, float *err, float *rc, void *cuda_stream)
{
    if (batch < 0 || heads < 0 || (long long)batch * heads > (1LL << 24) || ls_iters < 0 || ls_iters > 16)
        return fail(STEPQ_ERR_INVALID_ARG, "stepq_calib_row_error shape");
    stepq_status st = check_widths(n_widths, widths);
    if (st != STEPQ_OK) return st;
    if (batch == 0 || heads == 0) return STEPQ_OK;
    if ((st = check_dev(S, "S", 16)) != STEPQ_OK || (st = check_dev(rho, "rho", 4)) != STEPQ_OK ||
        (st = check_dev(err, "err", 4)) != STEPQ_OK || (st = check_dev(rc, "rc", 4)) != STEPQ_OK)
        return st;
    stepq::CalibArgs c{};
    c.batch = batch; c.heads = heads; c.n_widths = n_widths; c.ls_iters = ls_iters;
    for (int x = 0; x < n_widths; x++) c.widths[x] = widths[x];
    c.S = S; c.rho = rho; c.err = err; c.rc = rc;
    cudaError_t e = stepq::launch_calib_error(c, reinterpret_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_calib_row_error launch");
}

stepq_status stepq_calib_reduce(int batch, int heads, int n_widths, const float *err, double *err_sum,
                                void *cuda_stream)
{
    if (batch < 0 || heads < 0 || n_widths < 1 || n_widths > stepq::kCalibMaxWidths)
        return fail(STEPQ_ERR_INVALID_ARG, "stepq_calib_reduce shape");
    if (heads == 0) return STEPQ_OK;
    stepq_status st;
    if ((st = check_dev(err, "err", 4)) != STEPQ_OK || (st = check_dev(err_sum, "err_sum", 8)) != STEPQ_OK)
        return st;
    stepq::CalibArgs c{};
    c.batch = batch; c.heads = heads; c.n_widths = n_widths; c.err = const_cast<float *>(err); c.err_sum = err_sum;
    cudaError_t e = stepq::launch_calib_reduce(c, reinterpret_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_calib_reduce launch");
}

size_t stepq_calib_scratch_bytes(const stepq_calib_desc *cd)
{
    if (check_calib_desc(cd) != STEPQ_OK) return 0;
    return calib_layout(cd).total;
}

stepq_status stepq_calibrate(const stepq_calib_desc *cd, const float *S0, const float *q, const float *k,
                             const float *v, const float *alpha, const float *beta, void *scratch,
                             size_t scratch_bytes, void *cuda_stream, float *rho_out, uint8_t *bits_out)
{
    stepq_status st = check_calib_desc(cd);
    if (st != STEPQ_OK) return st;
    if (!rho_out || !bits_out) return fail(STEPQ_ERR_INVALID_ARG, "rho_out / bits_out is NULL");
    const CalibLayout L = calib_layout(cd);
    if (scratch_bytes < L.total)
        return fail(STEPQ_ERR_INVALID_ARG, "scratch of %zu bytes < %zu required", scratch_bytes, L.total);
    const bool kda = cd->variant == STEPQ_KDA;
    if ((st = check_dev(scratch, "scratch", 256)) != STEPQ_OK || (st = check_dev(S0, "S0", 16)) != STEPQ_OK ||
        (st = check_dev(q, "q", 16)) != STEPQ_OK || (st = check_dev(k, "k", 16)) != STEPQ_OK ||
        (st = check_dev(v, "v", 16)) != STEPQ_OK || (st = check_dev(alpha, "alpha", kda ? 16 : 4)) != STEPQ_OK ||
        (st = check_dev(beta, "beta", 4)) != STEPQ_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(cuda_stream);
    uint8_t *base = static_cast<uint8_t *>(scratch);
    const int B = cd->batch, H = cd->heads, nW = cd->n_widths;
    const size_t n = (size_t)B * H;
    const size_t qstep = n * kDK, vstep = n * kDV, astep = kda ? n * kDK : n;
    float *S = reinterpret_cast<float *>(base + L.S);
    float *out = reinterpret_cast<float *>(base + L.out);
    double *acc_q2 = reinterpret_cast<double *>(base + L.acc_q2);
    double *acc_loga = reinterpret_cast<double *>(base + L.acc_loga);
    double *err_sum = reinterpret_cast<double *>(base + L.err_sum);
    float *rho_dev = reinterpret_cast<float *>(base + L.rho);
    cudaError_t e = cudaSuccess;
    auto cuda_ok = [&](cudaError_t r) { e = r; return r == cudaSuccess; };
    // impact and retention sums over every step's inputs
    if (!cuda_ok(cudaMemsetAsync(acc_q2, 0, (size_t)H * kDK * 8, s)) ||
        !cuda_ok(cudaMemsetAsync(acc_loga, 0, (size_t)H * kDK * 8, s)))
        return cuda_fail(e, "stepq_calibrate clear");
    for (int t = 0; t < cd->steps; t++) {
        st = stepq_calib_accumulate(cd->variant, B, H, q + t * qstep, alpha + t * astep, acc_q2, acc_loga, s);
        if (st != STEPQ_OK) return st;
    }
    std::vector<double> h_q2((size_t)H * kDK), h_loga((size_t)H * kDK);
    if (!cuda_ok(cudaMemcpyAsync(h_q2.data(), acc_q2, h_q2.size() * 8, cudaMemcpyDeviceToHost, s)) ||
        !cuda_ok(cudaMemcpyAsync(h_loga.data(), acc_loga, h_loga.size() * 8, cudaMemcpyDeviceToHost, s)) ||
        !cuda_ok(cudaStreamSynchronize(s)))
        return cuda_fail(e, "stepq_calibrate read sums");
    const double n_samples = (double)B * cd->steps;
    if ((st = stepq_calib_rho(H, n_samples, h_q2.data(), rho_out)) != STEPQ_OK) return st;
    // the rollout, its sampled states' errors at every candidate width
    if (!cuda_ok(cudaMemcpyAsync(rho_dev, rho_out, (size_t)H * kDK * 4, cudaMemcpyHostToDevice, s)) ||
        !cuda_ok(cudaMemcpyAsync(S, S0, n * kDK * kDV * 4, cudaMemcpyDeviceToDevice, s)) ||
        !cuda_ok(cudaMemsetAsync(err_sum, 0, (size_t)H * nW * kDK * 8, s)))
        return cuda_fail(e, "stepq_calibrate setup");
    float *err = reinterpret_cast<float *>(base + L.err);
    float *rc = reinterpret_cast<float *>(base + L.rc);
    for (int t = 0; t < cd->steps; t++) {
        if (!cuda_ok(stepq::launch_fp32_step(S, q + t * qstep, k + t * qstep, v + t * vstep, alpha + t * astep,
                                             beta + t * n, out, (int)n, kda, s)))
            return cuda_fail(e, "stepq_calibrate rollout");
        if ((t + 1) % cd->sample_every != 0) continue;
        if ((st = stepq_calib_row_error(B, H, S, rho_dev, nW, cd->widths, cd->ls_iters, err, rc, s)) != STEPQ_OK ||
            (st = stepq_calib_reduce(B, H, nW, err, err_sum, s)) != STEPQ_OK)
            return st;
    }
    std::vector<double> h_err((size_t)H * nW * kDK);
    if (!cuda_ok(cudaMemcpyAsync(h_err.data(), err_sum, h_err.size() * 8, cudaMemcpyDeviceToHost, s)) ||
        !cuda_ok(cudaStreamSynchronize(s)))
        return cuda_fail(e, "stepq_calibrate read errors");
    return stepq_calib_bits(cd->variant, H, n_samples, h_loga.data(), rho_out, h_err.data(), nW, cd->widths,
                            cd->avg_bits, cd->pivot_frac, bits_out);
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

stepq_status stepq_decode_step_noalloc(const stepq_desc *desc, void *states, size_t state_bytes, const float *q,
                                       const float *k, const float *v, const float *alpha, const float *beta,
                                       float *out, void *cuda_stream)
{
    stepq_status st = check_desc(desc, true, nullptr);
    if (st != STEPQ_OK) return st;
    const int H = desc->heads, B = desc->batch;
    if (H > kNoAllocMaxHeads)
        return fail(STEPQ_ERR_UNSUPPORTED, "stepq_decode_step_noalloc takes at most %d heads (got %d)",
                    kNoAllocMaxHeads, H);
    const size_t n = (size_t)B * H;
    // per-head item layout, as in a pool
    long long item_bytes[kNoAllocMaxHeads], head_off[kNoAllocMaxHeads];
    int slab_words[kNoAllocMaxHeads], kind[kNoAllocMaxHeads];
    long long req = 0, max_staged = 0;
    int n_pivot_items = 0;
    for (int h = 0; h < H; h++) {
        const int W = stream_words(desc->bits + (size_t)h * kDK);
        int npiv = 0;
        for (int i = 0; i < kDK; i++) npiv += desc->bits[h * kDK + i] == STEPQ_PIVOT_BITS;
        slab_words[h] = W;
        item_bytes[h] = stepq::kHeaderBytes + 4LL * W * stepq::kStreams * stepq::kSlabs;
        kind[h] = npiv == 0 ? stepq::kHeadQuant : (npiv == kDK ? stepq::kHeadAllPivot : stepq::kHeadMixed);
        head_off[h] = req;
        req += item_bytes[h];
        if (kind[h] == stepq::kHeadAllPivot)
            n_pivot_items += B;
        else
            max_staged = std::max(max_staged, item_bytes[h]);
    }
    // scratch image layout
    size_t o = 0;
    const size_t off_rec = o;        o = align_up(o + sizeof(stepq::HeadRec) * (size_t)H, 256);
    const size_t off_head_off = o;   o = align_up(o + 8 * (size_t)H, 16);
    const size_t off_head_bytes = o; o = align_up(o + 4 * (size_t)H, 16);
    const size_t off_status = o;     o = align_up(o + 16, 16);
    const size_t off_order = o;      o = align_up(o + 4 * n, 16);
    const size_t off_stage = o;      o = align_up(o + 16 * n, 16);
    if (o > kNoAllocScratchBytes)
        return fail(STEPQ_ERR_UNSUPPORTED,
                    "stepq_decode_step_noalloc: the tables of %d requests x %d heads take %zu bytes, more than "
                    "its fixed %zu-byte scratch; use a pool", B, H, o, kNoAllocScratchBytes);
    if (state_bytes < (size_t)req * (size_t)B)
        return fail(STEPQ_ERR_INVALID_ARG, "states holds %zu bytes < %zu required", state_bytes,
                    (size_t)req * (size_t)B);
    if (n == 0) return STEPQ_OK;
    if ((st = check_dev(states, "states", 16)) != STEPQ_OK) return st;
    if ((st = check_step_tensors(desc->variant, n, q, k, v, alpha, beta, out)) != STEPQ_OK) return st;
    if (overlaps(out, n * kDV * 4, states, (size_t)req * (size_t)B))
        return fail(STEPQ_ERR_INVALID_ARG, "out overlaps the packed states");
    // staging slot geometry, as in a pool
    const int kda = desc->variant == STEPQ_KDA;
    int off = (int)align_up((size_t)max_staged, 16);
    const int off_q = off; off += 4 * kDK;
    const int off_k = off; off += 4 * kDK;
    const int off_v = off; off += 4 * kDV;
    const int off_alpha = off; off += kda ? 4 * kDK : 0;
    const int off_ab = off; off += 16;
    const int off_rec_slot = off; off += (int)sizeof(stepq::HeadRec);
    const int slot_bytes = (int)align_up((size_t)off, 128);
    int nslots = 0;
    for (int ns = stepq::kMaxSlots; ns >= 2 && nslots == 0; ns--)
        if (stepq::decode_ctas_per_sm(ns, slot_bytes) >= 2) nslots = ns;
    for (int ns = stepq::kMaxSlots; ns >= 2 && nslots == 0; ns--)
        if (stepq::decode_ctas_per_sm(ns, slot_bytes) >= 1) nslots = ns;
    if (nslots == 0 && max_staged > 0) return fail(STEPQ_ERR_CUDA, "no staging ring fits in shared memory");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "stepq_decode_step_noalloc: current device");
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return fail(STEPQ_ERR_UNSUPPORTED, "stepq_decode_step_noalloc supports device ordinals below %d",
                    kNoAllocMaxDevices);
    std::lock_guard<std::mutex> guard(g_noalloc_mu);
    if (!g_noalloc_dev[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "stepq_decode_step_noalloc: scratch address");
        g_noalloc_dev[dev] = p;
    }
    uint8_t *img = g_noalloc_host;
    std::memset(img, 0, o);
    stepq::HeadRec *rec = reinterpret_cast<stepq::HeadRec *>(img + off_rec);
    long long *t_head_off = reinterpret_cast<long long *>(img + off_head_off);
    int *t_head_bytes = reinterpret_cast<int *>(img + off_head_bytes);
    int *order = reinterpret_cast<int *>(img + off_order);
    int *stage = reinterpret_cast<int *>(img + off_stage);
    int max_n16 = 0;
    for (int h = 0; h < H; h++) {
        stepq::HeadRec &R = rec[h];
        fill_rows(desc, h, R);
        R.head_off = head_off[h];
        R.head_kind = kind[h];
        R.head_bytes = (int)item_bytes[h];
        R.slab_words = slab_words[h];
        t_head_off[h] = head_off[h];
        t_head_bytes[h] = (int)item_bytes[h];
        if (kind[h] != stepq::kHeadAllPivot) max_n16 = std::max(max_n16, R.n16);
    }
    // item order: all-pivot heads' items first, then the others, heaviest
    // heads first; items of equal weight in item order
    int hs[kNoAllocMaxHeads];
    for (int h = 0; h < H; h++) hs[h] = h;
    for (int x = 1; x < H; x++) {  // stable insertion sort of the heads
        const int hx = hs[x];
        int y = x;
        for (; y > 0; y--) {
            const int hy = hs[y - 1];
            const int px = kind[hx] == stepq::kHeadAllPivot, py = kind[hy] == stepq::kHeadAllPivot;
            const bool before = (px != py) ? (px > py) : (item_bytes[hx] > item_bytes[hy]);
            if (!before) break;
            hs[y] = hy;
        }
        hs[y] = hx;
    }
    size_t pos = 0;
    for (int c0 = 0; c0 < H;) {
        int c1 = c0 + 1;  // heads hs[c0 .. c1) share one key
        while (c1 < H && (kind[hs[c1]] == stepq::kHeadAllPivot) == (kind[hs[c0]] == stepq::kHeadAllPivot) &&
               item_bytes[hs[c1]] == item_bytes[hs[c0]])
            c1++;
        int lo = c0, hi = c1;  // within the class, item order: request-major, then head
        for (int x = lo + 1; x < hi; x++)
            for (int y = x; y > lo && hs[y] < hs[y - 1]; y--) std::swap(hs[y], hs[y - 1]);
        for (int b = 0; b < B; b++)
            for (int c = lo; c < hi; c++) {
                const int h = hs[c], item = b * H + h;
                const unsigned long long offb = (unsigned long long)b * (unsigned long long)req +
                                                (unsigned long long)head_off[h];
                order[pos] = item;
                stage[4 * pos + 0] = item;
                stage[4 * pos + 1] = (int)item_bytes[h] | (h << 16);
                stage[4 * pos + 2] = (int)(uint32_t)(offb >> 10);  // items start at multiples of 1024 bytes
                stage[4 * pos + 3] = b;
                pos++;
            }
        c0 = c1;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(cuda_stream);
    uint8_t *dsc = static_cast<uint8_t *>(g_noalloc_dev[dev]);
    e = cudaMemcpyAsync(dsc, img, o, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "stepq_decode_step_noalloc: table upload");
    stepq::StepArgs a{};
    a.pool = static_cast<uint8_t *>(states);
    a.t.rowrec = reinterpret_cast<const stepq::HeadRec *>(dsc + off_rec);
    a.t.head_off = reinterpret_cast<const long long *>(dsc + off_head_off);
    a.t.head_bytes = reinterpret_cast<const int *>(dsc + off_head_bytes);
    a.t.order = reinterpret_cast<const int *>(dsc + off_order);
    a.t.stage = reinterpret_cast<const int4 *>(dsc + off_stage);
    a.t.status = reinterpret_cast<int *>(dsc + off_status);
    a.req_bytes = req;
    a.heads = H;
    a.batch = B;
    a.state_bytes = req * (long long)B;
    a.n_items = (int)n;
    a.ls_iters = desc->ls_iters;
    a.kda = kda;
    a.nslots = nslots;
    a.slot_bytes = slot_bytes;
    a.off_q = off_q; a.off_k = off_k; a.off_v = off_v;
    a.off_alpha = off_alpha; a.off_ab = off_ab; a.off_rec = off_rec_slot;
    a.n_pivot_items = n_pivot_items;
    a.max_n16 = max_n16;
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.beta = beta; a.out = out;
    e = stepq::launch_decode_step(a, s);
    return e == cudaSuccess ? STEPQ_OK : cuda_fail(e, "stepq_decode_step_noalloc launch");
}


}  // extern "C"