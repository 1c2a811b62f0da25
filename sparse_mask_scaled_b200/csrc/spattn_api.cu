// C ABI of libspattn: argument checks, the stream-ordered memory pool, mask
// handles and kernel launches. Every numerical step runs in the kernels of
// fwd_gather.cu, fwd_tc.cu, mask_build.cu and plan.cu; this file only validates
// and schedules.
//
// Argument checks run before any CUDA call, so a rejected call touches no
// device state.
#include "spattn.h"
#include "spattn_internal.cuh"
#include "bsg_plan.cuh"

#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

using namespace spattn;

namespace spattn {
namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_allocs{0};

// Every allocation the library makes (stream-ordered pool, device, mapped
// host) goes through these, which count it for spattn_alloc_count().
template <typename T>
cudaError_t lib_malloc_async(T** ptr, size_t bytes, cudaMemPool_t pool, cudaStream_t s) {
    g_allocs.fetch_add(1, std::memory_order_relaxed);
    return cudaMallocFromPoolAsync(reinterpret_cast<void**>(ptr), bytes, pool, s);
}
template <typename T>
cudaError_t lib_malloc(T** ptr, size_t bytes) {
    g_allocs.fetch_add(1, std::memory_order_relaxed);
    return cudaMalloc(reinterpret_cast<void**>(ptr), bytes);
}
cudaError_t lib_host_alloc(void** ptr, size_t bytes, unsigned flags) {
    g_allocs.fetch_add(1, std::memory_order_relaxed);
    return cudaHostAlloc(ptr, bytes, flags);
}
}  // namespace
cudaStream_t counted(cudaStream_t s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return s;
}
}  // namespace spattn

struct spattn_mask_s {
    int device;
    cudaStream_t stream;
    int32_t n;
    int32_t num_masks;
    int64_t nnz;
    int32_t* row_ptr;
    int32_t* col_idx;
    int32_t* long_rows;
    int64_t n_long;
    // tile plan (tensor-core tiles + residual CSR); has_plan = false when no tile qualifies
    bool has_plan;
    int32_t nqb;
    int64_t n_tiles, res_nnz, n_mixed, n_tc_blocks, res_n_long;
    int32_t* block_tile_off;
    int32_t* tile_info;
    uint32_t* tile_bits;
    int32_t* res_row_ptr;
    int32_t* res_col_idx;
    int32_t* res_long;
    // owned pool blocks the arrays above are carved from
    void* block_csr;   // row_ptr, long_rows
    void* block_col;   // col_idx
    void* block_plan;  // block_tile_off, tile_info, tile_bits, res_row_ptr, res_col_idx, res_long
    // query blocks with more than kChunkTiles tiles, split into chunks for the
    // d = 128 tile kernel (see TcParams); block_chunk holds the three arrays
    void* block_chunk;
    int32_t* blk_nch;
    int32_t* blk_slot;
    int2* chunk_extra;
    int32_t n_extra, n_slots;
    // block + strided + global masks with strided entries outside the plan's
    // tiles: those entries as a mask of their own in residue-permuted order
    // (str_mask), the rest as a regular mask (reg_mask); see strided.cu
    spattn_mask str_mask, reg_mask;
    int32_t str_stride;
    // Implicit interval masks (SLIDING, VARWIN, DENSE): per-row runs and the
    // tile map are what the forward pass reads; row_ptr / col_idx and the
    // explicit plan arrays above are written only when asked for.
    bool implicit;
    int kind;
    int32_t window;
    int min_nnz;         // selection threshold, 0 = no tile plan
    int32_t nkt;
    int2* lohi;          // [rows]
    int32_t* tmap;       // [nblocks * nkt]: the block's tile number, or -1
    int32_t* itv_tiles;  // [nblocks * nkt]: block x's tiles at x * nkt ..
    int32_t* itv_ntiles; // [nblocks]
    int32_t* blk_res;    // [nblocks]
    void* block_itv;     // lohi, tmap, itv_tiles, itv_ntiles, blk_res, block statistics
    ItvCounters* cnt_host;  // mapped host memory the build writes its totals to
    ItvCounters* cnt_dev;   // the same memory as the device addresses it
    unsigned* done_dev;     // the slot's block counter
    cudaEvent_t built;      // recorded after the build
    bool counters_valid;    // cnt_host has been read into the fields above
    bool plan_written;      // the explicit plan arrays exist
    bool host_no_residual;  // known from the parameters: every entry lies in a selected tile
    // transpose for the backward column pass (written on the first backward call)
    int32_t* t_row_ptr;
    int32_t* t_col_idx;
    void* block_t;
    // interval masks: the long-row list, written when asked for (its count is n_long)
    void* block_long;
    // Block + strided + global masks in closed form (bsg_plan.cuh): nothing is
    // built on the device; the pattern's parameters are the plan. A CSR-built
    // copy of the same mask (generic) is made on first need: CSR or plan
    // inspection, the backward pass, fp32 inputs, additive terms, key lengths.
    bool closed;
    int32_t bsg_block, bsg_stride, bsg_ng;
    int64_t closed_tiles;  // tensor-core tiles of one forward per (b, h), over the masks
    spattn_mask generic;
};

namespace {

thread_local char g_msg[512] = "";

int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return status;
}

int cuda_fail(cudaError_t e, const char* what) {
    if (e == cudaErrorMemoryAllocation)
        return fail(SPATTN_ERR_OOM, "%s: %s", what, cudaGetErrorString(e));
    return fail(SPATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define CUDA_TRY(call, what)                      \
    do {                                          \
        cudaError_t e_ = (call);                  \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

constexpr int kMaxDevices = 64;
std::mutex g_mu;
cudaMemPool_t g_pool[kMaxDevices];
int g_num_sms[kMaxDevices];

// The library's stream-ordered pool on `dev` (memory is kept cached between
// calls rather than returned to the driver).
cudaError_t device_state(int dev, cudaMemPool_t* pool, int* num_sms) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_pool[dev]) {
        cudaMemPoolProps props;
        memset(&props, 0, sizeof props);
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p;
        cudaError_t e = cudaMemPoolCreate(&p, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = UINT64_MAX;
        e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) return e;
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        g_pool[dev] = p;
        g_num_sms[dev] = sms;
    }
    *pool = g_pool[dev];
    if (num_sms) *num_sms = g_num_sms[dev];
    return cudaSuccess;
}

template <typename T>
cudaError_t pool_alloc(T** ptr, int64_t elems, cudaMemPool_t pool, cudaStream_t s) {
    const size_t bytes = (size_t)(elems > 0 ? elems : 1) * sizeof(T);
    return lib_malloc_async(reinterpret_cast<void**>(ptr), bytes, pool, s);
}

// Mapped host slots for the totals of an interval-mask build, each with an
// event, recycled once the build that last wrote the slot has completed (a
// destroyed mask's build may still be running).
struct HostSlot {
    ItvCounters* host;
    ItvCounters* dev;
    unsigned* done;  // device counter of the build's finished blocks (left at 0)
    cudaEvent_t ev;
};
std::mutex g_slot_mu;
std::vector<HostSlot> g_slot_free[kMaxDevices], g_slot_pending[kMaxDevices];
constexpr int kSlotChunk = 64;

cudaError_t get_slot(int dev, HostSlot* out) {
    std::lock_guard<std::mutex> lk(g_slot_mu);
    std::vector<HostSlot>& pend = g_slot_pending[dev];
    std::vector<HostSlot>& fr = g_slot_free[dev];
    for (size_t x = 0; x < pend.size();) {
        if (cudaEventQuery(pend[x].ev) == cudaSuccess) {
            fr.push_back(pend[x]);
            pend[x] = pend.back();
            pend.pop_back();
        } else {
            ++x;
        }
    }
    (void)cudaGetLastError();  // a not-ready query is not an error of the next call
    if (fr.empty()) {
        void* h = nullptr;
        cudaError_t e = lib_host_alloc(&h, sizeof(ItvCounters) * kSlotChunk,
                                      cudaHostAllocMapped | cudaHostAllocPortable);
        if (e != cudaSuccess) return e;
        void* d = nullptr;
        if ((e = cudaHostGetDevicePointer(&d, h, 0)) != cudaSuccess) return e;
        unsigned* dn = nullptr;
        if ((e = lib_malloc(&dn, sizeof(unsigned) * kSlotChunk)) != cudaSuccess) return e;
        if ((e = cudaMemset(dn, 0, sizeof(unsigned) * kSlotChunk)) != cudaSuccess) return e;
        for (int x = 0; x < kSlotChunk; ++x) {
            HostSlot sl;
            sl.host = static_cast<ItvCounters*>(h) + x;
            sl.dev = static_cast<ItvCounters*>(d) + x;
            sl.done = dn + x;
            if ((e = cudaEventCreateWithFlags(&sl.ev, cudaEventDisableTiming)) != cudaSuccess) return e;
            fr.push_back(sl);
        }
    }
    *out = fr.back();
    fr.pop_back();
    return cudaSuccess;
}

void put_slot(int dev, const HostSlot& sl) {
    std::lock_guard<std::mutex> lk(g_slot_mu);
    g_slot_pending[dev].push_back(sl);
}

int elem_size(int32_t dtype) { return dtype == SPATTN_BF16 ? 2 : 4; }

bool dtype_ok(int32_t dtype) { return dtype == SPATTN_BF16 || dtype == SPATTN_F32; }

// q, k, v and out: [B, H, n, d] with stride 1 over d and 16-byte vector access.
int check_qkv(const spattn_tensor* t, const char* name, const int64_t* shape, int32_t dtype) {
    if (!t) return fail(SPATTN_ERR_INVALID_ARG, "%s is NULL", name);
    if (t->reserved != 0) return fail(SPATTN_ERR_INVALID_ARG, "%s.reserved must be 0", name);
    if (t->dtype != dtype)
        return fail(SPATTN_ERR_INVALID_ARG, "%s dtype %d differs from q's %d", name, t->dtype, dtype);
    for (int x = 0; x < 4; ++x)
        if (t->shape[x] != shape[x])
            return fail(SPATTN_ERR_INVALID_ARG, "%s shape[%d] = %lld, expected %lld", name, x,
                        (long long)t->shape[x], (long long)shape[x]);
    if (!t->data) return fail(SPATTN_ERR_INVALID_ARG, "%s.data is NULL", name);
    if (t->stride[3] != 1) return fail(SPATTN_ERR_UNSUPPORTED, "%s needs stride 1 over d", name);
    const int es = elem_size(dtype);
    if (((uintptr_t)t->data) % 16 != 0)
        return fail(SPATTN_ERR_UNSUPPORTED, "%s.data is not 16-byte aligned", name);
    for (int x = 0; x < 3; ++x) {
        if (t->shape[x] > 1 && ((t->stride[x] * es) % 16 != 0))
            return fail(SPATTN_ERR_UNSUPPORTED, "%s stride[%d] is not a multiple of 16 bytes", name, x);
        if (t->shape[x] > 1 && t->stride[x] < 0)
            return fail(SPATTN_ERR_UNSUPPORTED, "%s stride[%d] is negative", name, x);
    }
    return SPATTN_OK;
}

int check_addend(const spattn_tensor* t, const char* name, const int64_t* full, AddendView* view) {
    memset(view, 0, sizeof *view);
    if (!t) return SPATTN_OK;
    if (t->reserved != 0) return fail(SPATTN_ERR_INVALID_ARG, "%s.reserved must be 0", name);
    if (!dtype_ok(t->dtype)) return fail(SPATTN_ERR_UNSUPPORTED, "%s dtype %d", name, t->dtype);
    if (!t->data) return fail(SPATTN_ERR_INVALID_ARG, "%s.data is NULL", name);
    int64_t st[4];
    for (int x = 0; x < 4; ++x) {
        if (t->shape[x] != 1 && t->shape[x] != full[x])
            return fail(SPATTN_ERR_INVALID_ARG,
                        "%s shape[%d] = %lld does not broadcast to %lld", name, x,
                        (long long)t->shape[x], (long long)full[x]);
        st[x] = t->shape[x] == 1 ? 0 : t->stride[x];
    }
    if (((uintptr_t)t->data) % elem_size(t->dtype) != 0)
        return fail(SPATTN_ERR_INVALID_ARG, "%s.data is not element-aligned", name);
    view->data = t->data;
    view->dtype = t->dtype == SPATTN_BF16 ? 0 : 1;
    view->s0 = st[0];
    view->s1 = st[1];
    view->s2 = st[2];
    view->s3 = st[3];
    return SPATTN_OK;
}

// Shared argument checks of the two forward entry points. Fills everything in
// `p` except the CSR and the schedule.
int check_fwd(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
              const spattn_tensor* add_mask, const spattn_tensor* bias, float scale,
              const spattn_tensor* out, float* lse, FwdParams* p, int* dtype, int* d) {
    if (!q) return fail(SPATTN_ERR_INVALID_ARG, "q is NULL");
    if (!dtype_ok(q->dtype)) return fail(SPATTN_ERR_UNSUPPORTED, "q dtype %d", q->dtype);
    for (int x = 0; x < 4; ++x)
        if (q->shape[x] < 0) return fail(SPATTN_ERR_INVALID_ARG, "q shape[%d] < 0", x);
    const int64_t B = q->shape[0], H = q->shape[1], n = q->shape[2], D = q->shape[3];
    if (D != 32 && D != 64 && D != 128)
        return fail(SPATTN_ERR_UNSUPPORTED, "head dim %lld (supported: 32, 64, 128)", (long long)D);
    if (B > 0x7fffffff || H > 0x7fffffff || n > 0x7ffffffe || B * H > 0x7fffffff)
        return fail(SPATTN_ERR_UNSUPPORTED, "B, H or n too large");
    int r;
    if ((r = check_qkv(q, "q", q->shape, q->dtype))) return r;
    if ((r = check_qkv(k, "k", q->shape, q->dtype))) return r;
    if ((r = check_qkv(v, "v", q->shape, q->dtype))) return r;
    if ((r = check_qkv(out, "out", q->shape, q->dtype))) return r;
    if (lse && ((uintptr_t)lse) % 4 != 0) return fail(SPATTN_ERR_INVALID_ARG, "lse not aligned");
    if (!(scale == scale)) return fail(SPATTN_ERR_INVALID_ARG, "scale is NaN");
    const int64_t full[4] = {B, H, n, n};
    memset(p, 0, sizeof *p);
    if ((r = check_addend(add_mask, "add_mask", full, &p->mask))) return r;
    if ((r = check_addend(bias, "bias", full, &p->bias))) return r;
    auto bs = [](const spattn_tensor* t, int x) { return t->shape[x] == 1 ? 0 : t->stride[x]; };
    p->q = q->data;
    p->k = k->data;
    p->v = v->data;
    p->out = out->data;
    p->lse = lse;
    p->q_sb = bs(q, 0); p->q_sh = bs(q, 1); p->q_sn = bs(q, 2);
    p->k_sb = bs(k, 0); p->k_sh = bs(k, 1); p->k_sn = bs(k, 2);
    p->v_sb = bs(v, 0); p->v_sh = bs(v, 1); p->v_sn = bs(v, 2);
    p->o_sb = bs(out, 0); p->o_sh = bs(out, 1); p->o_sn = bs(out, 2);
    p->B = (int)B;
    p->H = (int)H;
    p->n = (int)n;
    p->has_extra = (p->mask.data || p->bias.data) ? 1 : 0;
    p->qk_scale_log2 = scale * kLog2e;
    *dtype = q->dtype == SPATTN_BF16 ? 0 : 1;
    *d = (int)D;
    return SPATTN_OK;
}

int launch_fwd(FwdParams& p, int dtype, int d, int num_sms, cudaStream_t s) {
    cudaError_t e = launch_fwd_long_rows(p, dtype, d, num_sms, s);
    if (e != cudaSuccess) return cuda_fail(e, "long-row kernel launch");
    e = launch_fwd_short_rows(p, dtype, d, s);
    if (e != cudaSuccess) return cuda_fail(e, "row kernel launch");
    return SPATTN_OK;
}

void free_plan(spattn_mask m) {
    if (m->block_plan) cudaFreeAsync(m->block_plan, m->stream);
    if (m->block_chunk) cudaFreeAsync(m->block_chunk, m->stream);
    m->block_plan = m->block_chunk = nullptr;
    m->blk_nch = m->blk_slot = nullptr;
    m->chunk_extra = nullptr;
    m->n_extra = m->n_slots = 0;
    m->block_tile_off = m->tile_info = m->res_row_ptr = m->res_col_idx = m->res_long = nullptr;
    m->tile_bits = nullptr;
    m->has_plan = false;
}

// Lays out arrays in one pool allocation (each start 256-byte aligned).
struct Carve {
    size_t off[16];
    size_t total = 0;
    int n = 0;
    int add(size_t bytes) {
        off[n] = total;
        total += (bytes + 255) & ~size_t(255);
        return n++;
    }
    template <typename T>
    T* at(void* base, int k) const {
        return reinterpret_cast<T*>(static_cast<char*>(base) + off[k]);
    }
};

unsigned* g_err_ptr[kMaxDevices];


int build_status(unsigned err) {
    if (err & (kBuildTooMany | kBuildRowTooLong)) {
        return fail(SPATTN_ERR_UNSUPPORTED, "%s",
                    (err & kBuildTooMany) ? "more than 2^31-1 nonzeros"
                                          : "a COO row has more than 1024 candidates and n > 1572864");
    }
    if (err & kBuildNegativeWidth) return fail(SPATTN_ERR_BAD_CSR, "negative half-width");
    if (err & kBuildBadRowPtr) return fail(SPATTN_ERR_BAD_CSR, "row_ptr is not a valid prefix sum");
    if (err & kBuildBadColumn) return fail(SPATTN_ERR_BAD_CSR, "a column index is outside [0, n)");
    if (err & kBuildUnsorted) return fail(SPATTN_ERR_BAD_CSR, "a CSR row is not strictly increasing");
    return SPATTN_OK;
}

// Device address of the device error flags, looked up once per device.
int err_flags_ptr(int dev, unsigned** out) {
    if (!g_err_ptr[dev]) {
        unsigned* ep = nullptr;
        CUDA_TRY(error_flag_address(&ep), "error flag address");
        g_err_ptr[dev] = ep;
    }
    *out = g_err_ptr[dev];
    return SPATTN_OK;
}

// ---------------------------------------------------------- interval masks

bool implicit_kind(int kind) {
    return kind == SPATTN_MASK_SLIDING || kind == SPATTN_MASK_VARWIN || kind == SPATTN_MASK_DENSE;
}

// Whether every entry of a SLIDING or DENSE mask lies in a tile of at least
// min_nnz entries -- then the forward pass needs no gather kernel. Exact (the
// build's tile counts, from the parameters); false when unknown or when
// telling would cost more than a few million steps.
bool interval_all_in_tiles(int kind, int64_t n, int64_t w, int min_nnz) {
    if (min_nnz <= 0) return false;
    const int64_t nqb = (n + kTileM - 1) / kTileM;
    if (kind == SPATTN_MASK_DENSE) {
        const int64_t last = n - kTileM * (nqb - 1);  // rows and keys of the ragged last tiles
        return last * last >= min_nnz;
    }
    if (kind != SPATTN_MASK_SLIDING) return false;
    const int64_t nkt = (n + kTileN - 1) / kTileN;
    const int64_t span = std::min<int64_t>(nkt, (2 * w) / kTileN + 3);
    if (nqb * span * kTileM > (int64_t(1) << 22)) return false;
    for (int64_t qb = 0; qb < nqb; ++qb) {
        const int64_t i0 = qb * kTileM, i1 = std::min<int64_t>(n, i0 + kTileM);
        const int64_t lo_min = std::max<int64_t>(0, i0 - w), hi_max = std::min<int64_t>(n, i1 + w);
        for (int64_t kt = lo_min / kTileN; kt <= (hi_max - 1) / kTileN; ++kt) {
            int64_t c = 0;
            for (int64_t i = i0; i < i1; ++i) {
                const int64_t lo = std::max<int64_t>(0, i - w), hi = std::min<int64_t>(n, i + w + 1);
                c += std::max<int64_t>(0, std::min<int64_t>(hi, kt * kTileN + kTileN) -
                                              std::max<int64_t>(lo, kt * kTileN));
            }
            if (c > 0 && c < min_nnz) return false;
        }
    }
    return true;
}

// The build's totals into the mask's fields. wait: block until the build has
// run; else only read them if it already has (*ready tells which).
int read_counters(spattn_mask m, bool wait, bool* ready = nullptr) {
    if (ready) *ready = true;
    if (!m->implicit || m->counters_valid) return SPATTN_OK;
    if (wait) {
        CUDA_TRY(cudaEventSynchronize(m->built), "waiting for the mask build");
    } else {
        const cudaError_t q = cudaEventQuery(m->built);
        if (q == cudaErrorNotReady) {
            (void)cudaGetLastError();
            if (ready) *ready = false;
            return SPATTN_OK;
        }
        if (q != cudaSuccess) return cuda_fail(q, "mask build");
    }
    const volatile ItvCounters* c = m->cnt_host;
    m->nnz = c->nnz;
    m->n_long = c->n_long;
    m->n_tiles = c->n_tiles;
    m->res_nnz = c->res_nnz;
    m->n_tc_blocks = c->n_tc_blocks;
    m->counters_valid = true;
    return SPATTN_OK;
}

int create_implicit(const spattn_mask_spec& sp, cudaStream_t s, int dev, cudaMemPool_t pool,
                    spattn_mask* out) {
    const bool async = (sp.flags & SPATTN_MASK_ASYNC) != 0;
    const int64_t rows = (int64_t)sp.n * sp.num_masks;
    const int nqb = (sp.n + kTileM - 1) / kTileM, nkt = (sp.n + kTileN - 1) / kTileN;
    const int64_t nblocks = (int64_t)sp.num_masks * nqb;
    const int min_nnz =
        sp.tile_min_nnz < 0 ? 0 : (sp.tile_min_nnz == 0 ? kTileMinNnzDefault : sp.tile_min_nnz);
    unsigned* ef = nullptr;
    if (async) {
        const int r = err_flags_ptr(dev, &ef);
        if (r) return r;
    }
    Carve c;
    const int k_lh = c.add(rows * 8), k_tm = c.add(nblocks * nkt * 4), k_ti = c.add(nblocks * nkt * 4),
              k_nt = c.add(nblocks * 4), k_br = c.add(nblocks * 4), k_bs = c.add(nblocks * sizeof(ItvBlockStat));
    void* blk = nullptr;
    CUDA_TRY(lib_malloc_async(&blk, c.total, pool, s), "mask allocation");
    HostSlot sl;
    cudaError_t e = get_slot(dev, &sl);
    if (e != cudaSuccess) {
        cudaFreeAsync(blk, s);
        return cuda_fail(e, "mapped host memory for the mask totals");
    }
    ItvSpec is;
    is.kind = sp.kind;
    is.n = sp.n;
    is.num_masks = sp.num_masks;
    is.window = sp.window;
    is.half_widths = sp.half_widths;
    is.nqb = nqb;
    is.nkt = nkt;
    is.err_flags = ef;
    e = itv_build(is, c.at<int2>(blk, k_lh), c.at<int32_t>(blk, k_tm), c.at<int32_t>(blk, k_ti),
                  c.at<int32_t>(blk, k_nt), c.at<int32_t>(blk, k_br), c.at<ItvBlockStat>(blk, k_bs), min_nnz,
                  sl.done, sl.dev, s);
    if (e == cudaSuccess) e = cudaEventRecord(sl.ev, s);
    if (e != cudaSuccess) {
        cudaFreeAsync(blk, s);
        put_slot(dev, sl);
        return cuda_fail(e, "interval mask build");
    }
    spattn_mask m = new spattn_mask_s;
    memset(m, 0, sizeof *m);
    m->device = dev;
    m->stream = s;
    m->n = sp.n;
    m->num_masks = sp.num_masks;
    m->implicit = true;
    m->kind = sp.kind;
    m->window = sp.window;
    m->min_nnz = min_nnz;
    m->nqb = nqb;
    m->nkt = nkt;
    m->lohi = c.at<int2>(blk, k_lh);
    m->tmap = c.at<int32_t>(blk, k_tm);
    m->itv_tiles = c.at<int32_t>(blk, k_ti);
    m->itv_ntiles = c.at<int32_t>(blk, k_nt);
    m->blk_res = c.at<int32_t>(blk, k_br);
    m->block_itv = blk;
    m->cnt_host = sl.host;
    m->cnt_dev = sl.dev;
    m->done_dev = sl.done;
    m->built = sl.ev;
    m->has_plan = min_nnz > 0;
    m->host_no_residual = interval_all_in_tiles(sp.kind, sp.n, sp.window, min_nnz);
    if (!async) {
        int r = read_counters(m, true);
        const unsigned err = static_cast<const volatile ItvCounters*>(m->cnt_host)->err;
        if (r == SPATTN_OK && err) r = build_status(err);
        if (r != SPATTN_OK) {
            spattn_destroy_mask(m);
            return r;
        }
    }
    *out = m;
    return SPATTN_OK;
}

// row_ptr and col_idx of an interval mask, written on first request.
int write_csr(spattn_mask m) {
    if (!m->implicit || m->row_ptr) return SPATTN_OK;
    int r = read_counters(m, true);
    if (r) return r;
    if (m->nnz > 0x7fffffffLL)
        return fail(SPATTN_ERR_UNSUPPORTED, "the mask has more than 2^31 - 1 nonzeros for a CSR");
    const int64_t rows = (int64_t)m->n * m->num_masks;
    cudaMemPool_t pool;
    CUDA_TRY(device_state(m->device, &pool, nullptr), "memory pool");
    cudaStream_t s = m->stream;
    Carve ct;
    const int k_cnt = ct.add(rows * 4), k_scan = ct.add(scan_tmp_elems(rows) * 8), k_tot = ct.add(16);
    void *a = nullptr, *t = nullptr, *col = nullptr;
    cudaError_t e = lib_malloc_async(&a, (size_t)(rows + 1) * 4, pool, s);
    if (e == cudaSuccess) e = lib_malloc_async(&t, ct.total, pool, s);
    if (e == cudaSuccess) e = lib_malloc_async(&col, (size_t)(m->nnz > 0 ? m->nnz : 1) * 4, pool, s);
    if (e == cudaSuccess) {
        int64_t* tot = ct.at<int64_t>(t, k_tot);
        e = itv_write_csr(m->lohi, rows, ct.at<int32_t>(t, k_cnt), static_cast<int32_t*>(a),
                          static_cast<int32_t*>(col), ct.at<int64_t>(t, k_scan), tot,
                          reinterpret_cast<unsigned*>(tot + 1), s);
    }
    if (t) cudaFreeAsync(t, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        if (a) cudaFreeAsync(a, s);
        if (col) cudaFreeAsync(col, s);
        return cuda_fail(e, "writing the mask's CSR");
    }
    m->block_csr = a;
    m->block_col = col;
    m->row_ptr = static_cast<int32_t*>(a);
    m->col_idx = static_cast<int32_t*>(col);
    return SPATTN_OK;
}

// The explicit plan arrays of an interval mask (tile bits, residual CSR) and
// its mixed-row count, written on first request.
int write_plan(spattn_mask m) {
    if (!m->implicit || m->plan_written) return SPATTN_OK;
    int r = read_counters(m, true);
    if (r) return r;
    if (m->n_tiles == 0) {
        m->plan_written = true;
        return SPATTN_OK;
    }
    const int64_t rows = (int64_t)m->n * m->num_masks;
    cudaMemPool_t pool;
    CUDA_TRY(device_state(m->device, &pool, nullptr), "memory pool");
    cudaStream_t s = m->stream;
    const int64_t nblocks = (int64_t)m->num_masks * m->nqb;
    Carve cp;
    const int k_bto = cp.add((nblocks + 1) * 4), k_ti = cp.add(m->n_tiles * 4),
              k_tb = cp.add(m->n_tiles * kTileM * 16), k_rrp = cp.add((rows + 1) * 4),
              k_rci = cp.add(m->res_nnz * 4), k_rl = cp.add(rows * 4);
    Carve ct;
    const int64_t scan_rows = rows > nblocks ? rows : nblocks;
    const int k_pc = ct.add(sizeof(PlanCounters)), k_rc = ct.add(rows * 4),
              k_st = ct.add(scan_tmp_elems(scan_rows) * 8);
    void *a = nullptr, *t = nullptr;
    PlanCounters hpc;
    cudaError_t e = lib_malloc_async(&a, cp.total, pool, s);
    if (e == cudaSuccess) e = lib_malloc_async(&t, ct.total, pool, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ct.at<PlanCounters>(t, k_pc), 0, sizeof(PlanCounters), s);
    if (e == cudaSuccess) {
        PlanBuffers pb;
        memset(&pb, 0, sizeof pb);
        pb.cnt_map = m->tmap;
        pb.block_tile_off = cp.at<int32_t>(a, k_bto);
        pb.tile_info = cp.at<int32_t>(a, k_ti);
        pb.tile_cap = m->n_tiles;
        pb.tile_bits = cp.at<uint32_t>(a, k_tb);
        pb.res_row_ptr = cp.at<int32_t>(a, k_rrp);
        pb.res_col_idx = cp.at<int32_t>(a, k_rci);
        pb.res_long = cp.at<int32_t>(a, k_rl);
        pb.res_cnt = ct.at<int32_t>(t, k_rc);
        pb.scan_tmp = ct.at<int64_t>(t, k_st);
        e = itv_write_plan(m->lohi, m->n, m->num_masks, m->itv_tiles, m->itv_ntiles, pb,
                           ct.at<PlanCounters>(t, k_pc), s);
    }
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&hpc, ct.at<PlanCounters>(t, k_pc), sizeof hpc, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (t) cudaFreeAsync(t, s);
    if (e != cudaSuccess) {
        if (a) cudaFreeAsync(a, s);
        return cuda_fail(e, "writing the mask's tile plan");
    }
    m->block_plan = a;
    m->block_tile_off = cp.at<int32_t>(a, k_bto);
    m->tile_info = cp.at<int32_t>(a, k_ti);
    m->tile_bits = cp.at<uint32_t>(a, k_tb);
    m->res_row_ptr = cp.at<int32_t>(a, k_rrp);
    m->res_col_idx = cp.at<int32_t>(a, k_rci);
    m->res_long = cp.at<int32_t>(a, k_rl);
    m->n_mixed = hpc.n_mixed;
    m->res_n_long = hpc.res_n_long;
    m->plan_written = true;
    return SPATTN_OK;
}


// Splits the query blocks of a CSR mask's tile plan that have more than
// kChunkTiles tiles into chunks of that many, so that one long block (rows
// that attend to every key, say) does not serialise the d = 128 tile kernel:
// per block its chunk count and first partial-state slot, and the list of
// (block, chunk >= 1) the extra thread blocks take. Synchronises the mask's
// stream (it runs right after the plan is built, which already does).
int write_chunks(spattn_mask m, cudaMemPool_t pool) {
    const int64_t nblocks = (int64_t)m->num_masks * m->nqb;
    std::vector<int32_t> off((size_t)nblocks + 1);
    cudaStream_t s = m->stream;
    CUDA_TRY(cudaMemcpyAsync(off.data(), m->block_tile_off, off.size() * 4, cudaMemcpyDeviceToHost, s),
             "plan read-back");
    CUDA_TRY(cudaStreamSynchronize(s), "plan read-back");
    std::vector<int32_t> nch((size_t)nblocks, 1), slot((size_t)nblocks, -1), extra;
    int64_t n_slots = 0;
    for (int64_t x = 0; x < nblocks; ++x) {
        const int64_t T = off[x + 1] - off[x];
        if (T <= kChunkTiles) continue;
        nch[x] = (int32_t)((T + kChunkTiles - 1) / kChunkTiles);
        slot[x] = (int32_t)n_slots;
        n_slots += nch[x];
        for (int32_t c = 1; c < nch[x]; ++c) {
            extra.push_back((int32_t)x);
            extra.push_back(c);
        }
    }
    if (n_slots == 0) return SPATTN_OK;
    Carve cp;
    const int k_n = cp.add(nblocks * 4), k_s = cp.add(nblocks * 4), k_e = cp.add(extra.size() * 4);
    void* a = nullptr;
    CUDA_TRY(lib_malloc_async(&a, cp.total, pool, s), "chunk plan allocation");
    cudaError_t e = cudaMemcpyAsync(cp.at<int32_t>(a, k_n), nch.data(), nblocks * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(cp.at<int32_t>(a, k_s), slot.data(), nblocks * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(cp.at<int32_t>(a, k_e), extra.data(), extra.size() * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // the host vectors go out of scope
    if (e != cudaSuccess) {
        cudaFreeAsync(a, s);
        return cuda_fail(e, "chunk plan upload");
    }
    m->block_chunk = a;
    m->blk_nch = cp.at<int32_t>(a, k_n);
    m->blk_slot = cp.at<int32_t>(a, k_s);
    m->chunk_extra = cp.at<int2>(a, k_e);
    m->n_extra = (int32_t)(extra.size() / 2);
    m->n_slots = (int32_t)n_slots;
    return SPATTN_OK;
}

// Moves the strided entries (j = i mod S) that a block + strided + global
// mask's tile plan leaves to the gather kernel into a mask of their own in
// residue-permuted order, whose plan covers them with dense tiles, and keeps
// the rest as a regular mask (both built like user CSR masks, with the same
// tile threshold). Synchronises the mask's stream.
int write_strided(spattn_mask m, int S, int32_t tile_min_nnz, cudaMemPool_t pool) {
    cudaStream_t s = m->stream;
    const int n = m->n;
    const int64_t rows = (int64_t)m->num_masks * n;
    const int nkt = (n + kTileN - 1) / kTileN;
    const int64_t nblocks = (int64_t)m->num_masks * m->nqb;
    Carve ct;
    const int k_cp = ct.add(rows * 4), k_cr = ct.add(rows * 4), k_cg = ct.add(rows * 4),
              k_sp = ct.add((rows + 1) * 4), k_gp = ct.add((rows + 1) * 4), k_sel = ct.add(nblocks * nkt),
              k_st = ct.add(scan_tmp_elems(rows) * 8), k_tot = ct.add(2 * 8), k_err = ct.add(4);
    void* t = nullptr;
    CUDA_TRY(lib_malloc_async(&t, ct.total, pool, s), "strided split scratch");
    int32_t *cnt_perm = ct.at<int32_t>(t, k_cp), *cnt_row = ct.at<int32_t>(t, k_cr),
            *cnt_reg = ct.at<int32_t>(t, k_cg), *srp = ct.at<int32_t>(t, k_sp), *grp = ct.at<int32_t>(t, k_gp);
    int64_t* tot = ct.at<int64_t>(t, k_tot);
    unsigned* err = ct.at<unsigned>(t, k_err);
    int64_t htot[2] = {0, 0};
    int32_t *sci = nullptr, *gci = nullptr;
    cudaError_t e = cudaMemsetAsync(err, 0, 4, s);
    if (e == cudaSuccess)
        e = strided_split_count(m->res_row_ptr, m->res_col_idx, rows, n, S, cnt_perm, cnt_row, s);
    if (e == cudaSuccess) e = scan_counts(cnt_perm, rows, srp, ct.at<int64_t>(t, k_st), tot, err, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&htot[0], tot, 8, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && htot[0] > 0) {
        e = lib_malloc_async(&sci, (size_t)htot[0] * 4, pool, s);
        if (e == cudaSuccess)
            e = strided_split_fill(m->res_row_ptr, m->res_col_idx, m->row_ptr, m->col_idx, m->block_tile_off,
                                   m->tile_info, rows, n, S, m->nqb, nkt, nblocks, cnt_row, cnt_reg,
                                   ct.at<uint8_t>(t, k_sel), srp, sci, s);
        if (e == cudaSuccess) e = scan_counts(cnt_reg, rows, grp, ct.at<int64_t>(t, k_st), tot + 1, err, s);
        if (e == cudaSuccess) e = cudaMemcpyAsync(&htot[1], tot + 1, 8, cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e == cudaSuccess) e = lib_malloc_async(&gci, (size_t)(htot[1] > 0 ? htot[1] : 1) * 4, pool, s);
        if (e == cudaSuccess)
            e = strided_reg_fill(m->row_ptr, m->col_idx, rows, n, S, m->nqb, nkt, ct.at<uint8_t>(t, k_sel), grp,
                                 gci, err, s);
    }
    int r = SPATTN_OK;
    if (e != cudaSuccess) {
        r = cuda_fail(e, "strided split");
    } else if (htot[0] > 0) {
        spattn_mask_spec sp;
        memset(&sp, 0, sizeof sp);
        sp.kind = SPATTN_MASK_CSR;
        sp.n = n;
        sp.num_masks = m->num_masks;
        sp.tile_min_nnz = tile_min_nnz;
        sp.in_row_ptr = srp;
        sp.in_col_idx = sci;
        sp.in_nnz = htot[0];
        r = spattn_create_csr_mask(&sp, s, &m->str_mask);
        if (!r) {
            sp.in_row_ptr = grp;
            sp.in_col_idx = gci;
            sp.in_nnz = htot[1];
            r = spattn_create_csr_mask(&sp, s, &m->reg_mask);
        }
        if (!r) {  // every row of the regular part must come out at the length its scan allotted
            unsigned herr = 0;
            cudaError_t e2 = cudaMemcpyAsync(&herr, err, 4, cudaMemcpyDeviceToHost, s);
            if (e2 == cudaSuccess) e2 = cudaStreamSynchronize(s);
            if (e2 != cudaSuccess) r = cuda_fail(e2, "strided split check");
            else if (herr & kBuildBadRowPtr) r = fail(SPATTN_ERR_BAD_CSR, "strided split: row lengths disagree");
            if (r) {
                spattn_destroy_mask(m->str_mask);
                spattn_destroy_mask(m->reg_mask);
                m->str_mask = m->reg_mask = nullptr;
            }
        }
        if (!r && !(m->str_mask->has_plan && m->reg_mask->has_plan)) {  // nothing to gain: keep the mask as is
            spattn_destroy_mask(m->str_mask);
            spattn_destroy_mask(m->reg_mask);
            m->str_mask = m->reg_mask = nullptr;
        }
        if (!r && m->str_mask) m->str_stride = S;
    }
    if (sci) cudaFreeAsync(sci, s);
    if (gci) cudaFreeAsync(gci, s);
    cudaFreeAsync(t, s);
    return r;
}

// The tensor-core kernel over a mask's tiles (below); perm_G: see TcParams.
int launch_tc(const FwdParams& p, int d, spattn_mask m, int dev, const int32_t* blk_res, cudaStream_t s,
              int perm_G = 0);

// Forward over a mask split by write_strided: the permuted part, then the
// regular part over Q, K, V as they are, then each row merged through the two
// log-sum-exps. For d = 128 with n/S a multiple of 128 and every permuted entry
// in a tile, the tile kernel reads the permuted rows of Q, K and V in place
// (five-dimensional maps, stride S); otherwise they are copied in permuted
// order first.
int fwd_strided(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v, spattn_mask m,
                float scale, const spattn_tensor* out, float* lse, cudaStream_t s, const FwdParams& p, int d,
                cudaMemPool_t pool, int dev) {
    const int B = p.B, H = p.H, n = p.n, S = m->str_stride, G = n / S;
    const int64_t rows = (int64_t)B * H * n, elems = rows * d;
    const spattn_mask sm = m->str_mask;
    const bool in_place = d == 128 && G % kTileM == 0 && sm->has_plan && sm->res_nnz == 0 && sm->n_tiles > 0;
    Carve c;
    const int k_o = c.add(elems * 2), k_l2 = c.add(rows * 4), k_l1 = c.add(rows * 4),
              k_q = c.add(in_place ? 0 : elems * 2), k_k = c.add(in_place ? 0 : elems * 2),
              k_v = c.add(in_place ? 0 : elems * 2);
    void* t = nullptr;
    CUDA_TRY(lib_malloc_async(&t, c.total, pool, s), "strided forward scratch");
    auto tensor = [&](int key) {  // contiguous [B, H, n, d] bf16 scratch
        spattn_tensor x;
        memset(&x, 0, sizeof x);
        x.data = c.at<uint8_t>(t, key);
        x.dtype = SPATTN_BF16;
        x.shape[0] = B;
        x.shape[1] = H;
        x.shape[2] = n;
        x.shape[3] = d;
        x.stride[0] = (int64_t)H * n * d;
        x.stride[1] = (int64_t)n * d;
        x.stride[2] = d;
        x.stride[3] = 1;
        return x;
    };
    const spattn_tensor to = tensor(k_o);
    float* l2 = c.at<float>(t, k_l2);
    // the regular part's lse always goes to scratch: the merge reads it and
    // writes the caller's lse, and the two must not alias
    float* l1 = c.at<float>(t, k_l1);
    int r = SPATTN_OK;
    if (in_place) {
        FwdParams p2 = p;
        p2.out = to.data;
        p2.o_sb = to.stride[0];
        p2.o_sh = to.stride[1];
        p2.o_sn = to.stride[2];
        p2.lse = l2;
        p2.ws_ml = p2.ws_acc = nullptr;
        r = launch_tc(p2, d, sm, dev, nullptr, s, G);
    } else {
        const spattn_tensor tq = tensor(k_q), tk = tensor(k_k), tv = tensor(k_v);
        cudaError_t e = strided_permute_rows(p.q, p.q_sb, p.q_sh, p.q_sn, tq.data, B, H, n, d, S, s);
        if (e == cudaSuccess) e = strided_permute_rows(p.k, p.k_sb, p.k_sh, p.k_sn, tk.data, B, H, n, d, S, s);
        if (e == cudaSuccess) e = strided_permute_rows(p.v, p.v_sb, p.v_sh, p.v_sn, tv.data, B, H, n, d, S, s);
        r = e == cudaSuccess ? SPATTN_OK : cuda_fail(e, "strided forward (permute)");
        if (!r) r = spattn_fwd_mask(&tq, &tk, &tv, sm, nullptr, nullptr, scale, &to, l2, s);
    }
    if (!r) r = spattn_fwd_mask(q, k, v, m->reg_mask, nullptr, nullptr, scale, out, l1, s);
    if (!r) {
        const cudaError_t e = strided_merge(p.out, p.o_sb, p.o_sh, p.o_sn, l1, to.data, l2, lse, B, H, n, d, S, s);
        if (e != cudaSuccess) r = cuda_fail(e, "strided forward (merge)");
    }
    cudaFreeAsync(t, s);
    return r;
}

// The tensor-core kernel over the mask's tiles; blk_res: interval masks whose
// gather kernel ran (its partial states are in p.ws_ml / p.ws_acc).
int launch_tc(const FwdParams& p, int d, spattn_mask m, int dev, const int32_t* blk_res,
              cudaStream_t s, int perm_G) {
    unsigned* ef = nullptr;
    int r = err_flags_ptr(dev, &ef);
    if (r) return r;
    TcParams tp;
    memset(&tp, 0, sizeof tp);
    tp.B = p.B;
    tp.H = p.H;
    tp.n = p.n;
    tp.num_masks = m->num_masks;
    tp.nqb = m->nqb;
    tp.block_tile_off = m->block_tile_off;
    tp.tile_info = m->tile_info;
    if (m->implicit) {
        tp.itv_lohi = m->lohi;
        tp.blk_res = blk_res;
        tp.tile_info = m->itv_tiles;
        tp.block_ntiles = m->itv_ntiles;
        tp.tile_stride = m->nkt;
    } else {
        tp.tile_bits = m->tile_bits;
        tp.res_row_ptr = m->res_row_ptr;
    }
    tp.ws_ml = p.ws_ml;
    tp.ws_acc = p.ws_acc;
    tp.out = p.out;
    tp.o_sb = p.o_sb;
    tp.o_sh = p.o_sh;
    tp.o_sn = p.o_sn;
    tp.lse = p.lse;
    tp.mask = p.mask;
    tp.bias = p.bias;
    tp.has_extra = p.has_extra;
    tp.qk_scale_log2 = p.qk_scale_log2;
    tp.seqlen_k = p.seqlen_k;
    tp.err = ef;
    tp.perm_G = perm_G;
    void* cws = nullptr;  // partial states and arrival counts of split query blocks
    if (d == 128 && !m->implicit && m->blk_nch) {
        cudaMemPool_t pool;
        CUDA_TRY(device_state(dev, &pool, nullptr), "memory pool");
        const int64_t bh = (int64_t)p.B * p.H, nblocks = (int64_t)m->num_masks * m->nqb;
        Carve cp;
        const int k_w = cp.add((size_t)bh * m->n_slots * (d + 2) * kTileM * 4), k_c = cp.add(bh * nblocks * 4);
        CUDA_TRY(lib_malloc_async(&cws, cp.total, pool, s), "chunk workspace");
        cudaError_t e = cudaMemsetAsync(cp.at<unsigned>(cws, k_c), 0, bh * nblocks * 4, s);
        if (e != cudaSuccess) {
            cudaFreeAsync(cws, s);
            return cuda_fail(e, "chunk workspace");
        }
        tp.blk_nch = m->blk_nch;
        tp.blk_slot = m->blk_slot;
        tp.chunk_extra = m->chunk_extra;
        tp.n_extra = m->n_extra;
        tp.n_slots = m->n_slots;
        tp.chunk_tiles = kChunkTiles;
        tp.cws = cp.at<float>(cws, k_w);
        tp.ccnt = cp.at<unsigned>(cws, k_c);
    }
    const TcOperand oq{p.q, p.q_sn, p.q_sh, p.q_sb}, ok{p.k, p.k_sn, p.k_sh, p.k_sb},
        ov{p.v, p.v_sn, p.v_sh, p.v_sb};
    const cudaError_t e = launch_fwd_tc(oq, ok, ov, d, tp, s);
    if (cws) cudaFreeAsync(cws, s);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core kernel launch");
    return SPATTN_OK;
}

// Limit of every wait in the persistent tile kernel, in SM cycles: about one
// second, unless SPATTN_DEBUG_WAIT_CYCLES gives another (tests use a tiny one
// to make the waits expire and check the error path).
long long pp_wait_cycles() {
    const char* e = getenv("SPATTN_DEBUG_WAIT_CYCLES");
    if (e && *e) {
        const long long v = atoll(e);
        if (v >= 0) return v;
    }
    return 2000000000LL;
}

void pp_common(PpParams& pp, const FwdParams& p, unsigned* ef) {
    pp.B = p.B;
    pp.H = p.H;
    pp.n = p.n;
    pp.nqb = (p.n + kTileM - 1) / kTileM;
    pp.nkt = (p.n + kTileN - 1) / kTileN;
    pp.out = p.out;
    pp.o_sb = p.o_sb;
    pp.o_sh = p.o_sh;
    pp.o_sn = p.o_sn;
    pp.lse = p.lse;
    pp.qk_scale_log2 = p.qk_scale_log2;
    pp.err = ef;
    pp.wait_cycles = pp_wait_cycles();
    pp.chunk_tiles = kChunkTiles;
}

// Forward over a block + strided + global mask in closed form: one launch of
// the persistent tile kernel over the regular and the residue-permuted blocks.
// Per call it takes the partial states of split blocks and of rows met by both
// kinds of block from the pool, and clears their counts.
int fwd_closed(const FwdParams& p, int d, spattn_mask m, cudaStream_t s, cudaMemPool_t pool, int dev, int sms) {
    unsigned* ef = nullptr;
    int r = err_flags_ptr(dev, &ef);
    if (r) return r;
    const bsg::Shape sh = bsg::shape(p.n, m->bsg_block, m->bsg_stride, m->bsg_ng, kChunkTiles);
    const int64_t bh = (int64_t)p.B * p.H, rows = bh * p.n;
    const bool chunks = sh.nch > 1, partner = sh.G > 0;
    // counts: claim counter (8 bytes), chunk counts [bh][4], permuted-block
    // arrival counts [bh][npqb][128]
    const size_t n_pflag = partner ? (size_t)bh * sh.npqb * 128 : 0,
                 cnt_bytes = 8 + (size_t)bh * 4 * 4 + n_pflag * 4;
    Carve c;
    const int k_cws = c.add(chunks ? (size_t)bh * sh.nch * (d + 2) * kTileM * 4 : 0),
              k_pml = c.add(partner ? (size_t)rows * 2 * 4 : 0), k_pacc = c.add(partner ? (size_t)rows * d * 4 : 0),
              k_cnt = c.add(cnt_bytes);
    void* ws = nullptr;
    CUDA_TRY(lib_malloc_async(&ws, c.total, pool, s), "tile-kernel workspace");
    cudaError_t e = cudaMemsetAsync(c.at<uint8_t>(ws, k_cnt), 0, cnt_bytes, s);
    if (e == cudaSuccess) {
        PpParams pp;
        memset(&pp, 0, sizeof pp);
        pp_common(pp, p, ef);
        pp.num_masks = m->num_masks;
        pp.mode = 1;
        pp.n_items = bh * sh.items_per_head;
        pp.blk = m->bsg_block;
        pp.S = m->bsg_stride;
        pp.ng = m->bsg_ng;
        uint8_t* cnt = c.at<uint8_t>(ws, k_cnt);
        pp.claim = reinterpret_cast<unsigned long long*>(cnt);
        pp.ccnt = reinterpret_cast<unsigned*>(cnt + 8);
        pp.pflag = partner ? reinterpret_cast<unsigned*>(cnt + 8) + bh * 4 : nullptr;
        pp.cws = chunks ? c.at<float>(ws, k_cws) : nullptr;
        pp.pml = partner ? c.at<float>(ws, k_pml) : nullptr;
        pp.pacc = partner ? c.at<float>(ws, k_pacc) : nullptr;
        const TcOperand oq{p.q, p.q_sn, p.q_sh, p.q_sb}, ok{p.k, p.k_sn, p.k_sh, p.k_sb},
            ov{p.v, p.v_sn, p.v_sh, p.v_sb};
        AddendView none;
        memset(&none, 0, sizeof none);
        e = launch_fwd_pp(oq, ok, ov, d, pp, none, none, sms, s);
    }
    cudaFreeAsync(ws, s);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core kernel (closed-form mask)");
    return SPATTN_OK;
}

// Whether the persistent tile kernel takes an interval-mask forward. By
// default d = 128 without additive terms: at d <= 64 the four-CTAs-per-SM tile
// kernel (k_fwd_tc_quad) is faster on the interval workloads (variable window
// 0.10 against 0.15 ms, the Evoformer shape 0.15 against 0.24 ms, on one
// B200), so it keeps them. SPATTN_DEBUG_PP_INTERVAL=1 sends d = 32 and 64
// (additive terms too, when TMA can stage them) to the persistent kernel as
// well; the tests use it to cover those paths.
bool pp_takes_interval(const FwdParams& p, int d) {
    const char* e = getenv("SPATTN_DEBUG_PP_INTERVAL");
    const bool all = e && e[0] == '1';
    if (d == 128) return !p.has_extra;
    if (!all || (d != 32 && d != 64)) return false;
    return !p.has_extra || (pp_addend_ok(p.mask) && pp_addend_ok(p.bias));
}

// The persistent tile kernel over an interval mask's tiles; blk_res: the
// gather kernel ran first and left partial states in p.ws_ml / p.ws_acc for
// the flagged blocks.
int launch_pp_interval(const FwdParams& p, int d, spattn_mask m, int dev, int sms, const int32_t* blk_res,
                       cudaStream_t s) {
    unsigned* ef = nullptr;
    int r = err_flags_ptr(dev, &ef);
    if (r) return r;
    PpParams pp;
    memset(&pp, 0, sizeof pp);
    pp_common(pp, p, ef);
    pp.num_masks = m->num_masks;
    pp.mode = 0;
    pp.n_items = (int64_t)p.B * p.H * m->nqb;
    pp.itv_lohi = m->lohi;
    pp.itv_tiles = m->itv_tiles;
    pp.itv_ntiles = m->itv_ntiles;
    pp.blk_res = blk_res;
    pp.ws_ml = p.ws_ml;
    pp.ws_acc = p.ws_acc;
    pp.seqlen_k = p.seqlen_k;
    const TcOperand oq{p.q, p.q_sn, p.q_sh, p.q_sb}, ok{p.k, p.k_sn, p.k_sh, p.k_sb}, ov{p.v, p.v_sn, p.v_sh, p.v_sb};
    const cudaError_t e = launch_fwd_pp(oq, ok, ov, d, pp, p.mask, p.bias, sms, s);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core kernel launch");
    return SPATTN_OK;
}

// Forward over an interval mask. Without tensor-core tiles (fp32, no plan, or
// none selected) the interval gather kernel does every entry. With tiles it
// runs first only when entries outside the tiles may exist -- known exactly
// once the build's totals are in (it does not wait for them) or, before that,
// from the pattern's parameters -- and hands partial states to the
// tensor-core kernel.
int fwd_interval(FwdParams& p, int dtype, int d, spattn_mask m, cudaStream_t s, cudaMemPool_t pool,
                 int dev, int num_sms) {
    p.itv_lohi = m->lohi;
    p.nkt = m->nkt;
    p.nqb = m->nqb;
    // split query blocks until there are about four thread blocks per SM
    const int64_t qblocks = (int64_t)p.B * p.H * p.nqb;
    p.itv_slices = 1;
    while (p.itv_slices < 16 && qblocks * p.itv_slices < 4LL * num_sms) p.itv_slices *= 2;
    bool ready = false;
    int r = read_counters(m, false, &ready);
    if (r) return r;
    const bool tc = m->min_nnz > 0 && dtype == 0 && !(ready && m->n_tiles == 0);
    if (!tc) {
        const cudaError_t e = launch_fwd_itv(p, dtype, d, s);
        if (e != cudaSuccess) return cuda_fail(e, "interval gather kernel launch");
        return SPATTN_OK;
    }
    const int64_t nblocks = (int64_t)m->num_masks * m->nqb;
    const bool gather = ready ? (m->res_nnz > 0 || m->n_tc_blocks < nblocks) : !m->host_no_residual;
    float* ws = nullptr;
    if (gather) {
        const int64_t rows_all = (int64_t)p.B * p.H * p.n;
        CUDA_TRY(pool_alloc(&ws, rows_all * (d + 2), pool, s), "partial-state workspace");
        p.ws_ml = ws;
        p.ws_acc = ws + rows_all * 2;
        p.tmap = m->tmap;
        p.qb_ntiles = m->itv_ntiles;
        p.blk_res = m->blk_res;
        const cudaError_t e = launch_fwd_itv(p, dtype, d, s);
        if (e != cudaSuccess) {
            cudaFreeAsync(ws, s);
            return cuda_fail(e, "interval gather kernel launch");
        }
    }
    if (pp_takes_interval(p, d))
        r = launch_pp_interval(p, d, m, dev, num_sms, gather ? m->blk_res : nullptr, s);
    else
        r = launch_tc(p, d, m, dev, gather ? m->blk_res : nullptr, s);
    if (ws) cudaFreeAsync(ws, s);
    return r;
}


// The transposed mask (rows m*n + j listing the i with j in S_i), written on the
// first backward call over this mask, on the mask's stream.
int write_transpose(spattn_mask m) {
    if (m->t_row_ptr) return SPATTN_OK;
    int r = write_csr(m);
    if (r) return r;
    if (m->n > 1572864) return fail(SPATTN_ERR_UNSUPPORTED, "backward needs n <= 1572864");
    const int64_t rows = (int64_t)m->n * m->num_masks;
    cudaMemPool_t pool;
    CUDA_TRY(device_state(m->device, &pool, nullptr), "memory pool");
    cudaStream_t s = m->stream;
    Carve c;
    const int k_rp = c.add((rows + 1) * 4), k_ci = c.add((m->nnz > 0 ? m->nnz : 1) * 4);
    void *blk = nullptr, *scratch = nullptr;
    cudaError_t e = lib_malloc_async(&blk, c.total, pool, s);
    if (e == cudaSuccess)
        e = lib_malloc_async(&scratch, (size_t)transpose_scratch_words(rows, m->nnz) * 4, pool, s);
    if (e == cudaSuccess)
        e = build_transpose(m->row_ptr, m->col_idx, m->n, m->num_masks, m->nnz, c.at<int32_t>(blk, k_rp),
                            c.at<int32_t>(blk, k_ci), static_cast<int32_t*>(scratch), s);
    if (scratch) cudaFreeAsync(scratch, s);
    if (e != cudaSuccess) {
        if (blk) cudaFreeAsync(blk, s);
        return cuda_fail(e, "transposing the mask");
    }
    m->block_t = blk;
    m->t_row_ptr = c.at<int32_t>(blk, k_rp);
    m->t_col_idx = c.at<int32_t>(blk, k_ci);
    return SPATTN_OK;
}

// A block + strided + global mask in closed form: no device work at all. Its
// size is counted here from the pattern (row i of one mask: every key for a
// global row, else the union of its block, its strided keys and the global
// keys), and the forward pass derives tiles and bits from the parameters.
int create_closed(const spattn_mask_spec& sp, cudaStream_t s, int dev, spattn_mask* out) {
    const bsg::Shape sh = bsg::shape(sp.n, sp.block, sp.stride, sp.n_global, kChunkTiles);
    const int64_t n = sp.n, ng = sp.n_global;
    int64_t per = 0, n_long = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t c;
        if (i < ng) {
            c = n;
        } else {
            const int64_t blk = sp.block;
            const int64_t strided = sp.stride ? n / sp.stride : 0;  // keys j = i (mod stride)
            c = blk + strided + ng;
            if (blk > 0 && sp.stride) c -= 1;                      // j = i: block and strided
            if (blk > 0 && ng > 0) {                                // block keys below ng
                const int64_t b0 = (i / blk) * blk;
                c -= std::max<int64_t>(0, std::min(b0 + blk, ng) - b0);
            }
            if (sp.stride && (i % sp.stride) < ng) c -= 1;         // the strided key below ng
        }
        per += c;
        n_long += c > kLongRowThreshold ? 1 : 0;
    }
    // tiles of one forward per (b, h): chunks of block 0, further regular
    // blocks, permuted blocks (each over every permuted key tile)
    int64_t tiles = 0;
    for (int64_t x = 0; x < sh.items_per_head; ++x) tiles += bsg::item(sh, x, 1).T;
    spattn_mask m = new spattn_mask_s;
    memset(m, 0, sizeof *m);
    m->device = dev;
    m->stream = s;
    m->n = sp.n;
    m->num_masks = sp.num_masks;
    m->kind = sp.kind;
    m->nnz = per * sp.num_masks;
    m->n_long = n_long * sp.num_masks;
    m->nqb = sh.nqb;
    m->closed = true;
    m->bsg_block = sp.block;
    m->bsg_stride = sp.stride;
    m->bsg_ng = sp.n_global;
    m->closed_tiles = tiles * sp.num_masks;
    *out = m;
    return SPATTN_OK;
}

int create_mask(const spattn_mask_spec* spec, void* stream_v, spattn_mask* out, bool allow_closed);

// The CSR-built copy of a closed-form mask, made on first need on the mask's
// stream (synchronises it, like any CSR build).
int ensure_generic(spattn_mask m) {
    if (m->generic) return SPATTN_OK;
    spattn_mask_spec sp;
    memset(&sp, 0, sizeof sp);
    sp.kind = SPATTN_MASK_BLOCK_STRIDED_GLOBAL;
    sp.n = m->n;
    sp.num_masks = m->num_masks;
    sp.block = m->bsg_block;
    sp.stride = m->bsg_stride;
    sp.n_global = m->bsg_ng;
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != m->device) cudaSetDevice(m->device);
    const int r = create_mask(&sp, m->stream, &m->generic, false);
    if (prev >= 0 && prev != m->device) cudaSetDevice(prev);
    return r;
}

int create_mask(const spattn_mask_spec* spec, void* stream_v, spattn_mask* out, bool allow_closed) {
    g_msg[0] = 0;
    if (!out) return fail(SPATTN_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!spec) return fail(SPATTN_ERR_INVALID_ARG, "spec is NULL");
    const spattn_mask_spec& sp = *spec;
    if (sp.kind < SPATTN_MASK_CSR || sp.kind > SPATTN_MASK_DENSE)
        return fail(SPATTN_ERR_INVALID_ARG, "unknown mask kind %d", sp.kind);
    if (sp.n < 1) return fail(SPATTN_ERR_INVALID_ARG, "n must be >= 1");
    if (sp.num_masks < 1) return fail(SPATTN_ERR_INVALID_ARG, "num_masks must be >= 1");
    const int64_t rows = (int64_t)sp.n * sp.num_masks;
    if (rows > 0x7ffffffe) return fail(SPATTN_ERR_UNSUPPORTED, "num_masks * n too large");
    if (sp.kind == SPATTN_MASK_SLIDING && sp.window < 0)
        return fail(SPATTN_ERR_INVALID_ARG, "window must be >= 0");
    if (sp.kind == SPATTN_MASK_VARWIN && !sp.half_widths)
        return fail(SPATTN_ERR_INVALID_ARG, "half_widths is NULL");
    if (sp.kind == SPATTN_MASK_BLOCK_STRIDED_GLOBAL &&
        (sp.block < 0 || sp.stride < 0 || sp.n_global < 0))
        return fail(SPATTN_ERR_INVALID_ARG, "block, stride and n_global must be >= 0");
    if (sp.flags & ~(uint32_t)SPATTN_MASK_ASYNC) return fail(SPATTN_ERR_INVALID_ARG, "unknown spec.flags bits");
    if (sp.kind == SPATTN_MASK_CSR || sp.kind == SPATTN_MASK_COO) {
        if (!sp.in_row_ptr) return fail(SPATTN_ERR_INVALID_ARG, "in_row_ptr is NULL");
        if (sp.in_nnz < 0 || sp.in_nnz > 0x7fffffff)
            return fail(SPATTN_ERR_INVALID_ARG, "in_nnz out of range");
        if (sp.in_nnz > 0 && !sp.in_col_idx) return fail(SPATTN_ERR_INVALID_ARG, "in_col_idx is NULL");
    }
    cudaStream_t s = (cudaStream_t)stream_v;
    int dev;
    CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    cudaMemPool_t pool;
    CUDA_TRY(device_state(dev, &pool, nullptr), "memory pool");

    const int nqb_i = (sp.n + kTileM - 1) / kTileM;
    if (implicit_kind(sp.kind) && nqb_i <= kItvMaxKeyTiles && (int64_t)sp.num_masks * nqb_i <= kItvMaxBlocks)
        return create_implicit(sp, s, dev, pool, out);
    if (allow_closed && sp.kind == SPATTN_MASK_BLOCK_STRIDED_GLOBAL && sp.tile_min_nnz == 0 &&
        bsg::supported(sp.n, sp.block, sp.stride, sp.n_global))
        return create_closed(sp, s, dev, out);

    BuildSpec bs;
    bs.kind = sp.kind;
    bs.n = sp.n;
    bs.num_masks = sp.num_masks;
    bs.window = sp.window;
    bs.block = sp.block;
    bs.stride = sp.stride;
    bs.n_global = sp.n_global;
    bs.add_diagonal = sp.add_diagonal ? 1 : 0;
    bs.half_widths = sp.half_widths;
    bs.in_row_ptr = sp.in_row_ptr;
    bs.in_col_idx = sp.in_col_idx;
    bs.in_nnz = sp.in_nnz;

    const bool coo = sp.kind == SPATTN_MASK_COO;
    const bool intervals = sp.kind == SPATTN_MASK_SLIDING || sp.kind == SPATTN_MASK_VARWIN ||
                           sp.kind == SPATTN_MASK_DENSE;
    const int min_nnz = sp.tile_min_nnz == 0 ? kTileMinNnzDefault : sp.tile_min_nnz;
    const int nqb = (sp.n + kTileM - 1) / kTileM, nkt = (sp.n + kTileN - 1) / kTileN;
    const int64_t nblocks = (int64_t)sp.num_masks * nqb;
    const bool plan_possible = sp.tile_min_nnz >= 0 && nblocks * nkt <= kPlanMaxTileGrid;
    // phase 1 memory: the mask's row_ptr + long-row list, and temporaries --
    // those of the build and, as their sizes do not depend on nnz, the tile
    // plan's (counters first, then the per-tile counts, so one run of words
    // clears both)
    Carve ca;
    const int k_rp = ca.add((rows + 1) * 4), k_long = ca.add(rows * 4);
    Carve ct;
    const int k_info = ct.add(sizeof(BuildInfo)), k_cnt = ct.add(rows * 4);
    const int k_scan = ct.add((scan_tmp_elems(rows) + (coo ? (rows + 6) / 2 + 1 : 0)) * 8);
    const int k_coo = ct.add(coo ? (sp.in_nnz + rows) * 4 : 0);
    const int64_t scan_rows = rows > nblocks ? rows : nblocks;
    const int64_t cnt_words = plan_possible ? nblocks * nkt : 0;
    const int k_pc = ct.add(plan_possible ? sizeof(PlanCounters) : 0),
              k_cm = ct.add(cnt_words * 4), k_bn = ct.add(plan_possible ? nblocks * 4 : 0),
              k_st = ct.add(plan_possible ? scan_tmp_elems(scan_rows) * 8 : 0),
              k_rc = ct.add(plan_possible ? rows * 4 : 0);
    void *blk_a = nullptr, *blk_t = nullptr;
    cudaError_t e = lib_malloc_async(&blk_a, ca.total, pool, s);
    if (e == cudaSuccess) e = lib_malloc_async(&blk_t, ct.total, pool, s);
    if (e != cudaSuccess) {
        if (blk_a) cudaFreeAsync(blk_a, s);
        return cuda_fail(e, "mask allocation");
    }
    int32_t* row_ptr = ca.at<int32_t>(blk_a, k_rp);
    int32_t* long_rows = ca.at<int32_t>(blk_a, k_long);
    BuildInfo* info = ct.at<BuildInfo>(blk_t, k_info);
    int32_t* counts = ct.at<int32_t>(blk_t, k_cnt);
    int64_t* scan_tmp = ct.at<int64_t>(blk_t, k_scan);
    int32_t* coo_tmp = coo ? ct.at<int32_t>(blk_t, k_coo) : nullptr;
    // words from the counters to the end of the count array
    const int64_t zero_words = plan_possible ? (int64_t)(ct.off[k_cm] - ct.off[k_pc]) / 4 + cnt_words : 0;
    bool zeroed = false;
    e = build_phase1(bs, row_ptr, counts, scan_tmp, coo_tmp, info, long_rows,
                     zero_words > 0 && zero_words <= kPlanZeroInline ? ct.at<int32_t>(blk_t, k_pc) : nullptr,
                     zero_words, &zeroed, s);
    BuildInfo hinfo;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&hinfo, info, sizeof hinfo, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    int st = e == cudaSuccess ? build_status(hinfo.err) : SPATTN_OK;
    if (e != cudaSuccess || st != SPATTN_OK) {
        cudaFreeAsync(blk_t, s);
        cudaFreeAsync(blk_a, s);
        return e != cudaSuccess ? cuda_fail(e, "mask build (phase 1)") : st;
    }
    spattn_mask m = new spattn_mask_s;
    memset(m, 0, sizeof *m);
    m->device = dev;
    m->stream = s;
    m->n = sp.n;
    m->num_masks = sp.num_masks;
    m->nnz = hinfo.nnz;
    m->n_long = hinfo.n_long;
    m->row_ptr = row_ptr;
    m->long_rows = long_rows;
    m->block_csr = blk_a;

    // phase 2 memory: col_idx and the tile plan
    const bool plan = plan_possible && hinfo.nnz > 0;
    // interval rows hand their per-tile counts to the plan while writing columns
    const bool precounted = plan && intervals && zeroed;
    PlanBuffers pb;
    memset(&pb, 0, sizeof pb);
    PlanCounters hpc;
    memset(&hpc, 0, sizeof hpc);
    e = lib_malloc_async(&m->block_col, (size_t)(hinfo.nnz > 0 ? hinfo.nnz : 1) * 4, pool, s);
    if (e == cudaSuccess) {
        m->col_idx = static_cast<int32_t*>(m->block_col);
        e = build_phase2(bs, row_ptr, coo_tmp, m->col_idx,
                         precounted ? ct.at<int32_t>(blk_t, k_cm) : nullptr, s);
    }
    if (plan && e == cudaSuccess) {
        m->nqb = nqb;
        pb.tile_cap = plan_tile_capacity(nblocks, nkt, hinfo.nnz, min_nnz);
        Carve cp;
        const int k_bto = cp.add((nblocks + 1) * 4), k_ti = cp.add(pb.tile_cap * 4),
                  k_tb = cp.add(pb.tile_cap * kTileM * 16), k_rrp = cp.add((rows + 1) * 4),
                  k_rci = cp.add(hinfo.nnz * 4), k_rl = cp.add(rows * 4);
        e = lib_malloc_async(&m->block_plan, cp.total, pool, s);
        if (e == cudaSuccess) {
            m->block_tile_off = pb.block_tile_off = cp.at<int32_t>(m->block_plan, k_bto);
            m->tile_info = pb.tile_info = cp.at<int32_t>(m->block_plan, k_ti);
            m->tile_bits = pb.tile_bits = cp.at<uint32_t>(m->block_plan, k_tb);
            m->res_row_ptr = pb.res_row_ptr = cp.at<int32_t>(m->block_plan, k_rrp);
            m->res_col_idx = pb.res_col_idx = cp.at<int32_t>(m->block_plan, k_rci);
            m->res_long = pb.res_long = cp.at<int32_t>(m->block_plan, k_rl);
            PlanCounters* pc = ct.at<PlanCounters>(blk_t, k_pc);
            pb.cnt_map = ct.at<int32_t>(blk_t, k_cm);
            pb.block_ntiles = ct.at<int32_t>(blk_t, k_bn);
            pb.scan_tmp = ct.at<int64_t>(blk_t, k_st);
            pb.res_cnt = ct.at<int32_t>(blk_t, k_rc);
            e = build_plan(row_ptr, m->col_idx, sp.n, sp.num_masks, hinfo.nnz, min_nnz, intervals,
                           zeroed, precounted, pb, pc, s);
            if (e == cudaSuccess) e = cudaMemcpyAsync(&hpc, pc, sizeof hpc, cudaMemcpyDeviceToHost, s);
            if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        }
    }
    cudaFreeAsync(blk_t, s);
    if (e != cudaSuccess) {
        spattn_destroy_mask(m);
        return cuda_fail(e, "mask build (phase 2)");
    }
    if (plan) {
        m->n_tiles = hpc.n_tiles;
        m->res_nnz = hpc.res_nnz;
        m->n_mixed = hpc.n_mixed;
        m->n_tc_blocks = hpc.n_tc_blocks;
        m->res_n_long = hpc.res_n_long;
        m->has_plan = hpc.n_tiles > 0;
        if (!m->has_plan) free_plan(m);
        int r = m->has_plan ? write_chunks(m, pool) : SPATTN_OK;
        if (!r && m->has_plan && m->res_nnz > 0 && sp.kind == SPATTN_MASK_BLOCK_STRIDED_GLOBAL &&
            sp.stride >= 2 && sp.n % sp.stride == 0)
            r = write_strided(m, sp.stride, sp.tile_min_nnz, pool);
        if (r) {
            spattn_destroy_mask(m);
            return r;
        }
    }
    *out = m;
    return SPATTN_OK;
}

}  // namespace

extern "C" {

const char* spattn_last_error(void) { return g_msg; }

int spattn_version(void) { return 100; /* 0.1.0 */ }

uint64_t spattn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

uint64_t spattn_alloc_count(void) { return g_allocs.load(std::memory_order_relaxed); }

int spattn_create_csr_mask(const spattn_mask_spec* spec, void* stream_v, spattn_mask* out) {
    return create_mask(spec, stream_v, out, true);
}

int spattn_mask_copy_plan(spattn_mask m, int32_t* block_tile_off, int32_t* tile_info,
                          uint32_t* tile_bits, int32_t* res_row_ptr, int32_t* res_col_idx,
                          void* stream_v) {
    g_msg[0] = 0;
    if (!m) return fail(SPATTN_ERR_INVALID_ARG, "mask is NULL");
    if (m->closed) {  // the CSR-built copy's plan
        const int rg = ensure_generic(m);
        if (rg) return rg;
        return spattn_mask_copy_plan(m->generic, block_tile_off, tile_info, tile_bits, res_row_ptr, res_col_idx,
                                     stream_v);
    }
    int r = write_plan(m);
    if (r) return r;
    if (!m->has_plan || m->n_tiles == 0) return fail(SPATTN_ERR_INVALID_ARG, "the mask has no tile plan");
    cudaStream_t s = (cudaStream_t)stream_v;
    const int64_t rows = (int64_t)m->n * m->num_masks;
    const int64_t nblocks = (int64_t)m->num_masks * m->nqb;
    struct Item {
        void* dst;
        const void* src;
        size_t bytes;
    } items[] = {
        {block_tile_off, m->block_tile_off, (size_t)(nblocks + 1) * 4},
        {tile_info, m->tile_info, (size_t)m->n_tiles * 4},
        {tile_bits, m->tile_bits, (size_t)m->n_tiles * kTileM * 4 * 4},
        {res_row_ptr, m->res_row_ptr, (size_t)(rows + 1) * 4},
        {res_col_idx, m->res_col_idx, (size_t)m->res_nnz * 4},
    };
    for (const Item& it : items)
        if (it.dst && it.bytes)
            CUDA_TRY(cudaMemcpyAsync(it.dst, it.src, it.bytes, cudaMemcpyDefault, s), "plan copy");
    return SPATTN_OK;
}

int spattn_mask_plan_info(spattn_mask m, int64_t* n_tiles, int64_t* residual_nnz,
                          int64_t* n_mixed_rows) {
    g_msg[0] = 0;
    if (!m) return fail(SPATTN_ERR_INVALID_ARG, "mask is NULL");
    if (m->closed) {
        const int rg = ensure_generic(m);
        if (rg) return rg;
        return spattn_mask_plan_info(m->generic, n_tiles, residual_nnz, n_mixed_rows);
    }
    int r = read_counters(m, true);
    if (r == SPATTN_OK && n_mixed_rows) r = write_plan(m);
    if (r) return r;
    if (n_tiles) *n_tiles = m->has_plan ? m->n_tiles : 0;
    if (residual_nnz) *residual_nnz = m->has_plan ? m->res_nnz : m->nnz;
    if (n_mixed_rows) *n_mixed_rows = m->has_plan ? m->n_mixed : 0;
    return SPATTN_OK;
}

int spattn_mask_tile_count(spattn_mask m, int64_t* tiles) {
    g_msg[0] = 0;
    if (!m || !tiles) return fail(SPATTN_ERR_INVALID_ARG, "mask or tiles is NULL");
    if (m->closed) {
        *tiles = m->closed_tiles;
        return SPATTN_OK;
    }
    const int r = read_counters(m, true);
    if (r) return r;
    if (m->str_mask)  // the residue-permuted part and the rest, each with its own plan
        *tiles = m->str_mask->n_tiles + m->reg_mask->n_tiles;
    else
        *tiles = m->has_plan ? m->n_tiles : 0;
    return SPATTN_OK;
}

int spattn_mask_info(spattn_mask m, int32_t* n, int32_t* num_masks, int64_t* nnz,
                     const int32_t** row_ptr, const int32_t** col_idx, int64_t* n_long) {
    g_msg[0] = 0;
    if (!m) return fail(SPATTN_ERR_INVALID_ARG, "mask is NULL");
    int r = SPATTN_OK;
    if (nnz || n_long) r = read_counters(m, true);
    if (r == SPATTN_OK && (row_ptr || col_idx)) r = m->closed ? ensure_generic(m) : write_csr(m);
    if (r) return r;
    const spattn_mask c = m->closed ? m->generic : m;  // who holds the CSR
    if (n) *n = m->n;
    if (num_masks) *num_masks = m->num_masks;
    if (nnz) *nnz = m->nnz;
    if (row_ptr) *row_ptr = c->row_ptr;
    if (col_idx) *col_idx = c->col_idx;
    if (n_long) *n_long = m->n_long;
    return SPATTN_OK;
}

int spattn_mask_csr(spattn_mask m, const int32_t** row_ptr, const int32_t** col_idx, int64_t* nnz_total) {
    g_msg[0] = 0;
    if (!m) return fail(SPATTN_ERR_INVALID_ARG, "mask is NULL");
    return spattn_mask_info(m, nullptr, nullptr, nnz_total, row_ptr, col_idx, nullptr);
}

int spattn_mask_copy_long_rows(spattn_mask m, int32_t* dst, void* stream_v) {
    g_msg[0] = 0;
    if (!m || !dst) return fail(SPATTN_ERR_INVALID_ARG, "mask or dst is NULL");
    if (m->closed) {
        const int rg = ensure_generic(m);
        if (rg) return rg;
        return spattn_mask_copy_long_rows(m->generic, dst, stream_v);
    }
    int r = read_counters(m, true);
    if (r) return r;
    if (m->implicit && !m->long_rows && m->n_long > 0) {  // list them from the CSR, once
        if ((r = write_csr(m))) return r;
        cudaMemPool_t pool;
        CUDA_TRY(device_state(m->device, &pool, nullptr), "memory pool");
        const int64_t rows = (int64_t)m->n * m->num_masks;
        int32_t* blk = nullptr;  // [0]: count, [1 ..]: rows
        CUDA_TRY(lib_malloc_async(&blk, (size_t)(rows + 1) * 4, pool, m->stream), "long-row list");
        cudaError_t e = cudaMemsetAsync(blk, 0, 4, m->stream);
        if (e == cudaSuccess) e = launch_classify_long_rows(m->row_ptr, rows, m->nnz, blk + 1, blk, m->stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(m->stream);
        if (e != cudaSuccess) {
            cudaFreeAsync(blk, m->stream);
            return cuda_fail(e, "listing long rows");
        }
        m->block_long = blk;
        m->long_rows = blk + 1;
    }
    if (m->n_long > 0)
        CUDA_TRY(cudaMemcpyAsync(dst, m->long_rows, (size_t)m->n_long * 4, cudaMemcpyDefault,
                                 (cudaStream_t)stream_v),
                 "long-row copy");
    return SPATTN_OK;
}

int spattn_mask_copy_csr(spattn_mask m, int32_t* row_ptr_dst, int32_t* col_idx_dst,
                         void* stream_v) {
    g_msg[0] = 0;
    if (!m) return fail(SPATTN_ERR_INVALID_ARG, "mask is NULL");
    if (m->closed && (row_ptr_dst || col_idx_dst)) {
        const int r = ensure_generic(m);
        if (r) return r;
        return spattn_mask_copy_csr(m->generic, row_ptr_dst, col_idx_dst, stream_v);
    }
    if (row_ptr_dst || col_idx_dst) {
        const int r = write_csr(m);
        if (r) return r;
    }
    cudaStream_t s = (cudaStream_t)stream_v;
    const int64_t rows = (int64_t)m->n * m->num_masks;
    if (row_ptr_dst)
        CUDA_TRY(cudaMemcpyAsync(row_ptr_dst, m->row_ptr, (size_t)(rows + 1) * sizeof(int32_t),
                                 cudaMemcpyDefault, s),
                 "row_ptr copy");
    if (col_idx_dst && m->nnz > 0)
        CUDA_TRY(cudaMemcpyAsync(col_idx_dst, m->col_idx, (size_t)m->nnz * sizeof(int32_t),
                                 cudaMemcpyDefault, s),
                 "col_idx copy");
    return SPATTN_OK;
}

int spattn_destroy_mask(spattn_mask m) {
    g_msg[0] = 0;
    if (!m) return SPATTN_OK;
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != m->device) cudaSetDevice(m->device);
    cudaError_t e = cudaSuccess, e2;
    if (m->block_csr && (e2 = cudaFreeAsync(m->block_csr, m->stream)) != cudaSuccess) e = e2;
    if (m->block_col && (e2 = cudaFreeAsync(m->block_col, m->stream)) != cudaSuccess) e = e2;
    free_plan(m);
    if (m->str_mask) spattn_destroy_mask(m->str_mask);
    if (m->reg_mask) spattn_destroy_mask(m->reg_mask);
    if (m->generic) spattn_destroy_mask(m->generic);
    if (m->block_itv && (e2 = cudaFreeAsync(m->block_itv, m->stream)) != cudaSuccess) e = e2;
    if (m->block_long && (e2 = cudaFreeAsync(m->block_long, m->stream)) != cudaSuccess) e = e2;
    if (m->block_t && (e2 = cudaFreeAsync(m->block_t, m->stream)) != cudaSuccess) e = e2;
    if (m->cnt_host) {
        HostSlot sl;
        sl.host = m->cnt_host;
        sl.dev = m->cnt_dev;
        sl.done = m->done_dev;
        sl.ev = m->built;
        put_slot(m->device, sl);
    }
    if (prev >= 0 && prev != m->device) cudaSetDevice(prev);
    delete m;
    if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
    return SPATTN_OK;
}

int spattn_fwd(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
               const int32_t* row_ptr, const int32_t* col_idx, int32_t num_masks, int64_t nnz,
               const spattn_tensor* add_mask, const spattn_tensor* bias, float scale,
               const spattn_tensor* out, float* lse, void* stream_v) {
    g_msg[0] = 0;
    FwdParams p;
    int dtype, d;
    int r = check_fwd(q, k, v, add_mask, bias, scale, out, lse, &p, &dtype, &d);
    if (r) return r;
    if (num_masks != 1 && num_masks != p.B)
        return fail(SPATTN_ERR_INVALID_ARG, "num_masks must be 1 or B");
    if (!row_ptr) return fail(SPATTN_ERR_INVALID_ARG, "row_ptr is NULL");
    if (nnz < 0) return fail(SPATTN_ERR_INVALID_ARG, "nnz < 0");
    if (nnz > 0 && !col_idx) return fail(SPATTN_ERR_INVALID_ARG, "col_idx is NULL");
    if ((int64_t)p.B * p.H * p.n == 0) return SPATTN_OK;
    cudaStream_t s = (cudaStream_t)stream_v;
    int dev, sms;
    CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    cudaMemPool_t pool;
    CUDA_TRY(device_state(dev, &pool, &sms), "memory pool");
    p.num_masks = num_masks;
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
    p.nnz = nnz;
    const int64_t rows = (int64_t)num_masks * p.n;
    int32_t* scratch = nullptr;  // [0]: long-row count, [1 ..]: long-row list
    CUDA_TRY(pool_alloc(&scratch, rows + 1, pool, s), "scratch allocation");
    cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = launch_classify_long_rows(row_ptr, rows, nnz, scratch + 1, scratch, s);
    if (e != cudaSuccess) {
        cudaFreeAsync(scratch, s);
        return cuda_fail(e, "long-row classification");
    }
    p.long_rows = scratch + 1;
    p.long_count_dev = scratch;
    p.long_count_host = -1;
    r = launch_fwd(p, dtype, d, sms, s);
    cudaError_t ef = cudaFreeAsync(scratch, s);
    if (r) return r;
    if (ef != cudaSuccess) return cuda_fail(ef, "cudaFreeAsync");
    return SPATTN_OK;
}

int spattn_fwd_mask(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                    spattn_mask mask, const spattn_tensor* add_mask, const spattn_tensor* bias,
                    float scale, const spattn_tensor* out, float* lse, void* stream_v) {
    return spattn_fwd_mask_kpad(q, k, v, mask, nullptr, add_mask, bias, scale, out, lse, stream_v);
}

int spattn_fwd_mask_kpad(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                         spattn_mask mask, const int32_t* seqlen_k, const spattn_tensor* add_mask,
                         const spattn_tensor* bias, float scale, const spattn_tensor* out, float* lse,
                         void* stream_v) {
    g_msg[0] = 0;
    FwdParams p;
    int dtype, d;
    int r = check_fwd(q, k, v, add_mask, bias, scale, out, lse, &p, &dtype, &d);
    if (r) return r;
    if (seqlen_k && ((uintptr_t)seqlen_k) % 4 != 0) return fail(SPATTN_ERR_INVALID_ARG, "seqlen_k not aligned");
    p.seqlen_k = seqlen_k;
    if (!mask) return fail(SPATTN_ERR_INVALID_ARG, "mask is NULL");
    if (mask->n != p.n) return fail(SPATTN_ERR_INVALID_ARG, "mask n %d != q n %d", mask->n, p.n);
    if (mask->num_masks != 1 && mask->num_masks != p.B)
        return fail(SPATTN_ERR_INVALID_ARG, "mask num_masks must be 1 or B");
    if ((int64_t)p.B * p.H * p.n == 0) return SPATTN_OK;
    cudaStream_t s = (cudaStream_t)stream_v;
    int dev, sms;
    CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev != mask->device) return fail(SPATTN_ERR_INVALID_ARG, "mask lives on another device");
    cudaMemPool_t pool;
    CUDA_TRY(device_state(dev, &pool, &sms), "memory pool");
    p.num_masks = mask->num_masks;
    p.long_count_dev = nullptr;
    if (mask->closed) {
        // the kernel numbers its items in 32 bits
        const bsg::Shape sh = bsg::shape(p.n, mask->bsg_block, mask->bsg_stride, mask->bsg_ng, kChunkTiles);
        const bool fits = (int64_t)p.B * p.H * sh.items_per_head < ((int64_t)1 << 31);
        if (dtype == 0 && !seqlen_k && !p.has_extra && (d == 64 || d == 128) && fits)
            return fwd_closed(p, d, mask, s, pool, dev, sms);
        if ((r = ensure_generic(mask))) return r;
        return spattn_fwd_mask_kpad(q, k, v, mask->generic, seqlen_k, add_mask, bias, scale, out, lse, stream_v);
    }
    if (mask->implicit) return fwd_interval(p, dtype, d, mask, s, pool, dev, sms);
    if (mask->str_mask && dtype == 0 && !seqlen_k && !p.has_extra)
        return fwd_strided(q, k, v, mask, scale, out, lse, s, p, d, pool, dev);
    if (!(mask->has_plan && dtype == 0)) {  // every entry on the gather kernel
        p.row_ptr = mask->row_ptr;
        p.col_idx = mask->col_idx;
        p.nnz = mask->nnz;
        p.long_rows = mask->long_rows;
        p.long_count_host = mask->n_long;
        return launch_fwd(p, dtype, d, sms, s);
    }
    // tile plan: residual entries on the gather kernel, tiles on tensor cores
    p.row_ptr = mask->res_row_ptr;
    p.col_idx = mask->res_col_idx;
    p.nnz = mask->res_nnz;
    p.long_rows = mask->res_long;
    p.long_count_host = mask->res_n_long;
    p.qb_tile_off = mask->block_tile_off;
    p.nqb = mask->nqb;
    float* ws = nullptr;
    const int64_t rows_all = (int64_t)p.B * p.H * p.n;
    if (mask->n_mixed > 0) {
        CUDA_TRY(pool_alloc(&ws, rows_all * (d + 2), pool, s), "partial-state workspace");
        p.ws_ml = ws;
        p.ws_acc = ws + rows_all * 2;
    }
    const int64_t nblocks = (int64_t)mask->num_masks * mask->nqb;
    if (mask->res_nnz > 0 || mask->n_tc_blocks < nblocks) {
        r = launch_fwd(p, dtype, d, sms, s);
        if (r) {
            if (ws) cudaFreeAsync(ws, s);
            return r;
        }
    }
    r = launch_tc(p, d, mask, dev, nullptr, s);
    if (ws) cudaFreeAsync(ws, s);
    return r;
}

int spattn_fwd_unfused(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                       const int32_t* row_ptr, const int32_t* col_idx, int32_t num_masks, int64_t nnz,
                       const spattn_tensor* add_mask, const spattn_tensor* bias, float scale,
                       const spattn_tensor* out, float* lse, void* stream_v) {
    g_msg[0] = 0;
    FwdParams p;
    int dtype, d;
    int r = check_fwd(q, k, v, add_mask, bias, scale, out, lse, &p, &dtype, &d);
    if (r) return r;
    if (num_masks != 1 && num_masks != p.B) return fail(SPATTN_ERR_INVALID_ARG, "num_masks must be 1 or B");
    if (!row_ptr) return fail(SPATTN_ERR_INVALID_ARG, "row_ptr is NULL");
    if (nnz < 0) return fail(SPATTN_ERR_INVALID_ARG, "nnz < 0");
    if (nnz > 0 && !col_idx) return fail(SPATTN_ERR_INVALID_ARG, "col_idx is NULL");
    if ((int64_t)p.B * p.H * p.n == 0) return SPATTN_OK;
    cudaStream_t s = (cudaStream_t)stream_v;
    int dev;
    CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    cudaMemPool_t pool;
    CUDA_TRY(device_state(dev, &pool, nullptr), "memory pool");
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
    p.nnz = nnz;
    p.num_masks = num_masks;
    float* scores = nullptr;
    const int64_t copies = num_masks == 1 ? (int64_t)p.B * p.H : (int64_t)p.H;
    CUDA_TRY(pool_alloc(&scores, copies * (nnz > 0 ? nnz : 1), pool, s), "score buffer");
    const cudaError_t e = launch_fwd_unfused(p, dtype, d, scores, s);
    cudaFreeAsync(scores, s);
    if (e != cudaSuccess) return cuda_fail(e, "unfused kernel launch");
    return SPATTN_OK;
}

int spattn_bwd_mask(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                    spattn_mask mask, const spattn_tensor* add_mask, const spattn_tensor* bias,
                    float scale, const spattn_tensor* out, const float* lse, const spattn_tensor* dout,
                    const spattn_tensor* dq, const spattn_tensor* dk, const spattn_tensor* dv,
                    const spattn_tensor* dbias, void* stream_v) {
    g_msg[0] = 0;
    FwdParams p;
    int dtype, d;
    int r = check_fwd(q, k, v, add_mask, bias, scale, out, nullptr, &p, &dtype, &d);
    if (r) return r;
    if (!mask) return fail(SPATTN_ERR_INVALID_ARG, "mask is NULL");
    if (!lse) return fail(SPATTN_ERR_INVALID_ARG, "lse is NULL");
    if (((uintptr_t)lse) % 4 != 0) return fail(SPATTN_ERR_INVALID_ARG, "lse not aligned");
    const int64_t shape[4] = {q->shape[0], q->shape[1], q->shape[2], q->shape[3]};
    if ((r = check_qkv(dout, "dout", shape, q->dtype))) return r;
    if ((r = check_qkv(dq, "dq", shape, q->dtype))) return r;
    if ((r = check_qkv(dk, "dk", shape, q->dtype))) return r;
    if ((r = check_qkv(dv, "dv", shape, q->dtype))) return r;
    if (dbias) {
        if (!bias) return fail(SPATTN_ERR_INVALID_ARG, "dbias needs bias");
        if (dbias->dtype != SPATTN_F32 || dbias->reserved != 0)
            return fail(SPATTN_ERR_INVALID_ARG, "dbias must be f32");
        if (!dbias->data) return fail(SPATTN_ERR_INVALID_ARG, "dbias.data is NULL");
        int64_t acc = 1;
        for (int x = 3; x >= 0; --x) {
            if (dbias->shape[x] != bias->shape[x])
                return fail(SPATTN_ERR_INVALID_ARG, "dbias shape differs from bias shape");
            if (dbias->shape[x] > 1 && dbias->stride[x] != acc)
                return fail(SPATTN_ERR_INVALID_ARG, "dbias must be contiguous");
            acc *= dbias->shape[x];
        }
        if (((uintptr_t)dbias->data) % 4 != 0) return fail(SPATTN_ERR_INVALID_ARG, "dbias not aligned");
    }
    if (mask->n != p.n) return fail(SPATTN_ERR_INVALID_ARG, "mask n %d != q n %d", mask->n, p.n);
    if (mask->num_masks != 1 && mask->num_masks != p.B)
        return fail(SPATTN_ERR_INVALID_ARG, "mask num_masks must be 1 or B");
    if ((int64_t)p.B * p.H * p.n == 0) return SPATTN_OK;
    cudaStream_t s = (cudaStream_t)stream_v;
    int dev;
    CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev != mask->device) return fail(SPATTN_ERR_INVALID_ARG, "mask lives on another device");
    cudaMemPool_t pool;
    CUDA_TRY(device_state(dev, &pool, nullptr), "memory pool");
    if (mask->closed) {  // the backward walks the CSR-built copy
        if ((r = ensure_generic(mask))) return r;
        return spattn_bwd_mask(q, k, v, mask->generic, add_mask, bias, scale, out, lse, dout, dq, dk, dv, dbias,
                               stream_v);
    }
    if ((r = write_transpose(mask))) return r;
    // the transpose was written on the mask's stream; order this stream after it
    if (mask->stream != s) CUDA_TRY(cudaStreamSynchronize(mask->stream), "mask stream");

    BwdParams bp;
    memset(&bp, 0, sizeof bp);
    auto bs = [](const spattn_tensor* t, int x) { return t->shape[x] == 1 ? 0 : t->stride[x]; };
    bp.q = q->data;
    bp.k = k->data;
    bp.v = v->data;
    bp.out = out->data;
    bp.dout = dout->data;
    bp.dq = dq->data;
    bp.dk = dk->data;
    bp.dv = dv->data;
    bp.lse = lse;
    bp.q_sb = p.q_sb; bp.q_sh = p.q_sh; bp.q_sn = p.q_sn;
    bp.k_sb = p.k_sb; bp.k_sh = p.k_sh; bp.k_sn = p.k_sn;
    bp.v_sb = p.v_sb; bp.v_sh = p.v_sh; bp.v_sn = p.v_sn;
    bp.o_sb = p.o_sb; bp.o_sh = p.o_sh; bp.o_sn = p.o_sn;
    bp.do_sb = bs(dout, 0); bp.do_sh = bs(dout, 1); bp.do_sn = bs(dout, 2);
    bp.dq_sb = bs(dq, 0); bp.dq_sh = bs(dq, 1); bp.dq_sn = bs(dq, 2);
    bp.dk_sb = bs(dk, 0); bp.dk_sh = bs(dk, 1); bp.dk_sn = bs(dk, 2);
    bp.dv_sb = bs(dv, 0); bp.dv_sh = bs(dv, 1); bp.dv_sn = bs(dv, 2);
    bp.B = p.B;
    bp.H = p.H;
    bp.n = p.n;
    bp.num_masks = mask->num_masks;
    bp.row_ptr = mask->row_ptr;
    bp.col_idx = mask->col_idx;
    bp.nnz = mask->nnz;
    bp.t_row_ptr = mask->t_row_ptr;
    bp.t_col_idx = mask->t_col_idx;
    bp.mask = p.mask;
    bp.bias = p.bias;
    bp.has_extra = p.has_extra;
    bp.scale = scale;
    bp.qk_scale_log2 = p.qk_scale_log2;
    if (dbias) {
        bp.dbias = static_cast<float*>(dbias->data);
        bp.db_s0 = bs(dbias, 0); bp.db_s1 = bs(dbias, 1); bp.db_s2 = bs(dbias, 2); bp.db_s3 = bs(dbias, 3);
        size_t elems = 1;
        for (int x = 0; x < 4; ++x) elems *= (size_t)dbias->shape[x];
        CUDA_TRY(cudaMemsetAsync(dbias->data, 0, elems * 4, s), "clearing dbias");
    }
    float* Dbuf = nullptr;
    CUDA_TRY(pool_alloc(&Dbuf, (int64_t)p.B * p.H * p.n, pool, s), "backward workspace");
    bp.D = Dbuf;
    const cudaError_t e = launch_bwd(bp, dtype, d, s);
    cudaFreeAsync(Dbuf, s);
    if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
    return SPATTN_OK;
}

// ---- allocation-free forward: its scratch is this fixed array, part of the
// library image on every device that loads it.
static __device__ __align__(256) int32_t g_noalloc_scratch[SPATTN_NOALLOC_MAX_ROWS + 1];

static std::mutex g_noalloc_mu;
static int32_t* g_noalloc_ptr[kMaxDevices];
static int g_noalloc_sms[kMaxDevices];

// Device address of the scratch array and the SM count, looked up once per
// device with that device current. In host code the array's name is only a
// host-side stand-in, so the kernels are always given the looked-up address.
static int noalloc_setup(int dev, int32_t** ptr, int* sms) {
    if (dev < 0 || dev >= kMaxDevices) return fail(SPATTN_ERR_CUDA, "device %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        int32_t* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
        int n_sms = 0;
        e = cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        g_noalloc_sms[dev] = n_sms;
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    *sms = g_noalloc_sms[dev];
    return SPATTN_OK;
}

int spattn_fwd_noalloc(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                       const int32_t* row_ptr, const int32_t* col_idx, int32_t num_masks,
                       int64_t nnz, const spattn_tensor* add_mask, const spattn_tensor* bias,
                       float scale, const spattn_tensor* out, float* lse, void* stream_v) {
    g_msg[0] = 0;
    FwdParams p;
    int dtype, d;
    int r = check_fwd(q, k, v, add_mask, bias, scale, out, lse, &p, &dtype, &d);
    if (r) return r;
    if (num_masks != 1 && num_masks != p.B)
        return fail(SPATTN_ERR_INVALID_ARG, "num_masks must be 1 or B");
    if (!row_ptr) return fail(SPATTN_ERR_INVALID_ARG, "row_ptr is NULL");
    if (nnz < 0) return fail(SPATTN_ERR_INVALID_ARG, "nnz < 0");
    if (nnz > 0 && !col_idx) return fail(SPATTN_ERR_INVALID_ARG, "col_idx is NULL");
    const int64_t rows = (int64_t)num_masks * p.n;
    if (rows > SPATTN_NOALLOC_MAX_ROWS)
        return fail(SPATTN_ERR_UNSUPPORTED,
                    "spattn_fwd_noalloc: num_masks * n = %lld exceeds its fixed scratch of %d rows",
                    (long long)rows, SPATTN_NOALLOC_MAX_ROWS);
    if ((int64_t)p.B * p.H * p.n == 0) return SPATTN_OK;
    cudaStream_t s = (cudaStream_t)stream_v;
    int dev, sms;
    CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    int32_t* scratch = nullptr;  // [0]: long-row count, [1 ..]: long-row list
    if ((r = noalloc_setup(dev, &scratch, &sms))) return r;
    p.num_masks = num_masks;
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
    p.nnz = nnz;
    // the array keeps the previous call's contents: the counter must restart at 0
    CUDA_TRY(cudaMemsetAsync(scratch, 0, sizeof(int32_t), s), "clearing the no-alloc counter");
    CUDA_TRY(launch_classify_long_rows(row_ptr, rows, nnz, scratch + 1, scratch, s),
             "long-row classification");
    p.long_rows = scratch + 1;
    p.long_count_dev = scratch;
    p.long_count_host = -1;
    return launch_fwd(p, dtype, d, sms, s);
}

int spattn_check_device_error(void* stream_v) { return spattn_device_error(stream_v, nullptr); }

int spattn_device_error(void* stream_v, uint32_t* flags) {
    g_msg[0] = 0;
    unsigned v = 0;
    cudaError_t e = read_and_clear_device_error(&v, (cudaStream_t)stream_v);
    if (flags) *flags = v;
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error flag");
    if (v & kErrTimeout) return fail(SPATTN_ERR_TIMEOUT, "a bounded wait in the tensor-core kernel expired");
    if (v & kErrBadColumn) return fail(SPATTN_ERR_BAD_CSR, "a column index outside [0, n) was skipped");
    return SPATTN_OK;
}

}  // extern "C"
