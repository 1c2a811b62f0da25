// Persistent, warp-specialised tensor-core forward for d = 32, 64 and 128
// (tcgen05 MMAs with TMEM accumulators, TMA tile loads without multicast,
// sm_100a).
//
// One CTA per SM works through items (a 128-row query block and its key
// tiles). Three warpgroups:
//   warp 0      additive-term producer (one thread): the blocks of the
//               additive terms per tile by TMA (only in the build with them)
//   warp 1      item taker and Q producer (one thread): takes each slot's next
//               item, hands it over through a small ring in shared memory, and
//               loads its Q tile
//   warps 2, 3  MMA issuers of slots 0 and 1 (one warp each, one elected lane
//               issuing), which also load their slot's K and V tiles
//   warps 4-7   softmax group of slot 0 (one query row per thread)
//   warps 8-11  softmax group of slot 1
// (the first warpgroup gives registers to the other two: 96 per thread
// against 200). The two slots hold one item each, with their own Q, K and V
// buffers in shared memory and their own S and O in tensor memory: slot s has
// S in two 64-key halves at columns [256 s, 256 s + 64) and [256 s + 64,
// 256 s + 128) and O at [256 s + 128, 256 s + 128 + d); P, in bf16, overwrites
// the first 32 columns of its half. For tile g the issuer computes S_h(g) =
// Q K_h(g)^T for both halves; once the softmax group has turned half h into
// P, O (+)= P_h V_h, and as soon as that product is complete, S_h(g + 1) into
// the freed half -- so while the softmax group works on one half, the tensor
// cores compute the other half's S (and the other slot's work): the softmax
// group waits for S only when the tensor cores or the loads fall behind.
// After an item's last tile the issuer starts the next item's S at once when
// its Q and K are in, else at that item's start. The build for closed-form
// masks (CF), whose items have one or two tiles, computes S of a tile as one
// N = 128 product once the previous tile's P_b V_b is complete instead. The producers poll with
// non-blocking barrier tests and sleep briefly when nothing is free (they
// share sub-partitions with softmax warps). Items come either from a counter
// shared by all CTAs, taken in order as slots free up, or from a fixed share
// per CTA. Every wait is bounded.
//
// The end of an item goes through the warps' staging buffers in shared
// memory, so that its global writes (and the reads of published states)
// cover whole 128-byte lines.
//
// Per half, each thread streams its row of S 32 keys at a time (the next
// chunk's TMEM load in flight): scale, entries the mask does not list to -inf,
// p = 2^(x - m_ref) against a running reference max, row sum, bf16 P back to
// TMEM. The reference only moves when a chunk's max exceeds it by more than
// 2^8; then the half's P chunk already written, the sum and O are rescaled by
// exp2(m_old - m_new) (the streaming-dataflow SDPA paper's delta rescaling,
// applied lazily; exact in exact arithmetic). A warp skips the 32-key chunks in
// which none of its rows has an entry (no TMEM load, no exp; P is zero there).
//
// With an additive mask or bias (d <= 64, interval masks), the producer also
// loads each tile's block of the additive terms into the slot's shared memory
// (by TMA, with the K tile's timing), and the softmax group adds it before the
// row max; with key lengths, tiles at or past a batch element's length are
// dropped from the end of each list and the cut tile is masked.
//
// Two sources of work items:
//   interval masks (sliding, variable window, dense): every (b, h, query
//     block) with tiles; per-row bits from the row's run; rows that also have
//     gathered entries merge the gather kernel's partial state;
//   block + strided + global masks in closed form (bsg_plan.cuh), taken from
//     the counter: residue-permuted blocks (read through five-dimensional
//     tensor maps) publish the fp32 state (m, l, O) of their rows and count
//     their four warps in; regular query blocks (block 0 of a mask with
//     global rows split into chunks, merged by the warp that completes a
//     per-(b, h, warp) count) start each row from the published state of its
//     permuted part -- O loaded into TMEM, m and l into registers -- so that
//     the rest of the row accumulates on top of it (the running-max /
//     running-sum combination of two partial states of the streaming-dataflow
//     SDPA paper, done inside the accumulator). The order of the items puts a
//     head's permuted blocks well ahead of its regular ones, and a block only
//     ever waits for earlier-taken ones.
#include "spattn_internal.cuh"
#include "sm100_ptx.cuh"
#include "bsg_plan.cuh"

#include <math.h>
#include <mutex>

namespace spattn {
namespace {

using namespace sm100;

constexpr int kPpThreads = 384;
// registers per thread after the split (launched with 168: 384 x 168 = 64,512
// >= 128 x 96 + 256 x 200 = 63,488; per SM sub-partition, warps w, w + 4,
// w + 8: (96 + 2 x 200) x 32 <= 16,384)
constexpr int kPpRegsLow = 96;
constexpr int kPpRegsHigh = 200;
constexpr uint32_t kPpTmemCols = 512;
constexpr float kPpRescale = 8.0f;               // log2 units
constexpr long long kPpDrainCycles = 200000000LL;  // ~0.1 s per drain wait

// mbarriers of slot s: kBarsPerSlot * s + one of these
// (S, P and their "free" barriers come per 64-key half: half h at + h)
enum : int {
    kQFull = 0, kQEmpty, kKFull, kKEmpty, kVFull, kVEmpty, kSFull, kSFullB, kPFull, kPFullB, kSFree, kSFreeB,
    kODone, kDrainS, kAFull, kAEmpty, kBarsPerSlot
};
constexpr int kNumBars = 2 * kBarsPerSlot;

template <int D, bool EXTRA>
struct PpCfg {
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
    static_assert(!EXTRA || D <= 64, "additive terms: d <= 64");
    static constexpr int CHUNK_ELEMS = D >= 64 ? 64 : D;  // bf16 per swizzled row
    static constexpr int ROW_BYTES = CHUNK_ELEMS * 2;     // 128 or 64
    static constexpr int NCHUNK = D / CHUNK_ELEMS;
    static constexpr int CHUNK_BYTES = 128 * ROW_BYTES;   // 128 rows of one column chunk
    static constexpr int TILE_BYTES = NCHUNK * CHUNK_BYTES;
    static constexpr int SBO = 8 * ROW_BYTES;
    static constexpr int KSTEPS_PER_CHUNK = CHUNK_ELEMS / 16;
    static constexpr cute::UMMA::LayoutType LAYOUT =
        D >= 64 ? cute::UMMA::LayoutType::SWIZZLE_128B : cute::UMMA::LayoutType::SWIZZLE_64B;
    static constexpr int OFF_Q = 0;                    // [slot]
    static constexpr int OFF_K = 2 * TILE_BYTES;       // [slot]
    static constexpr int OFF_V = 4 * TILE_BYTES;       // [slot]
    // additive terms: [slot][term] 128 rows x 128 keys bf16 as two 64-key
    // chunks of 128-byte rows (128-byte swizzle)
    static constexpr int A_BYTES = 2 * 128 * 128;
    static constexpr int OFF_A = 6 * TILE_BYTES;
    // per softmax warp a 4 KB buffer through which the epilogue's global
    // accesses go as whole lines (when it fits beside the tiles)
    static constexpr int STG_BYTES = 8 * 4096;
    // [slot][4] decoded items (8 words), [slot] counts; then per softmax warp a
    // FIFO of published permuted blocks: [8][4] count offsets, [8] pushed,
    // [8] counted in, one count of warps done
    static constexpr int RING_BYTES = 2 * 4 * 8 * 4 + 16 + 8 * 4 * 4 + 8 * 4 + 8 * 4 + 16;
    static constexpr bool STAGE = OFF_A + (EXTRA ? 4 * A_BYTES : 0) + STG_BYTES + kNumBars * 8 + 16 + RING_BYTES <= 227 * 1024;
    static constexpr int OFF_STG = OFF_A + (EXTRA ? 4 * A_BYTES : 0);
    static constexpr int OFF_BAR = OFF_STG + (STAGE ? STG_BYTES : 0);
    static constexpr int OFF_INT = OFF_BAR + kNumBars * 8;  // TMEM base, abort flag
    static constexpr int OFF_RING = OFF_INT + 16;
    // at least 116 KB, so that one CTA (which takes all 512 TMEM columns) runs per SM
    static constexpr int SMEM_BYTES = OFF_RING + RING_BYTES > 116 * 1024 ? OFF_RING + RING_BYTES : 116 * 1024;
};

// A work item as every role sees it.
struct PpItem {
    int bh, b, h;
    int perm;           // closed form: permuted block
    int qb;             // query block (permuted: residue)
    int pqb;            // permuted: block of positions
    int chunk;          // closed form: chunk of query block 0
    int u0;             // closed form: first tile of the chunk
    int T;              // tiles
    int64_t blk;        // interval masks: mask block (mask * nqb + qb)
};

// Keys of batch element b: [0, L), L = n without key lengths.
__device__ __forceinline__ int pp_key_limit(const PpParams& P, int b) {
    if (!P.seqlen_k) return P.n;
    const int L = __ldg(P.seqlen_k + b);
    return L < 0 ? 0 : (L > P.n ? P.n : L);
}

// Item x (below n_items, which stays below 2^31).
__device__ __forceinline__ PpItem pp_item(const PpParams& P, const bsg::Shape& sh, int64_t x) {
    PpItem it;
    it.perm = 0;
    it.pqb = 0;
    it.chunk = 0;
    it.u0 = 0;
    it.blk = 0;
    it.T = 0;
    if (P.mode == 0) {
        it.bh = (int)x / P.nqb;
        it.qb = (int)x - it.bh * P.nqb;
        it.b = it.bh / P.H;
        it.h = it.bh - it.b * P.H;
        const int mk = P.num_masks == 1 ? 0 : it.b;
        it.blk = (int64_t)mk * P.nqb + it.qb;
        it.T = __ldg(P.itv_ntiles + it.blk);
        if (P.seqlen_k && it.T > 1) {  // tiles past the key length go (ascending key tiles; one stays)
            const int L = pp_key_limit(P, it.b);
            while (it.T > 1 && (__ldg(P.itv_tiles + it.blk * P.nkt + it.T - 1) & 0x7fffffff) * 128 >= L) --it.T;
        }
    } else {
        const bsg::Item bi = bsg::item(sh, x, P.B * P.H);
        it.bh = bi.bh;
        it.b = bi.bh / P.H;
        it.h = bi.bh - it.b * P.H;
        it.perm = bi.perm;
        it.qb = bi.qb;
        it.pqb = bi.pqb;
        it.chunk = bi.chunk;
        it.u0 = bi.u0;
        it.T = bi.T;
    }
    return it;
}

// Ring entries: the decoded item as eight words (bh, b, h, qb, pqb, chunk,
// u0, T with the permuted flag in bit 30; word 7 = -1 after the last item).
__device__ __forceinline__ void ring_put(volatile int* e, const PpItem& it) {
    e[0] = it.bh;
    e[1] = it.b;
    e[2] = it.h;
    e[3] = it.qb;
    e[4] = it.pqb;
    e[5] = it.chunk;
    e[6] = it.u0;
    e[7] = it.T | (it.perm << 30);
}
__device__ __forceinline__ bool ring_get(const PpParams& P, const volatile int* e, PpItem& it) {
    const int w7 = e[7];
    if (w7 < 0) return false;
    it.bh = e[0];
    it.b = e[1];
    it.h = e[2];
    it.qb = e[3];
    it.pqb = e[4];
    it.chunk = e[5];
    it.u0 = e[6];
    it.T = w7 & 0x3fffffff;
    it.perm = (w7 >> 30) & 1;
    it.blk = (int64_t)(P.num_masks == 1 ? 0 : it.b) * P.nqb + it.qb;
    return true;
}

// Key tile u of the item: the key tile index, with kTileDenseBit set when
// every entry of the tile is present (interval masks only).
__device__ __forceinline__ int pp_tile(const PpParams& P, const bsg::Shape& sh, const PpItem& it, int u) {
    if (P.mode == 0) return __ldg(P.itv_tiles + it.blk * P.nkt + u);
    bsg::Item bi;
    bi.bh = it.bh;
    bi.perm = it.perm;
    bi.qb = it.qb;
    bi.pqb = it.pqb;
    bi.chunk = it.chunk;
    bi.u0 = it.u0;
    bi.T = it.T;
    return bsg::key_tile(sh, bi, u);
}

// Bounded wait that also gives up as soon as another thread of the CTA has.
__device__ __forceinline__ bool pp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            *abort_flag = 1;
            return false;
        }
    }
}

template <int R>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

__device__ __forceinline__ void st_release_cta(volatile int* p, int v) {
    asm volatile("st.release.cta.shared.b32 [%0], %1;" ::"r"(smem_u32((const void*)p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(volatile int* p) {
    int v;
    asm volatile("ld.acquire.cta.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32((const void*)p)) : "memory");
    return v;
}

// Bring `bytes` (a multiple of 16, 16-byte aligned) starting at p into L2.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Release / acquire fence at GPU scope (ordering, not sequential consistency).
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
    return v;
}

// Rows between registers (lane = row) and global memory through a warp's
// 4 KB shared-memory buffer, so that each global instruction of the warp
// covers whole lines (128 / (16 UNITS) rows of 16 UNITS bytes) instead of one
// 16-byte piece in each of 32 lines. Unit u of row r sits at
// r * 128 + ((u ^ (r & 7)) << 4), which keeps both the row-per-lane and the
// line-per-lane-group accesses free of bank conflicts. A row address of 0
// skips the row. All 32 lanes take part.
template <int UNITS>
__device__ __forceinline__ void rows_store(uint32_t stg, int lane, const uint32_t (&w)[4 * UNITS], uint64_t dst) {
    static_assert(UNITS == 4 || UNITS == 8, "row pieces of 64 or 128 bytes");
#pragma unroll
    for (int u = 0; u < UNITS; ++u)
        st_shared_v4(stg + lane * 128 + ((u ^ (lane & 7)) << 4), make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]));
    __syncwarp();
    constexpr int RPI = 32 / UNITS;  // rows per instruction
    const int u = lane % UNITS;
#pragma unroll
    for (int k = 0; k < UNITS; ++k) {
        const int r = RPI * k + lane / UNITS;
        const uint64_t p = __shfl_sync(0xffffffffu, dst, r);
        const uint4 v = ld_shared_v4(stg + r * 128 + ((u ^ (r & 7)) << 4));
        if (p) *reinterpret_cast<uint4*>(p + u * 16) = v;
    }
    __syncwarp();
}

// The D fp32 values of each of the warp's 32 rows (row address src per lane,
// 0: zeros) from global memory (read at L2, written by another CTA) into the
// TMEM columns tO .. tO + D - 1 of the lane's row. All of the warp's line
// loads are in flight together (one round trip to L2); each 32-column chunk
// then reaches its row's lane through the staging buffer. (The
// lines are read once, but dropping them from L2 unwritten corrupted reads
// of neighbouring lines still in flight, so they are left to age out.)
template <int D>
__device__ __forceinline__ void rows_to_tmem(uint32_t stg, int lane, uint64_t src, uint32_t tO) {
    constexpr int CB = D >= 64 ? 2 : 1;  // chunks whose loads are in flight together
    const int u = lane & 7;
    uint64_t p[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) p[k] = __shfl_sync(0xffffffffu, src, 4 * k + (lane >> 3));
#pragma unroll
    for (int c0 = 0; c0 < D / 32; c0 += CB) {
        uint4 v[CB][8];
#pragma unroll
        for (int c = 0; c < CB; ++c)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                v[c][k] = p[k] ? __ldcg(reinterpret_cast<const uint4*>(p[k] + (c0 + c) * 128 + u * 16))
                               : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int c = 0; c < CB; ++c) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int r = 4 * k + (lane >> 3);
                st_shared_v4(stg + r * 128 + ((u ^ (r & 7)) << 4), v[c][k]);
            }
            __syncwarp();
            uint32_t w[32];
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) {
                const uint4 x = ld_shared_v4(stg + lane * 128 + ((uu ^ (lane & 7)) << 4));
                w[4 * uu] = x.x;
                w[4 * uu + 1] = x.y;
                w[4 * uu + 2] = x.z;
                w[4 * uu + 3] = x.w;
            }
            __syncwarp();
            tmem_st32(tO + 32 * (c0 + c), w);
        }
    }
}

// 32 columns of this warp's rows of O (fp32, not yet divided by L) from TMEM.
__device__ __forceinline__ void o_chunk(uint32_t tO, int c, float (&x)[32]) {
    tmem_ld32f(tO + 32 * c, x);
    tmem_wait_ld_depf(x);
}

// Output piece p (64 columns, or 32 when D == 32) of the rows whose address
// orow is not 0: bf16(x * inv), round to nearest even.
template <int D, bool STAGE>
__device__ __forceinline__ void put_out_piece(uint64_t orow, int p, float inv, const float (&xa)[32], const float (&xb)[32],
                                              uint32_t stg, int lane) {
    constexpr int CW = D >= 64 ? 64 : 32;
    uint32_t w[CW / 2];
#pragma unroll
    for (int k = 0; k < CW / 2; ++k) {
        const float x0 = k < 16 ? xa[2 * k] : xb[2 * k - 32], x1 = k < 16 ? xa[2 * k + 1] : xb[2 * k - 31];
        __nv_bfloat162 hv = __floats2bfloat162_rn(x0 * inv, x1 * inv);
        w[k] = *reinterpret_cast<uint32_t*>(&hv);
    }
    const uint64_t dst = orow ? orow + (uint64_t)p * CW * 2 : 0ull;
    if (STAGE) {
        rows_store<CW / 8>(stg, lane, w, dst);
    } else if (dst) {
#pragma unroll
        for (int u = 0; u < CW / 8; ++u)
            *reinterpret_cast<uint4*>(dst + u * 16) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    }
}

// The end of one item for one warp's rows: state (M, L) in base 2 in
// registers, O (not yet divided by L) in TMEM at tO, streamed 32 columns at a
// time. Interval masks merge the gather kernel's partial state where there is
// one; chunks of a split block merge through the chunk states; a permuted
// block publishes its rows' state; the rest writes the rows. All 32 lanes
// take part; with STAGE the published rows and the output rows move as whole
// lines through the warp's staging buffer stg.
template <int D, bool STAGE>
__device__ __forceinline__ void pp_finish(const PpParams& P, const bsg::Shape& sh, const PpItem& it, int quarter, int t, int i,
                          bool row_ok, float M, float L, uint32_t tO, uint32_t stg, volatile int* pubq) {
    const int lane = threadIdx.x & 31;
    const int64_t bh = it.bh;
    const uint64_t orow_any = reinterpret_cast<uint64_t>(reinterpret_cast<__nv_bfloat16*>(P.out) + (int64_t)it.b * P.o_sb +
                                                         (int64_t)it.h * P.o_sh + (int64_t)(row_ok ? i : 0) * P.o_sn);
    if (P.mode == 0) {
        const int64_t wrow = bh * P.n + (row_ok ? i : 0);
        // rows that also have gathered entries: the gather kernel's partial state
        const bool gm = row_ok && P.blk_res && __ldg(P.blk_res + it.blk) && P.ws_ml[wrow * 2 + 1] > 0.f;
        float fa = 1.f, fg = 0.f;
        if (gm) {
            const float mg = P.ws_ml[wrow * 2], lg = P.ws_ml[wrow * 2 + 1];
            const float Mn = fmaxf(M, mg);
            const float Mu = Mn == -INFINITY ? 0.f : Mn;
            fa = ex2(M - Mu);
            fg = ex2(mg - Mu);
            L = L * fa + lg * fg;
            M = Mn;
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const float* acc = P.ws_acc + wrow * D;
#pragma unroll
        for (int p = 0; p < (D >= 64 ? D / 64 : 1); ++p) {
            float xa[32], xb[32];
            o_chunk(tO, (D >= 64 ? 2 : 1) * p, xa);
            if (D >= 64) o_chunk(tO, 2 * p + 1, xb);
            if (gm) {
#pragma unroll
                for (int z = 0; z < 32; ++z) {
                    xa[z] = fmaf(acc[(D >= 64 ? 64 : 32) * p + z], fg, xa[z] * fa);
                    if (D >= 64) xb[z] = fmaf(acc[64 * p + 32 + z], fg, xb[z] * fa);
                }
            }
            put_out_piece<D, STAGE>(row_ok ? orow_any : 0ull, p, inv, xa, xb, stg, lane);
        }
        if (row_ok && P.lse) P.lse[bh * P.n + i] = L > 0.f ? (M + lg2(L)) * kLn2 : -INFINITY;
        return;
    }

    if (!it.perm && sh.nch > 1 && it.qb == 0) {
        // one chunk of the global-row block: publish its state, and the warp
        // that completes this quarter's count merges all chunks' states into
        // its O (the layout (chunk, value, row) keeps the accesses on whole lines)
        float* mine = P.cws + ((bh * sh.nch + it.chunk) * (int64_t)(D + 2)) * 128 + t;
        mine[0] = M;
        mine[128] = L;
        if (__any_sync(0xffffffffu, L > 0.f)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                float x[32];
                o_chunk(tO, c, x);
                if (L > 0.f) {
#pragma unroll
                    for (int z = 0; z < 32; ++z) mine[(int64_t)(2 + 32 * c + z) * 128] = x[z];
                }
            }
        }
        __threadfence();
        __syncwarp();
        unsigned last = 0;
        if (lane == 0) last = atomicAdd(P.ccnt + bh * 4 + quarter, 1u) == (unsigned)(sh.nch - 1);
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) return;
        __threadfence();
        const float* base = P.cws + (bh * sh.nch * (int64_t)(D + 2)) * 128 + t;
        const int64_t rec = (int64_t)(D + 2) * 128;  // floats per chunk record
        float Mf = -INFINITY;
        for (int c = 0; c < sh.nch; ++c)
            if (__ldcg(base + c * rec + 128) > 0.f) Mf = fmaxf(Mf, __ldcg(base + c * rec));
        float Lf = 0.f;
        for (int c = 0; c < sh.nch; ++c) {
            const float lc = __ldcg(base + c * rec + 128);
            if (lc > 0.f) Lf += lc * ex2(__ldcg(base + c * rec) - Mf);
        }
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
            float acc[32];
#pragma unroll
            for (int z = 0; z < 32; ++z) acc[z] = 0.f;
            for (int c = 0; c < sh.nch; ++c) {
                const float lc = __ldcg(base + c * rec + 128);
                if (!(lc > 0.f)) continue;
                const float wgt = ex2(__ldcg(base + c * rec) - Mf);
                const float* src = base + c * rec + (int64_t)(2 + 32 * cc) * 128;
#pragma unroll
                for (int z = 0; z < 32; ++z) acc[z] = fmaf(__ldcg(src + (int64_t)z * 128), wgt, acc[z]);
            }
            uint32_t w[32];
#pragma unroll
            for (int z = 0; z < 32; ++z) w[z] = __float_as_uint(acc[z]);
            tmem_st32(tO + 32 * cc, w);
        }
        tmem_wait_st();
        M = Mf;
        L = Lf;
    }
    if (it.perm) {
        // a permuted block publishes the state of its rows (their regular
        // block starts from it); the count of its four warps releases it
        const bool pr = row_ok && bsg::has_perm(sh, i);
        const int64_t prow = bh * P.n + (pr ? i : 0);
        if (pr) {
            P.pml[prow * 2] = M;
            P.pml[prow * 2 + 1] = L;
        }
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            float x[32];
            o_chunk(tO, c, x);
            if (STAGE) {
                uint32_t w[32];
#pragma unroll
                for (int z = 0; z < 32; ++z) w[z] = __float_as_uint(x[z]);
                rows_store<8>(stg, lane, w, pr ? reinterpret_cast<uint64_t>(P.pacc + prow * D + 32 * c) : 0ull);
            } else if (pr) {
#pragma unroll
                for (int z = 0; z < 32; z += 4)
                    *reinterpret_cast<float4*>(P.pacc + prow * D + 32 * c + z) = make_float4(x[z], x[z + 1], x[z + 2], x[z + 3]);
            }
        }
        // queue the block's count for the item-taker thread, which counts this
        // warp in after a fence at GPU scope (off this warp's path): lane 0
        // releases the queue entry at CTA scope after the barrier that orders
        // every lane's stores (lanes wrote other rows' lines) before it
        __syncwarp();
        if (lane == 0) {
            const int w = (threadIdx.x >> 5) - 4;
            volatile int* pushed = pubq + 32 + w;
            volatile int* counted = pubq + 40 + w;
            const int n = *pushed;
            if (n - *counted >= 4) {  // the queue is full: wait (bounded) for the taker
                const long long t0 = clock64();
                while (n - ld_acquire_cta(counted) >= 4) {
                    if (clock64() - t0 > P.wait_cycles) {
                        atomicOr(P.err, kErrTimeout);
                        break;
                    }
                    __nanosleep(64);
                }
            }
            pubq[w * 4 + (n & 3)] = (int)((bh * sh.npqb + it.pqb) * 128 + it.qb);
            st_release_cta(pushed, n + 1);
        }
        __syncwarp();
        return;
    }
    // a regular block's rows: the output (their permuted part, if any, is in O already)
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll 1
    for (int p = 0; p < (D >= 64 ? D / 64 : 1); ++p) {
        float xa[32], xb[32];
        o_chunk(tO, (D >= 64 ? 2 : 1) * p, xa);
        if (D >= 64) o_chunk(tO, 2 * p + 1, xb);
        put_out_piece<D, STAGE>(row_ok ? orow_any : 0ull, p, inv, xa, xb, stg, lane);
    }
    if (row_ok && P.lse) P.lse[bh * P.n + i] = L > 0.f ? (M + lg2(L)) * kLn2 : -INFINITY;
}

template <int D, bool EXTRA, bool CF>
__global__ void __launch_bounds__(kPpThreads, 1)
    k_fwd_pp(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQp,
             const __grid_constant__ CUtensorMap tmKp, const __grid_constant__ CUtensorMap tmVp,
             const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
             const PpParams P) {
    using C = PpCfg<D, EXTRA>;
    // CF: the build for closed-form masks (no additive terms there)
    static_assert(!(CF && EXTRA), "closed-form masks carry no additive terms");
    constexpr int NSTREAM = EXTRA ? 4 : 3;  // producer streams: Q, K, V (, additive terms)
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (smem_u32(smem) & 1023u) {  // the swizzled layouts need a 1024-byte aligned base
        if (tid == 0) atomicOr(P.err, kErrTimeout);
        return;
    }
    const bsg::Shape sh = bsg::shape(P.n, P.blk, P.S, P.ng, P.chunk_tiles);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_INT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_INT + 4);
    auto bar = [&](int s, int which) { return smem_u32(bars + s * kBarsPerSlot + which); };
    const uint32_t sQ0 = smem_u32(smem + C::OFF_Q), sK0 = smem_u32(smem + C::OFF_K),
                   sV0 = smem_u32(smem + C::OFF_V);
    // per slot a ring of the items it has taken (the m-th at entry m & 3, -1
    // after the last), written by the producer before it arms the slot's QFull
    // barrier for that item and before it raises the slot's count of entries
    // (the softmax warps go by the count: the producer may be two Q loads
    // ahead of them, where a barrier's phase parity would not tell)
    volatile int* ring = reinterpret_cast<volatile int*>(smem + C::OFF_RING);  // [slot][4][8]
    volatile int* ring_n = reinterpret_cast<volatile int*>(smem + C::OFF_RING + 2 * 4 * 8 * 4);
    // per softmax warp w a queue of the permuted blocks it published: entries
    // pubq[4 w .. 4 w + 3] (count offsets), pushed pubq[32 + w], counted in
    // pubq[40 + w]; pubq[48]: softmax warps done
    volatile int* pubq = ring_n + 4;
    auto entry = [&](int s, uint32_t m) { return ring + (s * 4 + (int)(m & 3u)) * 8; };

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kPpTmemCols);
    if (tid == 0) {
        for (int s = 0; s < 2; ++s)
            for (int x = 0; x < kBarsPerSlot; ++x)
                mbar_init(bar(s, x), (x == kPFull || x == kPFullB || x == kAEmpty) ? 4u : 1u);
        *abort_flag = 0;
        ring_n[0] = ring_n[1] = 0;
        for (int x = 32; x < 49; ++x) pubq[x] = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        if (P.mode == 1 && P.S) {
            prefetch_tensormap(&tmQp);
            prefetch_tensormap(&tmKp);
            prefetch_tensormap(&tmVp);
        }
        if (EXTRA && P.extra[0]) prefetch_tensormap(&tmA0);
        if (EXTRA && P.extra[1]) prefetch_tensormap(&tmA1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        regs_dec<kPpRegsLow>();
    }
    if (warp == 1) {
        // ------------------------------------------------------------ Q producer
        if (lane == 0) {
            // per slot: items taken (qm), whether the end was reached
            int qm[2] = {0, 0};
            bool qend[2] = {false, false};
            int64_t scur[2] = {0, 0};  // static order: the slot's next position
            // the next item with tiles for slot s, or -1: from the claim counter
            // (items in order over all CTAs), else CTA c's static share
            auto take = [&](int s, PpItem& it) -> bool {
                while (true) {
                    int64_t x;
                    if (P.claim) {
                        x = (int64_t)atomicAdd(P.claim, 1ull);
                    } else {
                        x = (int64_t)blockIdx.x + (2 * scur[s] + s) * (int64_t)gridDim.x;
                        ++scur[s];
                    }
                    if (x >= P.n_items) return false;
                    it = pp_item(P, sh, x);
                    if (it.T > 0) return true;
                }
            };
            int counted[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // per softmax warp: blocks counted in
            long long t_last = clock64();
            while (true) {
                bool any = false, progress = false;
                // count in the permuted blocks the softmax warps published: one
                // fence at GPU scope after acquiring their queues, then the counts
                {
                    int pushed[8];
                    bool work = false;
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        pushed[w] = ld_acquire_cta(pubq + 32 + w);
                        work |= pushed[w] != counted[w];
                    }
                    if (work) {
                        fence_acq_rel_gpu();
#pragma unroll
                        for (int w = 0; w < 8; ++w) {
                            for (; counted[w] != pushed[w]; ++counted[w])
                                atomicAdd(P.pflag + pubq[4 * w + (counted[w] & 3)], 1u);
                            st_release_cta(pubq + 40 + w, counted[w]);
                        }
                        progress = true;
                    }
                }
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    if (qend[s]) continue;
                    any = true;
                    // take the slot's next item once its Q buffer is free
                    if (qm[s] != 0 && !mbar_test(bar(s, kQEmpty), (qm[s] - 1) & 1)) continue;
                    PpItem it;
                    const bool got = take(s, it);
                    volatile int* e = entry(s, qm[s]);
                    const uint32_t fb = bar(s, kQFull);
                    if (!got) {
                        e[7] = -1;
                        qend[s] = true;
                        mbar_arrive(fb);  // the phase completes: the end is read
                    } else {
                        ring_put(e, it);
                        if (C::STAGE && P.mode == 1 && sh.G > 0 && !it.perm && it.chunk == 0) {
                            // a regular block that starts from its rows' published
                            // states (written long before; they may have left L2):
                            // bring the 128 rows' states, contiguous, into L2 now,
                            // one item before they are read
                            const int64_t row0 = (int64_t)it.bh * P.n + (int64_t)it.qb * 128;
                            prefetch_l2_bulk(P.pacc + row0 * D, 128u * D * 4u);
                            prefetch_l2_bulk(P.pml + row0 * 2, 128u * 8u);
                        }
                        const uint32_t dst = sQ0 + s * C::TILE_BYTES;
                        mbar_expect_tx(fb, C::TILE_BYTES);
#pragma unroll
                        for (int c = 0; c < C::NCHUNK; ++c) {
                            if (it.perm)
                                tma_load_5d(dst + c * C::CHUNK_BYTES, &tmQp, fb, c * C::CHUNK_ELEMS, it.qb, it.pqb * 128,
                                            it.h, it.b);
                            else
                                tma_load_4d(dst + c * C::CHUNK_BYTES, &tmQ, fb, c * C::CHUNK_ELEMS, it.qb * 128, it.h,
                                            it.b);
                        }
                    }
                    ++qm[s];
                    __threadfence_block();
                    ring_n[s] = qm[s];
                    progress = true;
                }
                // done once every item is handed out and every softmax warp has
                // finished (its last publication counted in above)
                if (!any && ld_acquire_cta(pubq + 48) == 8) {
                    bool drained = true;
#pragma unroll
                    for (int w = 0; w < 8; ++w) drained &= ld_acquire_cta(pubq + 32 + w) == counted[w];
                    if (drained) break;
                    continue;
                }
                if (progress) {
                    t_last = clock64();
                } else {
                    // no back-off: a slot's next item goes out the moment its Q
                    // buffer frees (sleeping up to 256 ns here measured ~1 % slower)
                    if (*abort_flag) break;
                    if (clock64() - t_last > P.wait_cycles) {
                        *abort_flag = 1;
                        break;
                    }
                }
            }
            // no load may outlive the CTA (a slot that reached its end had its last Q consumed)
#pragma unroll
            for (int s = 0; s < 2; ++s)
                if (!qend[s] && qm[s]) mbar_wait_bounded(bar(s, kQFull), (qm[s] - 1) & 1, kPpDrainCycles);
        }
    } else if (warp == 0) {
        // ------------------------------------------------------------ additive-term producer
        if (lane == 0) {
            // per slot, the additive terms' blocks per tile (only with additive
            // terms; the stream index 3 of a per-slot set whose K and V streams
            // are left to the MMA issuers) walk the slot's items from the ring:
            // item km, tile ku, loads issued
            int km[2][NSTREAM], ku[2][NSTREAM];
            uint32_t cnt[2][NSTREAM];
            bool live[2][NSTREAM];
            // bytes of one tile's additive blocks (two 64-key chunks per term)
            const uint32_t a_bytes = EXTRA ? (uint32_t)((P.extra[0] ? P.a_rows[0] : 0) + (P.extra[1] ? P.a_rows[1] : 0)) *
                                                 256u
                                           : 0u;
#pragma unroll
            for (int s = 0; s < 2; ++s)
#pragma unroll
                for (int k = 0; k < NSTREAM; ++k) {
                    km[s][k] = ku[s][k] = 0;
                    cnt[s][k] = 0;
                    live[s][k] = k == 3;  // K and V are loaded by the slots' MMA issuers
                }
            long long t_last = clock64();
            unsigned nap = 0;  // back-off when a pass finds nothing to load
            while (true) {
                bool any = false, progress = false;
                const int rn[2] = {ring_n[0], ring_n[1]};
                __threadfence_block();  // the entries below the counts are written
#pragma unroll
                for (int s = 0; s < 2; ++s) {
#pragma unroll
                    for (int k = 1; k < NSTREAM; ++k) {
                        if (!live[s][k]) continue;
                        any = true;
                        if (km[s][k] >= rn[s]) continue;  // its next item is not taken yet
                        PpItem it;
                        if (!ring_get(P, entry(s, km[s][k]), it)) {
                            live[s][k] = false;
                            continue;
                        }
                        const int eb = k == 1 ? kKEmpty : (k == 2 ? kVEmpty : kAEmpty);
                        if (cnt[s][k] != 0 && !mbar_test(bar(s, eb), (cnt[s][k] - 1) & 1)) continue;
                        const uint32_t fb = bar(s, k == 1 ? kKFull : (k == 2 ? kVFull : kAFull));
                        const int kt = pp_tile(P, sh, it, ku[s][k]) & 0x7fffffff;
                        if (k < 3) {
                            const uint32_t dst = (k == 1 ? sK0 : sV0) + s * C::TILE_BYTES;
                            mbar_expect_tx(fb, C::TILE_BYTES);
                            const CUtensorMap* map = it.perm ? (k == 1 ? &tmKp : &tmVp) : (k == 1 ? &tmK : &tmV);
#pragma unroll
                            for (int c = 0; c < C::NCHUNK; ++c) {
                                if (it.perm)
                                    tma_load_5d(dst + c * C::CHUNK_BYTES, map, fb, c * C::CHUNK_ELEMS, it.qb, kt * 128,
                                                it.h, it.b);
                                else
                                    tma_load_4d(dst + c * C::CHUNK_BYTES, map, fb, c * C::CHUNK_ELEMS, kt * 128, it.h,
                                                it.b);
                            }
                        } else {
                            // the additive terms' blocks of this tile: term a at
                            // OFF_A + (2 s + a) A_BYTES, chunk c of a_rows[a] rows at
                            // c * a_rows[a] * 128 bytes
                            mbar_expect_tx(fb, a_bytes);
#pragma unroll
                            for (int a = 0; a < 2; ++a) {
                                if (!P.extra[a]) continue;
                                const uint32_t dst = smem_u32(smem + C::OFF_A + (2 * s + a) * C::A_BYTES);
                                const int r0 = P.a_rows[a] == 1 ? 0 : it.qb * 128;
                                const int hh = P.a_h[a] ? it.h : 0, bb = P.a_b[a] ? it.b : 0;
#pragma unroll
                                for (int c = 0; c < 2; ++c)
                                    tma_load_4d(dst + (uint32_t)(c * P.a_rows[a] * 128), a == 0 ? &tmA0 : &tmA1, fb,
                                                kt * 128 + c * 64, r0, hh, bb);
                            }
                        }
                        ++cnt[s][k];
                        if (++ku[s][k] == it.T) {
                            ku[s][k] = 0;
                            ++km[s][k];
                        }
                        progress = true;
                    }
                }
                if (!any) break;
                if (progress) {
                    t_last = clock64();
                    nap = 0;
                } else {
                    // a short sleep: the next buffer frees within microseconds, and
                    // spinning would take issue slots from the softmax warps
                    // sharing this sub-partition
                    nap = nap ? (nap < 64 ? 2 * nap : 64) : 16;
                    __nanosleep(nap);
                    if (*abort_flag) break;
                    if (clock64() - t_last > P.wait_cycles) {
                        *abort_flag = 1;
                        break;
                    }
                }
            }
            // no load may outlive the CTA: wait (bounded) for the last of each buffer
#pragma unroll
            for (int s = 0; s < 2; ++s)
#pragma unroll
                for (int k = 1; k < NSTREAM; ++k) {
                    const int full = k == 1 ? kKFull : (k == 2 ? kVFull : kAFull);
                    if (cnt[s][k]) mbar_wait_bounded(bar(s, full), (cnt[s][k] - 1) & 1, kPpDrainCycles);
                }
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------------------ MMA issuers
        // warp 2 issues slot 0's MMAs, warp 3 slot 1's (one thread each). Per
        // 128-key tile g and 64-key half h: S_h(g) = Q K_h(g)^T into the
        // half's S columns; once the softmax group has written P_h(g) (bf16, in
        // the first 32 of them), O (+)= P_h(g) V_h(g). S_h(g + 1) overwrites
        // P_h(g), so it waits for that product; it is issued right after it,
        // before the other half's product, so that the softmax group finds the
        // next half's S ready. The whole warp runs the loop (its values are
        // warp-uniform); one elected lane issues each MMA and commit, lane 0
        // each load.
        {
            const int s = warp - 2;
            const uint32_t tSm = tmem + (uint32_t)(s * 256), tOm = tSm + 128;
            // Items of the closed form have one or two tiles (a few have 8):
            // there S of a tile goes out as one N = 128 product after the
            // previous tile's P V, which issues fewer MMAs and measured
            // faster; the long items of interval masks gain more from S per
            // half, the next tile's first half computed during the softmax of
            // this tile's second
            constexpr bool full_s = CF;
            const uint32_t idS = idesc_bf16_f32(128, full_s ? 128 : 64, false);
            const uint32_t idO = idesc_bf16_f32(128, D, true);
            // shared-memory descriptors at the slot's Q and K buffers (K-major
            // operands) and V buffer (MN-major B); a k-step, a key half and a
            // column chunk add their byte offset / 16 to the start-address field
            const uint64_t dQK0 = smem_desc(sQ0, 16, C::SBO, C::LAYOUT);
            const uint64_t dQ = dQK0 + (uint64_t)((C::OFF_Q + s * C::TILE_BYTES) >> 4);
            const uint64_t dK = dQK0 + (uint64_t)((C::OFF_K + s * C::TILE_BYTES) >> 4);
            const uint64_t dV = smem_desc(sV0, C::CHUNK_BYTES, C::SBO, C::LAYOUT) + (uint64_t)((s * C::TILE_BYTES) >> 4);
            auto issue_s = [&](int h) {  // S_h of the tile whose K is in (full_s: both halves, h = 0)
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t off = (uint64_t)(((ks / C::KSTEPS_PER_CHUNK) * C::CHUNK_BYTES +
                                                     (ks % C::KSTEPS_PER_CHUNK) * 32) >> 4);
                    mma_bf16_ss_elect(tSm + (uint32_t)(64 * h), dQ + off, dK + off + (uint64_t)((64 * h * C::ROW_BYTES) >> 4),
                                      idS, ks > 0 ? 1u : 0u);
                }
                mma_commit_elect(bar(s, kSFull + h));
                if (full_s) mma_commit_elect(bar(s, kSFullB));
            };
            auto issue_pv = [&](int h, bool zero) {  // O (+)= P_h V_h (zero: O = the product)
                tc_fence_after();
#pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)  // 16 keys per step
                    mma_bf16_ts_elect(tOm, tSm + (uint32_t)(64 * h + 8 * ks),
                                     dV + (uint64_t)(((4 * h + ks) * 16 * C::ROW_BYTES) >> 4), idO,
                                     (zero && ks == 0) ? 0u : 1u);
                mma_commit_elect(bar(s, kSFree + h));
            };
            auto W = [&](int which, uint32_t phase) { return pp_wait(bar(s, which), phase & 1, abort_flag, P.wait_cycles); };
            // K or V tile u of item ti into the slot's buffer (its previous
            // contents already consumed)
            auto load = [&](bool isK, const PpItem& ti, int tu) {
                const uint32_t fb = bar(s, isK ? kKFull : kVFull);
                const uint32_t dst = (isK ? sK0 : sV0) + s * C::TILE_BYTES;
                const int kt = pp_tile(P, sh, ti, tu) & 0x7fffffff;
                const CUtensorMap* map = ti.perm ? (isK ? &tmKp : &tmVp) : (isK ? &tmK : &tmV);
                if (lane == 0) {
                    mbar_expect_tx(fb, C::TILE_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NCHUNK; ++c) {
                        if (ti.perm)
                            tma_load_5d(dst + c * C::CHUNK_BYTES, map, fb, c * C::CHUNK_ELEMS, ti.qb, kt * 128, ti.h, ti.b);
                        else
                            tma_load_4d(dst + c * C::CHUNK_BYTES, map, fb, c * C::CHUNK_ELEMS, kt * 128, ti.h, ti.b);
                    }
                }
                __syncwarp();
            };
            uint32_t g = 0;        // tiles of this slot so far
            uint32_t kc = 0, vc = 0;  // K and V tiles loaded so far (this thread issues them: it
                                      // knows the moment its MMAs free a buffer)
            bool s_ready = false;  // both halves of the current item's first S are issued
            bool alive = true;
            for (uint32_t m = 0; alive; ++m) {
                if (ring_n[s] <= (int)m) {
                    const long long t0 = clock64();
                    while (ring_n[s] <= (int)m) {
                        if (*abort_flag || clock64() - t0 > P.wait_cycles) {
                            *abort_flag = 1;
                            alive = false;
                            break;
                        }
                        __nanosleep(32);
                    }
                    if (!alive) break;
                }
                __threadfence_block();
                PpItem it;
                if (!ring_get(P, entry(s, m), it)) break;
                bsg::Item bi;
                bi.perm = it.perm;
                bi.chunk = it.chunk;
                const bool zero_first = !(C::STAGE && P.mode == 1 && bsg::starts_from_perm(sh, bi));
                // the first tile's K and V, unless loaded during the previous item
                if (kc == g) {
                    if (!(alive = g == 0 || W(kKEmpty, g - 1))) break;
                    load(true, it, 0);
                    ++kc;
                }
                if (vc == g) {
                    if (!(alive = g == 0 || W(kVEmpty, g - 1))) break;
                    load(false, it, 0);
                    ++vc;
                }
                if (!s_ready) {
                    alive = W(kQFull, m) && W(kKFull, g) && (g == 0 || W(full_s ? kSFreeB : kSFree, g - 1));
                    if (!alive) break;
                    issue_s(0);
                    if (!full_s) {
                        if (!(alive = g == 0 || W(kSFreeB, g - 1))) break;
                        issue_s(1);
                    }
                    mma_commit_elect(bar(s, kKEmpty));
                    if (it.T == 1) mma_commit_elect(bar(s, kQEmpty));
                }
                s_ready = false;
                for (int u = 0; u < it.T; ++u, ++g) {
                    // the next tile: this item's next one, or the next item's first
                    // once it is taken
                    PpItem tn;
                    int un = 0;
                    auto next_known = [&]() -> bool {
                        if (u + 1 < it.T) {
                            tn = it;
                            un = u + 1;
                            return true;
                        }
                        if (ring_n[s] <= (int)(m + 1)) return false;
                        __threadfence_block();
                        un = 0;
                        return ring_get(P, entry(s, m + 1), tn);
                    };
                    // K of the next tile as soon as S of this one is complete
                    if (kc == g + 1 && next_known()) {
                        if (!(alive = W(kKEmpty, g))) break;
                        load(true, tn, un);
                        ++kc;
                    }
                    if (!(alive = W(kPFull, g) && W(kVFull, g))) break;
                    issue_pv(0, u == 0 && zero_first);
                    if (kc == g + 1 && mbar_test(bar(s, kKEmpty), g & 1) && next_known()) {
                        load(true, tn, un);
                        ++kc;
                    }
                    // the next tile: this item's next one, or the next item's
                    // first when its Q and K are already in (else at its start)
                    bool nxt = false, nlast = false;
                    if (u + 1 < it.T) {
                        nxt = true;
                        nlast = u + 2 == it.T;
                    } else if (ring_n[s] > (int)(m + 1) && mbar_test(bar(s, kQFull), (m + 1) & 1) &&
                               mbar_test(bar(s, kKFull), (g + 1) & 1)) {
                        PpItem itn;
                        if (ring_get(P, entry(s, m + 1), itn)) {
                            nxt = true;
                            nlast = itn.T == 1;
                        }
                    }
                    // S_a(g + 1) before P_b V_b(g) when its K is already in (the
                    // softmax group turns to it next), else after
                    bool a_done = false;
                    if (nxt && !full_s) {
                        if (!(alive = W(kSFree, g))) break;
                        if (mbar_test(bar(s, kKFull), (g + 1) & 1)) {
                            issue_s(0);
                            a_done = true;
                        }
                    }
                    if (!(alive = W(kPFullB, g))) break;
                    issue_pv(1, false);
                    mma_commit_elect(bar(s, kVEmpty));
                    if (u + 1 == it.T) mma_commit_elect(bar(s, kODone));
                    if (nxt && full_s) {  // S(g + 1) once P_b V_b(g) has consumed the P it overwrites
                        if (!(alive = W(kKFull, g + 1) && W(kSFreeB, g))) break;
                        issue_s(0);
                        mma_commit_elect(bar(s, kKEmpty));
                        if (nlast) mma_commit_elect(bar(s, kQEmpty));
                        if (u + 1 == it.T) s_ready = true;
                    }
                    // V of the next tile as soon as P_b V_b of this one is complete
                    // (and K, if the next item was not taken earlier)
                    if (vc == g + 1 && next_known()) {
                        if (!(alive = W(kVEmpty, g))) break;
                        load(false, tn, un);
                        ++vc;
                        if (kc == g + 1) {
                            if (!(alive = W(kKEmpty, g))) break;
                            load(true, tn, un);
                            ++kc;
                        }
                    }
                    if (nxt && !full_s) {
                        if (!a_done) {
                            if (!(alive = W(kKFull, g + 1))) break;
                            issue_s(0);
                        }
                        if (!(alive = W(kSFreeB, g))) break;
                        issue_s(1);
                        mma_commit_elect(bar(s, kKEmpty));
                        if (nlast) mma_commit_elect(bar(s, kQEmpty));
                        if (u + 1 == it.T) s_ready = true;
                    }
                }
            }
            if (!alive) *abort_flag = 1;
            // every MMA this thread issued is complete before TMEM is released,
            // and no load it issued outlives the CTA
            mma_commit_elect(bar(s, kDrainS));
            mbar_wait_bounded(bar(s, kDrainS), 0u, kPpDrainCycles);
            if (kc) mbar_wait_bounded(bar(s, kKFull), (kc - 1) & 1, kPpDrainCycles);
            if (vc) mbar_wait_bounded(bar(s, kVFull), (vc - 1) & 1, kPpDrainCycles);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax groups
        regs_inc<kPpRegsHigh>();
        const int s = (warp - 4) >> 2;
        const int quarter = warp & 3;  // the TMEM lanes this warp may access
        const int t = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + (uint32_t)(s * 256) + lane_base, tO = tS + 128;
        const uint32_t stg = smem_u32(smem + C::OFF_STG) + (uint32_t)(warp - 4) * 4096u;
        uint32_t g = 0;            // tiles of this slot so far
        for (uint32_t m = 0;; ++m) {
            // the slot's m-th item, once the producer has taken it
            bool okq = true;
            if (ring_n[s] <= (int)m) {
                const long long t0 = clock64();
                while (ring_n[s] <= (int)m) {
                    if (*abort_flag || clock64() - t0 > P.wait_cycles) {
                        *abort_flag = 1;
                        okq = false;
                        break;
                    }
                    __nanosleep(32);
                }
            }
            if (!__all_sync(0xffffffffu, okq)) break;
            __threadfence_block();
            PpItem it;
            if (!ring_get(P, entry(s, m), it)) break;
            bsg::Item bi;
            bi.bh = it.bh;
            bi.perm = it.perm;
            bi.qb = it.qb;
            bi.pqb = it.pqb;
            bi.chunk = it.chunk;
            bi.u0 = it.u0;
            bi.T = it.T;
            int i;
            bool row_ok;
            int rlo = 0, rhi = 0;
            if (P.mode == 0) {
                i = it.qb * 128 + t;
                row_ok = i < P.n;
                if (row_ok) {
                    const int2 v = __ldg(P.itv_lohi + (it.blk / P.nqb) * P.n + i);
                    rlo = v.x;
                    rhi = v.y;
                }
            } else {
                i = bsg::row_of(sh, bi, t);
                row_ok = i >= 0;
            }
            float m_ref = -INFINITY, l = 0.f;
            // a regular block whose rows also have a permuted part starts from
            // that part's published state (m, l and O), loaded while S of its
            // first tile is computed; rows without one start from O = 0
            const bool init_o = C::STAGE && P.mode == 1 && bsg::starts_from_perm(sh, bi);
            if (C::STAGE && init_o) {
                const bool pr = row_ok && bsg::has_perm(sh, i);
                bool use = pr;
                const int64_t prow = (int64_t)it.bh * P.n + (pr ? i : 0);
                if (pr) {
                    // the permuted block (residue i mod 128, positions block
                    // (i / 128) / 128) is complete once all four of its warps arrived
                    const unsigned* f = P.pflag + ((int64_t)it.bh * sh.npqb + ((i >> 7) >> 7)) * 128 + (i & 127);
                    if (ld_acquire_u32(f) < 4u) {
                        const long long t0 = clock64();
                        while (ld_acquire_u32(f) < 4u) {
                            if (clock64() - t0 > P.wait_cycles || *abort_flag) {
                                atomicOr(P.err, kErrTimeout);
                                use = false;
                                break;
                            }
                            __nanosleep(128);
                        }
                    }
                }
                // each row's count is acquired by its own lane; the barrier and
                // a fence put every lane's loads (lanes load other rows) after them
                __syncwarp();
                fence_acq_rel_gpu();
                if (use) {
                    m_ref = __ldcg(P.pml + prow * 2);
                    l = __ldcg(P.pml + prow * 2 + 1);
                }
                rows_to_tmem<D>(stg, lane, use ? reinterpret_cast<uint64_t>(P.pacc + prow * D) : 0ull, tO);
                tmem_wait_st();
            }
            const int klim = pp_key_limit(P, it.b);
            bool alive = true;
            for (int u = 0; u < it.T && alive; ++u, ++g) {
                const int info = pp_tile(P, sh, it, u);
                const int kt = info & 0x7fffffff;
                bool dense = P.mode == 0 && info < 0;
                uint32_t w[4] = {0u, 0u, 0u, 0u};
                if (row_ok && !dense) {
                    if (P.mode == 0) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) w[q] = bsg::run_word(rlo, rhi, kt * 128 + 32 * q);
                    } else {
                        bsg::row_bits(sh, bi, kt, t, w);
                    }
                }
                if (klim - kt * 128 < 128) {  // the tile the key length cuts
                    if (dense) {
                        dense = false;
                        if (row_ok) w[0] = w[1] = w[2] = w[3] = 0xffffffffu;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) w[q] &= bsg::run_word(0, klim - kt * 128, 32 * q);
                }
                uint32_t need = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (dense || __any_sync(0xffffffffu, w[q] != 0u)) need |= 1u << q;
                if (EXTRA) {  // this tile's blocks of the additive terms are in shared memory
                    const bool oka = pp_wait(bar(s, kAFull), g & 1, abort_flag, P.wait_cycles);
                    if (!__all_sync(0xffffffffu, oka)) {
                        alive = false;
                        break;
                    }
                }
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    const bool ok = pp_wait(bar(s, kSFull + h), g & 1, abort_flag, P.wait_cycles);
                    if (!__all_sync(0xffffffffu, ok)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tSh = tS + (uint32_t)(64 * h);
                    // Stream the half 32 keys at a time (the second chunk's TMEM
                    // load in flight while the first is processed): scale,
                    // additive terms, entries not in the mask to -inf, then
                    // p = 2^(x - m_ref) against the running reference max, row
                    // sum, bf16 P into TMEM. When a chunk's max exceeds the
                    // reference by more than 2^8 the reference moves to it and
                    // the half's P chunk already written (and the sum) are
                    // rescaled in place; O is rescaled after the half. P of keys
                    // 64 h + 32 c .. + 31 goes to the half's columns 16 c ..
                    // 16 c + 15, which only hold S already consumed.
                    float alpha_h = 1.f;  // product of this half's rescales
                    float xa[32], xb[32];
                    if (need & (1u << (2 * h))) tmem_ld32f(tSh, xa);
                    tmem_wait_ld_depf(xa);
#pragma unroll
                    for (int hq = 0; hq < 2; ++hq) {
                        const int qq = 2 * h + hq;
                        float(&xc)[32] = hq == 0 ? xa : xb;
                        // the second chunk's load first (waited for at the end of the first)
                        if (hq == 0 && (need & (2u << qq))) tmem_ld32f(tSh + 32, xb);
                        uint32_t pk[16];
                        if (need & (1u << qq)) {
                            const uint32_t wq = qq == 0 ? w[0] : (qq == 1 ? w[1] : (qq == 2 ? w[2] : w[3]));
#pragma unroll
                            for (int k = 0; k < 32; ++k) xc[k] *= P.qk_scale_log2;
                            if (EXTRA) {
                                // + log2(e) * (mask + bias): 16-byte units 4 (qq & 1) ..
                                // + 3 of chunk qq / 2 of this row's line (128-byte
                                // swizzle: unit j of row r at j ^ (r & 7))
#pragma unroll
                                for (int a = 0; a < 2; ++a) {
                                    if (!P.extra[a]) continue;
                                    const int rows = P.a_rows[a], r0 = rows == 1 ? 0 : t;
                                    const uint8_t* base = smem + C::OFF_A + (2 * s + a) * C::A_BYTES +
                                                          (qq >> 1) * rows * 128 + r0 * 128;
#pragma unroll
                                    for (int uu = 0; uu < 4; ++uu) {
                                        const int j = 4 * (qq & 1) + uu;
                                        const int ph = rows == 1 ? j : (j ^ (r0 & 7));
                                        const uint4 v4 = *reinterpret_cast<const uint4*>(base + ph * 16);
                                        const uint32_t ws[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                                        for (int e = 0; e < 4; ++e) {
                                            xc[8 * uu + 2 * e] += kLog2e * __uint_as_float(ws[e] << 16);
                                            xc[8 * uu + 2 * e + 1] += kLog2e * __uint_as_float(ws[e] & 0xffff0000u);
                                        }
                                    }
                                }
                            }
                            if (!dense) {
#pragma unroll
                                for (int k = 0; k < 32; ++k) xc[k] = ((wq >> k) & 1u) ? xc[k] : -INFINITY;
                            }
                            float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
                            for (int k = 0; k < 16; k += 2) {
                                ma = fmax3(ma, xc[2 * k], xc[2 * k + 1]);
                                mb = fmax3(mb, xc[2 * k + 2], xc[2 * k + 3]);
                            }
                            const float mx = fmaxf(ma, mb);
                            const bool grow = mx > m_ref + kPpRescale;
                            if (__any_sync(0xffffffffu, grow)) {
                                // rare: new reference; the half's first P chunk (when
                                // this is its second) and the sum scale by alpha (1
                                // for rows that keep theirs)
                                float alpha = 1.f;
                                if (grow) {
                                    alpha = ex2(m_ref - mx);
                                    m_ref = mx;
                                    l *= alpha;
                                    alpha_h *= alpha;
                                }
                                if (hq == 1) {
                                    tmem_wait_st();  // the P chunk written, before reading it back
                                    uint32_t pw[16];
                                    tmem_ld16(tSh, pw);
                                    tmem_wait_ld_dep16(pw);
#pragma unroll
                                    for (int k = 0; k < 16; ++k) {
                                        __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(pw[k] << 16) * alpha,
                                                                                  __uint_as_float(pw[k] & 0xffff0000u) * alpha);
                                        pw[k] = *reinterpret_cast<uint32_t*>(&hv);
                                    }
                                    tmem_st16(tSh, pw);
                                }
                            }
                            const float mu = m_ref == -INFINITY ? 0.f : m_ref;
                            const uint64_t nmu2 = pack2(-mu, -mu);
                            uint64_t sa = pack2(0.f, 0.f), sb = sa;
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                float p0, p1;
                                unpack2(add2(pack2(xc[2 * k], xc[2 * k + 1]), nmu2), p0, p1);
                                p0 = ex2(p0);
                                p1 = ex2(p1);
                                if (k & 1)
                                    sb = add2(sb, pack2(p0, p1));
                                else
                                    sa = add2(sa, pack2(p0, p1));
                                __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
                                pk[k] = *reinterpret_cast<uint32_t*>(&hv);
                            }
                            float s0, s1, s2, s3;
                            unpack2(sa, s0, s1);
                            unpack2(sb, s2, s3);
                            l += (s0 + s1) + (s2 + s3);
                        } else {
#pragma unroll
                            for (int k = 0; k < 16; ++k) pk[k] = 0u;
                        }
                        tmem_st16(tSh + 16 * hq, pk);
                        if (hq == 0) tmem_wait_ld_depf(xb);  // the second chunk's S
                    }
                    if ((u > 0 || h > 0 || init_o) && __any_sync(0xffffffffu, alpha_h != 1.f)) {
                        // bring O (every product issued before this half's, once
                        // complete, or the published state it started from) to the
                        // new reference
                        if (u > 0 || h > 0) {
                            const bool ok2 = h > 0 ? pp_wait(bar(s, kSFree), g & 1, abort_flag, P.wait_cycles)
                                                   : pp_wait(bar(s, kSFreeB), (g - 1) & 1, abort_flag, P.wait_cycles);
                            if (!__all_sync(0xffffffffu, ok2)) {
                                alive = false;
                                break;
                            }
                            tc_fence_after();
                        }
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t ro[32];
                            tmem_ld32(tO + 32 * c, ro);
                            tmem_wait_ld_dep(ro);
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) ro[jj] = __float_as_uint(__uint_as_float(ro[jj]) * alpha_h);
                            tmem_st32(tO + 32 * c, ro);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(s, kPFull + h));
                }
                if (!alive) break;
                if (EXTRA) {  // the additive blocks are read: the producer may refill them
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(s, kAEmpty));
                }
            }
            if (!alive) break;
            // ---------------------------------------------------------- epilogue
            const bool ok = pp_wait(bar(s, kODone), m & 1, abort_flag, P.wait_cycles);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            pp_finish<D, C::STAGE>(P, sh, it, quarter, t, i, row_ok, m_ref, l, tO, stg, pubq);
            __syncwarp();
        }
        // this warp publishes nothing more (released after its last queue entry)
        __syncwarp();
        if (lane == 0) asm volatile("red.release.cta.shared.add.u32 [%0], 1;" ::"r"(smem_u32((const void*)(pubq + 48))) : "memory");
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicOr(P.err, kErrTimeout);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kPpTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn pp_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [B, H, n, d] bf16 as {d, n, H, B}, box {min(d, 64), 128, 1, 1}, 128-byte
// swizzle (64-byte for d = 32).
cudaError_t pp_map4(CUtensorMap* map, const TcOperand& t, int B, int H, int n, int d) {
    EncodeTiledFn fn = pp_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const int chunk = d >= 64 ? 64 : d;
    const uint64_t sn = (uint64_t)t.s_n * 2;
    const uint64_t sh = H > 1 ? (uint64_t)t.s_h * 2 : sn * (uint64_t)n;
    const uint64_t sb = B > 1 ? (uint64_t)t.s_b * 2 : sh * (uint64_t)H;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {sn, sh, sb};
    cuuint32_t box[4] = {(cuuint32_t)chunk, 128, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.data), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, chunk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The same tensor in residue-permuted order: {d, S, G, H, B} (row k S + r at
// (r, k)), box {64, 1, 128, 1, 1}: one load brings rows r, r + S, ... .
cudaError_t pp_map5(CUtensorMap* map, const TcOperand& t, int B, int H, int n, int d, int S) {
    EncodeTiledFn fn = pp_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const int G = n / S;
    const uint64_t sn = (uint64_t)t.s_n * 2;
    const uint64_t sh = H > 1 ? (uint64_t)t.s_h * 2 : sn * (uint64_t)n;
    const uint64_t sb = B > 1 ? (uint64_t)t.s_b * 2 : sh * (uint64_t)H;
    cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)S, (cuuint64_t)G, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[4] = {sn, sn * (uint64_t)S, sh, sb};
    cuuint32_t box[5] = {64, 1, 128, 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(t.data), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// An additive term [B or 1, H or 1, n or 1, n] (bf16, keys contiguous) as
// {keys, rows, heads, batch}, box {64, rows_box, 1, 1}: 128-byte swizzle for
// 128-row blocks, none for a term shared by all rows (rows_box 1). Dimensions
// the term broadcasts over have extent 1.
cudaError_t pp_map_addend(CUtensorMap* map, const AddendView& a, int B, int H, int n, int rows_box) {
    EncodeTiledFn fn = pp_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const uint64_t row_bytes = ((uint64_t)n * 2 + 15) & ~uint64_t(15);  // a valid stride for extent-1 dimensions
    cuuint64_t dims[4] = {(cuuint64_t)n, (cuuint64_t)(a.s2 ? n : 1), (cuuint64_t)(a.s1 ? H : 1),
                          (cuuint64_t)(a.s0 ? B : 1)};
    cuuint64_t strides[3] = {a.s2 ? (uint64_t)a.s2 * 2 : row_bytes, a.s1 ? (uint64_t)a.s1 * 2 : row_bytes,
                             a.s0 ? (uint64_t)a.s0 * 2 : row_bytes};
    cuuint32_t box[4] = {64, (cuuint32_t)rows_box, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(a.data), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    rows_box == 1 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, bool EXTRA, bool CF>
cudaError_t launch_pp_t(const TcOperand& q, const TcOperand& k, const TcOperand& v, const PpParams& p0,
                        const AddendView& mask, const AddendView& bias, int num_sms, cudaStream_t s) {
    using C = PpCfg<D, EXTRA>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, []() {
        attr_err = cudaFuncSetAttribute((const void*)k_fwd_pp<D, EXTRA, CF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
        // setmaxnreg.inc draws on the registers the CTA was launched with: the
        // split fits only when the launch holds at least 128 x 96 + 256 x 200
        // of them (fewer would leave the softmax warps waiting for registers
        // that never come), so refuse any build of the kernel launched with
        // fewer
        cudaFuncAttributes fa;
        if (attr_err == cudaSuccess) attr_err = cudaFuncGetAttributes(&fa, (const void*)k_fwd_pp<D, EXTRA, CF>);
        if (attr_err == cudaSuccess && fa.numRegs * kPpThreads < 128 * kPpRegsLow + 256 * kPpRegsHigh)
            attr_err = cudaErrorInvalidConfiguration;
    });
    if (attr_err != cudaSuccess) return attr_err;
    PpParams p = p0;
    CUtensorMap mq, mk, mv, mqp, mkp, mvp, ma0, ma1;
    cudaError_t e;
    if ((e = pp_map4(&mq, q, p.B, p.H, p.n, D)) != cudaSuccess) return e;
    if ((e = pp_map4(&mk, k, p.B, p.H, p.n, D)) != cudaSuccess) return e;
    if ((e = pp_map4(&mv, v, p.B, p.H, p.n, D)) != cudaSuccess) return e;
    if (p.mode == 1 && p.S) {
        if ((e = pp_map5(&mqp, q, p.B, p.H, p.n, D, p.S)) != cudaSuccess) return e;
        if ((e = pp_map5(&mkp, k, p.B, p.H, p.n, D, p.S)) != cudaSuccess) return e;
        if ((e = pp_map5(&mvp, v, p.B, p.H, p.n, D, p.S)) != cudaSuccess) return e;
    } else {
        mqp = mq;
        mkp = mk;
        mvp = mv;
    }
    ma0 = ma1 = mq;
    const AddendView* terms[2] = {&mask, &bias};
    for (int a = 0; a < 2; ++a) {
        p.extra[a] = EXTRA && terms[a]->data != nullptr;
        p.a_rows[a] = terms[a]->s2 ? 128 : 1;
        p.a_h[a] = terms[a]->s1 != 0;
        p.a_b[a] = terms[a]->s0 != 0;
        if (p.extra[a] &&
            (e = pp_map_addend(a == 0 ? &ma0 : &ma1, *terms[a], p.B, p.H, p.n, p.a_rows[a])) != cudaSuccess)
            return e;
    }
    if (p.n_items <= 0) return cudaSuccess;
    const int64_t grid = p.n_items < num_sms ? p.n_items : num_sms;
    k_fwd_pp<D, EXTRA, CF><<<(unsigned)grid, kPpThreads, C::SMEM_BYTES, counted(s)>>>(mq, mk, mv, mqp, mkp, mvp,
                                                                                       ma0, ma1, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_pp(const TcOperand& q, const TcOperand& k, const TcOperand& v, int d, const PpParams& p,
                          const AddendView& mask, const AddendView& bias, int num_sms, cudaStream_t s) {
    const bool extra = mask.data || bias.data;
    if (extra && (p.mode != 0 || d > 64 || !pp_addend_ok(mask) || !pp_addend_ok(bias))) return cudaErrorInvalidValue;
    // closed-form masks (mode 1) take the build whose S goes out per tile
    const bool cf = p.mode == 1;
    switch (d) {
    case 32: return extra ? launch_pp_t<32, true, false>(q, k, v, p, mask, bias, num_sms, s)
                          : cf ? launch_pp_t<32, false, true>(q, k, v, p, mask, bias, num_sms, s)
                               : launch_pp_t<32, false, false>(q, k, v, p, mask, bias, num_sms, s);
    case 64: return extra ? launch_pp_t<64, true, false>(q, k, v, p, mask, bias, num_sms, s)
                          : cf ? launch_pp_t<64, false, true>(q, k, v, p, mask, bias, num_sms, s)
                               : launch_pp_t<64, false, false>(q, k, v, p, mask, bias, num_sms, s);
    case 128: return cf ? launch_pp_t<128, false, true>(q, k, v, p, mask, bias, num_sms, s)
                        : launch_pp_t<128, false, false>(q, k, v, p, mask, bias, num_sms, s);
    }
    return cudaErrorInvalidValue;
}

bool pp_addend_ok(const AddendView& a) {
    if (!a.data) return true;
    const uintptr_t base = reinterpret_cast<uintptr_t>(a.data);
    return a.dtype == 0 && a.s3 == 1 && (base & 15) == 0 && (a.s2 * 2) % 16 == 0 && (a.s1 * 2) % 16 == 0 &&
           (a.s0 * 2) % 16 == 0;
}

}  // namespace spattn
