// Tensor-core forward for the mask's dense and near-dense 128 x 128 tiles
// (tcgen05 MMAs with TMEM accumulators, TMA tile loads, sm_100a).
//
// One CTA owns one 128-row query block of one (b, h) and walks the block's
// selected key tiles. Per tile:
//   S = Q K^T               tcgen05.mma (M = 128, N = 128 or two N = 64 halves,
//                           K = d), S in TMEM
//   s = scale*S + mask + bias, entries the mask does not list set to -inf
//   running max / sum       the streaming-dataflow SDPA paper's rescaling rule;
//                           the max used as reference only moves when a tile's
//                           max exceeds it by more than 2^8, and then the O
//                           accumulator in TMEM is rescaled by exp2(m_old - m_new)
//   O += P V                tcgen05.mma (M = 128, N = d), P from TMEM or smem
// K/V tiles are double-buffered and loaded by TMA (no multicast) while the
// previous tile's softmax and P V run. At the end O / l is written (bf16) and
// lse = m + log(l); rows that also have residual (gathered) entries first merge
// the gather kernel's partial (m, l, acc) with the same rescaling rule.
//
// Two kernels: k_fwd_tc<d> (d = 128, one thread per row) and
// k_fwd_tc_quad<d, EXTRA, STAGED> (d <= 64: one thread per row, 64-key
// sub-tiles, P in TMEM, four CTAs per SM; with an additive mask or bias the
// term that varies by row is staged in shared memory by TMA (STAGED, four CTAs
// per SM) or, for layouts TMA cannot fetch, prefetched into registers (three)).
//
// Every mbarrier wait is bounded: on expiry the CTA raises the device error
// flag, drains what it issued (bounded again), frees its TMEM and returns.
#include "spattn_internal.cuh"
#include "sm100_ptx.cuh"

#include <math.h>
#include <mutex>

namespace spattn {
namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr float kRescaleThreshold = 8.0f;       // log2 units
constexpr long long kWaitCycles = 2000000000LL;  // about one second at B200 clocks
constexpr uint32_t kTmemCols = 256;             // S: columns [0, 128), O: [128, 128 + d)

template <int D>
struct TcCfg {
    static constexpr int CHUNK_ELEMS = D >= 64 ? 64 : D;  // elements per swizzled row
    static constexpr int ROW_BYTES = CHUNK_ELEMS * 2;     // 64 or 128
    static constexpr int NCHUNK = D / CHUNK_ELEMS;        // column chunks of a tile
    static constexpr int CHUNK_BYTES = 128 * ROW_BYTES;
    static constexpr int TILE_BYTES = NCHUNK * CHUNK_BYTES;  // 128 x d bf16
    static constexpr int SBO = 8 * ROW_BYTES;                // 8-row swizzle atom
    static constexpr int KSTEPS_PER_CHUNK = CHUNK_ELEMS / 16;
    static constexpr cute::UMMA::LayoutType LAYOUT =
        D >= 64 ? cute::UMMA::LayoutType::SWIZZLE_128B : cute::UMMA::LayoutType::SWIZZLE_64B;
    static constexpr int P_BYTES = 128 * 128 * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE_BYTES;         // two buffers
    static constexpr int OFF_V = 3 * TILE_BYTES;     // two buffers
    static constexpr int OFF_P = 5 * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;  // mbarriers, tmem slot, abort flag, exchange
    static constexpr int BAR_BYTES = 10 * 8 + 14 * 4;
    // At least 100 KB so that no more than two CTAs (2 x 256 TMEM columns) share
    // an SM and tcgen05.alloc never has to wait; d = 64 fits two CTAs per SM.
    static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES > 100 * 1024 ? OFF_BAR + BAR_BYTES : 100 * 1024;
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
};

// Adds log2(e) * addend[b, h, i, c0 + j] to x[j] for j < ncols (an N-column run).
template <int N>
__device__ __forceinline__ void add_addend_run(const AddendView& a, int64_t rowbase, int c0, int ncols,
                                               float (&x)[N]) {
    const int64_t off0 = rowbase + (int64_t)c0 * a.s3;
    if (a.dtype == 0 && a.s3 == 1 && ncols == N &&
        ((reinterpret_cast<uintptr_t>(a.data) + (uintptr_t)off0 * 2) & 15) == 0) {
        const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.data) + off0);
#pragma unroll
        for (int c = 0; c < N / 8; ++c) {
            const uint4 w = __ldg(p + c);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                x[c * 8 + 2 * t] += kLog2e * __uint_as_float(ws[t] << 16);
                x[c * 8 + 2 * t + 1] += kLog2e * __uint_as_float(ws[t] & 0xffff0000u);
            }
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < N; ++j) {
        if (j < ncols) {
            const int64_t off = off0 + (int64_t)j * a.s3;
            const float v = a.dtype == 0
                                ? __bfloat162float(__ldg(reinterpret_cast<const __nv_bfloat16*>(a.data) + off))
                                : __ldg(reinterpret_cast<const float*>(a.data) + off);
            x[j] += kLog2e * v;
        }
    }
}

// Key padding: the keys of batch element b are [0, L) (L = n without it). Tiles
// are listed by ascending key tile, so the ones at or past L are dropped from
// the end; one is kept so that the epilogue still writes the rows.
__device__ __forceinline__ int key_limit_tc(const TcParams& P, int b) {
    if (!P.seqlen_k) return P.n;
    const int L = P.seqlen_k[b];
    return L < 0 ? 0 : (L > P.n ? P.n : L);
}
__device__ __forceinline__ int trim_tiles(const TcParams& P, int t_begin, int T, int L) {
    if (P.seqlen_k)
        while (T > 1 && (P.tile_info[t_begin + T - 1] & 0x7fffffff) * kTileN >= L) --T;
    return T;
}

// First tile and number of tiles of query block blk.
__device__ __forceinline__ void block_tiles(const TcParams& P, int64_t blk, int& t_begin, int& T) {
    if (P.block_ntiles) {
        t_begin = (int)(blk * P.tile_stride);
        T = P.block_ntiles[blk];
    } else {
        t_begin = P.block_tile_off[blk];
        T = P.block_tile_off[blk + 1] - t_begin;
    }
}

// Bits of the columns [c0, c0 + 32) that lie in the run [lo, hi).
__device__ __forceinline__ uint32_t run_word(int lo, int hi, int c0) {
    int a = lo - c0, z = hi - c0;
    a = a < 0 ? 0 : (a > 32 ? 32 : a);
    z = z < 0 ? 0 : (z > 32 ? 32 : z);
    if (z <= a) return 0u;
    const uint32_t top = z == 32 ? 0xffffffffu : ((1u << z) - 1u);
    return top & ~((1u << a) - 1u);  // a < 32 here
}

// Row `row` of tile t (key tile in `info`): its 128 mask bits, from the tile's
// stored bits or, for interval masks, from the row's run [lo, hi).
__device__ __forceinline__ uint4 tile_row_bits4(const TcParams& P, int t, int info, int row, int lo, int hi) {
    if (P.itv_lohi) {
        const int c0 = (info & 0x7fffffff) * kTileN;
        return make_uint4(run_word(lo, hi, c0), run_word(lo, hi, c0 + 32), run_word(lo, hi, c0 + 64),
                          run_word(lo, hi, c0 + 96));
    }
    return __ldg(reinterpret_cast<const uint4*>(P.tile_bits) + ((int64_t)t * 128 + row));
}

// Whether row (mrow of the mask, wrow of the output) has a partial state from
// the gather kernel to merge.
__device__ __forceinline__ bool has_partial(const TcParams& P, int64_t blk, int64_t mrow, int64_t wrow) {
    if (!P.ws_ml) return false;
    if (P.blk_res) return P.blk_res[blk] && P.ws_ml[wrow * 2 + 1] > 0.f;
    return P.res_row_ptr[mrow + 1] > P.res_row_ptr[mrow];
}

// Counts this warp in; true for lane 0 of the warp whose arrival is number
// `last` (0-based). Orders the warp's earlier shared-memory, async-proxy and
// tensor-memory accesses before the count and makes the others' visible to the
// winner.
__device__ __forceinline__ bool arrive_last(uint32_t* counter, uint32_t last) {
    tc_fence_before();
    __syncwarp();
    bool win = false;
    if ((threadIdx.x & 31) == 0) {
        __threadfence_block();
        win = atomicAdd(counter, 1u) == last;
        if (win) {
            __threadfence_block();
            tc_fence_after();
        }
    }
    return win;
}

// Writes row i of the output from its state (m, l, o) (log2 units, O not yet
// divided by l), first merging the gather kernel's partial when the row has
// one; lse = (m + log2 l) ln 2.
template <int D>
__device__ __forceinline__ void tc_write_row(const TcParams& P, int b, int h, int64_t bh, int mk, int64_t blk,
                                             int i, float m, float l, const float (&o)[D]) {
    if (i >= P.n) return;
    float M = m, L = l, fa = 1.f, fg = 0.f;
    const int64_t mrow = (int64_t)mk * P.n + i;
    const int64_t wrow = bh * P.n + i;
    const bool mixed = has_partial(P, blk, mrow, wrow);
    if (mixed) {
        const float mg = P.ws_ml[wrow * 2], lg = P.ws_ml[wrow * 2 + 1];
        M = fmaxf(m, mg);
        const float Mu = M == -INFINITY ? 0.f : M;
        fa = ex2(m - Mu);
        fg = ex2(mg - Mu);
        L = l * fa + lg * fg;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(P.out) + (int64_t)b * P.o_sb + (int64_t)h * P.o_sh +
                          (int64_t)i * P.o_sn;
    const float* acc = mixed ? P.ws_acc + wrow * D : nullptr;
#pragma unroll
    for (int e8 = 0; e8 < D / 8; ++e8) {
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float val = o[e8 * 8 + t] * fa;
            if (mixed) val = fmaf(acc[e8 * 8 + t], fg, val);
            v[t] = val * inv;
        }
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            __nv_bfloat162 hv = __floats2bfloat162_rn(v[2 * t], v[2 * t + 1]);
            w[t] = *reinterpret_cast<uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(orow + e8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (P.lse) P.lse[wrow] = L > 0.f ? (M + lg2(L)) * kLn2 : -INFINITY;
}

// A query block whose tile list is split into chunks (one thread block each):
// the chunk's partial state (m, l, O) of every row goes to its slot in
// P.cws ([slot][d + 2][128 rows], so each warp's stores are coalesced); the
// thread block whose arrival completes the block's count merges all chunks
// with the running max / sum rule and returns true with the merged state in
// (m, l, o); the others return false. flag: one int of shared memory.
template <int D>
__device__ bool chunk_merge(const TcParams& P, int64_t bh, int64_t blk, int chunk, int nch, int row, float& m,
                            float& l, float (&o)[D], volatile int* flag) {
    const int64_t slot0 = (bh * P.n_slots + P.blk_slot[blk]) * (int64_t)(D + 2);
    float* mine = P.cws + (slot0 + (int64_t)chunk * (D + 2)) * 128 + row;
    mine[0] = m;
    mine[128] = l;
#pragma unroll
    for (int j = 0; j < D; ++j) mine[(int64_t)(2 + j) * 128] = o[j];
    __threadfence();
    __syncthreads();
    if (row == 0) {
        const int64_t nblk = (int64_t)P.num_masks * P.nqb;
        *flag = atomicAdd(P.ccnt + bh * nblk + blk, 1u) == (unsigned)(nch - 1);
    }
    __syncthreads();
    if (!*flag) return false;
    __threadfence();
    float M = -INFINITY, L = 0.f;
#pragma unroll
    for (int j = 0; j < D; ++j) o[j] = 0.f;
    for (int c = 0; c < nch; ++c) {
        const float* pp = P.cws + (slot0 + (int64_t)c * (D + 2)) * 128 + row;
        const float mc = __ldcg(pp), lc = __ldcg(pp + 128);
        if (!(lc > 0.f)) continue;
        const float Mn = fmaxf(M, mc);
        const float fa = ex2(M - Mn), fb = ex2(mc - Mn);
#pragma unroll
        for (int j = 0; j < D; ++j) o[j] = fmaf(__ldcg(pp + (int64_t)(2 + j) * 128), fb, o[j] * fa);
        L = L * fa + lc * fb;
        M = Mn;
    }
    m = M;
    l = L;
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const TcParams P) {
    using C = TcCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int tid = threadIdx.x, warp = tid >> 5;
    // thread blocks [0, B*H*nqb) take query block (bh, qb) -- its first chunk
    // when it is split --; the rest take the further chunks P.chunk_extra lists
    const int64_t nbase = (int64_t)P.B * P.H * P.nqb;
    int bh, qb, chunk = 0;
    if ((int64_t)blockIdx.x < nbase) {
        bh = (int)(blockIdx.x / P.nqb);
        qb = (int)(blockIdx.x - (int64_t)bh * P.nqb);
    } else {
        const int64_t e = (int64_t)blockIdx.x - nbase;
        bh = (int)(e / P.n_extra);
        const int2 x = P.chunk_extra[e - (int64_t)bh * P.n_extra];
        if (P.num_masks > 1 && x.x / P.nqb != bh / P.H) return;  // a chunk of another batch element's mask
        qb = x.x % P.nqb;
        chunk = x.y;
    }
    const int b = bh / P.H, h = bh - b * P.H;
    const int mk = P.num_masks == 1 ? 0 : b;
    const int64_t blk = (int64_t)mk * P.nqb + qb;
    int t_begin, T;
    block_tiles(P, blk, t_begin, T);
    if (T <= 0) return;
    const int klim = key_limit_tc(P, b);
    T = trim_tiles(P, t_begin, T, klim);  // whole CTA: the gather kernel owns this block
    const int nch = P.blk_nch ? P.blk_nch[blk] : 1;
    if (nch > 1) {  // this chunk's tiles (none when the key length cut them all)
        t_begin += chunk * P.chunk_tiles;
        T -= chunk * P.chunk_tiles;
        T = T < P.chunk_tiles ? T : P.chunk_tiles;
    }
    if (smem_u32(smem) & 1023u) {  // the swizzled layouts need a 1024-byte aligned base
        if (tid == 0) atomicOr(P.err, kErrTimeout);
        return;
    }

    const uint32_t sQ = smem_u32(smem + C::OFF_Q);
    const uint32_t sK0 = smem_u32(smem + C::OFF_K), sV0 = smem_u32(smem + C::OFF_V);
    const uint32_t sP = smem_u32(smem + C::OFF_P);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    const uint32_t barQ = smem_u32(bars + 0), barKV0 = smem_u32(bars + 1), barS = smem_u32(bars + 3),
                   barO = smem_u32(bars + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* chunk_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

    float o[D];
    if (T <= 0) {  // an empty chunk still counts in, with an empty partial
        float m0 = -INFINITY, l0 = 0.f;
#pragma unroll
        for (int j = 0; j < D; ++j) o[j] = 0.f;
        if (chunk_merge<D>(P, bh, blk, chunk, nch, tid, m0, l0, o, chunk_flag))
            tc_write_row<D>(P, b, h, bh, mk, blk, qb * 128 + tid, m0, l0, o);
        return;
    }

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    if (tid == 0) {
        for (int x = 0; x < 5; ++x) mbar_init(smem_u32(bars + x), 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 128;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    // issue bookkeeping (thread 0), for draining after an expired wait
    int n_kv_issued = 0, n_s_issued = 0, n_pv_issued = 0;

    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait_bounded(bar, parity, kWaitCycles)) return true;
        *abort_flag = 1;
        return false;
    };
    auto issue_kv = [&](int u) {  // tile u -> buffer u & 1
        const int kt = P.tile_info[t_begin + u] & 0x7fffffff;
        const uint32_t bar = barKV0 + 8u * (u & 1);
        const uint32_t dK = sK0 + (uint32_t)((u & 1) * C::TILE_BYTES);
        const uint32_t dV = sV0 + (uint32_t)((u & 1) * C::TILE_BYTES);
        mbar_expect_tx(bar, 2u * C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c) {
            if (P.perm_G) {  // keys kt*128 .. in permuted order: residue r, positions k0 .. k0 + 127
                const int r = kt * 128 / P.perm_G, k0 = kt * 128 - r * P.perm_G;
                tma_load_5d(dK + c * C::CHUNK_BYTES, &tmK, bar, c * C::CHUNK_ELEMS, r, k0, h, b);
                tma_load_5d(dV + c * C::CHUNK_BYTES, &tmV, bar, c * C::CHUNK_ELEMS, r, k0, h, b);
            } else {
                tma_load_4d(dK + c * C::CHUNK_BYTES, &tmK, bar, c * C::CHUNK_ELEMS, kt * 128, h, b);
                tma_load_4d(dV + c * C::CHUNK_BYTES, &tmV, bar, c * C::CHUNK_ELEMS, kt * 128, h, b);
            }
        }
        ++n_kv_issued;
    };
    const uint32_t idS = idesc_bf16_f32(128, 128, false);
    const uint32_t idO = idesc_bf16_f32(128, D, true);
    auto issue_S = [&](int u) {
        const uint32_t sK = sK0 + (uint32_t)((u & 1) * C::TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int c = ks / C::KSTEPS_PER_CHUNK, kin = ks % C::KSTEPS_PER_CHUNK;
            const uint32_t off = (uint32_t)(c * C::CHUNK_BYTES + kin * 32);
            const uint64_t da = smem_desc(sQ + off, 16, C::SBO, C::LAYOUT);
            const uint64_t db = smem_desc(sK + off, 16, C::SBO, C::LAYOUT);
            mma_bf16_ss(tS, da, db, idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(barS);
        ++n_s_issued;
    };
    auto issue_PV = [&](int u) {
        const uint32_t sV = sV0 + (uint32_t)((u & 1) * C::TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // 16 keys per step
            const uint64_t da = smem_desc(sP + (uint32_t)((ks >> 2) * 16384 + (ks & 3) * 32), 16, 1024,
                                          cute::UMMA::LayoutType::SWIZZLE_128B);
            const uint64_t db = smem_desc(sV + (uint32_t)(ks * 16 * C::ROW_BYTES), C::CHUNK_BYTES, C::SBO,
                                          C::LAYOUT);
            mma_bf16_ss(tO, da, db, idO, (u > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(barO);
        ++n_pv_issued;
    };

    if (tid == 0) {
        mbar_expect_tx(barQ, (uint32_t)C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
            if (P.perm_G) {
                const int r = qb * 128 / P.perm_G, k0 = qb * 128 - r * P.perm_G;
                tma_load_5d(sQ + c * C::CHUNK_BYTES, &tmQ, barQ, c * C::CHUNK_ELEMS, r, k0, h, b);
            } else {
                tma_load_4d(sQ + c * C::CHUNK_BYTES, &tmQ, barQ, c * C::CHUNK_ELEMS, qb * 128, h, b);
            }
        issue_kv(0);
        if (T > 1) issue_kv(1);
        if (wait(barQ, 0) && wait(barKV0, 0)) {
            tc_fence_after();
            issue_S(0);
        }
    }

    const int row = tid;
    const int i = qb * 128 + row;
    const bool row_ok = i < P.n;
    const int64_t mask_rowbase = (int64_t)b * P.mask.s0 + (int64_t)h * P.mask.s1 + (int64_t)i * P.mask.s2;
    const int64_t bias_rowbase = (int64_t)b * P.bias.s0 + (int64_t)h * P.bias.s1 + (int64_t)i * P.bias.s2;
    float m_ref = -INFINITY, l = 0.f;
    int rlo = 0, rhi = 0;  // interval masks: the row's run
    if (P.itv_lohi && row_ok) {
        const int2 v = P.itv_lohi[(int64_t)mk * P.n + i];
        rlo = v.x;
        rhi = v.y;
    }

    // tile u's info and row bits are loaded one tile ahead
    int next_info = P.tile_info[t_begin];
    uint4 next_bits = make_uint4(0u, 0u, 0u, 0u);
    if (next_info >= 0 && row_ok && !P.itv_lohi) next_bits = tile_row_bits4(P, t_begin, next_info, row, rlo, rhi);
    const uint64_t c2 = pack2(P.qk_scale_log2, P.qk_scale_log2);

    for (int u = 0; u < T; ++u) {
        const int info = next_info;
        const uint4 wbits = next_bits;
        if (u + 1 < T) {
            next_info = P.tile_info[t_begin + u + 1];
            if (next_info >= 0 && row_ok && !P.itv_lohi)
                next_bits = tile_row_bits4(P, t_begin + u + 1, next_info, row, rlo, rhi);
        }
        const int kt = info & 0x7fffffff;
        const bool dense = info < 0;  // the same for the whole CTA
        const bool extra = P.has_extra && row_ok;
        const int jj0 = kt * 128;
        uint4 wb = P.itv_lohi && row_ok && !dense ? tile_row_bits4(P, 0, info, row, rlo, rhi) : wbits;
        const int lim = klim - jj0;  // keys of this tile that exist
        const bool cut = lim < 128;
        if (cut) {
            if (dense) wb = make_uint4(~0u, ~0u, ~0u, ~0u);
            wb.x &= run_word(0, lim, 0);
            wb.y &= run_word(0, lim, 32);
            wb.z &= run_word(0, lim, 64);
            wb.w &= run_word(0, lim, 96);
        }
        const uint32_t bw[4] = {wb.x, wb.y, wb.z, wb.w};

        wait(barS, (uint32_t)(u & 1));
        tc_fence_after();
        __syncwarp();
        // pass 1, 64 columns at a time: x = scale*log2(e)*S (+ log2(e)*(mask + bias)),
        // entries the CSR does not list -> -inf, row max; x goes back into TMEM
        float ma = -INFINITY, mb = -INFINITY, mc = -INFINITY, md = -INFINITY;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float xh[64];
            if (extra) {
#pragma unroll
                for (int j = 0; j < 64; ++j) xh[j] = 0.f;
                const int c0 = jj0 + half * 64;
                const int ncols = P.n - c0 < 64 ? P.n - c0 : 64;
                if (P.mask.data) add_addend_run<64>(P.mask, mask_rowbase, c0, ncols, xh);
                if (P.bias.data) add_addend_run<64>(P.bias, bias_rowbase, c0, ncols, xh);
            }
            uint32_t r0[32], r1[32];
            tmem_ld32(tS + lane_base + half * 64, r0);
            tmem_ld32(tS + lane_base + half * 64 + 32, r1);
            tmem_wait_ld_dep(r0);
            tmem_wait_ld_dep(r1);
            if (extra) {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    fma2_inplace(xh[2 * k], xh[2 * k + 1], r0[2 * k], r0[2 * k + 1], c2);
                    fma2_inplace(xh[32 + 2 * k], xh[33 + 2 * k], r1[2 * k], r1[2 * k + 1], c2);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    mul2(xh[2 * k], xh[2 * k + 1], r0[2 * k], r0[2 * k + 1], c2);
                    mul2(xh[32 + 2 * k], xh[33 + 2 * k], r1[2 * k], r1[2 * k + 1], c2);
                }
            }
            if (!dense || cut) {
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    xh[j] = ((bw[half * 2 + (j >> 5)] >> (j & 31)) & 1u) ? xh[j] : -INFINITY;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                ma = fmax3(ma, xh[8 * k + 0], xh[8 * k + 1]);
                mb = fmax3(mb, xh[8 * k + 2], xh[8 * k + 3]);
                mc = fmax3(mc, xh[8 * k + 4], xh[8 * k + 5]);
                md = fmax3(md, xh[8 * k + 6], xh[8 * k + 7]);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                r0[j] = __float_as_uint(xh[j]);
                r1[j] = __float_as_uint(xh[32 + j]);
            }
            tmem_st32(tS + lane_base + half * 64, r0);
            tmem_st32(tS + lane_base + half * 64 + 32, r1);
        }
        tmem_wait_st();
        const float mx = fmax3(ma, mb, fmaxf(mc, md));
        const bool need = mx > m_ref + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
            alpha = ex2(m_ref - mx);
            m_ref = mx;
            l *= alpha;
        }
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        const uint64_t nmu2 = pack2(-mu, -mu);
        uint64_t sa = pack2(0.f, 0.f), sb = sa;  // two running pair sums

        // pass 2, per 64-key chunk: p = exp2(x - m), row sum, P (bf16) into the K-major,
        // 128-byte-swizzled A operand layout of the P V MMA (chunk kc = keys 64kc ..)
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
            uint32_t r0[32], r1[32];
            tmem_ld32(tS + lane_base + kc * 64, r0);
            tmem_ld32(tS + lane_base + kc * 64 + 32, r1);
            tmem_wait_ld_dep(r0);
            tmem_wait_ld_dep(r1);
            uint32_t pk[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const uint32_t w0 = k < 16 ? r0[2 * k] : r1[2 * k - 32];
                const uint32_t w1 = k < 16 ? r0[2 * k + 1] : r1[2 * k - 31];
                float p0, p1;
                unpack2(add2(pack2(__uint_as_float(w0), __uint_as_float(w1)), nmu2), p0, p1);
                p0 = ex2(p0);
                p1 = ex2(p1);
                if (k & 1)
                    sb = add2(sb, pack2(p0, p1));
                else
                    sa = add2(sa, pack2(p0, p1));
                __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
                pk[k] = *reinterpret_cast<uint32_t*>(&hv);
            }
            if (kc == 0 && u > 0) {
                // P V of the previous tile reads sP: it must be done before sP is overwritten

                wait(barO, (uint32_t)((u - 1) & 1));
                tc_fence_after();
                if (tid == 0 && u + 1 < T && !*abort_flag) issue_kv(u + 1);  // its buffer is free now
                __syncwarp();
                if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t ro[32];
                        tmem_ld32(tO + lane_base + c * 32, ro);
                        tmem_wait_ld_dep(ro);
#pragma unroll
                        for (int j = 0; j < 32; ++j) ro[j] = __float_as_uint(__uint_as_float(ro[j]) * alpha);
                        tmem_st32(tO + lane_base + c * 32, ro);
                    }
                    tmem_wait_st();
                }
            }
#pragma unroll
            for (int piece = 0; piece < 8; ++piece) {
                const uint32_t addr = sP + (uint32_t)(kc * 16384 + row * 128 + ((piece ^ (row & 7)) << 4));
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[piece * 4]),
                             "r"(pk[piece * 4 + 1]), "r"(pk[piece * 4 + 2]), "r"(pk[piece * 4 + 3])
                             : "memory");
            }
        }
        {
            float s0, s1, s2, s3;
            unpack2(sa, s0, s1);
            unpack2(sb, s2, s3);
            l += (s0 + s1) + (s2 + s3);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && !*abort_flag) {
            tc_fence_after();
            issue_PV(u);
            if (u + 1 < T && wait(barKV0 + 8u * ((u + 1) & 1), (uint32_t)(((u + 1) >> 1) & 1))) {
                tc_fence_after();
                issue_S(u + 1);
            }
        }
    }

    // ------------------------------------------------------------ epilogue
    wait(barO, (uint32_t)((T - 1) & 1));
    tc_fence_after();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t ro[32];
        tmem_ld32(tO + lane_base + c * 32, ro);
        tmem_wait_ld_dep(ro);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[c * 32 + j] = __uint_as_float(ro[j]);
    }
    {
        float M = m_ref, L = l;
        __syncthreads();  // every wait is behind us: the abort flag is final and the same for all
        bool write = !*abort_flag;
        if (nch > 1 && write) write = chunk_merge<D>(P, bh, blk, chunk, nch, tid, M, L, o, chunk_flag);
        if (write) tc_write_row<D>(P, b, h, bh, mk, blk, i, M, L, o);
    }

    // ------------------------------------------------------------ teardown
    if (tid == 0 && *abort_flag) {
        // drain whatever was issued (bounded), so no async op outlives the CTA
        if (n_s_issued) mbar_wait_bounded(barS, (uint32_t)((n_s_issued - 1) & 1), kWaitCycles / 16);
        if (n_pv_issued) mbar_wait_bounded(barO, (uint32_t)((n_pv_issued - 1) & 1), kWaitCycles / 16);
        for (int bnum = 0; bnum < 2; ++bnum) {
            const int uses = (n_kv_issued - bnum + 1) / 2;  // loads into buffer bnum
            if (uses > 0)
                mbar_wait_bounded(barKV0 + 8u * bnum, (uint32_t)((uses - 1) & 1), kWaitCycles / 16);
        }
        atomicOr(P.err, kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ----------------------------------------------------------------------------
// Kernel for d <= 64: four warps, one query row per thread (the row's TMEM
// lane), 128 TMEM columns, so four CTAs share an SM (three when an additive
// mask or bias is added, EXTRA: its values take registers) and their per-tile
// dependency chains overlap. Each 128-key tile of the plan is walked as two
// 64-key sub-tiles s = 0, 1, ... TMEM: S(s) (fp32) in columns [0, 64); once
// every row has read it, P(s) (bf16, two per column) overwrites columns
// [0, 32); O in [64, 64 + d). Per sub-tile, every warp:
//   wait S(s) | (thread 0: TMA K(s+2) into K(s)'s buffer and V(s+1) into
//   V(s-1)'s buffer, both free now) | S(s) to registers, scale, add the
//   additive terms, drop the entries the mask does not list, row max | if the
//   max grew past the threshold, rescale O in TMEM (P V(s-1) is done: S(s)
//   was issued after it) | exp2, row sum, P(s) to TMEM | the warp whose
//   arrival completes "P written" issues O (+)= P(s) V(s) (A operand from
//   TMEM), waits for it (P must be consumed before S(s+1) overwrites it) and
//   issues S(s+1).
// No warp waits for another except through the data; the block epilogue
// reads O, divides by the row sum, merges the gather kernel's partial and
// writes out and lse.
constexpr int kQuadThreads = 128;
constexpr uint32_t kQuadCols = 128;

template <int D, bool EXTRA>
struct QuadCfg {
    using C = TcCfg<D>;
    static constexpr int Q_BYTES = C::TILE_BYTES;       // 128 rows x d
    static constexpr int KV_BYTES = C::TILE_BYTES / 2;  // 64 rows x d
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = Q_BYTES;               // two buffers
    static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;  // two buffers
    // with additive terms: the staged term's block of the current sub-tile,
    // 128 rows x 64 keys bf16 (128-byte rows, 128-byte swizzle)
    static constexpr int OFF_A = OFF_V + 2 * KV_BYTES;
    static constexpr int A_BYTES = EXTRA ? 128 * 128 : 0;
    static constexpr int OFF_BAR = OFF_A + A_BYTES;
    // mbarriers Q_full, K_full[2], V_full[2], S_full, O_done, A_full; TMEM slot,
    // abort flag, "P written" arrivals; issue counts (K, V loads, S, P V
    // commits, staged-term loads)
    static constexpr int BAR_BYTES = 8 * 8 + 3 * 4 + 5 * 4;
    // at most four CTAs per SM (4 x 128 TMEM columns)
    static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES > 46 * 1024 ? OFF_BAR + BAR_BYTES : 46 * 1024;
};

// Bounded wait that also gives up as soon as another warp of the CTA has.
__device__ __forceinline__ bool pers_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
            *abort_flag = 1;
            return false;
        }
    }
}

template <int D, bool EXTRA, bool STAGED>
__global__ void __launch_bounds__(kQuadThreads, EXTRA && !STAGED ? 3 : 4)
    k_fwd_tc_quad(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmA,
                  const TcParams P) {
    using C = TcCfg<D>;
    using L = QuadCfg<D, EXTRA>;
    static_assert(D == 32 || D == 64, "head dim");
    extern __shared__ __align__(1024) uint8_t smem[];

    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.x / P.nqb, qb = blockIdx.x - bh * P.nqb;
    const int b = bh / P.H, h = bh - b * P.H;
    const int mk = P.num_masks == 1 ? 0 : b;
    const int64_t blk = (int64_t)mk * P.nqb + qb;
    int t_begin, T;
    block_tiles(P, blk, t_begin, T);
    if (T <= 0) return;
    const int klim = key_limit_tc(P, b);
    T = trim_tiles(P, t_begin, T, klim);
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) atomicOr(P.err, kErrTimeout);
        return;
    }
    const int NS = 2 * T;  // 64-key sub-tiles

    const uint32_t sQ = smem_u32(smem + L::OFF_Q), sK0 = smem_u32(smem + L::OFF_K),
                   sV0 = smem_u32(smem + L::OFF_V), sA = smem_u32(smem + L::OFF_A);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    const uint32_t barQ = smem_u32(bars + 0), barK0 = smem_u32(bars + 1), barV0 = smem_u32(bars + 3),
                   barS = smem_u32(bars + 5), barO = smem_u32(bars + 6), barA = smem_u32(bars + 7);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    uint32_t* pcnt = tmem_slot + 2;    // "P written" arrivals
    uint32_t* issued = tmem_slot + 3;  // [0] K, [1] V loads, [2] S, [3] P V commits, [4] staged-term loads

    // the row's state first: these loads run while the CTA sets up and the
    // first tiles arrive
    const int i = qb * 128 + tid;
    const bool row_ok = i < P.n;
    int rlo = 0, rhi = 0;  // interval masks: the row's run
    if (P.itv_lohi && row_ok) {
        const int2 v = P.itv_lohi[(int64_t)mk * P.n + i];
        rlo = v.x;
        rhi = v.y;
    }
    int info_next = P.tile_info[t_begin];  // the plan entry of the next 128-key tile
    int info = info_next;

    // Additive mask and bias (EXTRA). One term that varies by row (the bias,
    // else the mask) is staged: when TMA can fetch it (P.a_tma), its 128-row x
    // 64-key block of each sub-tile comes into shared memory in one load, issued
    // as soon as every warp has used the previous block (by the warp that
    // completes "P written"), and each thread reads its row from there;
    // otherwise, when it is bf16 with unit column stride and 16-byte aligned
    // rows, the 64 values of the row's next sub-tile are fetched as raw words
    // one sub-tile ahead (after P is stored), so their latency overlaps P V and
    // the next S. The other term -- typically a key-padding mask shared by every
    // row, served from L1 -- and every other layout are loaded when used.
    const int64_t mrb = EXTRA ? (int64_t)b * P.mask.s0 + (int64_t)h * P.mask.s1 + (int64_t)i * P.mask.s2 : 0;
    const int64_t brb = EXTRA ? (int64_t)b * P.bias.s0 + (int64_t)h * P.bias.s1 + (int64_t)i * P.bias.s2 : 0;
    // the prefetched term: 2 = bias, 1 = mask, 0 = none
    const int pre = !EXTRA ? 0 : (P.bias.data && P.bias.s2 != 0) ? 2 : (P.mask.data && P.mask.s2 != 0) ? 1 : 0;
    const AddendView& pview = pre == 2 ? P.bias : P.mask;
    const int64_t prb = pre == 2 ? brb : mrb;
    uint4 praw[EXTRA ? 8 : 1];
    bool raw = false;  // praw holds the prefetched term's values for the current sub-tile
    // STAGED: the build for a term TMA can fetch (the launcher's P.a_tma)
    constexpr bool staged = EXTRA && STAGED;
    // the staged term's block of sub-tile keys c0 .. c0 + 63 (one thread)
    auto load_a = [&](int c0) {
        mbar_expect_tx(barA, (uint32_t)L::A_BYTES);
        tma_load_4d(sA, &tmA, barA, c0, qb * 128, pview.s1 ? h : 0, pview.s0 ? b : 0);
        issued[4] += 1u;
    };
    auto fetch = [&](int c0) {
        raw = false;
        if (!EXTRA || staged || pre == 0 || !row_ok || c0 + 64 > P.n || pview.dtype != 0 || pview.s3 != 1) return;
        const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(pview.data) + prb + c0;
        if (reinterpret_cast<uintptr_t>(src) & 15u) return;
#pragma unroll
        for (int k = 0; k < (EXTRA ? 8 : 1); ++k) praw[k] = __ldg(reinterpret_cast<const uint4*>(src) + k);
        raw = true;
    };
    if (EXTRA) fetch((info & 0x7fffffff) * kTileN);

    // K or V sub-tile s (first key `key`) into buffer s & 1
    auto load_k = [&](int s, int key) {
        const uint32_t bar = barK0 + 8u * (s & 1);
        mbar_expect_tx(bar, (uint32_t)L::KV_BYTES);
        tma_load_4d(sK0 + (uint32_t)((s & 1) * L::KV_BYTES), &tmK, bar, 0, key, h, b);
        issued[0] += 1u;
    };
    auto load_v = [&](int s, int key) {
        const uint32_t bar = barV0 + 8u * (s & 1);
        mbar_expect_tx(bar, (uint32_t)L::KV_BYTES);
        tma_load_4d(sV0 + (uint32_t)((s & 1) * L::KV_BYTES), &tmV, bar, 0, key, h, b);
        issued[1] += 1u;
    };

    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kQuadCols);
    if (tid == 0) {
        for (int x = 0; x < 8; ++x) mbar_init(smem_u32(bars + x), 1);
        *abort_flag = 0;
        for (int x = 0; x < 6; ++x) pcnt[x] = 0u;  // and issued[]
        fence_mbar_init();
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        if (staged) {
            prefetch_tensormap(&tmA);
            load_a((info & 0x7fffffff) * kTileN);
        }
        // Q and both halves of the first tile (every block has at least one)
        mbar_expect_tx(barQ, (uint32_t)L::Q_BYTES);
        tma_load_4d(sQ, &tmQ, barQ, 0, qb * 128, h, b);
        const int key = (info & 0x7fffffff) * kTileN;
        load_k(0, key);
        load_k(1, key + 64);
        load_v(0, key);
        load_v(1, key + 64);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tP = tmem, tO = tmem + 64;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    auto issue_s = [&](int s) -> bool {  // S(s) = Q K(s)^T once K(s) is loaded
        if (!pers_wait(barK0 + 8u * (s & 1), (uint32_t)((s >> 1) & 1), abort_flag)) return false;
        tc_fence_after();
        const uint32_t sK = sK0 + (uint32_t)((s & 1) * L::KV_BYTES);
        const uint32_t idS = idesc_bf16_f32(128, 64, false);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t da = smem_desc(sQ + ks * 32, 16, C::SBO, C::LAYOUT);
            const uint64_t db = smem_desc(sK + ks * 32, 16, C::SBO, C::LAYOUT);
            mma_bf16_ss_elect(tS, da, db, idS, ks > 0 ? 1u : 0u);
        }
        mma_commit_elect(barS);
        if ((tid & 31) == 0) issued[2] += 1u;
        return true;
    };
    auto issue_pv = [&](int s) -> bool {  // O (+)= P(s) V(s) once V(s) is loaded
        if (!pers_wait(barV0 + 8u * (s & 1), (uint32_t)((s >> 1) & 1), abort_flag)) return false;
        tc_fence_after();
        const uint32_t sV = sV0 + (uint32_t)((s & 1) * L::KV_BYTES);
        const uint32_t idO = idesc_bf16_f32(128, D, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t db =
                smem_desc(sV + (uint32_t)(ks * 16 * C::ROW_BYTES), C::CHUNK_BYTES, C::SBO, C::LAYOUT);
            mma_bf16_ts_elect(tO, tP + (uint32_t)(ks * 8), db, idO, (s > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit_elect(barO);
        if ((tid & 31) == 0) issued[3] += 1u;
        return true;
    };

    // MMAs are issued by a whole warp (one elected lane): warp 0 here, later
    // the warp whose arrival completes "P written"
    if (warp == 0 && pers_wait(barQ, 0u, abort_flag)) issue_s(0);
    __syncwarp();

    const uint64_t c2 = pack2(P.qk_scale_log2, P.qk_scale_log2);
    float m_ref = -INFINITY, l = 0.f;
    for (int s = 0; s < NS; ++s) {
        if ((s & 1) == 0) {  // a new 128-key tile; fetch the next one's entry early
            info = info_next;
            if ((s >> 1) + 1 < T) info_next = P.tile_info[t_begin + (s >> 1) + 1];
        }
        const int c0 = (info & 0x7fffffff) * kTileN + 64 * (s & 1);
        bool dense = info < 0;
        uint32_t wb0 = 0u, wb1 = 0u;
        if (!dense && row_ok) {
            if (P.itv_lohi) {
                wb0 = run_word(rlo, rhi, c0);
                wb1 = run_word(rlo, rhi, c0 + 32);
            } else {
                const uint2 v = __ldg(reinterpret_cast<const uint2*>(P.tile_bits) +
                                      ((int64_t)(t_begin + (s >> 1)) * 128 + tid) * 2 + (s & 1));
                wb0 = v.x;
                wb1 = v.y;
            }
        }
        const int kcut = klim - c0;  // keys of this sub-tile inside the key length
        if (kcut < 64) {
            if (dense) {
                dense = false;
                wb0 = wb1 = 0xffffffffu;
            }
            wb0 &= run_word(0, kcut, 0);
            wb1 &= run_word(0, kcut, 32);
        }

        const bool ok = pers_wait(barS, (uint32_t)(s & 1), abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        if (tid == 0) {  // S(s) done: K(s)'s buffer is free; P V(s-1) done: so is V(s-1)'s
            // sub-tile s + 2 is the next tile's half s & 1; s + 1 is this tile's
            // second half (s even) or the next tile's first (s odd)
            if (s + 2 < NS) load_k(s + 2, (info_next & 0x7fffffff) * kTileN + 64 * (s & 1));
            if (s >= 1 && s + 1 < NS)
                load_v(s + 1, (((s & 1) ? info_next : info) & 0x7fffffff) * kTileN + 64 * ((s + 1) & 1));
        }
        if (staged) {  // this sub-tile's block of the staged term, from shared memory
            const bool oka = pers_wait(barA, (uint32_t)(s & 1), abort_flag);
            if (!__all_sync(0xffffffffu, oka)) break;
            // unit u of row r at r * 128 + (u ^ (r & 7)) * 16 (128-byte swizzle)
            const uint32_t rowa = sA + (uint32_t)tid * 128u;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                uint4 v4;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v4.x), "=r"(v4.y), "=r"(v4.z), "=r"(v4.w)
                             : "r"(rowa + (uint32_t)((u ^ (tid & 7)) << 4))
                             : "memory");
                praw[u] = v4;
            }
            raw = row_ok;
        }
        float x[64];
        {
            uint32_t r0[32], r1[32];
            tmem_ld32(tS + lane_base, r0);
            tmem_ld32(tS + lane_base + 32, r1);
            tmem_wait_ld_dep(r0);
            tmem_wait_ld_dep(r1);
            if (EXTRA && raw) {  // x = scale*log2(e)*S + log2(e)*(prefetched term)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t w[4] = {praw[k].x, praw[k].y, praw[k].z, praw[k].w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int j = 8 * k + 2 * t;
                        const uint32_t s0 = j < 32 ? r0[j] : r1[j - 32], s1 = j < 32 ? r0[j + 1] : r1[j - 31];
                        x[j] = fmaf(__uint_as_float(s0), P.qk_scale_log2, kLog2e * __uint_as_float(w[t] << 16));
                        x[j + 1] = fmaf(__uint_as_float(s1), P.qk_scale_log2,
                                        kLog2e * __uint_as_float(w[t] & 0xffff0000u));
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    mul2(x[2 * k], x[2 * k + 1], r0[2 * k], r0[2 * k + 1], c2);
                    mul2(x[32 + 2 * k], x[33 + 2 * k], r1[2 * k], r1[2 * k + 1], c2);
                }
            }
            if (EXTRA && row_ok) {  // + log2(e) * (the terms not prefetched), loaded now
                const int ncols = P.n - c0 < 64 ? P.n - c0 : 64;
                if (P.mask.data && !(raw && pre == 1)) add_addend_run<64>(P.mask, mrb, c0, ncols, x);
                if (P.bias.data && !(raw && pre == 2)) add_addend_run<64>(P.bias, brb, c0, ncols, x);
            }
        }
        if (!dense) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                x[jj] = ((wb0 >> jj) & 1u) ? x[jj] : -INFINITY;
                x[32 + jj] = ((wb1 >> jj) & 1u) ? x[32 + jj] : -INFINITY;
            }
        }
        float ma = -INFINITY, mb = -INFINITY, mc = -INFINITY, md = -INFINITY;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            ma = fmax3(ma, x[8 * k + 0], x[8 * k + 1]);
            mb = fmax3(mb, x[8 * k + 2], x[8 * k + 3]);
            mc = fmax3(mc, x[8 * k + 4], x[8 * k + 5]);
            md = fmax3(md, x[8 * k + 6], x[8 * k + 7]);
        }
        const float mx = fmax3(ma, mb, fmaxf(mc, md));
        const bool need = mx > m_ref + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
            alpha = ex2(m_ref - mx);
            m_ref = mx;
            l *= alpha;
        }
        if (s > 0 && __any_sync(0xffffffffu, need)) {  // bring O (= P V(..s-1), complete) to the new max
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                uint32_t ro[16];
                tmem_ld16(tO + lane_base + 16 * c, ro);
                tmem_wait_ld_dep16(ro);
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) ro[jj] = __float_as_uint(__uint_as_float(ro[jj]) * alpha);
                tmem_st16(tO + lane_base + 16 * c, ro);
            }
        }
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        const uint64_t nmu2 = pack2(-mu, -mu);
        uint64_t sa = pack2(0.f, 0.f), sb = sa;
        uint32_t pk[32];  // P row, two bf16 per word
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            float p0, p1;
            unpack2(add2(pack2(x[2 * k], x[2 * k + 1]), nmu2), p0, p1);
            p0 = ex2(p0);
            p1 = ex2(p1);
            if (k & 1)
                sb = add2(sb, pack2(p0, p1));
            else
                sa = add2(sa, pack2(p0, p1));
            __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
            pk[k] = *reinterpret_cast<uint32_t*>(&hv);
        }
        {
            float s0, s1, s2, s3;
            unpack2(sa, s0, s1);
            unpack2(sb, s2, s3);
            l += (s0 + s1) + (s2 + s3);
        }
        tmem_st32(tP + lane_base, pk);
        tmem_wait_st();
        if (EXTRA && s + 1 < NS)  // the next sub-tile: this tile's second half or the next tile's first
            fetch((((s & 1) ? info_next : info) & 0x7fffffff) * kTileN + 64 * ((s + 1) & 1));
        const bool last = __shfl_sync(0xffffffffu, arrive_last(pcnt, 4u * (uint32_t)(s + 1) - 1u) ? 1 : 0, 0) != 0;
        if (last && !*abort_flag) {
            // every warp has used the staged term's block of sub-tile s: bring
            // in the next one
            if (staged && s + 1 < NS) {
                fence_proxy_async_smem();
                if ((tid & 31) == 0) load_a((((s & 1) ? info_next : info) & 0x7fffffff) * kTileN + 64 * ((s + 1) & 1));
                __syncwarp();
            }
            // every row has written P(s) (and rescaled O): P V(s), then S(s+1) once
            // P V(s) has consumed P (S(s+1) overwrites it)
            if (issue_pv(s) && s + 1 < NS && pers_wait(barO, (uint32_t)(s & 1), abort_flag)) issue_s(s + 1);
        }
        __syncwarp();
    }

    // ------------------------------------------------------------ epilogue
    const bool ok = pers_wait(barO, (uint32_t)((NS - 1) & 1), abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        float o[D];
        {
            uint32_t ro[32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                tmem_ld32(tO + lane_base + 32 * c, ro);
                tmem_wait_ld_dep(ro);
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) o[32 * c + jj] = __uint_as_float(ro[jj]);
            }
        }
        if (row_ok && !*abort_flag) {
            const int64_t mrow = (int64_t)mk * P.n + i, wrow = (int64_t)bh * P.n + i;
            float M = m_ref, Ls = l, fa = 1.f, fg = 0.f;
            const bool mixed = has_partial(P, blk, mrow, wrow);
            if (mixed) {
                const float mg = P.ws_ml[wrow * 2], lg = P.ws_ml[wrow * 2 + 1];
                M = fmaxf(m_ref, mg);
                const float Mu = M == -INFINITY ? 0.f : M;
                fa = ex2(m_ref - Mu);
                fg = ex2(mg - Mu);
                Ls = l * fa + lg * fg;
            }
            const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(P.out) + (int64_t)b * P.o_sb +
                                  (int64_t)h * P.o_sh + (int64_t)i * P.o_sn;
            const float* acc = mixed ? P.ws_acc + wrow * D : nullptr;
#pragma unroll
            for (int e8 = 0; e8 < D / 8; ++e8) {
                float v[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    float val = o[e8 * 8 + t] * fa;
                    if (mixed) val = fmaf(acc[e8 * 8 + t], fg, val);
                    v[t] = val * inv;
                }
                uint32_t w[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    __nv_bfloat162 hv = __floats2bfloat162_rn(v[2 * t], v[2 * t + 1]);
                    w[t] = *reinterpret_cast<uint32_t*>(&hv);
                }
                *reinterpret_cast<uint4*>(orow + e8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (P.lse) P.lse[wrow] = Ls > 0.f ? (M + lg2(Ls)) * kLn2 : -INFINITY;
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) {  // drain what was issued (bounded), then report
        const long long lim = kWaitCycles / 16;
        mbar_wait_bounded(barQ, 0u, lim);
        for (int x = 0; x < 2; ++x)
            for (int bnum = 0; bnum < 2; ++bnum) {
                const int uses = ((int)issued[x] - bnum + 1) / 2;  // loads into buffer bnum
                if (uses > 0)
                    mbar_wait_bounded(smem_u32(bars + 1 + 2 * x + bnum), (uint32_t)((uses - 1) & 1), lim);
            }
        if (issued[2]) mbar_wait_bounded(barS, (issued[2] - 1u) & 1u, lim);
        if (issued[3]) mbar_wait_bounded(barO, (issued[3] - 1u) & 1u, lim);
        if (issued[4]) mbar_wait_bounded(barA, (issued[4] - 1u) & 1u, lim);
        atomicOr(P.err, kErrTimeout);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kQuadCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 4-D map over a [B, H, n, d] bf16 tensor, box {chunk, rows, 1, 1}.
cudaError_t make_map(CUtensorMap* map, const TcOperand& t, int B, int H, int n, int d, int chunk,
                     int rows = 128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const uint64_t sn = (uint64_t)t.s_n * 2;
    const uint64_t sh = H > 1 ? (uint64_t)t.s_h * 2 : sn * (uint64_t)n;
    const uint64_t sb = B > 1 ? (uint64_t)t.s_b * 2 : sh * (uint64_t)H;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {sn, sh, sb};
    cuuint32_t box[4] = {(cuuint32_t)chunk, (cuuint32_t)rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw =
        chunk * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.data), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Whether TMA can fetch an additive term: bf16 with unit key stride, the base
// and every stride a multiple of 16 bytes.
bool addend_tma_ok(const AddendView& a) {
    const uintptr_t base = reinterpret_cast<uintptr_t>(a.data);
    return a.dtype == 0 && a.s3 == 1 && (base & 15) == 0 && (a.s2 * 2) % 16 == 0 && (a.s1 * 2) % 16 == 0 &&
           (a.s0 * 2) % 16 == 0;
}

// A per-row additive term [B or 1, H or 1, n, n] (bf16, keys contiguous) as
// {keys, rows, heads, batch}, box {64, 128, 1, 1}, 128-byte swizzle; the
// dimensions it broadcasts over have extent 1.
cudaError_t make_addend_map(CUtensorMap* map, const AddendView& a, int B, int H, int n) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const uint64_t row_bytes = ((uint64_t)n * 2 + 15) & ~uint64_t(15);  // a valid stride for extent-1 dimensions
    cuuint64_t dims[4] = {(cuuint64_t)n, (cuuint64_t)n, (cuuint64_t)(a.s1 ? H : 1), (cuuint64_t)(a.s0 ? B : 1)};
    cuuint64_t strides[3] = {(uint64_t)a.s2 * 2, a.s1 ? (uint64_t)a.s1 * 2 : row_bytes, a.s0 ? (uint64_t)a.s0 * 2 : row_bytes};
    cuuint32_t box[4] = {64, 128, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(a.data), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 5-D map over a [B, H, n, d] bf16 tensor read in residue-permuted order:
// dims {d, S, G, H, B} (row i = k S + r at (r, k)), box {chunk, 1, 128, 1, 1}:
// one load brings rows r, r + S, ..., r + 127 S.
cudaError_t make_perm_map(CUtensorMap* map, const TcOperand& t, int B, int H, int n, int d, int chunk, int G) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const int S = n / G;
    const uint64_t sn = (uint64_t)t.s_n * 2;
    const uint64_t sh = H > 1 ? (uint64_t)t.s_h * 2 : sn * (uint64_t)n;
    const uint64_t sb = B > 1 ? (uint64_t)t.s_b * 2 : sh * (uint64_t)H;
    cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)S, (cuuint64_t)G, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[4] = {sn, sn * (uint64_t)S, sh, sb};
    cuuint32_t box[5] = {(cuuint32_t)chunk, 1, 128, 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapSwizzle sw =
        chunk * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(t.data), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_tc_t(const TcOperand& q, const TcOperand& k, const TcOperand& v, const TcParams& p,
                        cudaStream_t s) {
    using C = TcCfg<D>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, []() {
        constexpr int DP = D <= 64 ? D : 64;
        if (D <= 64) {
            attr_err = cudaFuncSetAttribute((const void*)k_fwd_tc_quad<DP, true, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, QuadCfg<DP, true>::SMEM_BYTES);
            if (attr_err == cudaSuccess)
                attr_err = cudaFuncSetAttribute((const void*)k_fwd_tc_quad<DP, true, false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                QuadCfg<DP, true>::SMEM_BYTES);
            if (attr_err == cudaSuccess)
                attr_err = cudaFuncSetAttribute((const void*)k_fwd_tc_quad<DP, false, false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                QuadCfg<DP, false>::SMEM_BYTES);
        } else {
            attr_err = cudaFuncSetAttribute((const void*)k_fwd_tc<D>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        }
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mq, mk, mv;
    cudaError_t e;
    if (p.perm_G) {  // d = 128 only (k_fwd_tc), every load a permuted 128-row box
        if (D != 128 || p.perm_G % 128 != 0 || p.n % p.perm_G != 0) return cudaErrorInvalidValue;
        if ((e = make_perm_map(&mq, q, p.B, p.H, p.n, D, C::CHUNK_ELEMS, p.perm_G)) != cudaSuccess) return e;
        if ((e = make_perm_map(&mk, k, p.B, p.H, p.n, D, C::CHUNK_ELEMS, p.perm_G)) != cudaSuccess) return e;
        if ((e = make_perm_map(&mv, v, p.B, p.H, p.n, D, C::CHUNK_ELEMS, p.perm_G)) != cudaSuccess) return e;
        const int64_t grid = (int64_t)p.B * p.H * p.nqb + (p.blk_nch ? (int64_t)p.B * p.H * p.n_extra : 0);
        if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        k_fwd_tc<D><<<(unsigned)grid, kThreads, C::SMEM_BYTES, counted(s)>>>(mq, mk, mv, p);
        return cudaGetLastError();
    }
    if ((e = make_map(&mq, q, p.B, p.H, p.n, D, C::CHUNK_ELEMS)) != cudaSuccess) return e;
    // d <= 64: k_fwd_tc_quad loads K and V in 64-row sub-tiles
    const int kv_rows = D <= 64 ? 64 : 128;
    if ((e = make_map(&mk, k, p.B, p.H, p.n, D, C::CHUNK_ELEMS, kv_rows)) != cudaSuccess) return e;
    if ((e = make_map(&mv, v, p.B, p.H, p.n, D, C::CHUNK_ELEMS, kv_rows)) != cudaSuccess) return e;
    const int64_t grid = (int64_t)p.B * p.H * p.nqb;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    constexpr int DP = D <= 64 ? D : 64;
    if (D <= 64 && p.has_extra) {
        // the term that varies by row (the bias, else the mask) goes through
        // shared memory when TMA can fetch it
        TcParams pe = p;
        CUtensorMap ma = mq;
        const AddendView& t = (p.bias.data && p.bias.s2 != 0) ? p.bias : p.mask;
        pe.a_tma = t.data && t.s2 != 0 && addend_tma_ok(t) && make_addend_map(&ma, t, p.B, p.H, p.n) == cudaSuccess;
        if (pe.a_tma)
            k_fwd_tc_quad<DP, true, true><<<(unsigned)grid, kQuadThreads, QuadCfg<DP, true>::SMEM_BYTES, counted(s)>>>(
                mq, mk, mv, ma, pe);
        else
            k_fwd_tc_quad<DP, true, false><<<(unsigned)grid, kQuadThreads, QuadCfg<DP, true>::SMEM_BYTES, counted(s)>>>(
                mq, mk, mv, ma, pe);
    } else if (D <= 64) {
        k_fwd_tc_quad<DP, false, false><<<(unsigned)grid, kQuadThreads, QuadCfg<DP, false>::SMEM_BYTES, counted(s)>>>(mq, mk, mv, mq,
                                                                                                      p);
    } else {
        // one thread block per query block, plus one per further chunk of split blocks
        const int64_t grid2 = grid + (p.blk_nch ? (int64_t)p.B * p.H * p.n_extra : 0);
        if (grid2 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        k_fwd_tc<D><<<(unsigned)grid2, kThreads, C::SMEM_BYTES, counted(s)>>>(mq, mk, mv, p);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const TcOperand& q, const TcOperand& k, const TcOperand& v, int d,
                          const TcParams& p, cudaStream_t s) {
    switch (d) {
    case 32: return launch_tc_t<32>(q, k, v, p, s);
    case 64: return launch_tc_t<64>(q, k, v, p, s);
    case 128: return launch_tc_t<128>(q, k, v, p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace spattn
