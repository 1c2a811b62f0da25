// Tile plan of a built mask: which parts of the CSR go to the tensor-core
// kernel and which stay with the gather kernel.
//
// The n x n mask is cut into 128 x 128 tiles (128 query rows by 128 keys).
// A tile holding at least `tile_min_nnz` nonzeros becomes a tensor-core tile:
// the kernel computes all 128 x 128 scores with tcgen05 MMAs and a per-row
// 128-bit mask drops the entries the CSR does not list (the block-sparse idea
// of the gluon-nlp discussion -- whole blocks are cheaper than single
// entries -- applied per tile of an arbitrary CSR). The remaining nonzeros form
// the residual CSR, which the gather kernel processes. Rows that have entries
// in both are merged with the streaming-softmax rescaling rule.
#include "spattn.h"
#include "spattn_internal.cuh"

namespace spattn {
namespace {

// One warp per mask row: count the row's nonzeros per key tile (columns are
// sorted, so a tile's entries form one run per 32-entry chunk).
__global__ void k_tile_count(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                             int n, int64_t rows, int nqb, int nkt, int32_t* __restrict__ cnt) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const int64_t m = r / n, i = r - m * n;
        const int64_t base = (m * nqb + (i >> 7)) * nkt;
        const int64_t p0 = row_ptr[r], p1 = row_ptr[r + 1];
        for (int64_t c0 = p0; c0 < p1; c0 += 32) {
            const int64_t p = c0 + lane;
            const bool valid = p < p1;
            const int kt = valid ? (col_idx[p] >> 7) : -1;
            const int prev = __shfl_up_sync(0xffffffffu, kt, 1);
            const bool head = valid && (lane == 0 || prev != kt);
            const unsigned heads = __ballot_sync(0xffffffffu, head);
            if (head) {
                const unsigned above = lane == 31 ? 0u : (heads & (0xffffffffu << (lane + 1)));
                const int nvalid = (int)((p1 - c0) < 32 ? (p1 - c0) : 32);
                const int nxt = above ? __ffs(above) - 1 : nvalid;
                atomicAdd(&cnt[base + kt], nxt - lane);
            }
        }
    }
}

// One thread per (mask, query block): how many of its key tiles are selected.
__global__ void k_tile_select(const int32_t* __restrict__ cnt, int64_t nblocks, int nkt,
                              int min_nnz, int32_t* __restrict__ block_ntiles,
                              int32_t* __restrict__ n_tc_blocks) {
    for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < nblocks;
         x += (int64_t)gridDim.x * blockDim.x) {
        int c = 0;
        for (int kt = 0; kt < nkt; ++kt) c += cnt[x * nkt + kt] >= min_nnz;
        block_ntiles[x] = c;
        if (c > 0) atomicAdd(n_tc_blocks, 1);
    }
}

// Number the selected tiles (block-major, key tiles ascending) and turn the
// count array into a map (tile id, or -1). One warp per query block.
__global__ void k_tile_assign(int32_t* __restrict__ cnt_map, int64_t nblocks, int nkt, int min_nnz,
                              const int32_t* __restrict__ block_tile_off,
                              int32_t* __restrict__ tile_info) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t x = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); x < nblocks;
         x += warps) {
        int idx = block_tile_off[x];
        for (int k0 = 0; k0 < nkt; k0 += 32) {
            const int kt = k0 + lane;
            const int c = kt < nkt ? cnt_map[x * nkt + kt] : 0;
            const bool sel = kt < nkt && c >= min_nnz;
            const unsigned bal = __ballot_sync(0xffffffffu, sel);
            if (kt < nkt) {
                if (sel) {
                    const int id = idx + __popc(bal & ((1u << lane) - 1u));
                    tile_info[id] = kt | (c == kTileM * kTileN ? (int)kTileDenseBit : 0);
                    cnt_map[x * nkt + kt] = id;
                } else {
                    cnt_map[x * nkt + kt] = -1;
                }
            }
            idx += __popc(bal);
        }
    }
}

// One warp per row: set the bits of entries in selected (not dense) tiles, one
// atomic per 32-bit word (columns are sorted, so a word's entries are adjacent
// lanes), count the rest and list rows whose residual is long.
__global__ void k_tile_bits(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                            int n, int64_t rows, int nqb, int nkt, const int32_t* __restrict__ map,
                            const int32_t* __restrict__ tile_info, uint32_t* __restrict__ bits,
                            int32_t* __restrict__ res_cnt, int32_t* __restrict__ res_long,
                            int32_t* __restrict__ res_n_long) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const int64_t m = r / n, i = r - m * n;
        const int64_t base = (m * nqb + (i >> 7)) * nkt;
        const int row_in_tile = (int)(i & 127);
        int res = 0;
        const int64_t p1 = row_ptr[r + 1];
        for (int64_t c0 = row_ptr[r]; c0 < p1; c0 += 32) {
            const int64_t p = c0 + lane;
            int key = -1;
            uint32_t bit = 0u;
            bool residual = false;
            if (p < p1) {
                const int j = col_idx[p];
                const int id = map[base + (j >> 7)];
                if (id >= 0) {
                    if (tile_info[id] >= 0) {  // dense tiles need no bits
                        key = id * 4 + ((j & 127) >> 5);
                        bit = 1u << (j & 31);
                    }
                } else {
                    residual = true;
                }
            }
            res += __popc(__ballot_sync(0xffffffffu, residual));
            const unsigned grp = __match_any_sync(0xffffffffu, key);
            const uint32_t word = __reduce_or_sync(grp, bit);
            if (key >= 0 && lane == __ffs(grp) - 1)
                atomicOr(&bits[((int64_t)(key >> 2) * kTileM + row_in_tile) * 4 + (key & 3)], word);
        }
        if (lane == 0) {
            res_cnt[r] = res;
            if (res > kLongRowThreshold) res_long[atomicAdd(res_n_long, 1)] = (int32_t)r;
        }
    }
}

// One warp per row: copy the residual entries (ascending) and count the rows
// that mix tensor-core tiles and residual entries.
__global__ void k_residual_fill(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                                int n, int64_t rows, int nqb, int nkt, const int32_t* __restrict__ map,
                                const int32_t* __restrict__ block_tile_off,
                                const int32_t* __restrict__ res_row_ptr, int32_t* __restrict__ res_col,
                                int32_t* __restrict__ n_mixed) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const int64_t m = r / n, i = r - m * n;
        const int64_t blk = m * nqb + (i >> 7);
        const int64_t base = blk * nkt;
        int64_t o = res_row_ptr[r];
        if (res_row_ptr[r + 1] == o) continue;  // nothing left for the gather kernel
        const int64_t p1 = row_ptr[r + 1];
        for (int64_t c0 = row_ptr[r]; c0 < p1; c0 += 32) {
            const int64_t p = c0 + lane;
            int j = -1;
            bool keep = false;
            if (p < p1) {
                j = col_idx[p];
                keep = map[base + (j >> 7)] < 0;
            }
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            if (keep) res_col[o + __popc(bal & ((1u << lane) - 1u))] = j;
            o += __popc(bal);
        }
        if (lane == 0 && block_tile_off[blk + 1] > block_tile_off[blk]) atomicAdd(n_mixed, 1);
    }
}

// ---------------------------------------------------------------------------
// Interval rows (sliding window, variable window, dense): each row's columns are
// one run [lo, hi), read from the row's first and last CSR entry. Counts, bits
// and residual runs follow from the run's overlap with each tile, without
// reading the rest of col_idx.

// The run [lo, hi) of an interval row: from the mask's runs when given, else
// from its first and last CSR column.
__device__ __forceinline__ void row_run(const int32_t* __restrict__ row_ptr,
                                        const int32_t* __restrict__ col_idx,
                                        const int2* __restrict__ lohi, int64_t r, int& lo, int& hi) {
    if (lohi) {
        const int2 v = lohi[r];
        lo = v.x;
        hi = v.y;
        return;
    }
    const int64_t p0 = row_ptr[r], p1 = row_ptr[r + 1];
    if (p1 > p0) {
        lo = col_idx[p0];
        hi = col_idx[p1 - 1] + 1;
    } else {
        lo = hi = 0;
    }
}

__device__ __forceinline__ int overlap(int lo, int hi, int c0, int c1) {
    const int a = lo > c0 ? lo : c0, z = hi < c1 ? hi : c1;
    return z > a ? z - a : 0;
}

// One warp per 32 rows of a query block: per-tile counts, one atomic per tile.
__global__ void k_itv_count(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                            const int2* __restrict__ lohi, int n, int64_t nblocks, int nqb, int nkt, int32_t* __restrict__ cnt) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = nblocks * 4;
    for (int64_t w = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); w < nwarps;
         w += (int64_t)gridDim.x * (blockDim.x >> 5)) {
        const int64_t blk = w >> 2;
        const int64_t m = blk / nqb;
        const int i = (int)(blk - m * nqb) * kTileM + (int)(w & 3) * 32 + lane;
        int lo = 0, hi = 0;
        if (i < n) row_run(row_ptr, col_idx, lohi, m * n + i, lo, hi);
        const bool any = hi > lo;
        int k0 = any ? lo >> 7 : 0x7fffffff, k1 = any ? (hi - 1) >> 7 : -1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            k0 = min(k0, __shfl_xor_sync(0xffffffffu, k0, off));
            k1 = max(k1, __shfl_xor_sync(0xffffffffu, k1, off));
        }
        for (int kt = k0; kt <= k1; ++kt) {
            int c = overlap(lo, hi, kt * kTileN, kt * kTileN + kTileN);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
            if (lane == 0 && c) atomicAdd(&cnt[blk * nkt + kt], c);
        }
    }
}

// One thread per row slot of every query block: the row's bits in each
// selected (not dense) tile of its block -- zero words included, so the bit
// array needs no clearing -- and its residual count.
__global__ void k_itv_bits(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                           const int2* __restrict__ lohi, int n, int64_t nblocks, int nqb, const int32_t* __restrict__ block_tile_off,
                           const int32_t* __restrict__ tile_info, uint32_t* __restrict__ bits,
                           int32_t* __restrict__ res_cnt, int32_t* __restrict__ res_long,
                           int32_t* __restrict__ res_n_long) {
    for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < nblocks * kTileM;
         x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = x / kTileM;
        const int row = (int)(x - blk * kTileM);
        const int64_t m = blk / nqb;
        const int i = (int)(blk - m * nqb) * kTileM + row;
        int lo = 0, hi = 0;
        if (i < n) row_run(row_ptr, col_idx, lohi, m * n + i, lo, hi);
        int in_tiles = 0;
        for (int t = block_tile_off[blk]; t < block_tile_off[blk + 1]; ++t) {
            const int info = tile_info[t];
            const int c0 = (info & 0x7fffffff) * kTileN;
            in_tiles += overlap(lo, hi, c0, c0 + kTileN);
            uint4* dst = reinterpret_cast<uint4*>(bits + ((int64_t)t * kTileM + row) * 4);
            if (info < 0) {  // dense: the kernel reads no bits; store zero words
                *dst = make_uint4(0u, 0u, 0u, 0u);
                continue;
            }
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int a = c0 + 32 * q;
                const int lo2 = lo > a ? lo : a, hi2 = hi < a + 32 ? hi : a + 32;
                const int len = hi2 - lo2;
                w[q] = len <= 0 ? 0u : (len == 32 ? 0xffffffffu : (((1u << len) - 1u) << (lo2 - a)));
            }
            *dst = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (i < n) {
            const int res = (hi - lo) - in_tiles;
            res_cnt[m * n + i] = res;
            if (res > kLongRowThreshold) res_long[atomicAdd(res_n_long, 1)] = (int32_t)(m * n + i);
        }
    }
}

// One thread per row: the residual runs (parts of [lo, hi) in unselected tiles).
__global__ void k_itv_residual(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                               const int2* __restrict__ lohi, int n, int64_t rows, int nqb, int nkt, const int32_t* __restrict__ map,
                               const int32_t* __restrict__ block_tile_off,
                               const int32_t* __restrict__ res_row_ptr, int32_t* __restrict__ res_col,
                               int32_t* __restrict__ n_mixed) {
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows;
         r += (int64_t)gridDim.x * blockDim.x) {
        int64_t o = res_row_ptr[r];
        if (res_row_ptr[r + 1] == o) continue;
        const int64_t m = r / n, i = r - m * n;
        const int64_t blk = m * nqb + (i >> 7);
        int lo, hi;
        row_run(row_ptr, col_idx, lohi, r, lo, hi);
        for (int kt = lo >> 7; kt <= (hi - 1) >> 7; ++kt) {
            if (map[blk * nkt + kt] >= 0) continue;
            const int a = lo > kt * kTileN ? lo : kt * kTileN;
            const int z = hi < kt * kTileN + kTileN ? hi : kt * kTileN + kTileN;
            for (int j = a; j < z; ++j) res_col[o++] = j;
        }
        if (block_tile_off[blk + 1] > block_tile_off[blk]) atomicAdd(n_mixed, 1);
    }
}

// One block: select the tiles of every query block, number them (block-major,
// key tiles ascending), write block_tile_off and the tile map -- the work of
// k_tile_select + scan + k_tile_assign in one launch, for block grids up to
// kFusedSelectMax query blocks.
constexpr int kFusedSelectMax = 1 << 16;

__global__ void __launch_bounds__(1024)
    k_tile_select_fused(int32_t* __restrict__ cnt_map, int nblocks, int nkt, int min_nnz,
                        int32_t* __restrict__ block_tile_off, int32_t* __restrict__ tile_info,
                        PlanCounters* counters) {
    __shared__ int32_t wsum[32];
    __shared__ int32_t carry_s;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    int tc_blocks = 0;
    // pass 1: per-block selected counts, scanned into block_tile_off
    for (int x0 = 0; x0 < nblocks; x0 += 1024) {
        const int x = x0 + threadIdx.x;
        int c = 0;
        if (x < nblocks) {  // eight independent loads in flight per step
            const int32_t* row = cnt_map + (int64_t)x * nkt;
            int kt = 0;
            for (; kt + 8 <= nkt; kt += 8) {
                int32_t v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = row[kt + u];
#pragma unroll
                for (int u = 0; u < 8; ++u) c += v[u] >= min_nnz;
            }
            for (; kt < nkt; ++kt) c += row[kt] >= min_nnz;
        }
        tc_blocks += c > 0;
        int inc = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += y;
        }
        if (lane == 31) wsum[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            const int w = wsum[lane];
            int wi = w;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, wi, off);
                if (lane >= off) wi += y;
            }
            wsum[lane] = wi - w;
        }
        __syncthreads();
        const int carry = carry_s;
        if (x < nblocks) block_tile_off[x] = carry + wsum[warp] + inc - c;
        __syncthreads();
        if (threadIdx.x == 1023) carry_s = carry + wsum[warp] + inc;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        block_tile_off[nblocks] = carry_s;
        counters->n_tiles = carry_s;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) tc_blocks += __shfl_xor_sync(0xffffffffu, tc_blocks, off);
    if (lane == 0 && tc_blocks) atomicAdd(&counters->n_tc_blocks, tc_blocks);
    __syncthreads();
    // pass 2: one warp per block numbers its selected tiles
    for (int x = warp; x < nblocks; x += 32) {
        int idx = block_tile_off[x];
        for (int k0 = 0; k0 < nkt; k0 += 32) {
            const int kt = k0 + lane;
            const int c = kt < nkt ? cnt_map[(int64_t)x * nkt + kt] : 0;
            const bool sel = kt < nkt && c >= min_nnz;
            const unsigned bal = __ballot_sync(0xffffffffu, sel);
            if (kt < nkt) {
                if (sel) {
                    const int id = idx + __popc(bal & ((1u << lane) - 1u));
                    tile_info[id] = kt | (c == kTileM * kTileN ? (int)kTileDenseBit : 0);
                    cnt_map[(int64_t)x * nkt + kt] = id;
                } else {
                    cnt_map[(int64_t)x * nkt + kt] = -1;
                }
            }
            idx += __popc(bal);
        }
    }
}

// Clears the tile count array and the plan counters.
__global__ void k_plan_zero(int32_t* __restrict__ cnt, int64_t n_cnt, PlanCounters* counters) {
    for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < n_cnt;
         x += (int64_t)gridDim.x * blockDim.x)
        cnt[x] = 0;
    if (blockIdx.x == 0 && threadIdx.x < sizeof(PlanCounters) / 4)
        reinterpret_cast<uint32_t*>(counters)[threadIdx.x] = 0u;
}

// ------------------------------------------------- implicit interval masks
// One CTA of 128 threads per query block (128 rows of one mask): each row's run
// [lo, hi) from the pattern (a negative half-width leaves the row empty), the
// block's entry count per key tile accumulated in shared memory (a warp
// reduction and one shared atomic per tile and warp), the tile selection -- the
// tiles with at least min_nnz entries, listed in key order at tiles[blk * nkt ..]
// (bit 31: all 128 x 128 entries present), the map tmap[blk * nkt + kt] = local
// tile number or -1, whether entries stay outside the selected tiles -- and the
// block's statistics. The last CTA to finish (a self-resetting counter) adds the
// statistics up into the mask's totals.
__global__ void __launch_bounds__(kTileM)
    k_itv_build(ItvSpec s, int min_nnz, int2* __restrict__ lohi, int32_t* __restrict__ tmap,
                int32_t* __restrict__ tiles, int32_t* __restrict__ ntiles, int32_t* __restrict__ blk_res,
                ItvBlockStat* bstat, unsigned* done, ItvCounters* out) {
    extern __shared__ int32_t cs[];  // [nkt]
    __shared__ int32_t wsel[4];
    __shared__ long long wsum[2][4];
    __shared__ bool last_s;
    const int64_t nblocks = (int64_t)gridDim.x;
    const int64_t blk = blockIdx.x;
    const int64_t m = blk / s.nqb;
    const int qb = (int)(blk - m * s.nqb);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int kt = threadIdx.x; kt < s.nkt; kt += kTileM) cs[kt] = 0;
    __syncthreads();
    const int i = qb * kTileM + threadIdx.x;
    int lo = 0, hi = 0;
    bool bad = false;
    if (i < s.n) {
        const int64_t r = m * s.n + i;
        if (s.kind == SPATTN_MASK_DENSE) {
            hi = s.n;
        } else {
            const int64_t w = s.kind == SPATTN_MASK_SLIDING ? (int64_t)s.window : (int64_t)s.half_widths[r];
            if (w < 0) {
                bad = true;
            } else {
                lo = (int)(i - w < 0 ? 0 : i - w);
                hi = (int)(i + w + 1 > s.n ? s.n : i + w + 1);
            }
        }
        lohi[r] = make_int2(lo, hi);
    }
    {
        const bool any = hi > lo;
        int k0 = any ? lo >> 7 : 0x7fffffff, k1 = any ? (hi - 1) >> 7 : -1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            k0 = min(k0, __shfl_xor_sync(0xffffffffu, k0, off));
            k1 = max(k1, __shfl_xor_sync(0xffffffffu, k1, off));
        }
        for (int kt = k0; kt <= k1; ++kt) {
            int c = overlap(lo, hi, kt * kTileN, kt * kTileN + kTileN);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
            if (lane == 0 && c) atomicAdd(&cs[kt], c);
        }
    }
    const int n_long = __syncthreads_count(hi - lo > kLongRowThreshold);
    const int n_bad = __syncthreads_count(bad);
    // selection, 128 key tiles at a time, numbered in key order
    long long nnz = 0, res = 0;
    int base = 0;
    for (int c0 = 0; c0 < s.nkt; c0 += kTileM) {
        const int kt = c0 + threadIdx.x;
        const int v = kt < s.nkt ? cs[kt] : 0;
        const bool sel = min_nnz > 0 && v >= min_nnz;
        const unsigned bal = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) wsel[warp] = __popc(bal);
        __syncthreads();
        int off = base;
        for (int w = 0; w < warp; ++w) off += wsel[w];
        const int rank = off + __popc(bal & ((1u << lane) - 1u));
        if (kt < s.nkt) {
            tmap[blk * s.nkt + kt] = sel ? rank : -1;
            if (sel) tiles[blk * s.nkt + rank] = kt | (v == kTileM * kTileN ? (int)kTileDenseBit : 0);
        }
        nnz += v;
        res += sel ? 0 : v;
        base += wsel[0] + wsel[1] + wsel[2] + wsel[3];
        __syncthreads();
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        nnz += __shfl_xor_sync(0xffffffffu, nnz, o);
        res += __shfl_xor_sync(0xffffffffu, res, o);
    }
    if (lane == 0) {
        wsum[0][warp] = nnz;
        wsum[1][warp] = res;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        ItvBlockStat st;
        st.nnz = wsum[0][0] + wsum[0][1] + wsum[0][2] + wsum[0][3];
        st.res = wsum[1][0] + wsum[1][1] + wsum[1][2] + wsum[1][3];
        st.n_long = n_long;
        st.n_bad = n_bad;
        st.n_tiles = base;
        st.pad = 0;
        bstat[blk] = st;
        ntiles[blk] = base;
        blk_res[blk] = st.res > 0;
        __threadfence();
        last_s = atomicInc(done, (unsigned)(nblocks - 1)) == (unsigned)(nblocks - 1);
    }
    if (bad && s.err_flags) atomicOr(s.err_flags, kErrBadColumn);
    __syncthreads();
    if (!last_s) return;
    // the last block: every other block's statistics are written
    __threadfence();
    long long t_nnz = 0, t_res = 0, t_tiles = 0;
    int t_long = 0, t_bad = 0, t_tcb = 0;
    const volatile ItvBlockStat* vs = bstat;
    for (int64_t x = threadIdx.x; x < nblocks; x += kTileM) {
        t_nnz += vs[x].nnz;
        t_res += vs[x].res;
        t_tiles += vs[x].n_tiles;
        t_long += vs[x].n_long;
        t_bad += vs[x].n_bad;
        t_tcb += vs[x].n_tiles > 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        t_nnz += __shfl_xor_sync(0xffffffffu, t_nnz, o);
        t_res += __shfl_xor_sync(0xffffffffu, t_res, o);
        t_tiles += __shfl_xor_sync(0xffffffffu, t_tiles, o);
        t_long += __shfl_xor_sync(0xffffffffu, t_long, o);
        t_bad += __shfl_xor_sync(0xffffffffu, t_bad, o);
        t_tcb += __shfl_xor_sync(0xffffffffu, t_tcb, o);
    }
    __shared__ long long fin[6][4];
    if (lane == 0) {
        fin[0][warp] = t_nnz;
        fin[1][warp] = t_res;
        fin[2][warp] = t_tiles;
        fin[3][warp] = t_long;
        fin[4][warp] = t_bad;
        fin[5][warp] = t_tcb;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        long long f[6];
        for (int q = 0; q < 6; ++q) f[q] = fin[q][0] + fin[q][1] + fin[q][2] + fin[q][3];
        out->nnz = f[0];
        out->res_nnz = f[1];
        out->n_tiles = f[2];
        out->n_long = (int32_t)f[3];
        out->err = f[4] ? (unsigned)kBuildNegativeWidth : 0u;
        out->n_tc_blocks = (int32_t)f[5];
        out->pad = 0;
    }
}

// The per-block tile lists compacted in block order (one warp per query block).
__global__ void k_compact_tiles(const int32_t* __restrict__ tiles, const int32_t* __restrict__ ntiles,
                                const int32_t* __restrict__ block_tile_off, int64_t nblocks, int nkt,
                                int32_t* __restrict__ tile_info) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t x = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); x < nblocks; x += warps) {
        const int64_t o = block_tile_off[x];
        for (int r = lane; r < ntiles[x]; r += 32) tile_info[o + r] = tiles[x * nkt + r];
    }
}

__global__ void k_lohi_counts(const int2* __restrict__ lohi, int64_t rows, int32_t* __restrict__ counts) {
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows;
         r += (int64_t)gridDim.x * blockDim.x) {
        const int2 v = lohi[r];
        counts[r] = v.y > v.x ? v.y - v.x : 0;
    }
}

// One warp per row: columns lo, lo + 1, ..., hi - 1.
__global__ void k_lohi_fill(const int2* __restrict__ lohi, int64_t rows, const int32_t* __restrict__ row_ptr,
                            int32_t* __restrict__ col_idx) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int2 v = lohi[r];
        const int64_t o = row_ptr[r];
        for (int t = lane; t < v.y - v.x; t += 32) col_idx[o + t] = v.x + t;
    }
}

unsigned grid_for(int64_t work, int per_block, int64_t cap = 1 << 16) {
    int64_t g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return (unsigned)g;
}

}  // namespace

int64_t plan_tile_capacity(int64_t nblocks, int nkt, int64_t nnz, int min_nnz) {
    const int64_t by_grid = nblocks * nkt;
    const int64_t by_nnz = nnz / (min_nnz > 0 ? min_nnz : 1) + 1;
    return by_grid < by_nnz ? by_grid : by_nnz;
}

cudaError_t build_plan(const int32_t* row_ptr, const int32_t* col_idx, int n, int num_masks,
                       int64_t nnz, int min_nnz, bool intervals, bool zeroed, bool precounted,
                       const PlanBuffers& b, PlanCounters* counters, cudaStream_t s) {
    const int64_t rows = (int64_t)num_masks * n;
    const int nqb = (n + kTileM - 1) / kTileM, nkt = (n + kTileN - 1) / kTileN;
    const int64_t nblocks = (int64_t)num_masks * nqb;
    cudaError_t e;
    if (!zeroed) {
        k_plan_zero<<<grid_for(nblocks * nkt, 256, 1024), 256, 0, counted(s)>>>(b.cnt_map, nblocks * nkt, counters);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (intervals) {
        if (!precounted)
            k_itv_count<<<grid_for(nblocks * 4, 8), 256, 0, counted(s)>>>(row_ptr, col_idx, nullptr, n, nblocks, nqb, nkt,
                                                                b.cnt_map);
    } else {
        if ((e = cudaMemsetAsync(b.tile_bits, 0, sizeof(uint32_t) * b.tile_cap * kTileM * 4, s)) !=
            cudaSuccess)
            return e;
        k_tile_count<<<grid_for(rows, 8), 256, 0, counted(s)>>>(row_ptr, col_idx, n, rows, nqb, nkt, b.cnt_map);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (nblocks <= kFusedSelectMax) {
        k_tile_select_fused<<<1, 1024, 0, counted(s)>>>(b.cnt_map, (int)nblocks, nkt, min_nnz, b.block_tile_off,
                                               b.tile_info, counters);
    } else {
        k_tile_select<<<grid_for(nblocks, 128), 128, 0, counted(s)>>>(b.cnt_map, nblocks, nkt, min_nnz,
                                                            b.block_ntiles, &counters->n_tc_blocks);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = scan_counts(b.block_ntiles, nblocks, b.block_tile_off, b.scan_tmp, &counters->n_tiles,
                        &counters->err, s);
        if (e != cudaSuccess) return e;
        k_tile_assign<<<grid_for(nblocks, 8), 256, 0, counted(s)>>>(b.cnt_map, nblocks, nkt, min_nnz,
                                                          b.block_tile_off, b.tile_info);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (intervals)
        k_itv_bits<<<grid_for(nblocks * kTileM, 256), 256, 0, counted(s)>>>(
            row_ptr, col_idx, nullptr, n, nblocks, nqb, b.block_tile_off, b.tile_info, b.tile_bits, b.res_cnt,
            b.res_long, &counters->res_n_long);
    else
        k_tile_bits<<<grid_for(rows, 8), 256, 0, counted(s)>>>(row_ptr, col_idx, n, rows, nqb, nkt, b.cnt_map,
                                                     b.tile_info, b.tile_bits, b.res_cnt, b.res_long,
                                                     &counters->res_n_long);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = scan_counts(b.res_cnt, rows, b.res_row_ptr, b.scan_tmp, &counters->res_nnz, &counters->err, s);
    if (e != cudaSuccess) return e;
    if (intervals)
        k_itv_residual<<<grid_for(rows, 256), 256, 0, counted(s)>>>(row_ptr, col_idx, nullptr, n, rows, nqb, nkt, b.cnt_map,
                                                          b.block_tile_off, b.res_row_ptr, b.res_col_idx,
                                                          &counters->n_mixed);
    else
        k_residual_fill<<<grid_for(rows, 8), 256, 0, counted(s)>>>(row_ptr, col_idx, n, rows, nqb, nkt, b.cnt_map,
                                                         b.block_tile_off, b.res_row_ptr, b.res_col_idx,
                                                         &counters->n_mixed);
    return cudaGetLastError();
}


cudaError_t itv_build(const ItvSpec& s, int2* lohi, int32_t* tmap, int32_t* tiles, int32_t* ntiles,
                      int32_t* blk_res, ItvBlockStat* bstat, int min_nnz, unsigned* done,
                      ItvCounters* counters, cudaStream_t stream) {
    const int64_t nblocks = (int64_t)s.num_masks * s.nqb;
    if (s.nkt > kItvMaxKeyTiles || nblocks > kItvMaxBlocks || nblocks < 1) return cudaErrorInvalidValue;
    k_itv_build<<<(unsigned)nblocks, kTileM, (size_t)s.nkt * 4, counted(stream)>>>(
        s, min_nnz, lohi, tmap, tiles, ntiles, blk_res, bstat, done, counters);
    return cudaGetLastError();
}

cudaError_t itv_write_csr(const int2* lohi, int64_t rows, int32_t* counts, int32_t* row_ptr,
                          int32_t* col_idx, int64_t* scan_tmp, int64_t* total, unsigned* err,
                          cudaStream_t stream) {
    k_lohi_counts<<<grid_for(rows, 256), 256, 0, counted(stream)>>>(lohi, rows, counts);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if ((e = scan_counts(counts, rows, row_ptr, scan_tmp, total, err, stream)) != cudaSuccess) return e;
    if (col_idx) {
        k_lohi_fill<<<grid_for(rows, 8), 256, 0, counted(stream)>>>(lohi, rows, row_ptr, col_idx);
        e = cudaGetLastError();
    }
    return e;
}

cudaError_t itv_write_plan(const int2* lohi, int n, int num_masks, const int32_t* tiles,
                           const int32_t* ntiles, const PlanBuffers& b, PlanCounters* counters,
                           cudaStream_t s) {
    const int64_t rows = (int64_t)num_masks * n;
    const int nqb = (n + kTileM - 1) / kTileM, nkt = (n + kTileN - 1) / kTileN;
    const int64_t nblocks = (int64_t)num_masks * nqb;
    cudaError_t e = scan_counts(ntiles, nblocks, b.block_tile_off, b.scan_tmp, &counters->n_tiles,
                                &counters->err, s);
    if (e != cudaSuccess) return e;
    k_compact_tiles<<<grid_for(nblocks, 8), 256, 0, counted(s)>>>(tiles, ntiles, b.block_tile_off, nblocks, nkt,
                                                                  b.tile_info);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_itv_bits<<<grid_for(nblocks * kTileM, 256), 256, 0, counted(s)>>>(
        nullptr, nullptr, lohi, n, nblocks, nqb, b.block_tile_off, b.tile_info, b.tile_bits, b.res_cnt,
        b.res_long, &counters->res_n_long);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = scan_counts(b.res_cnt, rows, b.res_row_ptr, b.scan_tmp, &counters->res_nnz, &counters->err, s);
    if (e != cudaSuccess) return e;
    k_itv_residual<<<grid_for(rows, 256), 256, 0, counted(s)>>>(nullptr, nullptr, lohi, n, rows, nqb, nkt,
                                                               b.cnt_map, b.block_tile_off, b.res_row_ptr,
                                                               b.res_col_idx, &counters->n_mixed);
    return cudaGetLastError();
}

}  // namespace spattn
