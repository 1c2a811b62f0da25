// Mask builder: an attention-mask pattern -> a sorted, duplicate-free CSR.
//
// The gluon-nlp sparse-attention proposal reduces every attention scheme to
// "generate the corresponding mask" and hand it to one CSR kernel; the pattern
// list (local / sliding window, global tokens, block or strided) is the one of
// the "Sparse Attention" notes page, with the per-token variable window of the
// proposal's discussion, plus user COO candidates and user CSR.
//
// Two phases on the device:
//   phase 1  per-row counts (O(1) for interval rows, an ordered walk for block +
//            strided + global rows, a sort + merge of duplicates for COO rows,
//            validation for user CSR), then row_ptr by an exclusive scan;
//   phase 2  (after the host has read the total and allocated col_idx) the
//            columns, written in ascending order.
#include "spattn.h"
#include "spattn_internal.cuh"

#include <limits.h>
#include <string.h>

namespace spattn {
namespace {

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;
constexpr int kScanTile = kScanThreads * kScanItems;
constexpr int kCooWarpCap = 1024;   // candidates a warp sorts in shared memory
constexpr int kCooWarps = 4;        // warps per block in the COO sort kernel
constexpr int kBitmapMaxBytes = 192 * 1024;

__device__ __forceinline__ void raise(BuildInfo* info, unsigned bit) { atomicOr(&info->err, bit); }

// Interval rows: [lo, hi) for SLIDING / VARWIN / DENSE and the global rows of
// BLOCK_STRIDED_GLOBAL. Returns false when the row is not an interval.
__device__ __forceinline__ bool row_interval(const BuildSpec& s, int64_t r, int64_t& lo,
                                             int64_t& hi, BuildInfo* info) {
    const int64_t i = r % s.n;
    switch (s.kind) {
    case SPATTN_MASK_SLIDING:
    case SPATTN_MASK_VARWIN: {
        int64_t w = s.kind == SPATTN_MASK_SLIDING ? s.window : s.half_widths[r];
        if (w < 0) {
            if (info) raise(info, kBuildNegativeWidth);
            lo = hi = 0;
            return true;
        }
        lo = i - w < 0 ? 0 : i - w;
        hi = i + w + 1 > s.n ? s.n : i + w + 1;
        return true;
    }
    case SPATTN_MASK_DENSE:
        lo = 0;
        hi = s.n;
        return true;
    case SPATTN_MASK_BLOCK_STRIDED_GLOBAL:
        if (i < s.n_global) {
            lo = 0;
            hi = s.n;
            return true;
        }
        return false;
    default:
        return false;
    }
}

// Smallest column >= j of a non-global BLOCK_STRIDED_GLOBAL row i, or n.
__device__ __forceinline__ int64_t bsg_next(const BuildSpec& s, int64_t i, int64_t j) {
    int64_t c = s.n;
    if (j < s.n_global) c = j;
    if (s.block > 0) {
        const int64_t bs = (i / s.block) * s.block;
        const int64_t be = bs + s.block < s.n ? bs + s.block : s.n;
        if (j < be) {
            const int64_t x = j > bs ? j : bs;
            if (x < c) c = x;
        }
    }
    if (s.stride > 0) {
        const int64_t r0 = i % s.stride;
        const int64_t x = j <= r0 ? r0 : r0 + ((j - r0 + s.stride - 1) / s.stride) * s.stride;
        if (x < c) c = x;
    }
    return c;
}

__global__ void k_count(BuildSpec s, int32_t* __restrict__ counts, BuildInfo* info,
                        int32_t* __restrict__ long_rows) {
    const int64_t rows = (int64_t)s.num_masks * s.n;
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows;
         r += (int64_t)gridDim.x * blockDim.x) {
        int64_t cnt = 0, lo, hi;
        if (s.kind == SPATTN_MASK_CSR) {
            const int64_t p0 = s.in_row_ptr[r], p1 = s.in_row_ptr[r + 1];
            bool ok = p0 >= 0 && p1 >= p0 && p1 <= s.in_nnz;
            if (r == 0 && p0 != 0) ok = false;
            if (r == rows - 1 && p1 != s.in_nnz) ok = false;
            if (!ok) raise(info, kBuildBadRowPtr);
            cnt = ok ? p1 - p0 : 0;
        } else if (row_interval(s, r, lo, hi, info)) {
            cnt = hi - lo;
        } else {  // non-global row of BLOCK_STRIDED_GLOBAL
            const int64_t i = r % s.n;
            for (int64_t j = bsg_next(s, i, 0); j < s.n; j = bsg_next(s, i, j + 1)) ++cnt;
        }
        counts[r] = (int32_t)cnt;
        if (cnt > kLongRowThreshold && long_rows) long_rows[atomicAdd(&info->n_long, 1)] = (int32_t)r;
    }
}

// Rows longer than kLongRowThreshold, from per-row counts (COO kind).
__global__ void k_classify_counts(const int32_t* __restrict__ counts, int64_t rows,
                                  int32_t* __restrict__ long_rows, BuildInfo* info) {
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows;
         r += (int64_t)gridDim.x * blockDim.x)
        if (counts[r] > kLongRowThreshold) long_rows[atomicAdd(&info->n_long, 1)] = (int32_t)r;
}

// User CSR: every row strictly increasing with columns in [0, n).
__global__ void k_check_csr(BuildSpec s, BuildInfo* info) {
    const int64_t rows = (int64_t)s.num_masks * s.n;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        int64_t p0 = s.in_row_ptr[r], p1 = s.in_row_ptr[r + 1];
        if (p0 < 0 || p1 < p0 || p1 > s.in_nnz) continue;  // reported by k_count
        for (int64_t p = p0 + lane; p < p1; p += 32) {
            const int c = s.in_col_idx[p];
            if ((unsigned)c >= (unsigned)s.n) raise(info, kBuildBadColumn);
            if (p > p0 && s.in_col_idx[p - 1] >= c) raise(info, kBuildUnsorted);
        }
    }
}

// COO rows of at most kCooWarpCap candidates (diagonal included): one warp
// sorts the row in shared memory (bitonic network), drops repeats and writes
// the result to coo_tmp at in_row_ptr[r] + r. Longer rows are queued.
__global__ void __launch_bounds__(kCooWarps * 32)
    k_coo_sort(BuildSpec s, int32_t* __restrict__ counts, int32_t* __restrict__ coo_tmp,
               int32_t* __restrict__ big_list, int32_t* __restrict__ big_count, BuildInfo* info) {
    __shared__ int32_t buf[kCooWarps][kCooWarpCap];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t* a = buf[warp];
    const int64_t rows = (int64_t)s.num_masks * s.n;
    for (int64_t r = (int64_t)blockIdx.x * kCooWarps + warp; r < rows;
         r += (int64_t)gridDim.x * kCooWarps) {
        const int64_t p0 = s.in_row_ptr[r], p1 = s.in_row_ptr[r + 1];
        bool ok = p0 >= 0 && p1 >= p0 && p1 <= s.in_nnz;
        if (r == 0 && p0 != 0) ok = false;
        if (r == rows - 1 && p1 != s.in_nnz) ok = false;
        if (!ok) {
            if (lane == 0) {
                raise(info, kBuildBadRowPtr);
                counts[r] = 0;
            }
            continue;
        }
        const int64_t ncand = p1 - p0;
        const int64_t cnt = ncand + (s.add_diagonal ? 1 : 0);
        if (cnt > kCooWarpCap) {
            if (lane == 0) {
                counts[r] = 0;
                big_list[atomicAdd(big_count, 1)] = (int32_t)r;
            }
            continue;
        }
        int P = 32;
        while (P < cnt) P <<= 1;
        const int i = (int)(r % s.n);
        for (int t = lane; t < P; t += 32) {
            int v = INT_MAX;
            if (t < ncand) {
                v = s.in_col_idx[p0 + t];
                if ((unsigned)v >= (unsigned)s.n) {
                    raise(info, kBuildBadColumn);
                    v = INT_MAX;
                }
            } else if (t == ncand && s.add_diagonal) {
                v = i;
            }
            a[t] = v;
        }
        __syncwarp();
        for (int k = 2; k <= P; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int t = lane; t < P; t += 32) {
                    const int u = t ^ j;
                    if (u > t) {
                        const int x = a[t], y = a[u];
                        const bool up = (t & k) == 0;
                        if ((x > y) == up) {
                            a[t] = y;
                            a[u] = x;
                        }
                    }
                }
                __syncwarp();
            }
        }
        const int64_t base = p0 + r;
        int written = 0;
        for (int t0 = 0; t0 < P; t0 += 32) {
            const int t = t0 + lane;
            const int v = a[t];
            const bool keep = v != INT_MAX && (t == 0 || a[t - 1] != v);
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            if (keep) coo_tmp[base + written + __popc(bal & ((1u << lane) - 1u))] = v;
            written += __popc(bal);
        }
        if (lane == 0) counts[r] = written;
        __syncwarp();
    }
}

// Queued long COO rows: one block per row marks the columns in an n-bit map in
// shared memory and writes the set bits in order.
__global__ void __launch_bounds__(1024)
    k_coo_big(BuildSpec s, int32_t* __restrict__ counts, int32_t* __restrict__ coo_tmp,
              const int32_t* __restrict__ big_list, const int32_t* __restrict__ big_count,
              BuildInfo* info) {
    extern __shared__ uint32_t bits[];
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    const int words = (s.n + 31) >> 5;
    const int nb = *big_count;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int q = blockIdx.x; q < nb; q += gridDim.x) {
        const int64_t r = big_list[q];
        const int64_t p0 = s.in_row_ptr[r], p1 = s.in_row_ptr[r + 1];
        for (int w = threadIdx.x; w < words; w += blockDim.x) bits[w] = 0u;
        if (threadIdx.x == 0) carry = 0;
        __syncthreads();
        for (int64_t p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
            const int c = s.in_col_idx[p];
            if ((unsigned)c >= (unsigned)s.n) {
                raise(info, kBuildBadColumn);
                continue;
            }
            atomicOr(&bits[c >> 5], 1u << (c & 31));
        }
        if (threadIdx.x == 0 && s.add_diagonal) {
            const int i = (int)(r % s.n);
            atomicOr(&bits[i >> 5], 1u << (i & 31));
        }
        __syncthreads();
        const int64_t base = p0 + r;
        for (int w0 = 0; w0 < words; w0 += blockDim.x) {
            const int w = w0 + threadIdx.x;
            const uint32_t m = w < words ? bits[w] : 0u;
            const int c = __popc(m);
            int inc = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, off);
                if (lane >= off) inc += y;
            }
            if (lane == 31) warp_tot[warp] = inc;
            __syncthreads();
            if (warp == 0) {
                const int nw = blockDim.x >> 5;
                const int x = lane < nw ? warp_tot[lane] : 0;
                int xi = x;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, xi, off);
                    if (lane >= off) xi += y;
                }
                if (lane < nw) warp_tot[lane] = xi - x;
            }
            __syncthreads();
            int pos = carry + warp_tot[warp] + inc - c;
            uint32_t mm = m;
            while (mm) {
                const int bit = __ffs(mm) - 1;
                coo_tmp[base + pos++] = w * 32 + bit;
                mm &= mm - 1;
            }
            __syncthreads();
            if (threadIdx.x == blockDim.x - 1) carry = pos;
            __syncthreads();
        }
        if (threadIdx.x == 0) counts[r] = carry;
        __syncthreads();
    }
}

__global__ void k_flag_big_rows(const int32_t* big_count, BuildInfo* info) {
    if (threadIdx.x == 0 && *big_count > 0) raise(info, kBuildRowTooLong);
}

__device__ __forceinline__ int64_t block_exclusive_scan(int64_t x, int64_t* total) {
    __shared__ int64_t wsum[32];
    __shared__ int64_t tot;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t inc = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, (long long)inc, off);
        if (lane >= off) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        const int64_t w = lane < nw ? wsum[lane] : 0;
        int64_t wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, (long long)wi, off);
            if (lane >= off) wi += y;
        }
        if (lane < nw) wsum[lane] = wi - w;
        if (lane == 31) tot = wi;
    }
    __syncthreads();
    const int64_t res = wsum[warp] + inc - x;
    *total = tot;
    __syncthreads();
    return res;
}

// Arrays up to kScanSmallMax: a single block scans them in passes of
// kPassRows values, carrying the running total from pass to pass. Values go
// through shared memory so that global loads and stores are coalesced (value
// t0 + j * 1024 + tid by thread tid), while the scan itself takes kPassItems
// consecutive values per thread (one pad word per 32 keeps those reads free of
// bank conflicts).
constexpr int kPassItems = 8;
constexpr int kPassRows = kScanThreads * kPassItems;
constexpr int64_t kScanSmallMax = 8 * (int64_t)kPassRows;

__device__ __forceinline__ int pad32(int i) { return i + (i >> 5); }

// out[r] = sum of get(0 .. r-1) for r < rows, clamped to INT_MAX; returns the
// total. With kLong, rows whose value exceeds kLongRowThreshold are listed in
// row order in long_rows and counted in *n_long.
template <bool kLong, class Get>
__device__ __forceinline__ int64_t block_scan_rows(int64_t rows, Get get, int32_t* __restrict__ out,
                                                   int32_t* __restrict__ long_rows, int64_t* n_long) {
    __shared__ int32_t sv[kPassRows + kPassRows / 32];
    const int tid = threadIdx.x;
    int64_t carry = 0, long_carry = 0;
    for (int64_t t0 = 0; t0 < rows; t0 += kPassRows) {
        int32_t g[kPassItems];
#pragma unroll
        for (int j = 0; j < kPassItems; ++j) {
            const int64_t r = t0 + j * kScanThreads + tid;
            g[j] = r < rows ? get(r) : 0;
        }
#pragma unroll
        for (int j = 0; j < kPassItems; ++j) sv[pad32(j * kScanThreads + tid)] = g[j];
        __syncthreads();
        int32_t v[kPassItems];
        int64_t sum = 0, nl = 0;
#pragma unroll
        for (int t = 0; t < kPassItems; ++t) {
            v[t] = sv[pad32(tid * kPassItems + t)];
            sum += v[t];
            nl += v[t] > kLongRowThreshold;
        }
        int64_t tot, ltot = 0, lrun = 0;
        int64_t run = carry + block_exclusive_scan(sum, &tot);  // ends with a barrier
        if (kLong) lrun = long_carry + block_exclusive_scan(nl, &ltot);
#pragma unroll
        for (int t = 0; t < kPassItems; ++t) {
            sv[pad32(tid * kPassItems + t)] = run > INT_MAX ? INT_MAX : (int32_t)run;
            if (kLong && v[t] > kLongRowThreshold) long_rows[lrun++] = (int32_t)(t0 + tid * kPassItems + t);
            run += v[t];
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kPassItems; ++j) {
            const int64_t r = t0 + j * kScanThreads + tid;
            if (r < rows) out[r] = sv[pad32(j * kScanThreads + tid)];
        }
        carry += tot;
        long_carry += ltot;
        __syncthreads();  // the next pass refills sv
    }
    if (kLong) *n_long = long_carry;
    return carry;
}

__global__ void __launch_bounds__(kScanThreads)
    k_scan_small(const int32_t* __restrict__ counts, int64_t rows, int32_t* __restrict__ out,
                 int64_t* total_out, unsigned* err) {
    const int64_t carry =
        block_scan_rows<false>(rows, [&](int64_t r) { return counts[r]; }, out, nullptr, nullptr);
    if (threadIdx.x == 0) {
        out[rows] = carry > INT_MAX ? INT_MAX : (int32_t)carry;
        *total_out = carry;
        if (carry > INT_MAX) atomicOr(err, kBuildTooMany);
    }
}

// Entries of row r for one mask kind (not COO); bad user row pointers and
// negative half-widths count 0 and set their bit in err.
template <int K>
__device__ __forceinline__ int32_t row_count(const BuildSpec& s, int64_t r, int64_t rows, unsigned& err) {
    if (K == SPATTN_MASK_CSR) {
        const int64_t p0 = s.in_row_ptr[r], p1 = s.in_row_ptr[r + 1];
        bool ok = p0 >= 0 && p1 >= p0 && p1 <= s.in_nnz;
        if (r == 0 && p0 != 0) ok = false;
        if (r == rows - 1 && p1 != s.in_nnz) ok = false;
        if (!ok) err |= kBuildBadRowPtr;
        return ok ? (int32_t)(p1 - p0) : 0;
    } else if (K == SPATTN_MASK_DENSE) {
        return s.n;
    } else if (K == SPATTN_MASK_SLIDING || K == SPATTN_MASK_VARWIN) {
        const int64_t i = r % s.n;
        const int64_t w = K == SPATTN_MASK_SLIDING ? s.window : s.half_widths[r];
        if (w < 0) {
            err |= kBuildNegativeWidth;
            return 0;
        }
        const int64_t lo = i - w < 0 ? 0 : i - w;
        const int64_t hi = i + w + 1 > s.n ? s.n : i + w + 1;
        return (int32_t)(hi - lo);
    } else {  // BLOCK_STRIDED_GLOBAL: global rows are full, the others walk their columns
        const int64_t i = r % s.n;
        if (i < s.n_global) return s.n;
        int32_t cnt = 0;
        for (int64_t j = bsg_next(s, i, 0); j < s.n; j = bsg_next(s, i, j + 1)) ++cnt;
        return cnt;
    }
}

// Phase 1 in one launch for masks of at most kSingleMax rows (every kind but
// COO): per-row counts, their exclusive scan into row_ptr, the list of rows
// longer than kLongRowThreshold (in row order) and the info block -- written,
// not accumulated, so it needs no clearing -- and, optionally, the clearing of
// zero_words int32 words at zero_buf (the tile plan's counters and counts).
constexpr int64_t kSingleMax = kScanSmallMax;

template <int K>
__global__ void __launch_bounds__(kScanThreads)
    k_count_scan_single(BuildSpec s, int32_t* __restrict__ row_ptr, int32_t* __restrict__ long_rows,
                        BuildInfo* info, int32_t* __restrict__ zero_buf, int64_t zero_words) {
    __shared__ unsigned err_s;
    if (threadIdx.x == 0) err_s = 0u;
    for (int64_t x = threadIdx.x; x < zero_words; x += blockDim.x) zero_buf[x] = 0;
    const int64_t rows = (int64_t)s.num_masks * s.n;
    unsigned err = 0u;
    int64_t n_long = 0;
    const int64_t total = block_scan_rows<true>(
        rows, [&](int64_t r) { return row_count<K>(s, r, rows, err); }, row_ptr, long_rows, &n_long);
    if (err) atomicOr(&err_s, err);  // err_s was set before the scan's barriers
    __syncthreads();
    if (threadIdx.x == 0) {
        row_ptr[rows] = total > INT_MAX ? INT_MAX : (int32_t)total;
        info->nnz = total;
        info->n_long = (int32_t)n_long;
        info->err = err_s | (total > INT_MAX ? (unsigned)kBuildTooMany : 0u);
        info->pad = 0u;
        info->pad2 = 0;
    }
}

// Tile t of kScanTile counts: local exclusive prefixes + the tile's total.
__global__ void __launch_bounds__(kScanThreads)
    k_scan_tiles(const int32_t* __restrict__ counts, int64_t rows, int64_t* __restrict__ pref,
                 int64_t* __restrict__ tile_sums) {
    const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
    int64_t v[kScanItems], sum = 0;
#pragma unroll
    for (int t = 0; t < kScanItems; ++t) {
        v[t] = base + t < rows ? counts[base + t] : 0;
        sum += v[t];
    }
    int64_t total;
    int64_t run = block_exclusive_scan(sum, &total);
#pragma unroll
    for (int t = 0; t < kScanItems; ++t) {
        if (base + t < rows) pref[base + t] = run;
        run += v[t];
    }
    if (threadIdx.x == 0) tile_sums[blockIdx.x] = total;
}

// One block: exclusive scan of the tile totals in place; the grand total -> *total
// (and the kBuildTooMany bit of *err when it does not fit int32).
__global__ void __launch_bounds__(kScanThreads)
    k_scan_tile_sums(int64_t* __restrict__ tile_sums, int64_t ntiles, int64_t* total_out,
                     unsigned* err) {
    int64_t carry = 0;
    for (int64_t t0 = 0; t0 < ntiles; t0 += kScanThreads) {
        const int64_t t = t0 + threadIdx.x;
        const int64_t v = t < ntiles ? tile_sums[t] : 0;
        int64_t total;
        const int64_t ex = block_exclusive_scan(v, &total);
        if (t < ntiles) tile_sums[t] = carry + ex;
        carry += total;
    }
    if (threadIdx.x == 0) {
        *total_out = carry;
        if (carry > INT_MAX) atomicOr(err, kBuildTooMany);
    }
}

__global__ void k_scan_finalize(const int64_t* __restrict__ pref,
                                const int64_t* __restrict__ tile_sums, int64_t rows,
                                const int64_t* total, int32_t* __restrict__ row_ptr) {
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r <= rows;
         r += (int64_t)gridDim.x * blockDim.x) {
        const int64_t v = r < rows ? pref[r] + tile_sums[r / kScanTile] : *total;
        row_ptr[r] = v > INT_MAX ? INT_MAX : (int32_t)v;
    }
}

// Phase 2, one warp per row: interval rows, COO rows (copied from coo_tmp) and
// user CSR rows (copied).
__global__ void k_fill_warp(BuildSpec s, const int32_t* __restrict__ row_ptr,
                            const int32_t* __restrict__ coo_tmp, int32_t* __restrict__ col_idx,
                            int32_t* __restrict__ tile_cnt, int nqb, int nkt) {
    const int64_t rows = (int64_t)s.num_masks * s.n;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const int64_t o0 = row_ptr[r], o1 = row_ptr[r + 1];
        int64_t lo, hi;
        if (s.kind == SPATTN_MASK_COO) {
            const int32_t* src = coo_tmp + s.in_row_ptr[r] + r;
            for (int64_t t = lane; t < o1 - o0; t += 32) col_idx[o0 + t] = src[t];
        } else if (s.kind == SPATTN_MASK_CSR) {
            const int32_t* src = s.in_col_idx + s.in_row_ptr[r];
            for (int64_t t = lane; t < o1 - o0; t += 32) col_idx[o0 + t] = src[t];
        } else if (row_interval(s, r, lo, hi, nullptr)) {
            for (int64_t t = lane; t < o1 - o0; t += 32) col_idx[o0 + t] = (int32_t)(lo + t);
            if (tile_cnt && hi > lo) {  // the row's share of each 128 x 128 tile it touches
                const int64_t m = r / s.n, i = r - m * s.n;
                const int64_t base = (m * nqb + (i >> 7)) * nkt;
                for (int64_t kt = (lo >> 7) + lane; kt <= (hi - 1) >> 7; kt += 32) {
                    const int64_t a = lo > kt * 128 ? lo : kt * 128;
                    const int64_t z = hi < kt * 128 + 128 ? hi : kt * 128 + 128;
                    atomicAdd(&tile_cnt[base + kt], (int)(z - a));
                }
            }
        }
    }
}

// Phase 2, one thread per non-global BLOCK_STRIDED_GLOBAL row: ordered walk.
__global__ void k_fill_bsg(BuildSpec s, const int32_t* __restrict__ row_ptr,
                           int32_t* __restrict__ col_idx) {
    const int64_t rows = (int64_t)s.num_masks * s.n;
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows;
         r += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = r % s.n;
        if (i < s.n_global) continue;
        int64_t o = row_ptr[r];
        const int64_t o1 = row_ptr[r + 1];
        for (int64_t j = bsg_next(s, i, 0); j < s.n && o < o1; j = bsg_next(s, i, j + 1))
            col_idx[o++] = (int32_t)j;
    }
}

unsigned grid_for(int64_t work, int per_block, int64_t cap = 1 << 16) {
    int64_t g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return (unsigned)g;
}

// Transpose helpers: per-column counts and the unsorted fill (one warp per row).
__global__ void k_tcount(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int n,
                         int64_t rows, int32_t* __restrict__ cnt) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int64_t m = r / n;
        for (int64_t p = row_ptr[r] + lane; p < row_ptr[r + 1]; p += 32) atomicAdd(&cnt[m * n + col_idx[p]], 1);
    }
}

__global__ void k_tfill(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int n,
                        int64_t rows, const int32_t* __restrict__ cand_row_ptr, int32_t* __restrict__ cursor,
                        int32_t* __restrict__ cand_col) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int64_t m = r / n, i = r - m * n;
        for (int64_t p = row_ptr[r] + lane; p < row_ptr[r + 1]; p += 32) {
            const int64_t t = m * n + col_idx[p];
            cand_col[cand_row_ptr[t] + atomicAdd(&cursor[t], 1)] = (int32_t)i;
        }
    }
}

}  // namespace

int64_t scan_tmp_elems(int64_t rows) { return rows + 1 + (rows + kScanTile - 1) / kScanTile + 1; }

cudaError_t build_phase1(const BuildSpec& s, int32_t* row_ptr, int32_t* counts,
                         int64_t* scan_tmp, int32_t* coo_tmp, BuildInfo* info,
                         int32_t* long_rows, int32_t* zero_buf, int64_t zero_words,
                         bool* zeroed, cudaStream_t stream) {
    const int64_t rows = (int64_t)s.num_masks * s.n;
    cudaError_t e;
    *zeroed = false;
    // block + strided + global rows walk their columns to count them: one
    // block only takes the small ones
    const bool single = s.kind == SPATTN_MASK_BLOCK_STRIDED_GLOBAL ? rows <= kPassRows / 2
                                                                  : s.kind != SPATTN_MASK_COO && rows <= kSingleMax;
    if (single) {
        const int64_t zw = zero_buf ? zero_words : 0;
        switch (s.kind) {
        case SPATTN_MASK_CSR:
            k_count_scan_single<SPATTN_MASK_CSR><<<1, kScanThreads, 0, counted(stream)>>>(
                s, row_ptr, long_rows, info, zero_buf, zw);
            break;
        case SPATTN_MASK_SLIDING:
            k_count_scan_single<SPATTN_MASK_SLIDING><<<1, kScanThreads, 0, counted(stream)>>>(
                s, row_ptr, long_rows, info, zero_buf, zw);
            break;
        case SPATTN_MASK_VARWIN:
            k_count_scan_single<SPATTN_MASK_VARWIN><<<1, kScanThreads, 0, counted(stream)>>>(
                s, row_ptr, long_rows, info, zero_buf, zw);
            break;
        case SPATTN_MASK_DENSE:
            k_count_scan_single<SPATTN_MASK_DENSE><<<1, kScanThreads, 0, counted(stream)>>>(
                s, row_ptr, long_rows, info, zero_buf, zw);
            break;
        default:
            k_count_scan_single<SPATTN_MASK_BLOCK_STRIDED_GLOBAL><<<1, kScanThreads, 0, counted(stream)>>>(
                s, row_ptr, long_rows, info, zero_buf, zw);
            break;
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        *zeroed = zero_buf != nullptr;
        if (s.kind == SPATTN_MASK_CSR) {
            k_check_csr<<<grid_for(rows, 8), 256, 0, counted(stream)>>>(s, info);
            e = cudaGetLastError();
        }
        return e;
    }
    if ((e = cudaMemsetAsync(info, 0, sizeof(BuildInfo), stream)) != cudaSuccess) return e;
    if (s.kind == SPATTN_MASK_COO) {
        // big-row queue lives after the scan area
        int32_t* big_count = reinterpret_cast<int32_t*>(scan_tmp + scan_tmp_elems(rows));
        int32_t* big_list = big_count + 4;
        e = cudaMemsetAsync(big_count, 0, sizeof(int32_t), stream);
        if (e != cudaSuccess) return e;
        k_coo_sort<<<grid_for(rows, kCooWarps), kCooWarps * 32, 0, counted(stream)>>>(
            s, counts, coo_tmp, big_list, big_count, info);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (s.in_nnz + (s.add_diagonal ? 1 : 0) > kCooWarpCap) {
            const int words = (s.n + 31) / 32;
            const size_t smem = (size_t)words * 4;
            if (smem <= (size_t)kBitmapMaxBytes) {
                e = cudaFuncSetAttribute(k_coo_big, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
                if (e != cudaSuccess) return e;
                k_coo_big<<<grid_for(rows, 1, 512), 1024, smem, counted(stream)>>>(s, counts, coo_tmp,
                                                                         big_list, big_count, info);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            } else {
                // the n-bit map does not fit in shared memory: queued rows are an error
                k_flag_big_rows<<<1, 32, 0, counted(stream)>>>(big_count, info);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
        }
    } else {
        k_count<<<grid_for(rows, 256), 256, 0, counted(stream)>>>(s, counts, info, long_rows);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (s.kind == SPATTN_MASK_CSR) {
            k_check_csr<<<grid_for(rows, 8), 256, 0, counted(stream)>>>(s, info);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
    }
    if (s.kind == SPATTN_MASK_COO) {
        k_classify_counts<<<grid_for(rows, 256), 256, 0, counted(stream)>>>(counts, rows, long_rows, info);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return scan_counts(counts, rows, row_ptr, scan_tmp, &info->nnz, &info->err, stream);
}

cudaError_t scan_counts(const int32_t* counts, int64_t rows, int32_t* out, int64_t* scan_tmp,
                        int64_t* total, unsigned* err, cudaStream_t stream) {
    if (rows <= kScanSmallMax) {  // one block walks the tiles with a running carry
        k_scan_small<<<1, kScanThreads, 0, counted(stream)>>>(counts, rows, out, total, err);
        return cudaGetLastError();
    }
    const int64_t ntiles = (rows + kScanTile - 1) / kScanTile;
    int64_t* pref = scan_tmp;
    int64_t* tile_sums = scan_tmp + rows + 1;
    cudaError_t e;
    k_scan_tiles<<<(unsigned)ntiles, kScanThreads, 0, counted(stream)>>>(counts, rows, pref, tile_sums);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_scan_tile_sums<<<1, kScanThreads, 0, counted(stream)>>>(tile_sums, ntiles, total, err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_scan_finalize<<<grid_for(rows + 1, 256), 256, 0, counted(stream)>>>(pref, tile_sums, rows, total, out);
    return cudaGetLastError();
}

cudaError_t build_phase2(const BuildSpec& s, const int32_t* row_ptr, const int32_t* coo_tmp,
                         int32_t* col_idx, int32_t* tile_cnt, cudaStream_t stream) {
    const int64_t rows = (int64_t)s.num_masks * s.n;
    const int nqb = (s.n + kTileM - 1) / kTileM, nkt = (s.n + kTileN - 1) / kTileN;
    k_fill_warp<<<grid_for(rows, 8), 256, 0, counted(stream)>>>(s, row_ptr, coo_tmp, col_idx, tile_cnt, nqb, nkt);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (s.kind == SPATTN_MASK_BLOCK_STRIDED_GLOBAL) {
        k_fill_bsg<<<grid_for(rows, 128), 128, 0, counted(stream)>>>(s, row_ptr, col_idx);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace spattn

namespace spattn {

// Scratch layout (int32 words, each part 64-word aligned): cnt [rows], cursor
// [rows], cand_row_ptr [rows + 1], cand_col [nnz], counts [rows], long_rows
// [rows], coo_tmp [nnz + rows], info (BuildInfo), scan_tmp (int64, with the COO
// queue of long rows).
namespace {
int64_t al64(int64_t w) { return (w + 63) & ~int64_t(63); }
}  // namespace

int64_t transpose_scratch_words(int64_t rows, int64_t nnz) {
    const int64_t scan64 = scan_tmp_elems(rows) + (rows + 6) / 2 + 1;
    return 2 * al64(rows) + al64(rows + 1) + al64(nnz) + 2 * al64(rows) + al64(nnz + rows) + 64 +
           2 * scan64;
}

cudaError_t build_transpose(const int32_t* row_ptr, const int32_t* col_idx, int n, int num_masks,
                            int64_t nnz, int32_t* t_row_ptr, int32_t* t_col_idx, int32_t* scratch,
                            cudaStream_t stream) {
    const int64_t rows = (int64_t)num_masks * n;
    int32_t* cnt = scratch;
    int32_t* cursor = cnt + al64(rows);
    int32_t* cand_row_ptr = cursor + al64(rows);
    int32_t* cand_col = cand_row_ptr + al64(rows + 1);
    int32_t* counts = cand_col + al64(nnz);
    int32_t* long_rows = counts + al64(rows);
    int32_t* coo_tmp = long_rows + al64(rows);
    BuildInfo* info = reinterpret_cast<BuildInfo*>(coo_tmp + al64(nnz + rows));
    int64_t* scan_tmp = reinterpret_cast<int64_t*>(reinterpret_cast<int32_t*>(info) + 64);
    cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * (size_t)(2 * al64(rows)), stream);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(info, 0, sizeof(BuildInfo), stream)) != cudaSuccess) return e;
    k_tcount<<<grid_for(rows, 8), 256, 0, counted(stream)>>>(row_ptr, col_idx, n, rows, cnt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = scan_counts(cnt, rows, cand_row_ptr, scan_tmp, &info->nnz, &info->err, stream);
    if (e != cudaSuccess) return e;
    k_tfill<<<grid_for(rows, 8), 256, 0, counted(stream)>>>(row_ptr, col_idx, n, rows, cand_row_ptr, cursor,
                                                            cand_col);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // sort each transposed row: the COO builder's path (no repeats to merge)
    BuildSpec bs;
    memset(&bs, 0, sizeof bs);
    bs.kind = SPATTN_MASK_COO;
    bs.n = n;
    bs.num_masks = num_masks;
    bs.in_row_ptr = cand_row_ptr;
    bs.in_col_idx = cand_col;
    bs.in_nnz = nnz;
    bool zeroed = false;
    e = build_phase1(bs, t_row_ptr, counts, scan_tmp, coo_tmp, info, long_rows, nullptr, 0, &zeroed, stream);
    if (e != cudaSuccess) return e;
    return build_phase2(bs, t_row_ptr, coo_tmp, t_col_idx, nullptr, stream);
}

}  // namespace spattn
