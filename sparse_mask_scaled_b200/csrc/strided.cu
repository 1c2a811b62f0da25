// Strided entries of a block + strided + global mask as dense tiles.
//
// In residue-permuted order -- row or key i at position perm(i) = (i mod S) G
// + i div S, G = n / S -- the entries j = i (mod S) of the strided pattern
// (row i attends to every S-th key from its own residue) fall into G x G
// blocks on the diagonal, which the tile plan of a mask built from them
// covers with dense tensor-core tiles. The mask's strided entries that its own
// plan leaves to the gather kernel are moved into such a permuted mask; the
// rest forms a regular mask. The forward runs both over Q, K, V with rows
// permuted for the first, and merges the two results row by row through
// their log-sum-exps (the softmax over a union of disjoint entry sets).
#include "spattn_internal.cuh"

namespace spattn {
namespace {

__device__ __forceinline__ int perm_of(int i, int S, int G) { return (i % S) * G + i / S; }

// Per residual row r = mk * n + i: its entries j = i (mod S), counted at the
// row's permuted position (cnt_perm) and at its own (cnt_row).
__global__ void k_str_count(const int32_t* rrp, const int32_t* rci, int64_t rows, int n, int S, int G,
                            int32_t* cnt_perm, int32_t* cnt_row) {
    const int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int64_t mk = r / n;
    const int i = (int)(r - mk * n);
    int c = 0;
    for (int p = rrp[r]; p < rrp[r + 1]; ++p) c += (rci[p] % S) == (i % S);
    cnt_perm[mk * n + perm_of(i, S, G)] = c;
    cnt_row[r] = c;
}

// Those entries in permuted order: row mk * n + perm(i), columns perm(j)
// (ascending: they share j's residue, so perm(j) grows with j).
__global__ void k_str_fill(const int32_t* rrp, const int32_t* rci, int64_t rows, int n, int S, int G,
                           const int32_t* srp, int32_t* sci) {
    const int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int64_t mk = r / n;
    const int i = (int)(r - mk * n);
    int o = srp[mk * n + perm_of(i, S, G)];
    for (int p = rrp[r]; p < rrp[r + 1]; ++p) {
        const int j = rci[p];
        if (j % S == i % S) sci[o++] = perm_of(j, S, G);
    }
}

// sel[block * nkt + kt] = 1 for the plan's tiles.
__global__ void k_sel_map(const int32_t* bto, const int32_t* tinfo, int nkt, uint8_t* sel) {
    const int64_t blk = blockIdx.x;
    for (int t = bto[blk] + threadIdx.x; t < bto[blk + 1]; t += blockDim.x)
        sel[blk * nkt + (tinfo[t] & 0x7fffffff)] = 1;
}

// Row lengths of the regular part: the mask's row minus its strided residual entries.
__global__ void k_reg_count(const int32_t* rp, const int32_t* cnt_row, int64_t rows, int32_t* cnt_reg) {
    const int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (r < rows) cnt_reg[r] = (rp[r + 1] - rp[r]) - cnt_row[r];
}

// The regular part: every entry but those j = i (mod S) outside the plan's
// tiles. One warp per row, 32 entries at a time, compacted by ballot (rows of
// global tokens hold every key).
__global__ void k_reg_fill(const int32_t* rp, const int32_t* ci, int64_t rows, int n, int S, int nqb, int nkt,
                           const uint8_t* sel, const int32_t* grp, int32_t* gci, unsigned* err) {
    const int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const int64_t mk = r / n;
    const int i = (int)(r - mk * n);
    const int ri = i % S;
    const uint8_t* srow = sel + (mk * nqb + (i >> 7)) * nkt;
    int o = grp[r];
    const int o_end = grp[r + 1];  // (the count allotted from the residual; never written past)
    for (int p0 = rp[r]; p0 < rp[r + 1]; p0 += 32) {
        const int p = p0 + lane;
        bool keep = false;
        int j = 0;
        if (p < rp[r + 1]) {
            j = ci[p];
            keep = !(j % S == ri && !srow[j >> 7]);
        }
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        const int at = o + __popc(bal & ((1u << lane) - 1u));
        if (keep && at < o_end) gci[at] = j;
        o += __popc(bal);
    }
    // the entries kept must fill exactly the slots the count pass allotted
    // (k_str_count and this selection agree), else the part is unusable
    if (lane == 0 && o != o_end) atomicOr(err, (unsigned)kBuildBadRowPtr);
}

// dst[b, h, perm(i), :] = src[b, h, i, :] (bf16; dst contiguous [B, H, n, d]),
// one thread per 16-byte chunk (d / 8 consecutive threads per row).
__global__ void k_perm_rows(const uint4* src, int64_t s_b, int64_t s_h, int64_t s_n, uint4* dst, int H, int n,
                            int d, int S, int G, int64_t rows) {
    const int vec = d / 8;  // 16-byte chunks per row
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t w = t / vec;
    const int c = (int)(t - w * vec);
    if (w >= rows) return;
    const int64_t bh = w / n;
    const int i = (int)(w - bh * n);
    const int64_t b = bh / H, h = bh - b * H;
    dst[(bh * n + perm_of(i, S, G)) * vec + c] = src[(b * s_b + h * s_h + (int64_t)i * s_n) / 8 + c];
}

// out[b, h, i, :] and lse[b, h, i] from the regular part's (out, lse1) and the
// permuted part's (o2, lse2) at row perm(i): weights exp(lse - L), L their
// log-sum-exp. One thread per 8 elements (d / 8 consecutive threads per row).
__global__ void k_merge_perm(uint4* out, int64_t o_sb, int64_t o_sh, int64_t o_sn, const float* lse1,
                             const uint4* o2, const float* lse2, float* lse, int H, int n, int d, int S, int G,
                             int64_t rows) {
    const int vec = d / 8;
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t w = t / vec;
    const int c = (int)(t - w * vec);
    if (w >= rows) return;
    const int64_t bh = w / n;
    const int i = (int)(w - bh * n);
    const int64_t b = bh / H, h = bh - b * H;
    const int64_t pr = bh * n + perm_of(i, S, G);
    const float l1 = lse1[w], l2 = lse2[pr];
    const float L = fmaxf(l1, l2);
    float w1 = 0.f, w2 = 0.f, tot = 0.f;
    if (L != -INFINITY) {
        w1 = expf(l1 - L);
        w2 = expf(l2 - L);
        tot = w1 + w2;
        w1 /= tot;
        w2 /= tot;
    }
    uint4* op = out + (b * o_sb + h * o_sh + (int64_t)i * o_sn) / 8 + c;
    const uint4 a = *op, q = o2[pr * vec + c];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, qw[4] = {q.x, q.y, q.z, q.w};
    uint32_t rw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float lo = __uint_as_float(aw[k] << 16) * w1 + __uint_as_float(qw[k] << 16) * w2;
        const float hi = __uint_as_float(aw[k] & 0xffff0000u) * w1 + __uint_as_float(qw[k] & 0xffff0000u) * w2;
        __nv_bfloat162 hv = __floats2bfloat162_rn(lo, hi);
        rw[k] = *reinterpret_cast<uint32_t*>(&hv);
    }
    *op = make_uint4(rw[0], rw[1], rw[2], rw[3]);
    if (lse && c == 0) lse[w] = L == -INFINITY ? -INFINITY : L + logf(tot);
}

unsigned blocks_for(int64_t threads, int per) { return (unsigned)((threads + per - 1) / per); }

}  // namespace

cudaError_t strided_split_count(const int32_t* rrp, const int32_t* rci, int64_t rows, int n, int S,
                                int32_t* cnt_perm, int32_t* cnt_row, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    k_str_count<<<blocks_for(rows, 256), 256, 0, counted(s)>>>(rrp, rci, rows, n, S, n / S, cnt_perm, cnt_row);
    return cudaGetLastError();
}

cudaError_t strided_split_fill(const int32_t* rrp, const int32_t* rci, const int32_t* rp, const int32_t* ci,
                               const int32_t* bto, const int32_t* tinfo, int64_t rows, int n, int S, int nqb,
                               int nkt, int64_t nblocks, const int32_t* cnt_row, int32_t* cnt_reg,
                               uint8_t* sel, const int32_t* srp, int32_t* sci, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(sel, 0, (size_t)nblocks * nkt, s);
    if (e != cudaSuccess) return e;
    if (nblocks > 0) k_sel_map<<<(unsigned)nblocks, 128, 0, counted(s)>>>(bto, tinfo, nkt, sel);
    k_str_fill<<<blocks_for(rows, 256), 256, 0, counted(s)>>>(rrp, rci, rows, n, S, n / S, srp, sci);
    k_reg_count<<<blocks_for(rows, 256), 256, 0, counted(s)>>>(rp, cnt_row, rows, cnt_reg);
    return cudaGetLastError();
}

cudaError_t strided_reg_fill(const int32_t* rp, const int32_t* ci, int64_t rows, int n, int S, int nqb, int nkt,
                             const uint8_t* sel, const int32_t* grp, int32_t* gci, unsigned* err, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    k_reg_fill<<<blocks_for(rows * 32, 256), 256, 0, counted(s)>>>(rp, ci, rows, n, S, nqb, nkt, sel, grp, gci,
                                                                   err);
    return cudaGetLastError();
}

cudaError_t strided_permute_rows(const void* src, int64_t s_b, int64_t s_h, int64_t s_n, void* dst, int B, int H,
                                 int n, int d, int S, cudaStream_t s) {
    const int64_t rows = (int64_t)B * H * n;
    if (rows == 0) return cudaSuccess;
    k_perm_rows<<<blocks_for(rows * (d / 8), 256), 256, 0, counted(s)>>>(
        static_cast<const uint4*>(src), s_b, s_h, s_n, static_cast<uint4*>(dst), H, n, d, S, n / S, rows);
    return cudaGetLastError();
}

cudaError_t strided_merge(void* out, int64_t o_sb, int64_t o_sh, int64_t o_sn, const float* lse1, const void* o2,
                          const float* lse2, float* lse, int B, int H, int n, int d, int S, cudaStream_t s) {
    const int64_t rows = (int64_t)B * H * n;
    if (rows == 0) return cudaSuccess;
    k_merge_perm<<<blocks_for(rows * (d / 8), 256), 256, 0, counted(s)>>>(
        static_cast<uint4*>(out), o_sb, o_sh, o_sn, lse1, static_cast<const uint4*>(o2), lse2, lse, H, n, d, S,
        n / S, rows);
    return cudaGetLastError();
}

}  // namespace spattn
