// Internal declarations of libspattn (not installed; the public ABI is include/spattn.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spattn {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// device error flag bits (read by spattn_device_error)
constexpr unsigned kErrBadColumn = 1u;
constexpr unsigned kErrTimeout = 2u;  // a bounded wait of the tensor-core kernel expired

// Tensor-core tiling: 128 query rows by 128 keys.
constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr unsigned kTileDenseBit = 0x80000000u;  // tile_info flag: all 128 x 128 entries present
constexpr int kTileMinNnzDefault = 512;
// The d = 128 tile kernel splits a query block with more tiles than this into
// chunks of this many, one thread block each.
constexpr int kChunkTiles = 8;
// Tile planning is skipped when num_masks * (n/128)^2 exceeds this (count array size).
constexpr int64_t kPlanZeroInline = 1 << 18;  // words the single-launch build clears
constexpr int64_t kPlanMaxTileGrid = int64_t(1) << 26;

// Rows with more nonzeros than this are processed by a whole thread block
// (eight warps) instead of one warp.
constexpr int kLongRowThreshold = 1024;

// An additive term over (b, h, i, j): the attention mask or the attention bias.
struct AddendView {
    const void* data;  // nullptr = absent
    int dtype;         // 0 bf16, 1 f32
    int64_t s0, s1, s2, s3;  // element strides over (b, h, i, j); 0 broadcasts
};

struct FwdParams {
    const void* q;
    const void* k;
    const void* v;
    void* out;
    float* lse;  // nullable
    int64_t q_sb, q_sh, q_sn;
    int64_t k_sb, k_sh, k_sn;
    int64_t v_sb, v_sh, v_sn;
    int64_t o_sb, o_sh, o_sn;
    int B, H, n;
    int num_masks;
    const int32_t* row_ptr;
    const int32_t* col_idx;
    int64_t nnz;
    AddendView mask, bias;
    int has_extra;          // mask or bias present
    float qk_scale_log2;    // scale * log2(e)
    // rows longer than kLongRowThreshold, as mask-row ids (m * n + i)
    const int32_t* long_rows;
    const int32_t* long_count_dev;  // device count (used when long_count_host < 0)
    int64_t long_count_host;        // host count, or -1
    // With a tensor-core plan: rows of query blocks that have tensor-core tiles
    // write their partial state (m in base 2, l, unnormalised acc) to ws_ml /
    // ws_acc instead of the output (only when they have gathered entries).
    const int32_t* qb_tile_off;  // [num_masks * nqb + 1] or nullptr
    int nqb;
    float* ws_ml;   // [B*H*n*2]
    float* ws_acc;  // [B*H*n*d]
    // Interval masks (k_fwd_itv): row m*n + i is the run [lo, hi) of itv_lohi.
    // With a tile plan (tmap != nullptr) only the parts in unselected key tiles
    // (tmap[blk * nkt + kt] < 0) are gathered; the rows of a query block with
    // tiles hand their partial state to the tensor-core kernel, and only blocks
    // flagged in blk_res have any.
    const int2* itv_lohi;
    const int32_t* tmap;
    const int32_t* blk_res;
    const int32_t* qb_ntiles;  // tensor-core tiles per query block
    int nkt;
    const int32_t* seqlen_k;  // nullable, [B]: keys j >= seqlen_k[b] are left out (key padding)
    int itv_slices;  // 1, 2, 4, 8 or 16 thread blocks per 128-row query block
};

// Backward pass (fwd_gather.cu): gradients of sum(dout * out) for the same
// attention, recomputing each score from q, k and the saved lse. The row pass
// (one warp per query row) writes dq and D_i = <dout_i, out_i>; the column pass
// (one warp per key, over the transposed mask) writes dk and dv.
struct BwdParams {
    const void *q, *k, *v, *out, *dout;
    void *dq, *dk, *dv;
    const float* lse;  // natural log, [B*H*n]
    float* D;          // [B*H*n], written by the row pass
    float* dbias;      // nullable: f32, accumulated (atomics), element strides db_s*
    int64_t db_s0, db_s1, db_s2, db_s3;
    int64_t q_sb, q_sh, q_sn, k_sb, k_sh, k_sn, v_sb, v_sh, v_sn, o_sb, o_sh, o_sn;
    int64_t do_sb, do_sh, do_sn, dq_sb, dq_sh, dq_sn, dk_sb, dk_sh, dk_sn, dv_sb, dv_sh, dv_sn;
    int B, H, n, num_masks;
    const int32_t* row_ptr;    // the mask
    const int32_t* col_idx;
    int64_t nnz;
    const int32_t* t_row_ptr;  // its transpose: row m*n + j lists the i with j in S_i
    const int32_t* t_col_idx;
    AddendView mask, bias;
    int has_extra;
    float scale;
    float qk_scale_log2;
};
cudaError_t launch_bwd(const BwdParams& p, int dtype, int d, cudaStream_t stream);
// The unfused three-stage forward (SDDMM -> row softmax -> SpMM); scores: fp32
// [(num_masks == 1 ? B*H : H) * nnz].
cudaError_t launch_fwd_unfused(const FwdParams& p, int dtype, int d, float* scores, cudaStream_t stream);

// Tensor-core kernel (fwd_tc.cu).
struct TcOperand {
    const void* data;  // bf16 [B, H, n, d], stride 1 over d
    int64_t s_n, s_h, s_b;
};
struct TcParams {
    int B, H, n, num_masks, nqb;
    const int32_t* block_tile_off;  // [num_masks * nqb + 1]
    const int32_t* tile_info;       // key tile | kTileDenseBit
    // Instead of block_tile_off: block x's tiles are tile_info[x * tile_stride ..
    // x * tile_stride + block_ntiles[x] - 1] (interval masks).
    const int32_t* block_ntiles;
    int tile_stride;
    const int32_t* seqlen_k;  // nullable, [B]: keys j >= seqlen_k[b] are left out
    const uint32_t* tile_bits;      // [tiles][128 rows][4 words]
    const int32_t* res_row_ptr;     // residual CSR (a row with entries has a partial)
    // Interval masks: masks come from the row runs instead of tile_bits, and the
    // rows of blocks flagged in blk_res have a partial (used when its l > 0).
    const int2* itv_lohi;
    const int32_t* blk_res;
    const float* ws_ml;             // partials from the gather kernel, or nullptr
    const float* ws_acc;
    // Query blocks whose tile lists are split into chunks of chunk_tiles tiles
    // (d = 128; nullptr blk_nch: none): block x has blk_nch[x] chunks, whose
    // partial states take slots blk_slot[x] + c of the n_slots of each (b, h)
    // in cws; chunks c >= 1 run on extra thread blocks, one per entry of
    // chunk_extra ((block, c); n_extra per (b, h)); ccnt[bh * blocks + x]
    // counts the chunks done (zero before the launch).
    const int32_t* blk_nch;
    const int32_t* blk_slot;
    const int2* chunk_extra;
    int n_extra, n_slots, chunk_tiles;
    float* cws;
    unsigned* ccnt;
    // d = 128 only: rows and keys are numbered in residue-permuted order --
    // position p = (i mod S) perm_G + i div S holds row / key i of the Q, K, V
    // tensors (S = n / perm_G, perm_G a multiple of 128) -- and the tile loads
    // fetch their 128 rows with stride S (five-dimensional maps); 0 = off.
    int perm_G;
    void* out;
    int64_t o_sb, o_sh, o_sn;
    float* lse;
    AddendView mask, bias;
    int has_extra;
    // set by the launcher (d <= 64): the additive term that varies by row is
    // staged into shared memory by TMA, one 128-row x 64-key block per sub-tile
    int a_tma;
    float qk_scale_log2;
    unsigned* err;
};
cudaError_t launch_fwd_tc(const TcOperand& q, const TcOperand& k, const TcOperand& v, int d,
                          const TcParams& p, cudaStream_t stream);

// Persistent ping-pong tensor-core kernel (fwd_pp.cu), d = 32, 64 or 128,
// bf16; additive terms (d <= 64) and key lengths for interval masks.
struct PpParams {
    int B, H, n, num_masks, nqb, nkt;
    int mode;         // 0: interval-mask tiles; 1: block + strided + global in closed form
    int64_t n_items;  // work items (mode 0: B*H*nqb; mode 1: B*H*items per head)
    // mode 0: the interval mask's runs and tile lists, and the gather kernel's
    // partial states of rows in flagged blocks (blk_res; ws_ml / ws_acc)
    const int2* itv_lohi;
    const int32_t* itv_tiles;   // [blocks][nkt]: key tile | kTileDenseBit
    const int32_t* itv_ntiles;  // [blocks]
    const int32_t* blk_res;     // nullable
    const float* ws_ml;
    const float* ws_acc;
    // mode 1: pattern parameters (bsg_plan.cuh), chunk partial states
    // [B*H][nch][d + 2][128] with counts [B*H][4], the permuted parts' states
    // [B*H*n][2] (m, l) and [B*H*n][d] (O) with per permuted block arrival
    // counts [B*H][npqb][128] (counts zero before the launch)
    int blk, S, ng, chunk_tiles;
    float* cws;
    unsigned* ccnt;
    float* pml;
    float* pacc;
    unsigned* pflag;
    // nullable: items are taken from this counter (zero before the launch) in
    // order; else CTA c takes items c, c + grid, ... (slots alternating)
    unsigned long long* claim;
    void* out;
    int64_t o_sb, o_sh, o_sn;
    float* lse;  // nullable
    float qk_scale_log2;
    unsigned* err;
    long long wait_cycles;  // limit of every wait (SM cycles)
    // mode 0, d <= 64: additive terms (bf16, keys contiguous, 16-byte aligned
    // rows) staged tile by tile through shared memory by TMA; extra[a] != 0
    // when term a (0: mask, 1: bias) is present, a_rows[a] = 1 when it is the
    // same for every query row, else 128; a_h / a_b: it varies with h / b
    int extra[2], a_rows[2], a_h[2], a_b[2];
    const int32_t* seqlen_k;  // nullable, [B]: keys j >= seqlen_k[b] are left out
};
cudaError_t launch_fwd_pp(const TcOperand& q, const TcOperand& k, const TcOperand& v, int d, const PpParams& p,
                          const AddendView& mask, const AddendView& bias, int num_sms, cudaStream_t stream);
// Whether an additive term can be staged through shared memory by TMA.
bool pp_addend_ok(const AddendView& a);
cudaError_t error_flag_address(unsigned** p);
// Every kernel launch of the library passes its stream through counted(),
// which adds one to the count spattn_launch_count() reports.
cudaStream_t counted(cudaStream_t s);

// Tile plan (plan.cu).
struct PlanBuffers {
    int32_t* cnt_map;         // [nblocks * nkt] (temporary)
    int32_t* block_ntiles;    // [nblocks] (temporary)
    int32_t* block_tile_off;  // [nblocks + 1]
    int64_t* scan_tmp;        // [scan_tmp_elems(max(rows, nblocks))] (temporary)
    int32_t* tile_info;       // [tile_cap]
    uint32_t* tile_bits;      // [tile_cap * 128 * 4]
    int64_t tile_cap;
    int32_t* res_cnt;         // [rows] (temporary)
    int32_t* res_row_ptr;     // [rows + 1]
    int32_t* res_col_idx;     // [nnz]
    int32_t* res_long;        // [rows]
};
struct PlanCounters {  // device-side results
    int64_t n_tiles;
    int64_t res_nnz;
    int32_t n_mixed;      // rows with entries on both paths
    int32_t res_n_long;   // long rows of the residual CSR
    int32_t n_tc_blocks;  // query blocks with at least one tile
    unsigned err;
};
int64_t plan_tile_capacity(int64_t nblocks, int nkt, int64_t nnz, int min_nnz);
// intervals: every row's columns form one contiguous run (sliding window,
// variable window, dense), which lets the plan skip reading col_idx.
// zeroed: the count array and the counters are already clear; precounted: the count
// array already holds the per-tile counts (interval rows, from build_phase2).
cudaError_t build_plan(const int32_t* row_ptr, const int32_t* col_idx, int n, int num_masks,
                       int64_t nnz, int min_nnz, bool intervals, bool zeroed, bool precounted,
                       const PlanBuffers& b, PlanCounters* counters, cudaStream_t s);

// Implicit interval masks (plan.cu). SLIDING, VARWIN and DENSE rows are single
// runs [lo, hi); such a mask keeps the runs (int2 per row) and its tile plan,
// and writes a CSR only when one is asked for.
struct ItvSpec {
    int kind, n, num_masks, window;
    const int32_t* half_widths;  // VARWIN
    int nqb, nkt;
    unsigned* err_flags;  // nullable: negative half-widths also raise kErrBadColumn here
};
// Results of the build, written by the last thread block of the build kernel.
struct ItvCounters {
    int64_t nnz;
    int64_t n_tiles;
    int64_t res_nnz;      // entries outside tensor-core tiles
    int32_t n_long;       // rows with more than kLongRowThreshold entries
    int32_t n_tc_blocks;  // query blocks with at least one tile
    unsigned err;         // kBuildNegativeWidth
    int32_t pad;
};
// Per query block, for the totals.
struct ItvBlockStat {
    int64_t nnz, res;
    int32_t n_long, n_bad, n_tiles, pad;
};
constexpr int kItvMaxKeyTiles = 8192;       // per-block tile counts live in shared memory
constexpr int64_t kItvMaxBlocks = 1 << 16;  // query blocks of one build
// One launch, no host synchronisation: per query block (one thread block each)
// the rows' runs, the entry counts per key tile, the selected tiles (count >=
// min_nnz; min_nnz <= 0 selects none) listed at tiles[blk * nkt ..] with their
// number in ntiles[blk], the tile map tmap[blk * nkt + kt] (local tile number or
// -1) and blk_res[blk] (entries outside the selected tiles); the last block to
// finish writes the totals. done: a device counter that is 0 and is left 0.
cudaError_t itv_build(const ItvSpec& s, int2* lohi, int32_t* tmap, int32_t* tiles, int32_t* ntiles,
                      int32_t* blk_res, ItvBlockStat* bstat, int min_nnz, unsigned* done,
                      ItvCounters* counters, cudaStream_t stream);
// CSR of an interval mask: counts (scratch int32 [rows]) -> row_ptr [rows + 1]
// -> col_idx [nnz]. scan_tmp: int64 [scan_tmp_elems(rows)], total/err: device scalars.
cudaError_t itv_write_csr(const int2* lohi, int64_t rows, int32_t* counts, int32_t* row_ptr,
                          int32_t* col_idx, int64_t* scan_tmp, int64_t* total, unsigned* err,
                          cudaStream_t stream);
// The explicit plan of an interval mask, as build_plan writes it for CSR masks:
// b.block_tile_off and b.tile_info (compacted from tiles / ntiles), tile_bits,
// the residual CSR and the mixed-row count. b.cnt_map is the tile map;
// counters->res_n_long, n_mixed must start at 0.
cudaError_t itv_write_plan(const int2* lohi, int n, int num_masks, const int32_t* tiles,
                           const int32_t* ntiles, const PlanBuffers& b, PlanCounters* counters,
                           cudaStream_t stream);

// ---------------------------------------------------------------- launchers
// All launchers enqueue on `stream` and return the cudaGetLastError() result.

// Forward pass kernels (fwd_gather.cu). dtype: 0 bf16, 1 f32.
cudaError_t launch_fwd_short_rows(const FwdParams& p, int dtype, int d, cudaStream_t stream);
cudaError_t launch_fwd_long_rows(const FwdParams& p, int dtype, int d, int num_sms,
                                 cudaStream_t stream);
// Collect rows longer than kLongRowThreshold (clamped to [0, nnz]) into
// `list`, counting them in *count (which must start at 0).
cudaError_t launch_classify_long_rows(const int32_t* row_ptr, int64_t rows, int64_t nnz,
                                      int32_t* list, int32_t* count, cudaStream_t stream);
cudaError_t read_and_clear_device_error(unsigned* flags, cudaStream_t stream);
// Interval-mask gather (fields itv_lohi / tmap / blk_res / nkt of p).
cudaError_t launch_fwd_itv(const FwdParams& p, int dtype, int d, cudaStream_t stream);

// Mask builder (mask_build.cu).
struct BuildSpec {
    int kind, n, num_masks, window, block, stride, n_global, add_diagonal;
    const int32_t* half_widths;
    const int32_t* in_row_ptr;
    const int32_t* in_col_idx;
    int64_t in_nnz;
};

// Device-side result block written by the builder.
struct BuildInfo {
    unsigned err;      // BuildErr bits
    unsigned pad;
    int64_t nnz;       // total nonzeros
    int32_t n_long;    // long rows
    int32_t pad2;
};
enum BuildErr : unsigned {
    kBuildBadColumn = 1u,
    kBuildUnsorted = 2u,
    kBuildBadRowPtr = 4u,
    kBuildNegativeWidth = 8u,
    kBuildTooMany = 16u,    // nnz above INT32_MAX
    kBuildRowTooLong = 32u, // COO row above the builder's candidate limit
};

// COO rows with more than 1024 candidates are merged through an n-bit map in
// shared memory, which limits such rows to n <= 1,572,864.
// Phase 1: per-row counts (and, for COO, sorted unique rows in `coo_tmp`,
// row r at offset in_row_ptr[r] + r), then row_ptr by an exclusive scan.
// Writes info->err and info->nnz. Scratch: `counts` int32 [rows];
// `scan_tmp` int64 [scan_tmp_elems(rows)] followed, for COO, by int32
// [rows + 4] (the queue of long COO rows); coo_tmp int32 [in_nnz + rows]
// (COO only).
// Also lists rows with more than kLongRowThreshold entries in long_rows [rows],
// counted in info->n_long. Writes (or clears, then accumulates) *info. When
// the single-launch path is taken and zero_buf is given, also clears
// zero_words int32 words there and sets *zeroed.
cudaError_t build_phase1(const BuildSpec& s, int32_t* row_ptr, int32_t* counts,
                         int64_t* scan_tmp, int32_t* coo_tmp, BuildInfo* info,
                         int32_t* long_rows, int32_t* zero_buf, int64_t zero_words, bool* zeroed,
                         cudaStream_t stream);
int64_t scan_tmp_elems(int64_t rows);
// Exclusive scan of int32 counts [rows] into out int32 [rows + 1]; the total goes
// to *total (device) and overflow past INT32_MAX sets kBuildTooMany in *err.
// scan_tmp: int64 [scan_tmp_elems(rows)].
cudaError_t scan_counts(const int32_t* counts, int64_t rows, int32_t* out, int64_t* scan_tmp,
                        int64_t* total, unsigned* err, cudaStream_t stream);
// Phase 2: write col_idx from the pattern (or copy it from coo_tmp / in_col_idx).
// With tile_cnt (cleared, [num_masks * nqb * nkt]), interval rows also add their
// per-tile counts for the tile plan.
cudaError_t build_phase2(const BuildSpec& s, const int32_t* row_ptr, const int32_t* coo_tmp,
                         int32_t* col_idx, int32_t* tile_cnt, cudaStream_t stream);

// Transpose of a CSR mask set: t_row_ptr [rows + 1] / t_col_idx [nnz], row
// m*n + j listing, ascending, the i with j in row m*n + i. Scratch sizes in
// int32 words: transpose_scratch_words(rows, nnz). No host synchronisation.
int64_t transpose_scratch_words(int64_t rows, int64_t nnz);
cudaError_t build_transpose(const int32_t* row_ptr, const int32_t* col_idx, int n, int num_masks,
                            int64_t nnz, int32_t* t_row_ptr, int32_t* t_col_idx, int32_t* scratch,
                            cudaStream_t stream);

// Strided entries of a block + strided + global mask (strided.cu). perm(i) =
// (i mod S) n/S + i div S; n is a multiple of S.
// Per residual row, its entries j = i (mod S): counted at the row's permuted
// position (cnt_perm, [rows]) and at its own (cnt_row).
cudaError_t strided_split_count(const int32_t* res_row_ptr, const int32_t* res_col_idx, int64_t rows, int n,
                                int S, int32_t* cnt_perm, int32_t* cnt_row, cudaStream_t s);
// Writes those entries in permuted order (columns perm(j)) at str_row_ptr, and
// the regular part's row lengths (the mask's rows minus them) to cnt_reg; sel:
// [nblocks * nkt] bytes of scratch (the plan's tiles).
cudaError_t strided_split_fill(const int32_t* res_row_ptr, const int32_t* res_col_idx, const int32_t* row_ptr,
                               const int32_t* col_idx, const int32_t* block_tile_off, const int32_t* tile_info,
                               int64_t rows, int n, int S, int nqb, int nkt, int64_t nblocks,
                               const int32_t* cnt_row, int32_t* cnt_reg, uint8_t* sel,
                               const int32_t* str_row_ptr, int32_t* str_col_idx, cudaStream_t s);
// The regular part: every entry of the mask but those moved to the permuted one.
// A row whose kept entries do not fill exactly its allotted slots raises
// kBuildBadRowPtr in *err.
cudaError_t strided_reg_fill(const int32_t* row_ptr, const int32_t* col_idx, int64_t rows, int n, int S, int nqb,
                             int nkt, const uint8_t* sel, const int32_t* reg_row_ptr, int32_t* reg_col_idx,
                             unsigned* err, cudaStream_t s);
// dst (contiguous [B, H, n, d] bf16) row perm(i) = src (strides in elements) row i.
cudaError_t strided_permute_rows(const void* src, int64_t s_b, int64_t s_h, int64_t s_n, void* dst, int B, int H,
                                 int n, int d, int S, cudaStream_t s);
// out / lse (nullable) of each row from the regular part's (out, lse1) and the
// permuted part's (o2, lse2) at the row's permuted position.
cudaError_t strided_merge(void* out, int64_t o_sb, int64_t o_sh, int64_t o_sn, const float* lse1, const void* o2,
                          const float* lse2, float* lse, int B, int H, int n, int d, int S, cudaStream_t s);

}  // namespace spattn
