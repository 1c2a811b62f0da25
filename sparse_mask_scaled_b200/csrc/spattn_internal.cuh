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
};

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
// (COO only). info->err must start at 0.
cudaError_t build_phase1(const BuildSpec& s, int32_t* row_ptr, int32_t* counts,
                         int64_t* scan_tmp, int32_t* coo_tmp, BuildInfo* info,
                         cudaStream_t stream);
int64_t scan_tmp_elems(int64_t rows);
// Phase 2: write col_idx from the pattern (or copy it from coo_tmp / in_col_idx).
cudaError_t build_phase2(const BuildSpec& s, const int32_t* row_ptr, const int32_t* coo_tmp,
                         int32_t* col_idx, cudaStream_t stream);

}  // namespace spattn
