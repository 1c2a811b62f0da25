/*
 * spattn.h -- C ABI of the sparse-mask scaled dot-product attention library
 * (libspattn.so, CUDA, sm_100a).
 *
 * The operation. For batch b, head h and query row i, let S_i be the column set
 * of row i of an n x n attention mask given in CSR form: token i attends to
 * token j exactly when j is in S_i ("[Proposal] Unified Interface/Implementation
 * for Sparse Attention", gluon-nlp issue 1407, opening post: a user-defined
 * CSR/COO mask of shape (n, n)). Then
 *
 *     s_ij   = scale * <q_i, k_j> + mask[b,h,i,j] + bias[b,h,i,j]      (j in S_i)
 *     out_i  = sum_{j in S_i} softmax_j(s_i.) * v_j
 *     lse_i  = log(sum_{j in S_i} exp(s_ij))                             (natural log)
 *
 * The proposal computes this as an SDDMM over the mask's nonzeros, a sparse
 * row softmax and an SpMM with V. The additive mask and the additive bias
 * follow "support attentions in AlphaFold2" (flash-attention PR 57, the
 * attention mask and attention bias shape rules); the scale multiplies the dot
 * product only. This library fuses the three stages in one pass per row with a
 * running max and a running sum rescaled by exp(m_old - m_new), dividing by the
 * sum once at the end ("Implementing and Optimizing the Scaled Dot-Product
 * Attention on Streaming Dataflow", proposed method), so no nnz-sized score
 * buffer is ever written.
 *
 * A row with no nonzeros, or whose scores are all -inf, gives out = 0 and
 * lse = -inf.
 *
 * Conventions shared by every entry point:
 *   - Every pointer named "device" must point to GPU memory of the current
 *     device; "host" pointers to CPU memory. The caller owns everything it
 *     passes in; the library keeps no reference after a call returns, except
 *     inside a spattn_mask handle, which owns the memory it allocated.
 *   - Calls are stream-ordered: they enqueue work on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream) and return without waiting, except
 *     where a function says it synchronises.
 *   - Every function returns a spattn_status. On failure nothing has been
 *     enqueued unless the function says otherwise, and spattn_last_error()
 *     returns a message for the calling thread.
 */
#ifndef SPATTN_H
#define SPATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPATTN_OK = 0,
    SPATTN_ERR_INVALID_ARG = 1, /* null pointer, bad shape, stride or size */
    SPATTN_ERR_UNSUPPORTED = 2, /* valid request outside what is implemented (dtype, head dim, alignment) */
    SPATTN_ERR_BAD_CSR = 3,     /* CSR/COO content invalid (see spattn_create_csr_mask) */
    SPATTN_ERR_CUDA = 4,        /* a CUDA runtime call failed; spattn_last_error() names it */
    SPATTN_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
    SPATTN_ERR_OOM = 6          /* device memory allocation failed */
} spattn_status;

typedef enum { SPATTN_BF16 = 0, SPATTN_F32 = 1 } spattn_dtype;

/* A strided 4-D view of device memory. Strides are in elements. A dimension of
 * size 1 may have any stride (it is read as 0, i.e. broadcast). */
typedef struct {
    void* data;        /* device */
    int32_t dtype;     /* spattn_dtype */
    int32_t reserved;  /* must be 0 */
    int64_t shape[4];
    int64_t stride[4];
} spattn_tensor;

/* ------------------------------------------------------------------ masks */

/* Mask patterns. The pattern list follows the "Sparse Attention" notes page
 * (local / sliding window, global tokens, block or strided patterns) and the
 * gluon-nlp proposal (user-defined CSR/COO masks; a per-token variable window
 * length in the discussion). Row i of mask m lists, ascending and without
 * duplicates:
 *   SLIDING              j with |i - j| <= window
 *   VARWIN               j with i - w_i <= j <= i + w_i, w_i = half_widths[m*n + i] >= 0
 *   BLOCK_STRIDED_GLOBAL j in the same block of `block` tokens as i (block > 0), or
 *                        (j - i) a multiple of `stride` (stride > 0), or
 *                        i < n_global (global tokens attend to all), or
 *                        j < n_global (and are attended to by all)
 *   COO                  the candidate columns of row m*n + i (duplicates merged,
 *                        any order), plus i itself when add_diagonal != 0
 *   CSR                  the caller's CSR, which must already be sorted and unique
 *   DENSE                every j (an all-ones mask)
 * Columns are clipped to [0, n). */
typedef enum {
    SPATTN_MASK_CSR = 0,
    SPATTN_MASK_SLIDING = 1,
    SPATTN_MASK_VARWIN = 2,
    SPATTN_MASK_BLOCK_STRIDED_GLOBAL = 3,
    SPATTN_MASK_COO = 4,
    SPATTN_MASK_DENSE = 5
} spattn_mask_kind;

typedef struct {
    int32_t kind;         /* spattn_mask_kind */
    int32_t n;            /* sequence length, >= 1 */
    int32_t num_masks;    /* masks stacked row-wise: rows m*n .. m*n + n - 1 belong to mask m */
    int32_t window;       /* SLIDING: half-width, >= 0 */
    int32_t block;        /* BLOCK_STRIDED_GLOBAL: block size (0 = no block part) */
    int32_t stride;       /* BLOCK_STRIDED_GLOBAL: stride (0 = no strided part) */
    int32_t n_global;     /* BLOCK_STRIDED_GLOBAL: number of global tokens (0 = none) */
    int32_t add_diagonal; /* COO: also include (i, i) */
    const int32_t* half_widths; /* VARWIN: device, [num_masks * n], each >= 0 */
    const int32_t* in_row_ptr;  /* CSR, COO: device, [num_masks * n + 1], starts at 0, non-decreasing */
    const int32_t* in_col_idx;  /* CSR, COO: device, [in_nnz], each in [0, n) */
    int64_t in_nnz;             /* CSR, COO: in_row_ptr[num_masks * n] */
    int32_t tile_min_nnz;       /* tensor-core tiles: a 128 x 128 tile with at least this many
                                   nonzeros is computed on tensor cores (bf16 inputs);
                                   0 = default (512; for BLOCK_STRIDED_GLOBAL it also
                                   allows the closed form, see spattn_create_csr_mask),
                                   < 0 = never */
    uint32_t flags;             /* SPATTN_MASK_* flags below, or 0 */
} spattn_mask_spec;

/* spec.flags: SLIDING, VARWIN and DENSE masks are built without waiting for
 * the device (no host synchronisation; see spattn_create_csr_mask). Other
 * kinds ignore it. */
#define SPATTN_MASK_ASYNC 1u

/* A built mask: its CSR (row_ptr int32 [num_masks*n + 1], col_idx int32 [nnz]),
 * plus the schedule the forward pass uses: rows long enough to be split over a
 * whole thread block, and the tile plan -- the 128 x 128 tiles (128 query rows
 * by 128 keys) that hold at least tile_min_nnz nonzeros, each with a per-row
 * bit mask, and the residual CSR of the entries outside those tiles. (Blocks
 * are cheaper than single entries: the block-sparse remark of the gluon-nlp
 * discussion, applied tile by tile to any CSR.) Owns its device memory.
 *
 * Interval masks. Every row of a SLIDING, VARWIN or DENSE mask is one run of
 * columns [lo, hi), so such a mask (up to 1,048,576 keys and 65,536 query
 * blocks of 128 rows) keeps the runs and its tile selection instead: the
 * forward pass derives columns and tile bits from the runs, and the CSR, the
 * tile bits and the residual CSR are written only when a call below asks for
 * them (that call synchronises the mask's stream once, and the arrays are then
 * kept until the mask is destroyed). */
typedef struct spattn_mask_s* spattn_mask;

/* Build a CSR mask on the device from a pattern (the proposal's "generate the
 * corresponding attention mask" step, then the row schedule).
 * Synchronises `stream` (twice for CSR, COO and BLOCK_STRIDED_GLOBAL masks, to
 * size col_idx and the schedule; once for interval masks, to check the
 * half-widths; not at all for interval masks with SPATTN_MASK_ASYNC). With
 * SPATTN_MASK_ASYNC the call only enqueues the build: a negative half-width is
 * then not reported here -- its row is left empty and the device error flag
 * bit 0 is raised (see spattn_device_error) -- and the size queries below wait
 * for the build. Memory comes from the library's stream-ordered pool and is
 * released by spattn_destroy_mask.
 * A BLOCK_STRIDED_GLOBAL mask with tile_min_nnz == 0 whose block divides 128,
 * stride is 0 or 128, n_global <= 128, n is a multiple of 128 and block or
 * n_global is positive is kept in closed form: the call does no device work
 * and never synchronises; the forward pass derives every tensor-core tile and
 * every row's bits from the four parameters, the strided entries outside the
 * regular tiles running as residue-permuted dense tiles (token i at
 * (i mod 128) n/128 + i div 128) in the same launch: each row's regular
 * part starts from the fp32 partial state (m, l, O) its permuted part
 * published, the running max / sum combination of the two. Its CSR, tile plan,
 * the backward pass and forward calls the closed form does not take (fp32
 * inputs, additive terms, key lengths, d = 32) use a CSR-built copy of the
 * mask made on first need (one build on the mask's stream, with its
 * synchronisations; kept until the mask is destroyed).
 * Any other BLOCK_STRIDED_GLOBAL mask whose n is a multiple of `stride` also keeps the
 * strided entries that fall outside its tensor-core tiles as a second mask in
 * residue-permuted order (token i at (i mod stride) n/stride + i div stride),
 * where they form dense tiles, plus the remaining entries as a third. That is
 * two more CSR builds (and syncs) and about the CSR's size again in memory.
 * spattn_fwd_mask uses them for bf16 inputs without additive terms; the results
 * are the same within rounding (each part's output is rounded to bf16 once
 * before the two are merged).
 * Errors: INVALID_ARG (bad kind, parameters or flags), BAD_CSR (CSR not
 * sorted/unique, a column outside [0, n), row_ptr not a valid prefix sum, or a
 * negative half-width), UNSUPPORTED (more than 2^31 - 1 nonzeros, or a COO row
 * with more candidates than the builder's limit), OOM, CUDA. On error *out is
 * NULL. */
int spattn_create_csr_mask(const spattn_mask_spec* spec, void* stream, spattn_mask* out);

/* Read a mask's sizes and device CSR pointers (owned by the mask). Any output
 * pointer may be NULL. n_long: rows with more than 1024 nonzeros (handled by
 * a whole thread block). nnz and n_long wait for an asynchronous build; asking
 * for row_ptr or col_idx of an interval mask writes its CSR first (synchronises;
 * UNSUPPORTED above 2^31 - 1 nonzeros). */
int spattn_mask_info(spattn_mask mask, int32_t* n, int32_t* num_masks, int64_t* nnz,
                     const int32_t** row_ptr, const int32_t** col_idx, int64_t* n_long);

/* The user-visible CSR of a mask: row_ptr int32 [num_masks * n + 1] (global
 * offsets, row m*n + i of mask m), col_idx int32 [nnz_total], both device
 * pointers owned by the mask and valid until spattn_destroy_mask, and the
 * total number of nonzeros over all num_masks masks. Any output pointer may be
 * NULL. This is the n x n CSR attention mask that "[Proposal] Unified
 * Interface/Implementation for Sparse Attention" (gluon-nlp issue 1407,
 * opening post) has the user hand to the operation; the same as
 * spattn_mask_info with only these outputs (an interval or closed-form mask
 * writes its CSR first and synchronises the mask's stream once; nnz_total
 * waits for an asynchronous build). Errors: INVALID_ARG (mask NULL),
 * UNSUPPORTED (more than 2^31 - 1 nonzeros), OOM, CUDA. */
int spattn_mask_csr(spattn_mask mask, const int32_t** row_ptr, const int32_t** col_idx,
                    int64_t* nnz_total);

/* Copy a mask's CSR into caller buffers (device or host memory, any mix):
 * row_ptr_dst int32 [num_masks * n + 1], col_idx_dst int32 [nnz]; either may be
 * NULL to skip it. Stream-ordered on `stream`; host destinations should be
 * pinned for the copy to be asynchronous. Interval masks write their CSR first
 * (as spattn_mask_info). */
int spattn_mask_copy_csr(spattn_mask mask, int32_t* row_ptr_dst, int32_t* col_idx_dst,
                         void* stream);

/* Copy the mask's list of long rows -- the n_long rows (mask-row ids
 * m * n + i) with more than 1024 nonzeros, which the gather kernel gives a
 * whole thread block -- into dst (device or host, int32 [n_long]; the order is
 * unspecified). Stream-ordered on `stream`; an interval mask lists them from
 * its CSR on first request, and a closed-form mask from its CSR-built copy
 * (both synchronise once). Errors: INVALID_ARG (NULL argument), OOM, CUDA. */
int spattn_mask_copy_long_rows(spattn_mask mask, int32_t* dst, void* stream);

/* The tile plan's sizes: tensor-core tiles, residual nonzeros (the entries the
 * gather kernel processes on bf16 inputs) and rows with entries on both paths.
 * Any output pointer may be NULL. Waits for an asynchronous build; n_mixed_rows
 * of an interval mask writes its explicit plan first (synchronises). */
int spattn_mask_plan_info(spattn_mask mask, int64_t* n_tiles, int64_t* residual_nnz,
                          int64_t* n_mixed_rows);

/* Diagnostic with no counterpart in the method: the number of 128 x 128
 * tensor-core tiles one forward pass over this mask computes per (b, h),
 * summed over the mask's num_masks masks (as nnz is), for bf16 inputs without
 * additive terms; each tile is two 128 x 128 x d MMAs (S = Q K^T and P V).
 * For a closed-form block + strided + global mask this counts its regular and
 * residue-permuted tiles. Waits for an asynchronous build. Errors:
 * INVALID_ARG (NULL argument). */
int spattn_mask_tile_count(spattn_mask mask, int64_t* tiles);

/* Copy the tile plan into caller buffers (device or host, any may be NULL):
 * block_tile_off int32 [num_masks * ceil(n/128) + 1] (tiles of query block x are
 * tile ids block_tile_off[x] .. block_tile_off[x+1]-1), tile_info int32 [n_tiles]
 * (key tile index, bit 31 set when all 128 x 128 entries are present),
 * tile_bits uint32 [n_tiles * 128 * 4] (row r of a tile: 4 words, bit c of word
 * c/32 = column c; left zero for dense tiles, whose entries are all present), residual row_ptr int32 [num_masks * n + 1] and col_idx
 * int32 [residual_nnz]. Returns SPATTN_ERR_INVALID_ARG when the mask has no
 * tile plan. Stream-ordered on `stream`; interval masks write these arrays
 * first (synchronises). */
int spattn_mask_copy_plan(spattn_mask mask, int32_t* block_tile_off, int32_t* tile_info,
                          uint32_t* tile_bits, int32_t* res_row_ptr, int32_t* res_col_idx,
                          void* stream);

/* Release a mask. Stream-ordered on the stream it was created on. NULL is a no-op. */
int spattn_destroy_mask(spattn_mask mask);

/* --------------------------------------------------------------- forward */

/* Fused masked attention over a raw device CSR.
 *   q, k, v  [B, H, n, d], dtype bf16 or f32 (all three the same), stride 1 over d,
 *            d in {32, 64, 128}, base pointers and row strides 16-byte aligned.
 *   row_ptr  device int32 [num_masks * n + 1]; num_masks is 1 (shared by every b)
 *            or B (mask b for batch b). Entries are clamped to [0, nnz].
 *   col_idx  device int32 [nnz]. Columns need not be sorted. A column outside
 *            [0, n) is skipped and raises the device error flag (read it with
 *            spattn_device_error). Duplicate columns count once per occurrence.
 *   add_mask, bias  optional (NULL) 4-D tensors broadcastable to [B, H, n, n]
 *            (each dimension equal or 1), dtype bf16 or f32; values are added to
 *            the scaled scores (-inf removes an entry).
 *   scale    softmax scale applied to <q_i, k_j> only (commonly 1/sqrt(d)).
 *   out      [B, H, n, d], same dtype as q, stride 1 over d, rounded to nearest even.
 *   lse      optional device float [B * H * n]; lse[(b*H + h)*n + i].
 * Uses scratch memory (a list of long rows, O(num_masks * n)) taken from the
 * library's stream-ordered pool and returned before the call's work completes. */
int spattn_fwd(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
               const int32_t* row_ptr, const int32_t* col_idx, int32_t num_masks, int64_t nnz,
               const spattn_tensor* add_mask, const spattn_tensor* bias, float scale,
               const spattn_tensor* out, float* lse, void* stream);

/* The same operation over a mask built by spattn_create_csr_mask, using its
 * prebuilt schedule. The mask's num_masks must be 1 or B and its n must match q.
 * With bf16 inputs and a tile plan, the plan's tiles run on tensor cores
 * (tcgen05) and the residual entries on the gather kernel; rows with entries
 * on both paths are merged with the running max/sum rule. Those rows need a
 * workspace of B*H*n*(d+2) floats, taken from the library's stream-ordered
 * pool for the duration of the call (only when the plan may have such rows:
 * for an interval mask whose build has not completed when the call is made,
 * whenever its parameters do not rule them out). Never synchronises.
 * fp32 inputs use the gather kernel for every entry.
 * A bounded wait in the tensor-core kernel that expires raises device error
 * flag bit 1 (see spattn_device_error). */
int spattn_fwd_mask(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                    spattn_mask mask, const spattn_tensor* add_mask, const spattn_tensor* bias,
                    float scale, const spattn_tensor* out, float* lse, void* stream);

/* The same operation as spattn_fwd computed as the proposal's three separate
 * stages ("[Proposal] Unified Interface/Implementation for Sparse Attention",
 * opening post: SDDMM, sparse softmax, SpMM): every score goes to an fp32 buffer
 * of (num_masks == 1 ? B*H : H) * nnz floats taken from the library's pool, a
 * second kernel turns the scores into softmax weights in place (and writes
 * lse), a third multiplies the weights with V. It exists to measure what the
 * fused pass saves (time, and the nnz-sized buffer) on the same inputs.
 * Arguments and errors as spattn_fwd; OOM when the buffer cannot be had. */
int spattn_fwd_unfused(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                       const int32_t* row_ptr, const int32_t* col_idx, int32_t num_masks, int64_t nnz,
                       const spattn_tensor* add_mask, const spattn_tensor* bias, float scale,
                       const spattn_tensor* out, float* lse, void* stream);

/* Backward pass over a built mask: the gradients of L = sum(dout * out) with
 * respect to q, k, v and (optionally) the bias, given the forward's out and lse
 * (the chain rule of the operation above; the pages discuss bias gradients in
 * "support attentions in AlphaFold2", flash-attention PR 57, the backward
 * discussion). With P_ij = exp(s_ij - lse_i) and D_i = <dout_i, out_i>:
 *   dS_ij = P_ij (<dout_i, v_j> - D_i)
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij dout_i,      dbias[b,h,i,j] = dS_ij summed over the bias's
 *                                  broadcast dimensions.
 *   q, k, v, add_mask, bias, scale  as given to the forward.
 *   out, lse  the forward's outputs (lse required).
 *   dout      [B, H, n, d], q's dtype.
 *   dq, dk, dv  [B, H, n, d], q's dtype, written (not accumulated).
 *   dbias     optional (NULL): f32, contiguous, the bias's shape; cleared and then
 *             accumulated with atomics (the order of the additions varies).
 * Every entry runs on CUDA cores: a row pass (one warp per query row: dq and
 * D_i) and a column pass (one warp per key over the transposed mask: dk, dv).
 * The first call over a mask writes its CSR (interval masks) and its transpose,
 * kept until the mask is destroyed, on the mask's stream, and synchronises that
 * stream when it differs from `stream`. Uses a workspace of B*H*n floats from
 * the library's pool. Errors as spattn_fwd_mask; UNSUPPORTED for n > 1,572,864. */
int spattn_bwd_mask(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                    spattn_mask mask, const spattn_tensor* add_mask, const spattn_tensor* bias,
                    float scale, const spattn_tensor* out, const float* lse, const spattn_tensor* dout,
                    const spattn_tensor* dq, const spattn_tensor* dk, const spattn_tensor* dv,
                    const spattn_tensor* dbias, void* stream);

/* spattn_fwd_mask with key padding given as lengths: for batch element b only
 * keys j < seqlen_k[b] exist (seqlen_k: device int32 [B], clamped to [0, n]),
 * as if every score with j >= seqlen_k[b] were -inf -- the seqlen_k form of the
 * key-padding mask in "support attentions in AlphaFold2" (flash-attention PR
 * 57, the discussion of varlen key padding). One int per batch element is read
 * instead of a mask row, and tensor-core tiles wholly past the length are
 * skipped. seqlen_k may be NULL (no padding); add_mask and bias still apply.
 * Arguments and errors otherwise as spattn_fwd_mask. */
int spattn_fwd_mask_kpad(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                         spattn_mask mask, const int32_t* seqlen_k, const spattn_tensor* add_mask,
                         const spattn_tensor* bias, float scale, const spattn_tensor* out, float* lse,
                         void* stream);

/* The same operation as spattn_fwd, but the call allocates no device memory.
 * For callers that cannot call cudaMalloc or take memory from a pool at run
 * time: for example a host program or plug-in whose memory manager owns the
 * whole device memory budget and forbids allocations inside its execute step,
 * or code that must not meet an allocation failure or the synchronisation an
 * allocation may bring in the middle of its work. The pages describe no such
 * variant; it has no counterpart there.
 * The scratch it needs (the list of rows above 1024 nonzeros and its counter)
 * lives in one fixed array inside the library: SPATTN_NOALLOC_MAX_ROWS + 1
 * int32 (1 MiB), which every GPU that loads the library holds until the process
 * exits. num_masks * n must be <= SPATTN_NOALLOC_MAX_ROWS, else the call
 * returns SPATTN_ERR_UNSUPPORTED without enqueuing anything. The first call on
 * each device looks up the array's device address (once per device, with that
 * device current); make that first call before any stream capture. Every call
 * on a device shares the one array and clears its counter first: calls whose
 * work can overlap on the GPU (other streams, other host threads) race on it
 * and must be serialised by the caller. Arguments and errors otherwise as
 * spattn_fwd. */
#define SPATTN_NOALLOC_MAX_ROWS 262143
int spattn_fwd_noalloc(const spattn_tensor* q, const spattn_tensor* k, const spattn_tensor* v,
                       const int32_t* row_ptr, const int32_t* col_idx, int32_t num_masks,
                       int64_t nnz, const spattn_tensor* add_mask, const spattn_tensor* bias,
                       float scale, const spattn_tensor* out, float* lse, void* stream);

/* ------------------------------------------------------------- utilities */

/* Message of the last failed call on this thread ("" if none). Valid until the
 * thread's next call into the library. */
const char* spattn_last_error(void);

/* Synchronise `stream`, then read and clear the current device's error flags
 * raised by kernels (bit 0: a column index outside [0, n) was skipped, or an
 * asynchronous interval-mask build met a negative half-width; bit 1:
 * a bounded wait in the tensor-core kernel expired and its rows are invalid).
 * *flags may be NULL. Returns SPATTN_OK, SPATTN_ERR_TIMEOUT if bit 1 was set,
 * else SPATTN_ERR_BAD_CSR if bit 0 was set. */
int spattn_device_error(void* stream, uint32_t* flags);

/* spattn_device_error without the flag word: synchronises `stream`, reads and
 * clears the error flags, and returns SPATTN_ERR_TIMEOUT if a bounded
 * device-side wait expired, SPATTN_ERR_BAD_CSR if a column outside [0, n) was
 * skipped (or an asynchronous build met a negative half-width), SPATTN_OK
 * otherwise (SPATTN_ERR_CUDA if the synchronisation itself fails). */
int spattn_check_device_error(void* stream);

/* Library version: major * 10000 + minor * 100 + patch. */
int spattn_version(void);

/* Number of kernels this library has enqueued since it was loaded, over all
 * threads and devices (a diagnostic with no counterpart in the method: it lets
 * a caller count the launches a sequence of calls costs). Never fails. */
uint64_t spattn_launch_count(void);

/* Number of memory allocations this library has made since it was loaded
 * (stream-ordered pool blocks, device memory, mapped host memory), over all
 * threads and devices: a diagnostic with no counterpart in the method, so that
 * a caller can check that a sequence of calls allocates nothing. Never fails. */
uint64_t spattn_alloc_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SPATTN_H */
