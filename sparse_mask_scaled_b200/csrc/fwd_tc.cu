// Tensor-core forward for the mask's dense and near-dense 128 x 128 tiles
// (tcgen05 MMAs with TMEM accumulators, TMA tile loads, sm_100a).
//
// One CTA of 128 threads owns one 128-row query block of one (b, h) and walks
// the block's selected key tiles. Per tile:
//   S = Q K^T               tcgen05.mma (M = 128, N = 128, K = d), S in TMEM
//   s = scale*S + mask + bias, entries the CSR does not list set to -inf
//                           (thread t owns query row t = TMEM lane t)
//   running max / sum       the streaming-dataflow SDPA paper's rescaling rule;
//                           the max used as reference only moves when a tile's
//                           max exceeds it by more than 2^8, and then the O
//                           accumulator in TMEM is rescaled by exp2(m_old - m_new)
//   O += P V                tcgen05.mma (M = 128, N = d, K = 128), P from smem
// K/V tiles are double-buffered and loaded by TMA (no multicast) while the
// previous tile's softmax and P V run. At the end O / l is written (bf16) and
// lse = m + log(l); rows that also have residual (gathered) entries first merge
// the gather kernel's partial (m, l, acc) with the same rescaling rule.
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

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Makes every use of r[] depend on the TMEM load having completed.
__device__ __forceinline__ void tmem_wait_ld_dep(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

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
    static constexpr int OFF_BAR = OFF_P + P_BYTES;  // 5 mbarriers + tmem slot + abort flag
    // At least 100 KB so that no more than two CTAs (2 x 256 TMEM columns) share
    // an SM and tcgen05.alloc never has to wait; d = 64 fits two CTAs per SM.
    static constexpr int SMEM_BYTES = OFF_BAR + 64 > 100 * 1024 ? OFF_BAR + 64 : 100 * 1024;
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
};

// Adds log2(e) * addend[b, h, i, jj0 + j] to x[j] for j < ncols.
__device__ __forceinline__ void add_addend_row(const AddendView& a, int64_t rowbase, int jj0,
                                               int ncols, float (&x)[128]) {
    const int64_t off0 = rowbase + (int64_t)jj0 * a.s3;
    if (a.dtype == 0 && a.s3 == 1 && ncols == 128 &&
        ((reinterpret_cast<uintptr_t>(a.data) + (uintptr_t)off0 * 2) & 15) == 0) {
        const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.data) + off0);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
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
    for (int j = 0; j < 128; ++j) {
        if (j < ncols) {
            const int64_t off = off0 + (int64_t)j * a.s3;
            const float v = a.dtype == 0
                                ? __bfloat162float(__ldg(reinterpret_cast<const __nv_bfloat16*>(a.data) + off))
                                : __ldg(reinterpret_cast<const float*>(a.data) + off);
            x[j] += kLog2e * v;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const TcParams P) {
    using C = TcCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];

    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.x / P.nqb, qb = blockIdx.x - bh * P.nqb;
    const int b = bh / P.H, h = bh - b * P.H;
    const int mk = P.num_masks == 1 ? 0 : b;
    const int64_t blk = (int64_t)mk * P.nqb + qb;
    const int t_begin = P.block_tile_off[blk];
    const int T = P.block_tile_off[blk + 1] - t_begin;
    if (T <= 0) return;  // whole CTA: the gather kernel owns this block
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
            tma_load_4d(dK + c * C::CHUNK_BYTES, &tmK, bar, c * C::CHUNK_ELEMS, kt * 128, h, b);
            tma_load_4d(dV + c * C::CHUNK_BYTES, &tmV, bar, c * C::CHUNK_ELEMS, kt * 128, h, b);
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
            tma_load_4d(sQ + c * C::CHUNK_BYTES, &tmQ, barQ, c * C::CHUNK_ELEMS, qb * 128, h, b);
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

    for (int u = 0; u < T; ++u) {
        const int info = P.tile_info[t_begin + u];
        const int kt = info & 0x7fffffff;
        const bool dense = info < 0;
        uint32_t bits[4] = {0u, 0u, 0u, 0u};
        if (dense) {
            bits[0] = bits[1] = bits[2] = bits[3] = 0xffffffffu;
        } else if (row_ok) {
            const uint4 w = __ldg(reinterpret_cast<const uint4*>(P.tile_bits) + ((int64_t)(t_begin + u) * 128 + row));
            bits[0] = w.x;
            bits[1] = w.y;
            bits[2] = w.z;
            bits[3] = w.w;
        }
        float x[128];
#pragma unroll
        for (int j = 0; j < 128; ++j) x[j] = 0.f;
        const int jj0 = kt * 128;
        const int ncols = P.n - jj0 < 128 ? P.n - jj0 : 128;
        if (P.has_extra && row_ok) {
            if (P.mask.data) add_addend_row(P.mask, mask_rowbase, jj0, ncols, x);
            if (P.bias.data) add_addend_row(P.bias, bias_rowbase, jj0, ncols, x);
        }

        wait(barS, (uint32_t)(u & 1));
        tc_fence_after();
        __syncwarp();
        {
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tmem_ld32(tS + lane_base + 0, r0);
            tmem_ld32(tS + lane_base + 32, r1);
            tmem_ld32(tS + lane_base + 64, r2);
            tmem_ld32(tS + lane_base + 96, r3);
            tmem_wait_ld_dep(r0);
            tmem_wait_ld_dep(r1);
            tmem_wait_ld_dep(r2);
            tmem_wait_ld_dep(r3);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                x[j] = fmaf(__uint_as_float(r0[j]), P.qk_scale_log2, x[j]);
                x[32 + j] = fmaf(__uint_as_float(r1[j]), P.qk_scale_log2, x[32 + j]);
                x[64 + j] = fmaf(__uint_as_float(r2[j]), P.qk_scale_log2, x[64 + j]);
                x[96 + j] = fmaf(__uint_as_float(r3[j]), P.qk_scale_log2, x[96 + j]);
            }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 128; ++j) {
            const bool on = (bits[j >> 5] >> (j & 31)) & 1u;
            x[j] = on ? x[j] : -INFINITY;
            mx = fmaxf(mx, x[j]);
        }
        const bool need = mx > m_ref + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
            alpha = ex2(m_ref - mx);
            m_ref = mx;
            l *= alpha;
        }
        const float mu = m_ref == -INFINITY ? 0.f : m_ref;
        uint32_t pk[64];
        float lsum = 0.f;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
            const float p0 = ex2(x[2 * k] - mu), p1 = ex2(x[2 * k + 1] - mu);
            lsum += p0 + p1;
            __nv_bfloat162 hv = __floats2bfloat162_rn(p0, p1);
            pk[k] = *reinterpret_cast<uint32_t*>(&hv);
        }
        l += lsum;

        // P V of the previous tile must be done before sP is overwritten and O rescaled
        if (u > 0) {
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
        // P (bf16) into the K-major, 128-byte-swizzled A operand layout
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
            for (int piece = 0; piece < 8; ++piece) {
                const int k = kc * 32 + piece * 4;
                const uint32_t addr = sP + (uint32_t)(kc * 16384 + row * 128 + ((piece ^ (row & 7)) << 4));
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[k]),
                             "r"(pk[k + 1]), "r"(pk[k + 2]), "r"(pk[k + 3])
                             : "memory");
            }
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
    float o[D];
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t ro[32];
        tmem_ld32(tO + lane_base + c * 32, ro);
        tmem_wait_ld_dep(ro);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[c * 32 + j] = __uint_as_float(ro[j]);
    }
    if (row_ok && !*abort_flag) {
        float M = m_ref, L = l, fa = 1.f;
        const int64_t mrow = (int64_t)mk * P.n + i;
        const int64_t wrow = (int64_t)bh * P.n + i;
        const bool mixed = P.ws_ml && P.res_row_ptr[mrow + 1] > P.res_row_ptr[mrow];
        float mg = -INFINITY, lg = 0.f, fg = 0.f;
        if (mixed) {
            mg = P.ws_ml[wrow * 2];
            lg = P.ws_ml[wrow * 2 + 1];
            M = fmaxf(m_ref, mg);
            const float Mu = M == -INFINITY ? 0.f : M;
            fa = ex2(m_ref - Mu);
            fg = ex2(mg - Mu);
            L = l * fa + lg * fg;
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
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
        if (P.lse) P.lse[wrow] = L > 0.f ? (M + lg2(L)) * kLn2 : -INFINITY;
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

// 4-D map over a [B, H, n, d] bf16 tensor, box {chunk, 128 rows, 1, 1}.
cudaError_t make_map(CUtensorMap* map, const TcOperand& t, int B, int H, int n, int d, int chunk) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const uint64_t sn = (uint64_t)t.s_n * 2;
    const uint64_t sh = H > 1 ? (uint64_t)t.s_h * 2 : sn * (uint64_t)n;
    const uint64_t sb = B > 1 ? (uint64_t)t.s_b * 2 : sh * (uint64_t)H;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {sn, sh, sb};
    cuuint32_t box[4] = {(cuuint32_t)chunk, 128, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw =
        chunk * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.data), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
        attr_err = cudaFuncSetAttribute(k_fwd_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap mq, mk, mv;
    cudaError_t e;
    if ((e = make_map(&mq, q, p.B, p.H, p.n, D, C::CHUNK_ELEMS)) != cudaSuccess) return e;
    if ((e = make_map(&mk, k, p.B, p.H, p.n, D, C::CHUNK_ELEMS)) != cudaSuccess) return e;
    if ((e = make_map(&mv, v, p.B, p.H, p.n, D, C::CHUNK_ELEMS)) != cudaSuccess) return e;
    const int64_t grid = (int64_t)p.B * p.H * p.nqb;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    k_fwd_tc<D><<<(unsigned)grid, kThreads, C::SMEM_BYTES, s>>>(mq, mk, mv, p);
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
