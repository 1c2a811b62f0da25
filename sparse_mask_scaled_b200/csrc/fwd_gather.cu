// Fused sparse-mask attention forward on CUDA cores: for each query row, gather
// the K and V rows named by the row's CSR columns, take the dot products (the
// SDDMM of the gluon-nlp sparse-attention proposal), keep a running max and a
// running sum rescaled by exp(m_old - m_new) (the streaming-dataflow SDPA
// paper's proposed method) and accumulate the weighted V rows (the SpMM), then
// divide once by the sum. No per-nonzero score is ever stored.
//
// Work split. A warp owns one query row. A K/V row of d elements is covered by
// LPR = d * sizeof(T) / 16 lanes (one 16-byte vector each), so a warp holds
// G = 32 / LPR groups; group g takes nonzeros p = base + u*G + g (u < U) of each
// step of STEP = G*U nonzeros and keeps its own running (max, sum, acc); the
// groups merge with the same rescaling rule at the end of the row. Rows with
// more than kLongRowThreshold nonzeros go to a second kernel in which eight
// warps share a row and merge through shared memory.
//
// Scores are kept in the base-2 domain: q is pre-multiplied by scale*log2(e)
// and the additive mask/bias by log2(e), so every exponential is one ex2.
#include "spattn_internal.cuh"

#include <math.h>

namespace spattn {

__device__ unsigned int g_error_flags = 0;

namespace {

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

__device__ __forceinline__ uint4 ldg16(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// Two fp32 lanes per instruction (fma.rn.f32x2 / mul.rn.f32x2): each lane is
// the plain fp32 operation, rounded to nearest even.
__device__ __forceinline__ uint64_t f2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void split2(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

template <typename T>
struct Elem;

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int VEC = 8;
    __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            f[2 * t] = __uint_as_float(w[t] << 16);
            f[2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * t], f[2 * t + 1]);
            w[t] = *reinterpret_cast<uint32_t*>(&h);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ __forceinline__ static void store1(void* base, int64_t idx, float x) {
        reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(x);
    }
};

template <>
struct Elem<float> {
    static constexpr int VEC = 4;
    __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
        f[0] = __uint_as_float(r.x);
        f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z);
        f[3] = __uint_as_float(r.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
    __device__ __forceinline__ static void store1(void* base, int64_t idx, float x) {
        reinterpret_cast<float*>(base)[idx] = x;
    }
};

template <typename T, int D>
struct Cfg {
    static constexpr int VEC = Elem<T>::VEC;
    static constexpr int LPR = D / VEC;  // lanes per K/V row
    static constexpr int G = 32 / LPR;   // nonzeros loaded per vector instruction
    static constexpr int U = (32 / G) < 8 ? (32 / G) : 8;  // nonzeros per group per step
    static constexpr int STEP = G * U;   // nonzeros per warp step (<= 32)
    static_assert(D % VEC == 0 && LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "unsupported head dim");
};

template <int VEC>
struct State {
    float m;  // running max (base-2 domain)
    float l;  // running sum of ex2(s - m)
    float acc[VEC];
};

__device__ __forceinline__ float load_addend(const AddendView& a, int64_t off) {
    if (a.dtype == 0)
        return __bfloat162float(__ldg(reinterpret_cast<const __nv_bfloat16*>(a.data) + off));
    return __ldg(reinterpret_cast<const float*>(a.data) + off);
}

__device__ __forceinline__ void clamp_row(const FwdParams& P, int64_t mrow, int64_t& p0,
                                          int64_t& p1) {
    p0 = P.row_ptr[mrow];
    p1 = P.row_ptr[mrow + 1];
    p0 = p0 < 0 ? 0 : (p0 > P.nnz ? P.nnz : p0);
    p1 = p1 < p0 ? p0 : (p1 > P.nnz ? P.nnz : p1);
}

// Keys of batch element b that exist: [0, seqlen_k[b]) with key padding, else [0, n).
__device__ __forceinline__ int key_limit(const FwdParams& P, int b) {
    if (!P.seqlen_k) return P.n;
    const int L = P.seqlen_k[b];
    return L < 0 ? 0 : (L > P.n ? P.n : L);
}

template <typename T, int D>
struct RowCtx {
    const T* kb;   // K of (b, h)
    const T* vb;   // V of (b, h)
    int klim;      // keys >= klim are padding
    int64_t mask_base, bias_base;  // addend offsets of (b, h, i, 0)
    float qf[Cfg<T, D>::VEC];      // this lane's slice of q_i * scale * log2(e)
};

template <typename T, int D>
__device__ __forceinline__ void init_row(const FwdParams& P, int b, int h, int i, int lane,
                                         RowCtx<T, D>& rc, State<Cfg<T, D>::VEC>& st) {
    using C = Cfg<T, D>;
    const int c = lane % C::LPR;
    const T* q = reinterpret_cast<const T*>(P.q) + b * P.q_sb + h * P.q_sh + i * P.q_sn;
    rc.kb = reinterpret_cast<const T*>(P.k) + b * P.k_sb + h * P.k_sh;
    rc.vb = reinterpret_cast<const T*>(P.v) + b * P.v_sb + h * P.v_sh;
    rc.mask_base = b * P.mask.s0 + h * P.mask.s1 + i * P.mask.s2;
    rc.bias_base = b * P.bias.s0 + h * P.bias.s1 + i * P.bias.s2;
    rc.klim = key_limit(P, b);
    Elem<T>::unpack(ldg16(q + c * C::VEC), rc.qf);
#pragma unroll
    for (int e = 0; e < C::VEC; ++e) rc.qf[e] *= P.qk_scale_log2;
    st.m = -INFINITY;
    st.l = 0.f;
#pragma unroll
    for (int e = 0; e < C::VEC; ++e) st.acc[e] = 0.f;
}

// Process the steps of STEP nonzeros starting at first, first + stride, ...
// (below p1) of one row into `st`. kRun: the positions are the columns
// themselves (a run of an interval row), else indices into col_idx.
template <typename T, int D, bool kRun = false>
__device__ __forceinline__ void row_steps(const FwdParams& P, const RowCtx<T, D>& rc,
                                          int64_t first, int64_t p1, int64_t stride, int lane,
                                          State<Cfg<T, D>::VEC>& st) {
    using C = Cfg<T, D>;
    const int g = lane / C::LPR, c = lane % C::LPR;
    for (int64_t pb = first; pb < p1; pb += stride) {
        // one coalesced read of this step's columns (and additive terms)
        int col = -1;
        float extra = 0.f;
        const int64_t mp = pb + lane;
        if (lane < C::STEP && mp < p1) {
            const int j = kRun ? (int)mp : __ldg(P.col_idx + mp);
            if ((unsigned)j >= (unsigned)P.n) {
                atomicOr(&g_error_flags, kErrBadColumn);
            } else if (j < rc.klim) {  // padded keys are left out
                col = j;
                if (P.has_extra) {
                    float e = 0.f;
                    if (P.mask.data) e += load_addend(P.mask, rc.mask_base + j * P.mask.s3);
                    if (P.bias.data) e += load_addend(P.bias, rc.bias_base + j * P.bias.s3);
                    extra = e * kLog2e;
                }
            }
        }
        int js[C::U];
        float es[C::U];
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            js[u] = __shfl_sync(0xffffffffu, col, u * C::G + g);
            es[u] = __shfl_sync(0xffffffffu, extra, u * C::G + g);
        }
        uint4 kr[C::U], vr[C::U];
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            if (js[u] >= 0) {
                kr[u] = ldg16(rc.kb + (int64_t)js[u] * P.k_sn + c * C::VEC);
                vr[u] = ldg16(rc.vb + (int64_t)js[u] * P.v_sn + c * C::VEC);
            } else {
                kr[u] = make_uint4(0u, 0u, 0u, 0u);
                vr[u] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        float s[C::U];
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            float kf[C::VEC];
            Elem<T>::unpack(kr[u], kf);
            // even and odd elements in the two lanes of one packed FMA
            uint64_t a2 = f2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < C::VEC / 2; ++e) a2 = ffma2(f2(rc.qf[2 * e], rc.qf[2 * e + 1]), f2(kf[2 * e], kf[2 * e + 1]), a2);
            float ae, ao;
            split2(a2, ae, ao);
            s[u] = ae + ao;
        }
#pragma unroll
        for (int off = 1; off < C::LPR; off <<= 1) {
#pragma unroll
            for (int u = 0; u < C::U; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], off);
        }
        float mx = st.m;
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            s[u] = js[u] >= 0 ? s[u] + es[u] : -INFINITY;
            mx = fmaxf(mx, s[u]);
        }
        const float mu = (mx == -INFINITY) ? 0.f : mx;
        const float alpha = ex2(st.m - mu);
        st.l *= alpha;
        uint64_t acc2[C::VEC / 2];
#pragma unroll
        for (int e = 0; e < C::VEC / 2; ++e) acc2[e] = fmul2(f2(st.acc[2 * e], st.acc[2 * e + 1]), f2(alpha, alpha));
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            const float pw = ex2(s[u] - mu);
            st.l += pw;
            float vf[C::VEC];
            Elem<T>::unpack(vr[u], vf);
            const uint64_t pw2 = f2(pw, pw);
#pragma unroll
            for (int e = 0; e < C::VEC / 2; ++e) acc2[e] = ffma2(pw2, f2(vf[2 * e], vf[2 * e + 1]), acc2[e]);
        }
#pragma unroll
        for (int e = 0; e < C::VEC / 2; ++e) split2(acc2[e], st.acc[2 * e], st.acc[2 * e + 1]);
        st.m = mx;
    }
}

// Merge the warp's G group states (same rescaling rule); every group ends
// holding the merged state.
template <int VEC, int LPR>
__device__ __forceinline__ void merge_groups(State<VEC>& st) {
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, st.m, off);
        const float lo = __shfl_xor_sync(0xffffffffu, st.l, off);
        const float mx = fmaxf(st.m, mo);
        const float mu = (mx == -INFINITY) ? 0.f : mx;
        const float a = ex2(st.m - mu), bo = ex2(mo - mu);
        st.l = st.l * a + lo * bo;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const float ao = __shfl_xor_sync(0xffffffffu, st.acc[e], off);
            st.acc[e] = st.acc[e] * a + ao * bo;
        }
        st.m = mx;
    }
}

template <int VEC>
__device__ __forceinline__ void write_partial(float* dst, const float (&acc)[VEC]) {
#pragma unroll
    for (int e = 0; e < VEC; e += 4)
        *reinterpret_cast<float4*>(dst + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
}

template <typename T, int D>
__global__ void __launch_bounds__(256) k_fwd_short(const FwdParams P) {
    using C = Cfg<T, D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blocks_per_bh = (P.n + 7) >> 3;
    const int bh = blockIdx.x / blocks_per_bh;
    const int i = (blockIdx.x - bh * blocks_per_bh) * 8 + warp;
    if (i >= P.n) return;
    const int b = bh / P.H, h = bh - b * P.H;
    const int64_t mrow = (int64_t)(P.num_masks == 1 ? 0 : b) * P.n + i;
    int64_t p0, p1;
    clamp_row(P, mrow, p0, p1);
    if (p1 - p0 > kLongRowThreshold) return;  // the long-row kernel owns it

    RowCtx<T, D> rc;
    State<C::VEC> st;
    init_row<T, D>(P, b, h, i, lane, rc, st);
    row_steps<T, D>(P, rc, p0, p1, C::STEP, lane, st);
    merge_groups<C::VEC, C::LPR>(st);

    if (P.qb_tile_off) {
        const int64_t blk = (int64_t)(P.num_masks == 1 ? 0 : b) * P.nqb + (i >> 7);
        if (P.qb_tile_off[blk + 1] > P.qb_tile_off[blk]) {
            // the tensor-core kernel finishes this row; hand over the partial state
            if (p1 > p0) {
                const int64_t wrow = (int64_t)bh * P.n + i;
                if (lane < C::LPR)
                    write_partial<C::VEC>(P.ws_acc + wrow * D + lane * C::VEC, st.acc);
                if (lane == 0) {
                    P.ws_ml[wrow * 2] = st.m;
                    P.ws_ml[wrow * 2 + 1] = st.l;
                }
            }
            return;
        }
    }
    if (lane < C::LPR) {
        const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
        float o[C::VEC];
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) o[e] = st.acc[e] * inv;
        T* orow = reinterpret_cast<T*>(P.out) + b * P.o_sb + h * P.o_sh + i * P.o_sn;
        *reinterpret_cast<uint4*>(orow + lane * C::VEC) = Elem<T>::pack(o);
    }
    if (lane == 0 && P.lse)
        P.lse[((int64_t)bh) * P.n + i] = st.l > 0.f ? (st.m + lg2(st.l)) * kLn2 : -INFINITY;
}

// The warp-uniform runs of an interval row [lo, hi) that lie in unselected key
// tiles (tm[kt] < 0), merged across neighbouring tiles up to 32 tiles at a
// time; the whole run when tm is null. fn(a, z) is called by every lane.
template <class F>
__device__ __forceinline__ void for_each_run(const int32_t* __restrict__ tm, int lo, int hi, int lane,
                                             F&& fn) {
    if (hi <= lo) return;
    if (!tm) {
        fn(lo, hi);
        return;
    }
    const int k0 = lo >> 7, k1 = (hi - 1) >> 7;
    for (int c0 = k0; c0 <= k1; c0 += 32) {
        const int kt = c0 + lane;
        unsigned bits = __ballot_sync(0xffffffffu, kt <= k1 && __ldg(tm + kt) < 0);
        while (bits) {
            const int s = __ffs(bits) - 1;
            const unsigned inv = ~(bits >> s);
            const int len = inv ? __ffs(inv) - 1 : 32 - s;
            const int ta = c0 + s, tz = ta + len;
            fn(lo > ta * kTileN ? lo : ta * kTileN, hi < tz * kTileN ? hi : tz * kTileN);
            bits = s + len >= 32 ? 0u : (bits & (0xffffffffu << (s + len)));
        }
    }
}

// Final output of a row (out = acc / l, lse), or its partial state for the
// tensor-core kernel. Lanes < LPR hold the row's acc slices.
template <typename T, int D>
__device__ __forceinline__ void finish_row(const FwdParams& P, int b, int h, int i, int lane,
                                           const State<Cfg<T, D>::VEC>& st, bool partial) {
    using C = Cfg<T, D>;
    const int64_t wrow = ((int64_t)b * P.H + h) * P.n + i;
    if (partial) {
        if (lane < C::LPR) write_partial<C::VEC>(P.ws_acc + wrow * D + lane * C::VEC, st.acc);
        if (lane == 0) {
            P.ws_ml[wrow * 2] = st.m;
            P.ws_ml[wrow * 2 + 1] = st.l;
        }
        return;
    }
    if (lane < C::LPR) {
        const float inv = st.l > 0.f ? 1.f / st.l : 0.f;
        float o[C::VEC];
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) o[e] = st.acc[e] * inv;
        T* orow = reinterpret_cast<T*>(P.out) + b * P.o_sb + h * P.o_sh + i * P.o_sn;
        *reinterpret_cast<uint4*>(orow + lane * C::VEC) = Elem<T>::pack(o);
    }
    if (lane == 0 && P.lse) P.lse[wrow] = st.l > 0.f ? (st.m + lg2(st.l)) * kLn2 : -INFINITY;
}

// Eight rows i0 .. i0 + 7 of (b, h) (see k_fwd_itv).
template <typename T, int D>
__device__ __forceinline__ void itv_rows8(const FwdParams& P, int b, int h, int mk, int i0,
                                          const int32_t* __restrict__ tm, bool partial) {
    using C = Cfg<T, D>;
    __shared__ float sm_m[8], sm_l[8];
    __shared__ float sm_acc[8][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = i0 + warp;
    const int klim = key_limit(P, b);
    int lo = 0, hi = 0;
    if (i < P.n) {
        const int2 v = P.itv_lohi[(int64_t)mk * P.n + i];
        lo = v.x;
        hi = v.y < klim ? v.y : klim;
    }
    int len = 0;
    for_each_run(tm, lo, hi, lane, [&](int a, int z) { len += z - a; });
    if (!__syncthreads_or(len > kLongRowThreshold)) {
        if (i >= P.n) return;  // the caller's loop ends with this group
        RowCtx<T, D> rc;
        State<C::VEC> st;
        init_row<T, D>(P, b, h, i, lane, rc, st);
        for_each_run(tm, lo, hi, lane,
                     [&](int a, int z) { row_steps<T, D, true>(P, rc, a, z, C::STEP, lane, st); });
        merge_groups<C::VEC, C::LPR>(st);
        finish_row<T, D>(P, b, h, i, lane, st, partial);
        return;
    }
    for (int rr = 0; rr < 8 && i0 + rr < P.n; ++rr) {
        const int ii = i0 + rr;
        int2 v = P.itv_lohi[(int64_t)mk * P.n + ii];
        v.y = v.y < klim ? v.y : klim;
        RowCtx<T, D> rc;
        State<C::VEC> st;
        init_row<T, D>(P, b, h, ii, lane, rc, st);
        for_each_run(tm, v.x, v.y, lane, [&](int a, int z) {
            row_steps<T, D, true>(P, rc, a + warp * C::STEP, z, 8 * C::STEP, lane, st);
        });
        merge_groups<C::VEC, C::LPR>(st);
        if (lane == 0) {
            sm_m[warp] = st.m;
            sm_l[warp] = st.l;
        }
        if (lane < C::LPR) {
#pragma unroll
            for (int e = 0; e < C::VEC; ++e) sm_acc[warp][lane * C::VEC + e] = st.acc[e];
        }
        __syncthreads();
        if (warp == 0) {  // merge the eight warps' states; lanes < LPR own acc slices
            float mx = -INFINITY;
#pragma unroll
            for (int w = 0; w < 8; ++w) mx = fmaxf(mx, sm_m[w]);
            const float mu = (mx == -INFINITY) ? 0.f : mx;
            State<C::VEC> t;
            t.m = mx;
            t.l = 0.f;
#pragma unroll
            for (int e = 0; e < C::VEC; ++e) t.acc[e] = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const float f = ex2(sm_m[w] - mu);
                t.l = fmaf(sm_l[w], f, t.l);
                if (lane < C::LPR) {
#pragma unroll
                    for (int e = 0; e < C::VEC; ++e) t.acc[e] = fmaf(sm_acc[w][lane * C::VEC + e], f, t.acc[e]);
                }
            }
            finish_row<T, D>(P, b, h, ii, lane, t, partial);
        }
        __syncthreads();
    }
}

// Interval masks. A block takes 128 / itv_slices rows of one 128-row query
// block of one (b, h), eight at a time: eight warps, one row each; when any of
// the eight has more than kLongRowThreshold entries to gather, the warps take
// those rows one after the other together instead (merging through shared
// memory). In a query block with tensor-core tiles every row hands over its
// partial state (l = 0 when it gathered nothing), and query blocks without
// entries outside their tiles return at once.
template <typename T, int D>
__global__ void __launch_bounds__(256, 2) k_fwd_itv(const FwdParams P) {
    const int slices = P.itv_slices, rows_per = kTileM / slices;
    const int per_bh = P.nqb * slices;
    const int bh = blockIdx.x / per_bh;
    const int rem = blockIdx.x - bh * per_bh;
    const int qb = rem / slices;
    const int b = bh / P.H, h = bh - b * P.H;
    const int mk = P.num_masks == 1 ? 0 : b;
    const int64_t blk = (int64_t)mk * P.nqb + qb;
    const int32_t* tm = nullptr;
    bool partial = false;
    if (P.tmap) {
        tm = P.tmap + blk * P.nkt;
        if (P.qb_ntiles[blk] > 0) {
            if (!P.blk_res[blk]) return;  // the tensor-core kernel does every row alone
            partial = true;
        }
    }
    const int r0 = qb * kTileM + (rem - qb * slices) * rows_per;
    const int r1 = min(r0 + rows_per, P.n);
    for (int i0 = r0; i0 < r1; i0 += 8) itv_rows8<T, D>(P, b, h, mk, i0, tm, partial);
}

// ------------------------------------------------------------------ unfused
// The proposal's three separate stages, for comparison with the fused kernels:
// an SDDMM that writes every score to memory, a row softmax over those scores
// (in place, plus lse), and an SpMM of the weights with V. scores: fp32, one
// copy of the mask's nnz per (b, h) (per h when every b has its own mask),
// indexed by the mask's CSR position.
__device__ __forceinline__ int64_t unf_index(const FwdParams& P, int b, int h, int64_t p) {
    return (P.num_masks == 1 ? (int64_t)b * P.H + h : (int64_t)h) * P.nnz + p;
}

template <typename T, int D>
__global__ void __launch_bounds__(256) k_unf_sddmm(const FwdParams P, float* __restrict__ scores) {
    using C = Cfg<T, D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane / C::LPR, c = lane % C::LPR;
    const int per_bh = (P.n + 7) >> 3;
    const int bh = blockIdx.x / per_bh;
    const int i = (blockIdx.x - bh * per_bh) * 8 + warp;
    if (i >= P.n) return;
    const int b = bh / P.H, h = bh - b * P.H;
    const int64_t mrow = (int64_t)(P.num_masks == 1 ? 0 : b) * P.n + i;
    int64_t p0, p1;
    clamp_row(P, mrow, p0, p1);
    const T* kb = reinterpret_cast<const T*>(P.k) + b * P.k_sb + h * P.k_sh;
    float qf[C::VEC];
    Elem<T>::unpack(ldg16(reinterpret_cast<const T*>(P.q) + b * P.q_sb + h * P.q_sh + i * P.q_sn + c * C::VEC), qf);
    const int64_t mask_base = b * P.mask.s0 + h * P.mask.s1 + i * P.mask.s2;
    const int64_t bias_base = b * P.bias.s0 + h * P.bias.s1 + i * P.bias.s2;
    const float scale = P.qk_scale_log2 / kLog2e;
    for (int64_t pb = p0; pb < p1; pb += C::G) {  // one nonzero per group, same trip count for all
        const int64_t p = pb + g;
        const bool in = p < p1;
        const int j = in ? __ldg(P.col_idx + p) : 0;
        const bool ok = in && (unsigned)j < (unsigned)P.n;
        float kf[C::VEC];
        if (ok) Elem<T>::unpack(ldg16(kb + (int64_t)j * P.k_sn + c * C::VEC), kf);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) a = ok ? fmaf(qf[e], kf[e], a) : 0.f;
#pragma unroll
        for (int off = 1; off < C::LPR; off <<= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        if (in && c == 0) {
            float sc = -INFINITY;
            if (ok) {
                sc = scale * a;
                if (P.mask.data) sc += load_addend(P.mask, mask_base + j * P.mask.s3);
                if (P.bias.data) sc += load_addend(P.bias, bias_base + j * P.bias.s3);
            } else {
                atomicOr(&g_error_flags, kErrBadColumn);
            }
            scores[unf_index(P, b, h, p)] = sc;
        }
    }
}

// One warp per row: max, then exp and sum, then the weights in place; lse.
__global__ void __launch_bounds__(256) k_unf_softmax(const FwdParams P, float* __restrict__ scores) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_bh = (P.n + 7) >> 3;
    const int bh = blockIdx.x / per_bh;
    const int i = (blockIdx.x - bh * per_bh) * 8 + warp;
    if (i >= P.n) return;
    const int b = bh / P.H, h = bh - b * P.H;
    const int64_t mrow = (int64_t)(P.num_masks == 1 ? 0 : b) * P.n + i;
    int64_t p0, p1;
    clamp_row(P, mrow, p0, p1);
    float* row = scores + unf_index(P, b, h, 0);
    float m = -INFINITY;
    for (int64_t p = p0 + lane; p < p1; p += 32) m = fmaxf(m, row[p]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float mu = m == -INFINITY ? 0.f : m;
    float l = 0.f;
    for (int64_t p = p0 + lane; p < p1; p += 32) {
        const float e = ex2((row[p] - mu) * kLog2e);
        row[p] = e;
        l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int64_t p = p0 + lane; p < p1; p += 32) row[p] *= inv;
    if (lane == 0 && P.lse) P.lse[(int64_t)bh * P.n + i] = l > 0.f ? m + lg2(l) * kLn2 : -INFINITY;
}

template <typename T, int D>
__global__ void __launch_bounds__(256) k_unf_spmm(const FwdParams P, const float* __restrict__ weights) {
    using C = Cfg<T, D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane / C::LPR, c = lane % C::LPR;
    const int per_bh = (P.n + 7) >> 3;
    const int bh = blockIdx.x / per_bh;
    const int i = (blockIdx.x - bh * per_bh) * 8 + warp;
    if (i >= P.n) return;
    const int b = bh / P.H, h = bh - b * P.H;
    const int64_t mrow = (int64_t)(P.num_masks == 1 ? 0 : b) * P.n + i;
    int64_t p0, p1;
    clamp_row(P, mrow, p0, p1);
    const T* vb = reinterpret_cast<const T*>(P.v) + b * P.v_sb + h * P.v_sh;
    const float* w = weights + unf_index(P, b, h, 0);
    float acc[C::VEC];
#pragma unroll
    for (int e = 0; e < C::VEC; ++e) acc[e] = 0.f;
    for (int64_t p = p0 + g; p < p1; p += C::G) {
        const int j = __ldg(P.col_idx + p);
        if ((unsigned)j >= (unsigned)P.n) continue;
        const float wp = w[p];
        float vf[C::VEC];
        Elem<T>::unpack(ldg16(vb + (int64_t)j * P.v_sn + c * C::VEC), vf);
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) acc[e] = fmaf(wp, vf[e], acc[e]);
    }
#pragma unroll
    for (int off = C::LPR; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
    if (lane < C::LPR) {
        T* orow = reinterpret_cast<T*>(P.out) + b * P.o_sb + h * P.o_sh + i * P.o_sn;
        *reinterpret_cast<uint4*>(orow + lane * C::VEC) = Elem<T>::pack(acc);
    }
}

template <typename T, int D>
cudaError_t launch_unfused_t(const FwdParams& p, float* scores, cudaStream_t s) {
    const int64_t blocks = (int64_t)p.B * p.H * ((p.n + 7) / 8);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    k_unf_sddmm<T, D><<<(unsigned)blocks, 256, 0, counted(s)>>>(p, scores);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_unf_softmax<<<(unsigned)blocks, 256, 0, counted(s)>>>(p, scores);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_unf_spmm<T, D><<<(unsigned)blocks, 256, 0, counted(s)>>>(p, scores);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ backward
// Gradients of L = sum(dout * out) (the chain rule of the forward's definition):
// with P_ij = exp(s_ij - lse_i) and D_i = <dout_i, out_i> = sum_j P_ij <dout_i, v_j>,
//   dS_ij = P_ij (<dout_i, v_j> - D_i),  dq_i = scale sum_j dS_ij k_j,
//   dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dout_i,  dbias_ij += dS_ij.
// Scores are recomputed in the base-2 domain as in the forward.

template <typename T, int D>
__device__ __forceinline__ void load_slice(const T* base, int c, float (&f)[Cfg<T, D>::VEC]) {
    Elem<T>::unpack(ldg16(base + c * Cfg<T, D>::VEC), f);
}

// Dot product of a lane's VEC slices, summed over the LPR lanes of its group.
template <typename T, int D>
__device__ __forceinline__ float group_dot(const float* a, const float* b) {
    using C = Cfg<T, D>;
    // even and odd elements in the two lanes of one packed FMA
    uint64_t a2 = f2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < C::VEC / 2; ++e) a2 = ffma2(f2(a[2 * e], a[2 * e + 1]), f2(b[2 * e], b[2 * e + 1]), a2);
    float ae, ao;
    split2(a2, ae, ao);
    float acc = ae + ao;
#pragma unroll
    for (int off = 1; off < C::LPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    return acc;
}

// y += a * x on N floats, two per packed FMA.
template <int N>
__device__ __forceinline__ void axpy2(float (&y)[N], float a, const float (&x)[N]) {
    const uint64_t a2 = f2(a, a);
#pragma unroll
    for (int e = 0; e < N / 2; ++e) split2(ffma2(a2, f2(x[2 * e], x[2 * e + 1]), f2(y[2 * e], y[2 * e + 1])), y[2 * e], y[2 * e + 1]);
}

template <typename T, int D>
__device__ __forceinline__ void store_slice(void* base, int64_t off, const float (&f)[Cfg<T, D>::VEC]) {
    *reinterpret_cast<uint4*>(reinterpret_cast<T*>(base) + off) = Elem<T>::pack(f);
}

// Sums a per-group VEC accumulator over the warp's groups (every lane ends with the sum).
template <int VEC, int LPR>
__device__ __forceinline__ void sum_groups(float (&acc)[VEC]) {
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
}

// Row pass for query row i of (b, h), one warp: dq_i, D_i and the score
// gradients -- added to dbias with atomics, or, with db_row, to that shared-memory
// row of n floats (indexed by key).
template <typename T, int D>
__device__ __forceinline__ void bwd_row(const BwdParams& P, int b, int h, int i, float* db_row) {
    using C = Cfg<T, D>;
    const int lane = threadIdx.x & 31;
    const int g = lane / C::LPR, c = lane % C::LPR;
    const int bh = b * P.H + h;
    const int64_t mrow = (int64_t)(P.num_masks == 1 ? 0 : b) * P.n + i;
    const int64_t wrow = (int64_t)bh * P.n + i;
    const T* kb = reinterpret_cast<const T*>(P.k) + b * P.k_sb + h * P.k_sh;
    const T* vb = reinterpret_cast<const T*>(P.v) + b * P.v_sb + h * P.v_sh;
    float qf[C::VEC], dof[C::VEC], of[C::VEC];
    load_slice<T, D>(reinterpret_cast<const T*>(P.q) + b * P.q_sb + h * P.q_sh + i * P.q_sn, c, qf);
    load_slice<T, D>(reinterpret_cast<const T*>(P.dout) + b * P.do_sb + h * P.do_sh + i * P.do_sn, c, dof);
    load_slice<T, D>(reinterpret_cast<const T*>(P.out) + b * P.o_sb + h * P.o_sh + i * P.o_sn, c, of);
    const float Di = group_dot<T, D>(dof, of);
#pragma unroll
    for (int e = 0; e < C::VEC; ++e) qf[e] *= P.qk_scale_log2;
    const float lse2 = P.lse[wrow] * kLog2e;
    const int64_t mask_base = b * P.mask.s0 + h * P.mask.s1 + i * P.mask.s2;
    const int64_t bias_base = b * P.bias.s0 + h * P.bias.s1 + i * P.bias.s2;
    const int64_t db_base = b * P.db_s0 + h * P.db_s1 + i * P.db_s2;
    float dq[C::VEC];
#pragma unroll
    for (int e = 0; e < C::VEC; ++e) dq[e] = 0.f;
    int64_t p0 = P.row_ptr[mrow], p1 = P.row_ptr[mrow + 1];
    p0 = p0 < 0 ? 0 : (p0 > P.nnz ? P.nnz : p0);
    p1 = p1 < p0 ? p0 : (p1 > P.nnz ? P.nnz : p1);
    if (lse2 == -INFINITY) p1 = p0;  // a degenerate row has no weights
    for (int64_t pb = p0; pb < p1; pb += C::STEP) {
        int col = -1;
        float extra = 0.f;
        if (lane < C::STEP && pb + lane < p1) {
            const int j = __ldg(P.col_idx + pb + lane);
            if ((unsigned)j < (unsigned)P.n) {
                col = j;
                if (P.has_extra) {
                    float ex = 0.f;
                    if (P.mask.data) ex += load_addend(P.mask, mask_base + j * P.mask.s3);
                    if (P.bias.data) ex += load_addend(P.bias, bias_base + j * P.bias.s3);
                    extra = ex * kLog2e;
                }
            } else {
                atomicOr(&g_error_flags, kErrBadColumn);
            }
        }
        constexpr int UB = 1;  // (more loads in flight cost registers, and occupancy, than they gain)
#pragma unroll
        for (int u0 = 0; u0 < C::U; u0 += UB) {
            int js[UB];
            float ess[UB];
            uint4 kr[UB], vr[UB];
#pragma unroll
            for (int t = 0; t < UB; ++t) {
                js[t] = __shfl_sync(0xffffffffu, col, (u0 + t) * C::G + g);
                ess[t] = __shfl_sync(0xffffffffu, extra, (u0 + t) * C::G + g);
                kr[t] = vr[t] = make_uint4(0u, 0u, 0u, 0u);
                if (js[t] >= 0) {
                    kr[t] = ldg16(kb + (int64_t)js[t] * P.k_sn + c * C::VEC);
                    vr[t] = ldg16(vb + (int64_t)js[t] * P.v_sn + c * C::VEC);
                }
            }
#pragma unroll
            for (int t = 0; t < UB; ++t) {
                const int j = js[t];
                float kf[C::VEC], vf[C::VEC];
                Elem<T>::unpack(kr[t], kf);
                Elem<T>::unpack(vr[t], vf);
                const float sc = group_dot<T, D>(qf, kf);
                const float dp = group_dot<T, D>(dof, vf);
                const float pw = j >= 0 ? ex2(sc + ess[t] - lse2) : 0.f;
                const float ds = pw * (dp - Di);
                axpy2(dq, ds, kf);
                if (P.dbias && j >= 0 && c == 0 && ds != 0.f) {
                    if (db_row)
                        db_row[j] += ds;  // one row per warp, one lane per key
                    else
                        atomicAdd(P.dbias + db_base + (int64_t)j * P.db_s3, ds);
                }
            }
        }
    }
    sum_groups<C::VEC, C::LPR>(dq);
    if (lane < C::LPR) {
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) dq[e] *= P.scale;
        store_slice<T, D>(P.dq, b * P.dq_sb + h * P.dq_sh + i * P.dq_sn + lane * C::VEC, dq);
    }
    if (lane == 0) P.D[wrow] = lse2 == -INFINITY ? 0.f : Di;
}

// Row pass: one warp per query row i of (b, h).
template <typename T, int D>
__global__ void __launch_bounds__(256) k_bwd_rows(const BwdParams P) {
    const int warp = threadIdx.x >> 5;
    const int per_bh = (P.n + 7) >> 3;
    const int bh = blockIdx.x / per_bh;
    const int i = (blockIdx.x - bh * per_bh) * 8 + warp;
    if (i >= P.n) return;
    bwd_row<T, D>(P, bh / P.H, bh - (bh / P.H) * P.H, i, nullptr);
}

// Row pass when the bias gradient is broadcast over the batch (a pair bias
// shared by every b): one warp per (h, i) walks every b and adds the score
// gradients up in a shared-memory row of n floats, then stores it -- one store
// per element instead of B contending atomics. kDbRowMax keys at most.
constexpr int kDbRowMax = 1536;

template <typename T, int D>
__global__ void __launch_bounds__(256) k_bwd_rows_dbb(const BwdParams P) {
    extern __shared__ float db_rows[];  // [8][n]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_h = (P.n + 7) >> 3;
    const int h = blockIdx.x / per_h;
    const int i = (blockIdx.x - h * per_h) * 8 + warp;
    float* row = db_rows + warp * P.n;
    for (int j = lane; j < P.n; j += 32) row[j] = 0.f;
    __syncwarp();
    if (i >= P.n) return;
    for (int b = 0; b < P.B; ++b) {
        bwd_row<T, D>(P, b, h, i, row);
        __syncwarp();
    }
    float* dst = P.dbias + h * P.db_s1 + (int64_t)i * P.db_s2;
    for (int j = lane; j < P.n; j += 32) dst[(int64_t)j * P.db_s3] = row[j];
}

// Column pass: one warp per key j of (b, h), over the rows i with j in S_i.
template <typename T, int D>
__global__ void __launch_bounds__(256, 3) k_bwd_cols(const BwdParams P) {
    using C = Cfg<T, D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane / C::LPR, c = lane % C::LPR;
    const int per_bh = (P.n + 7) >> 3;
    const int bh = blockIdx.x / per_bh;
    const int j = (blockIdx.x - bh * per_bh) * 8 + warp;
    if (j >= P.n) return;
    const int b = bh / P.H, h = bh - b * P.H;
    const int64_t mcol = (int64_t)(P.num_masks == 1 ? 0 : b) * P.n + j;
    const T* qb = reinterpret_cast<const T*>(P.q) + b * P.q_sb + h * P.q_sh;
    const T* dob = reinterpret_cast<const T*>(P.dout) + b * P.do_sb + h * P.do_sh;
    float kf[C::VEC], vf[C::VEC];
    load_slice<T, D>(reinterpret_cast<const T*>(P.k) + b * P.k_sb + h * P.k_sh + j * P.k_sn, c, kf);
    load_slice<T, D>(reinterpret_cast<const T*>(P.v) + b * P.v_sb + h * P.v_sh + j * P.v_sn, c, vf);
#pragma unroll
    for (int e = 0; e < C::VEC; ++e) kf[e] *= P.qk_scale_log2;
    float dk[C::VEC], dv[C::VEC];
#pragma unroll
    for (int e = 0; e < C::VEC; ++e) dk[e] = dv[e] = 0.f;
    const int64_t p0 = P.t_row_ptr[mcol], p1 = P.t_row_ptr[mcol + 1];
    for (int64_t pb = p0; pb < p1; pb += C::STEP) {
        int row = -1;
        float extra = 0.f, lse2 = -INFINITY, Di = 0.f;
        if (lane < C::STEP && pb + lane < p1) {
            const int i = __ldg(P.t_col_idx + pb + lane);
            row = i;
            const int64_t wrow = (int64_t)bh * P.n + i;
            lse2 = P.lse[wrow] * kLog2e;
            Di = P.D[wrow];
            if (P.has_extra) {
                float ex = 0.f;
                if (P.mask.data) ex += load_addend(P.mask, b * P.mask.s0 + h * P.mask.s1 + i * P.mask.s2 + j * P.mask.s3);
                if (P.bias.data) ex += load_addend(P.bias, b * P.bias.s0 + h * P.bias.s1 + i * P.bias.s2 + j * P.bias.s3);
                extra = ex * kLog2e;
            }
        }
#pragma unroll
        for (int u = 0; u < C::U; ++u) {
            const int i = __shfl_sync(0xffffffffu, row, u * C::G + g);
            const float es = __shfl_sync(0xffffffffu, extra, u * C::G + g);
            const float ls = __shfl_sync(0xffffffffu, lse2, u * C::G + g);
            const float di = __shfl_sync(0xffffffffu, Di, u * C::G + g);
            float qf[C::VEC], dof[C::VEC];
            if (i >= 0) {
                load_slice<T, D>(qb + (int64_t)i * P.q_sn, c, qf);
                load_slice<T, D>(dob + (int64_t)i * P.do_sn, c, dof);
            } else {
#pragma unroll
                for (int e = 0; e < C::VEC; ++e) qf[e] = dof[e] = 0.f;
            }
            const float sc = group_dot<T, D>(qf, kf);
            const float dp = group_dot<T, D>(dof, vf);
            const float pw = (i >= 0 && ls != -INFINITY) ? ex2(sc + es - ls) : 0.f;
            const float ds = pw * (dp - di);
            axpy2(dv, pw, dof);
            axpy2(dk, ds, qf);
        }
    }
    sum_groups<C::VEC, C::LPR>(dk);
    sum_groups<C::VEC, C::LPR>(dv);
    if (lane < C::LPR) {
#pragma unroll
        for (int e = 0; e < C::VEC; ++e) dk[e] *= P.scale;
        store_slice<T, D>(P.dk, b * P.dk_sb + h * P.dk_sh + j * P.dk_sn + lane * C::VEC, dk);
        store_slice<T, D>(P.dv, b * P.dv_sb + h * P.dv_sh + j * P.dv_sn + lane * C::VEC, dv);
    }
}

template <typename T, int D>
cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t s) {
    const int64_t blocks = (int64_t)p.B * p.H * ((p.n + 7) / 8);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // every (h, i) must own its dbias row for the batch-walking pass
    const bool own_rows = (p.db_s1 != 0 || p.H == 1) && (p.db_s2 != 0 || p.n == 1);
    if (p.dbias && p.db_s0 == 0 && p.B > 1 && own_rows && p.n <= kDbRowMax) {
        const int64_t hb = (int64_t)p.H * ((p.n + 7) / 8);
        const size_t smem = (size_t)8 * p.n * sizeof(float);
        if (smem > 48 * 1024) {
            cudaError_t a = cudaFuncSetAttribute(k_bwd_rows_dbb<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (a != cudaSuccess) return a;
        }
        k_bwd_rows_dbb<T, D><<<(unsigned)hb, 256, smem, counted(s)>>>(p);
    } else {
        k_bwd_rows<T, D><<<(unsigned)blocks, 256, 0, counted(s)>>>(p);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_bwd_cols<T, D><<<(unsigned)blocks, 256, 0, counted(s)>>>(p);
    return cudaGetLastError();
}

constexpr int kLongWarps = 8;

template <typename T, int D>
__global__ void __launch_bounds__(256) k_fwd_long(const FwdParams P) {
    using C = Cfg<T, D>;
    __shared__ float sm_m[kLongWarps], sm_l[kLongWarps];
    __shared__ float sm_acc[kLongWarps][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t count = P.long_count_host >= 0 ? P.long_count_host : (int64_t)*P.long_count_dev;
    const int64_t per_row = P.num_masks == 1 ? (int64_t)P.B * P.H : (int64_t)P.H;
    const int64_t items = count * per_row;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int64_t slot = it % count, rep = it / count;
        const int mrow = P.long_rows[slot];
        const int i = mrow % P.n;
        int b, h;
        if (P.num_masks == 1) {
            b = (int)(rep / P.H);
            h = (int)(rep - (int64_t)b * P.H);
        } else {
            b = mrow / P.n;
            h = (int)rep;
        }
        int64_t p0, p1;
        clamp_row(P, mrow, p0, p1);

        RowCtx<T, D> rc;
        State<C::VEC> st;
        init_row<T, D>(P, b, h, i, lane, rc, st);
        row_steps<T, D>(P, rc, p0 + (int64_t)warp * C::STEP, p1, (int64_t)kLongWarps * C::STEP,
                        lane, st);
        merge_groups<C::VEC, C::LPR>(st);
        if (lane == 0) {
            sm_m[warp] = st.m;
            sm_l[warp] = st.l;
        }
        if (lane < C::LPR) {
#pragma unroll
            for (int e = 0; e < C::VEC; ++e) sm_acc[warp][lane * C::VEC + e] = st.acc[e];
        }
        __syncthreads();
        if (threadIdx.x < D) {
            float mx = -INFINITY;
#pragma unroll
            for (int w = 0; w < kLongWarps; ++w) mx = fmaxf(mx, sm_m[w]);
            const float mu = (mx == -INFINITY) ? 0.f : mx;
            float l = 0.f, a = 0.f;
#pragma unroll
            for (int w = 0; w < kLongWarps; ++w) {
                const float f = ex2(sm_m[w] - mu);
                l = fmaf(sm_l[w], f, l);
                a = fmaf(sm_acc[w][threadIdx.x], f, a);
            }
            bool partial = false;
            if (P.qb_tile_off) {
                const int64_t blk = (int64_t)(P.num_masks == 1 ? 0 : b) * P.nqb + (i >> 7);
                partial = P.qb_tile_off[blk + 1] > P.qb_tile_off[blk];
            }
            const int64_t wrow = ((int64_t)b * P.H + h) * P.n + i;
            if (partial) {
                P.ws_acc[wrow * D + threadIdx.x] = a;
                if (threadIdx.x == 0) {
                    P.ws_ml[wrow * 2] = mx;
                    P.ws_ml[wrow * 2 + 1] = l;
                }
            } else {
                T* orow = reinterpret_cast<T*>(P.out) + b * P.o_sb + h * P.o_sh + i * P.o_sn;
                Elem<T>::store1(orow, threadIdx.x, l > 0.f ? a / l : 0.f);
                if (threadIdx.x == 0 && P.lse)
                    P.lse[wrow] = l > 0.f ? (mx + lg2(l)) * kLn2 : -INFINITY;
            }
        }
        __syncthreads();
    }
}

__global__ void k_classify_long(const int32_t* __restrict__ row_ptr, int64_t rows, int64_t nnz,
                                int32_t* __restrict__ list, int32_t* __restrict__ count) {
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows;
         r += (int64_t)gridDim.x * blockDim.x) {
        int64_t p0 = row_ptr[r], p1 = row_ptr[r + 1];
        p0 = p0 < 0 ? 0 : (p0 > nnz ? nnz : p0);
        p1 = p1 < p0 ? p0 : (p1 > nnz ? nnz : p1);
        if (p1 - p0 > kLongRowThreshold) list[atomicAdd(count, 1)] = (int32_t)r;
    }
}

template <typename T, int D>
cudaError_t launch_short_t(const FwdParams& p, cudaStream_t s) {
    const int64_t blocks = (int64_t)p.B * p.H * ((p.n + 7) / 8);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    k_fwd_short<T, D><<<(unsigned)blocks, 256, 0, counted(s)>>>(p);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_itv_t(const FwdParams& p, cudaStream_t s) {
    if (p.itv_slices < 1 || p.itv_slices > 16 || (p.itv_slices & (p.itv_slices - 1)))
        return cudaErrorInvalidValue;
    const int64_t blocks = (int64_t)p.B * p.H * p.nqb * p.itv_slices;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    k_fwd_itv<T, D><<<(unsigned)blocks, 256, 0, counted(s)>>>(p);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_long_t(const FwdParams& p, int num_sms, cudaStream_t s) {
    int64_t grid = (int64_t)num_sms * 4;
    if (p.long_count_host >= 0) {
        const int64_t items =
            p.long_count_host * (p.num_masks == 1 ? (int64_t)p.B * p.H : (int64_t)p.H);
        if (items == 0) return cudaSuccess;
        if (items < grid) grid = items;
    }
    k_fwd_long<T, D><<<(unsigned)grid, 256, 0, counted(s)>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_short_rows(const FwdParams& p, int dtype, int d, cudaStream_t s) {
    if (dtype == 0) {
        switch (d) {
        case 32: return launch_short_t<__nv_bfloat16, 32>(p, s);
        case 64: return launch_short_t<__nv_bfloat16, 64>(p, s);
        case 128: return launch_short_t<__nv_bfloat16, 128>(p, s);
        }
    } else {
        switch (d) {
        case 32: return launch_short_t<float, 32>(p, s);
        case 64: return launch_short_t<float, 64>(p, s);
        case 128: return launch_short_t<float, 128>(p, s);
        }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_unfused(const FwdParams& p, int dtype, int d, float* scores, cudaStream_t s) {
    if (dtype == 0) {
        switch (d) {
        case 32: return launch_unfused_t<__nv_bfloat16, 32>(p, scores, s);
        case 64: return launch_unfused_t<__nv_bfloat16, 64>(p, scores, s);
        case 128: return launch_unfused_t<__nv_bfloat16, 128>(p, scores, s);
        }
    } else {
        switch (d) {
        case 32: return launch_unfused_t<float, 32>(p, scores, s);
        case 64: return launch_unfused_t<float, 64>(p, scores, s);
        case 128: return launch_unfused_t<float, 128>(p, scores, s);
        }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_bwd(const BwdParams& p, int dtype, int d, cudaStream_t s) {
    if (dtype == 0) {
        switch (d) {
        case 32: return launch_bwd_t<__nv_bfloat16, 32>(p, s);
        case 64: return launch_bwd_t<__nv_bfloat16, 64>(p, s);
        case 128: return launch_bwd_t<__nv_bfloat16, 128>(p, s);
        }
    } else {
        switch (d) {
        case 32: return launch_bwd_t<float, 32>(p, s);
        case 64: return launch_bwd_t<float, 64>(p, s);
        case 128: return launch_bwd_t<float, 128>(p, s);
        }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_itv(const FwdParams& p, int dtype, int d, cudaStream_t s) {
    if (dtype == 0) {
        switch (d) {
        case 32: return launch_itv_t<__nv_bfloat16, 32>(p, s);
        case 64: return launch_itv_t<__nv_bfloat16, 64>(p, s);
        case 128: return launch_itv_t<__nv_bfloat16, 128>(p, s);
        }
    } else {
        switch (d) {
        case 32: return launch_itv_t<float, 32>(p, s);
        case 64: return launch_itv_t<float, 64>(p, s);
        case 128: return launch_itv_t<float, 128>(p, s);
        }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_long_rows(const FwdParams& p, int dtype, int d, int num_sms,
                                 cudaStream_t s) {
    if (dtype == 0) {
        switch (d) {
        case 32: return launch_long_t<__nv_bfloat16, 32>(p, num_sms, s);
        case 64: return launch_long_t<__nv_bfloat16, 64>(p, num_sms, s);
        case 128: return launch_long_t<__nv_bfloat16, 128>(p, num_sms, s);
        }
    } else {
        switch (d) {
        case 32: return launch_long_t<float, 32>(p, num_sms, s);
        case 64: return launch_long_t<float, 64>(p, num_sms, s);
        case 128: return launch_long_t<float, 128>(p, num_sms, s);
        }
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_classify_long_rows(const int32_t* row_ptr, int64_t rows, int64_t nnz,
                                      int32_t* list, int32_t* count, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    int64_t grid = (rows + 255) / 256;
    if (grid > 4096) grid = 4096;
    k_classify_long<<<(unsigned)grid, 256, 0, counted(s)>>>(row_ptr, rows, nnz, list, count);
    return cudaGetLastError();
}

cudaError_t error_flag_address(unsigned** p) {
    return cudaGetSymbolAddress(reinterpret_cast<void**>(p), g_error_flags);
}

cudaError_t read_and_clear_device_error(unsigned* flags, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    unsigned v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_error_flags, sizeof v);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_error_flags, &zero, sizeof zero);
    if (flags) *flags = v;
    return e;
}

}  // namespace spattn
