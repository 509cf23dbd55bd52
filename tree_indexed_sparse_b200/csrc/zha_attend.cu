// zha_attend.cu -- exact attention over the routed token set, and the dense
// flash-decode comparison kernel (sm_100a).
//
// Attention ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢":
// the first token is always kept as the attention sink; rit.work article,
// section "Дерево сокращает сам поиск нужных ключей": the main attention reads
// the raw keys of the found leaves):
//   o_h = sum_{i in T_h} softmax_i(q_h.k_i / sqrt(d)) v_i,
//   T_h = tokens of the leaf chunks head h kept  U  {0},  fp32 accumulation.
//
// Split-K flash decode.  The union leaf list of each KV head (every leaf kept
// by any of its G query heads, with the head bitmask) is flattened into token
// blocks; the grid's CTAs take contiguous ranges of blocks over all KV heads
// and each warp streams a contiguous sub-range.  Every K and V row is read
// from HBM once and serves all G heads of its group (GQA sharing): each lane
// loads one 16-byte slice of a row, the G partial dot products are
// reduce-scattered over the lanes of the row, and an online softmax keeps
// (max, sum, output) per head.  Per-CTA partials are merged by the last CTA
// of each KV head (fence + ticket), which also adds the sink token.
// The dense kernel is the same warp loop over all rows 0 .. N-1.
#include <algorithm>

#include "zha_device.cuh"
#include "zha_internal.cuh"

namespace zha {

constexpr float LOG2E = 1.4426950408889634f;

template <typename KT, int HD, int G>
struct AttnCfg {
    static constexpr int ES = (int)sizeof(KT);
    static constexpr int LPR = HD * ES / 16;   // lanes per row
    static constexpr int RPL = 32 / LPR;       // rows per warp-wide load
    static constexpr int EPL = 16 / ES;        // elements per lane per row
    static constexpr int RPB = LPR / G;        // rows per lane per block
    static constexpr int TB = RPB * RPL;       // tokens per block
    static_assert(LPR >= G && LPR % G == 0, "row slices must cover the heads");
};

// Online-softmax state of one warp for the G heads of one KV head.
template <typename KT, int HD, int G>
struct WarpAttn {
    using C = AttnCfg<KT, HD, G>;
    float m[G];          // running max (log2 domain), replicated over lanes
    float l;             // partial denominator of this lane's head (lane % G)
    float o[G][C::EPL];  // partial outputs of this lane's column slice

    __device__ void init() {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY;
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) o[h][e] = 0.f;
        }
        l = 0.f;
    }

    // One block of C::TB tokens.  rowinfo(t, row, ok, msk) maps a block token
    // index t in [0, TB) to a cache row.
    template <typename RowFn>
    __device__ void block(const KT *__restrict__ Kh, const KT *__restrict__ Vh, const float (&qs)[G][C::EPL],
                          RowFn rowinfo, float *pw, int lane) {
        const int grp = lane / C::LPR, col = (lane % C::LPR) * C::EPL;
        float k[C::RPB][C::EPL], vv[C::RPB][C::EPL];
        bool okr[C::RPB];
        uint32_t mr[C::RPB];
#pragma unroll
        for (int r = 0; r < C::RPB; ++r) {
            int64_t row;
            rowinfo(r * C::RPL + grp, row, okr[r], mr[r]);
            if (okr[r]) {
                VecStream<KT, C::EPL>::load(Kh + row * HD + col, k[r]);
                VecStream<KT, C::EPL>::load(Vh + row * HD + col, vv[r]);
            } else {
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) { k[r][e] = 0.f; vv[r][e] = 0.f; }
            }
        }
        float v[C::RPB * G];
#pragma unroll
        for (int r = 0; r < C::RPB; ++r)
#pragma unroll
            for (int h = 0; h < G; ++h) v[r * G + h] = lane_dot<C::EPL>(qs[h], k[r]);
        reduce_scatter<C::RPB * G, C::LPR>(v, lane);
        const int my = lane % C::LPR;
        const int my_r = my / G, my_h = my % G;
        // eligibility of this lane's (row, head)
        bool ok_me = false;
        uint32_t m_me = 0;
#pragma unroll
        for (int r = 0; r < C::RPB; ++r)
            if (r == my_r) { ok_me = okr[r]; m_me = mr[r]; }
        float s = (ok_me && ((m_me >> my_h) & 1u)) ? v[0] : -INFINITY;
        float bmax = s;
#pragma unroll
        for (int off = G; off < 32; off <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(FULL, bmax, off));
        float alpha[G];
        float mnew_me = 0.f, alpha_me = 1.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float mn = fmaxf(m[h], __shfl_sync(FULL, bmax, h));
            alpha[h] = (mn == -INFINITY) ? 1.f : exp2f(m[h] - mn);
            m[h] = mn;
            if (h == my_h) { mnew_me = mn; alpha_me = alpha[h]; }
        }
        const float pr = (s == -INFINITY) ? 0.f : exp2f(s - mnew_me);
        l = l * alpha_me + pr;
        pw[lane] = pr;
        __syncwarp();
        float pp[C::RPB * G];
#pragma unroll
        for (int i = 0; i < C::RPB * G; ++i) pp[i] = pw[grp * C::LPR + i];
        __syncwarp();
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) {
                float acc = o[h][e] * alpha[h];
#pragma unroll
                for (int r = 0; r < C::RPB; ++r) acc = fmaf(pp[r * G + h], vv[r][e], acc);
                o[h][e] = acc;
            }
        }
    }

    // Fold the row groups and lanes; afterwards lanes [0, LPR) hold o for the
    // columns [lane*EPL, ...) and every lane holds lsum[h].
    __device__ void finish(float (&lsum)[G], int lane) {
#pragma unroll
        for (int off = C::LPR; off < 32; off <<= 1)
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) o[h][e] += __shfl_xor_sync(FULL, o[h][e], off);
        float lt = l;
#pragma unroll
        for (int off = G; off < 32; off <<= 1) lt += __shfl_xor_sync(FULL, lt, off);
#pragma unroll
        for (int h = 0; h < G; ++h) lsum[h] = __shfl_sync(FULL, lt, h);
    }
};

// Shared memory of the CTA-level merge: per warp, G x (HD + 2) floats, plus
// the per-warp probability exchange.
template <int HD, int G>
struct AttnSmem {
    static constexpr int NW = ATTN_THREADS / 32;
    static constexpr int PER_WARP = G * (HD + 2);
    static constexpr size_t bytes = (size_t)NW * PER_WARP * 4 + NW * 32 * 4 + 256;
};

// Write a warp's state into the CTA merge area.
template <typename KT, int HD, int G>
__device__ void stash_warp(WarpAttn<KT, HD, G> &st, float *wsm, int lane) {
    using C = AttnCfg<KT, HD, G>;
    float lsum[G];
    st.finish(lsum, lane);
    if (lane < C::LPR) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) wsm[h * (HD + 2) + lane * C::EPL + e] = st.o[h][e];
    }
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            wsm[h * (HD + 2) + HD] = st.m[h];
            wsm[h * (HD + 2) + HD + 1] = lsum[h];
        }
    }
}

// Merge the CTA's warps (fixed order) into one partial per head.
template <int HD, int G>
__device__ void merge_warps(const float *sm, float *dst /* [G][HD+2] */) {
    constexpr int NW = ATTN_THREADS / 32;
    for (int idx = threadIdx.x; idx < G * (HD + 2); idx += blockDim.x) {
        const int h = idx / (HD + 2), e = idx % (HD + 2);
        float M = -INFINITY;
        for (int w = 0; w < NW; ++w) M = fmaxf(M, sm[w * G * (HD + 2) + h * (HD + 2) + HD]);
        float r;
        if (e == HD) {
            r = M;
        } else if (M == -INFINITY) {
            r = 0.f;
        } else {
            r = 0.f;
            for (int w = 0; w < NW; ++w) {
                const float mw = sm[w * G * (HD + 2) + h * (HD + 2) + HD];
                if (mw == -INFINITY) continue;
                r = fmaf(sm[w * G * (HD + 2) + h * (HD + 2) + e], exp2f(mw - M), r);
            }
        }
        dst[idx] = r;
    }
}

// Combine the partials of CTAs [b0, b1) for the G heads of KV head kh (one
// warp per head), add the sink token when asked, and write the outputs.
template <typename KT, int HD, int G>
__device__ void combine_kvh(const Decode &a, int kh, int b0, int b1, const float (&qs)[G][HD / 32], bool gather) {
    constexpr int CPL = HD / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp >= G) return;
    const int h = warp;
    const int hq = kh * G + h;
    float M = -INFINITY, L = 0.f, O[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) O[e] = 0.f;
    auto merge = [&](float mb, float lb, const float (&ob)[CPL]) {
        if (mb == -INFINITY) return;
        const float mn = fmaxf(M, mb);
        const float a1 = (M == -INFINITY) ? 0.f : exp2f(M - mn);
        const float a2 = exp2f(mb - mn);
        L = L * a1 + lb * a2;
#pragma unroll
        for (int e = 0; e < CPL; ++e) O[e] = O[e] * a1 + ob[e] * a2;
        M = mn;
    };
    for (int b = b0; b < b1; ++b) {
        const float *pb = a.part + (((int64_t)b * a.t.h_kv + kh) * G + h) * (HD + 2);
        const float mb = __ldcg(pb + HD);
        if (mb == -INFINITY) continue;
        const float lb = __ldcg(pb + HD + 1);
        float ob[CPL];
#pragma unroll
        for (int e = 0; e < CPL; ++e) ob[e] = __ldcg(pb + lane * CPL + e);
        merge(mb, lb, ob);
    }
    if (gather) {
        // sink token 0 unless leaf 0 is already in this head's set
        const int64_t kbase = (int64_t)kh * a.t.node_cap[0];
        const int32_t first = __ldcg(a.kept_ids[0] + kbase);
        const uint32_t fm = __ldcg(a.kept_mask[0] + kbase);
        const bool has0 = (__ldcg(a.kept_cnt + kh) > 0) && first == 0 && ((fm >> h) & 1u);
        if (!has0) {
            const KT *Kh = reinterpret_cast<const KT *>(a.t.K) + (int64_t)kh * a.t.kv_cap * HD;
            const KT *Vh = reinterpret_cast<const KT *>(a.t.V) + (int64_t)kh * a.t.kv_cap * HD;
            float k0[CPL], v0[CPL];
#pragma unroll
            for (int e = 0; e < CPL; ++e) {
                if constexpr (sizeof(KT) == 2) {
                    k0[e] = __uint_as_float(((uint32_t)Kh[lane * CPL + e]) << 16);
                    v0[e] = __uint_as_float(((uint32_t)Vh[lane * CPL + e]) << 16);
                } else {
                    k0[e] = Kh[lane * CPL + e];
                    v0[e] = Vh[lane * CPL + e];
                }
            }
            const float s0 = warp_sum(lane_dot<CPL>(qs[h], k0));
            merge(s0, 1.f, v0);
        }
    }
    const float inv = 1.f / L;
    float *dst = a.out + (int64_t)hq * HD + lane * CPL;
#pragma unroll
    for (int e = 0; e < CPL; ++e) dst[e] = O[e] * inv;
}

template <typename KT, int HD, int G>
__global__ void __launch_bounds__(ATTN_THREADS) k_attend(Decode a) {
    using C = AttnCfg<KT, HD, G>;
    extern __shared__ __align__(16) float asm_[];
    constexpr int NW = ATTN_THREADS / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h_kv = a.t.h_kv, c = a.t.c;
    float *wsm = asm_;
    float *pw = asm_ + NW * G * (HD + 2) + warp * 32;
    __shared__ int64_t s_pref[65];
    __shared__ int s_last[64];
    // unit (token block) counts per KV head and their prefix
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int kh = 0; kh < h_kv; ++kh) {
            s_pref[kh] = acc;
            const int64_t ntok = (int64_t)__ldcg(a.kept_cnt + kh) * c;
            acc += (ntok + C::TB - 1) / C::TB;
        }
        s_pref[h_kv] = acc;
    }
    __syncthreads();
    const int64_t U = s_pref[h_kv];
    const int nb = gridDim.x, b = blockIdx.x;
    const int64_t u0 = U * b / nb, u1 = U * (b + 1) / nb;
    for (int kh = 0; kh < h_kv; ++kh) {
        const int64_t p0 = s_pref[kh], p1 = s_pref[kh + 1];
        const int64_t lo = max(u0, p0), hi = min(u1, p1);
        float *dst = a.part + ((int64_t)b * h_kv + kh) * G * (HD + 2);
        if (lo >= hi) {
            for (int h = threadIdx.x; h < G; h += blockDim.x) dst[h * (HD + 2) + HD] = -INFINITY;
            continue;
        }
        // this CTA's segment of kh: local units [lo - p0, hi - p0)
        const int64_t ls = lo - p0, le = hi - p0, len = le - ls;
        const int64_t w0 = ls + len * warp / NW, w1 = ls + len * (warp + 1) / NW;
        float qs[G][C::EPL];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float *qh = a.q + (int64_t)(kh * G + h) * HD + (lane % C::LPR) * C::EPL;
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) qs[h][e] = qh[e] * (a.t.scale * LOG2E);
        }
        const KT *Kh = reinterpret_cast<const KT *>(a.t.K) + (int64_t)kh * a.t.kv_cap * HD;
        const KT *Vh = reinterpret_cast<const KT *>(a.t.V) + (int64_t)kh * a.t.kv_cap * HD;
        const int64_t kbase = (int64_t)kh * a.t.node_cap[0];
        const int64_t L = __ldcg(a.kept_cnt + kh);
        const int64_t N = a.t.n_tokens;
        const int clog = a.t.c_log2;
        WarpAttn<KT, HD, G> st;
        st.init();
        for (int64_t u = w0; u < w1; ++u) {
            const int64_t tb0 = u * C::TB;
            auto rowinfo = [&](int t, int64_t &row, bool &ok, uint32_t &msk) {
                const int64_t tok = tb0 + t;
                const int64_t k = clog >= 0 ? (tok >> clog) : tok / c;
                if (k >= L) { ok = false; row = 0; msk = 0; return; }
                const int64_t o = tok - k * c;
                row = (int64_t)__ldcg(a.kept_ids[0] + kbase + k) * c + o;
                ok = row < N;
                msk = ok ? (uint32_t)__ldcg(a.kept_mask[0] + kbase + k) : 0u;
            };
            st.block(Kh, Vh, qs, rowinfo, pw, lane);
        }
        stash_warp<KT, HD, G>(st, wsm + warp * G * (HD + 2), lane);
        __syncthreads();
        merge_warps<HD, G>(wsm, dst);
        __syncthreads();
    }
    // tickets: the last CTA touching a KV head combines it
    __threadfence();
    __syncthreads();
    if (threadIdx.x < h_kv) {
        const int kh = threadIdx.x;
        const int64_t p0 = s_pref[kh], p1 = s_pref[kh + 1];
        // CTA bb covers units [U*bb/nb, U*(bb+1)/nb); unit u lies in CTA
        // ((u+1)*nb - 1) / U.  Every CTA in [bf, bl] takes a ticket.
        int bf = 0, bl = -1;
        if (p1 > p0) {
            bf = (int)(((p0 + 1) * nb - 1) / U);
            bl = (int)((p1 * nb - 1) / U);
        }
        int last = 0;
        if (bl >= 0 && b >= bf && b <= bl) {
            const unsigned expected = (unsigned)(bl - bf + 1);
            const unsigned tk = atomicAdd(a.done + MAXD * h_kv + kh, 1u);
            last = (tk == expected - 1);
            if (last) a.done[MAXD * h_kv + kh] = 0u;
        }
        s_last[kh] = last ? (bf | (bl << 16)) + 1 : 0;
    }
    __syncthreads();
    for (int kh = 0; kh < h_kv; ++kh) {
        if (!s_last[kh]) continue;
        __threadfence();
        const int code = s_last[kh] - 1;
        const int bf = code & 0xffff, bl = code >> 16;
        float qs[G][HD / 32];
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < HD / 32; ++e) qs[h][e] = a.q[(int64_t)(kh * G + h) * HD + lane * (HD / 32) + e] * (a.t.scale * LOG2E);
        combine_kvh<KT, HD, G>(a, kh, bf, bl + 1, qs, true);
        __syncthreads();
    }
}

// Dense flash decode: CTA b serves KV head b % h_kv over its share of all rows.
template <typename KT, int HD, int G>
__global__ void __launch_bounds__(ATTN_THREADS) k_dense(Decode a) {
    using C = AttnCfg<KT, HD, G>;
    extern __shared__ __align__(16) float asm_[];
    constexpr int NW = ATTN_THREADS / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h_kv = a.t.h_kv;
    const int kh = blockIdx.x % h_kv, bi = blockIdx.x / h_kv, nbk = gridDim.x / h_kv;
    float *wsm = asm_;
    float *pw = asm_ + NW * G * (HD + 2) + warp * 32;
    __shared__ int s_last;
    const int64_t N = a.t.n_tokens;
    const int64_t U = (N + C::TB - 1) / C::TB;
    const int64_t u0 = U * bi / nbk, u1 = U * (bi + 1) / nbk, len = u1 - u0;
    const int64_t w0 = u0 + len * warp / NW, w1 = u0 + len * (warp + 1) / NW;
    float qs[G][C::EPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float *qh = a.q + (int64_t)(kh * G + h) * HD + (lane % C::LPR) * C::EPL;
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) qs[h][e] = qh[e] * (a.t.scale * LOG2E);
    }
    const KT *Kh = reinterpret_cast<const KT *>(a.t.K) + (int64_t)kh * a.t.kv_cap * HD;
    const KT *Vh = reinterpret_cast<const KT *>(a.t.V) + (int64_t)kh * a.t.kv_cap * HD;
    WarpAttn<KT, HD, G> st;
    st.init();
    for (int64_t u = w0; u < w1; ++u) {
        const int64_t tb0 = u * C::TB;
        auto rowinfo = [&](int t, int64_t &row, bool &ok, uint32_t &msk) {
            row = tb0 + t;
            ok = row < N;
            msk = 0xffffffffu;
        };
        st.block(Kh, Vh, qs, rowinfo, pw, lane);
    }
    stash_warp<KT, HD, G>(st, wsm + warp * G * (HD + 2), lane);
    __syncthreads();
    merge_warps<HD, G>(wsm, a.part + ((int64_t)bi * h_kv + kh) * G * (HD + 2));
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned tk = atomicAdd(a.done + MAXD * h_kv + h_kv + kh, 1u);
        s_last = (tk == (unsigned)(nbk - 1));
        if (s_last) a.done[MAXD * h_kv + h_kv + kh] = 0u;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float q2[G][HD / 32];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < HD / 32; ++e) q2[h][e] = a.q[(int64_t)(kh * G + h) * HD + lane * (HD / 32) + e] * (a.t.scale * LOG2E);
    combine_kvh<KT, HD, G>(a, kh, 0, nbk, q2, false);
}

// ---- dispatch ----------------------------------------------------------------

template <typename KT, int HD, int G>
static cudaError_t attend_impl(const Decode &dc, int n_cta, cudaStream_t s, bool dense) {
    const size_t smem = AttnSmem<HD, G>::bytes;
    if (dense) {
        cudaError_t err = cudaFuncSetAttribute(k_dense<KT, HD, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        k_dense<KT, HD, G><<<n_cta, ATTN_THREADS, smem, s>>>(dc);
    } else {
        cudaError_t err = cudaFuncSetAttribute(k_attend<KT, HD, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        k_attend<KT, HD, G><<<n_cta, ATTN_THREADS, smem, s>>>(dc);
    }
    return cudaGetLastError();
}

static cudaError_t attend_dispatch(const Decode &dc, int n_cta, cudaStream_t s, bool dense) {
    const Tree &t = dc.t;
    if (t.kv_dtype == 1) {
        if (t.d == 128 && t.G == 4) return attend_impl<uint16_t, 128, 4>(dc, n_cta, s, dense);
        if (t.d == 128 && t.G == 1) return attend_impl<uint16_t, 128, 1>(dc, n_cta, s, dense);
        if (t.d == 64 && t.G == 4) return attend_impl<uint16_t, 64, 4>(dc, n_cta, s, dense);
        if (t.d == 64 && t.G == 1) return attend_impl<uint16_t, 64, 1>(dc, n_cta, s, dense);
    } else {
        if (t.d == 128 && t.G == 4) return attend_impl<float, 128, 4>(dc, n_cta, s, dense);
        if (t.d == 128 && t.G == 1) return attend_impl<float, 128, 1>(dc, n_cta, s, dense);
        if (t.d == 64 && t.G == 4) return attend_impl<float, 64, 4>(dc, n_cta, s, dense);
        if (t.d == 64 && t.G == 1) return attend_impl<float, 64, 1>(dc, n_cta, s, dense);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attend(const Decode &dc, int n_cta, cudaStream_t s) { return attend_dispatch(dc, n_cta, s, false); }
cudaError_t launch_dense(const Decode &dc, int n_cta, cudaStream_t s) { return attend_dispatch(dc, n_cta, s, true); }

bool compiled_combo(int kv_dtype, int d, int R, int G) {
    (void)kv_dtype;
    return (d == 64 || d == 128) && (R == 1 || R == 16) && (G == 1 || G == 4);
}

}  // namespace zha
