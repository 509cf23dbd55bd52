// zha_attend.cuh -- exact attention over a token set, split over the CTAs of a
// grid with a warp-specialised bulk-copy pipeline (sm_100a).
//
// Attention ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢":
// the first token is always kept as the attention sink; rit.work article,
// section "Дерево сокращает сам поиск нужных ключей": the main attention reads
// the raw keys of the found leaves):
//   o_h = sum_{i in T_h} softmax_i(q_h.k_i / sqrt(d)) v_i,
//   T_h = tokens of the leaf chunks head h kept  U  {0},  fp32 accumulation.
//
// The union leaf list of each KV head (every leaf kept by any of its G query
// heads, with the head bitmask) is flattened into stages of TT tokens; the
// grid's CTAs take contiguous ranges of stages over all KV heads.  In each CTA
// one producer warp (warp 8) turns a stage into runs of contiguous K/V rows,
// writes the per-token head masks, and issues one cp.async.bulk per run into
// a ring of shared-memory stages guarded by mbarriers; warps 0-7 take TT/8
// tokens each per stage.  Every K and V row crosses HBM once and serves all G
// heads of its group (GQA sharing).  Each CTA leaves one partial (max, sum,
// output) per head per KV head it touched; combine_kvh merges them.
#pragma once

#include <algorithm>

#include "zha_device.cuh"
#include "zha_internal.cuh"
#include "zha_tma.cuh"

namespace zha {

constexpr float LOG2E = 1.4426950408889634f;
constexpr int ACW = 8;                         // consumer warps
constexpr int A_THREADS = (ACW + 1) * 32;      // + one producer warp
constexpr int TT = 64;                         // tokens per stage
constexpr int TW = TT / ACW;                   // tokens per consumer warp per stage
constexpr int LEAF_WIN = 2048;                 // leaf ids the producer keeps in shared memory

// One partial record: o[HD], max, sum, two pads (16-byte aligned records).
template <int HD>
constexpr int prec() { return HD + 4; }

template <typename KT, int HD, int G>
struct AttnCfg {
    static constexpr int ES = (int)sizeof(KT);
    static constexpr int RB = HD * ES;            // row bytes
    static constexpr int LPR = RB / 16;           // lanes per row (16-byte slices)
    static constexpr int RPL = 32 / LPR;          // rows per warp-wide access
    static constexpr int EPL = 16 / ES;           // elements per lane per row
    static constexpr int RPB = TW / RPL;          // rows per lane per stage
    static constexpr int NV = RPB * G;            // partial dots per lane
    static constexpr int NVP = NV > LPR ? NV : LPR;  // padded to the reduce width
    static constexpr int STAGE_BYTES = 2 * TT * RB;
    static constexpr int STAGES = (128 * 1024) / STAGE_BYTES > 4 ? 4 : (128 * 1024) / STAGE_BYTES;
    static_assert(LPR >= 1 && LPR <= 32 && RPB >= 1, "row layout");
    static_assert(LPR % G == 0, "row slices must cover the heads");
};

template <typename KT, int HD, int G>
struct ASmem {
    using C = AttnCfg<KT, HD, G>;
    static constexpr size_t off_meta = (size_t)C::STAGES * C::STAGE_BYTES;
    static constexpr size_t off_bar = off_meta + C::STAGES * TT;            // full[ST], empty[ST]
    static constexpr size_t off_abort = off_bar + 2 * C::STAGES * 8;
    static constexpr size_t off_merge = (off_abort + 16 + 15) / 16 * 16;
    static constexpr size_t off_pw = off_merge + (size_t)ACW * G * (HD + 2) * 4;
    static constexpr size_t off_win = off_pw + ACW * 32 * 4;               // producer's leaf-id window
    static constexpr size_t bytes = off_win + (size_t)LEAF_WIN * 5;
};

// Online-softmax state of one consumer warp for the G heads of one KV head.
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

    // The warp's TW tokens of one stage: K rows sK[t], V rows sV[t], head
    // masks msk[t] (0 = not a token of any head) for t in [0, TW).
    __device__ void tokens(const KT *sK, const KT *sV, const uint8_t *msk, const float (&qs)[G][C::EPL],
                           float *pw, int lane) {
        const int grp = lane / C::LPR, col = (lane % C::LPR) * C::EPL;
        float v[C::NVP];
        uint32_t mr[C::RPB];
#pragma unroll
        for (int r = 0; r < C::RPB; ++r) {
            const int t = r * C::RPL + grp;
            mr[r] = msk[t];
            float k[C::EPL];
            Vec<KT, C::EPL>::load(sK + t * HD + col, k);
#pragma unroll
            for (int h = 0; h < G; ++h) v[r * G + h] = mr[r] ? lane_dot<C::EPL>(qs[h], k) : 0.f;
        }
#pragma unroll
        for (int i = C::NV; i < C::NVP; ++i) v[i] = 0.f;
        reduce_scatter<C::NVP, C::LPR>(v, lane);
        const int my = lane % C::LPR;
        const int my_r = my / G, my_h = my % G;
        uint32_t m_me = 0;
#pragma unroll
        for (int r = 0; r < C::RPB; ++r)
            if (r == my_r) m_me = mr[r];
        const float s = ((m_me >> my_h) & 1u) ? v[0] : -INFINITY;
        float bmax = s;
#pragma unroll
        for (int off = G; off < 32; off <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(FULL, bmax, off));
        float alpha[G];
        float mnew_me = 0.f, alpha_me = 1.f;
        bool rescale = false;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float mn = fmaxf(m[h], __shfl_sync(FULL, bmax, h));
            alpha[h] = (mn == -INFINITY) ? 1.f : exp2f(m[h] - mn);
            rescale |= (mn != m[h]);
            m[h] = mn;
            if (h == my_h) { mnew_me = mn; alpha_me = alpha[h]; }
        }
        const float pr = (s == -INFINITY) ? 0.f : exp2f(s - mnew_me);
        l = l * alpha_me + pr;
        pw[lane] = pr;
        __syncwarp();
        float pp[C::NV];
#pragma unroll
        for (int i = 0; i < C::NV; ++i) pp[i] = pw[grp * C::LPR + i];
        __syncwarp();
        if (rescale) {  // uniform across the warp: m is replicated
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) o[h][e] *= alpha[h];
        }
#pragma unroll
        for (int r = 0; r < C::RPB; ++r) {
            if (!mr[r]) continue;
            float vv[C::EPL];
            Vec<KT, C::EPL>::load(sV + (r * C::RPL + grp) * HD + col, vv);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) o[h][e] = fmaf(pp[r * G + h], vv[e], o[h][e]);
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

// Merge the consumer warps' states (fixed order) into one partial per head
// and store it at dst [G][HD+4] = (o[HD], m, l, pad).  Consumer threads only.
template <typename KT, int HD, int G>
__device__ __noinline__ void flush_partial(WarpAttn<KT, HD, G> &st, float *merge, float *dst, int warp, int lane) {
    using C = AttnCfg<KT, HD, G>;
    float lsum[G];
    st.finish(lsum, lane);
    float *wsm = merge + warp * G * (HD + 2);
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
    gsync();
#pragma unroll 1
    for (int idx = warp * 32 + lane; idx < G * (HD + 2); idx += ACW * 32) {
        const int h = idx / (HD + 2), e = idx % (HD + 2);
        float M = -INFINITY;
        for (int w = 0; w < ACW; ++w) M = fmaxf(M, merge[(w * G + h) * (HD + 2) + HD]);
        float r = 0.f;
        if (e == HD) {
            r = M;
        } else if (M != -INFINITY) {
            for (int w = 0; w < ACW; ++w) {
                const float mw = merge[(w * G + h) * (HD + 2) + HD];
                if (mw == -INFINITY) continue;
                r = fmaf(merge[(w * G + h) * (HD + 2) + e], exp2f(mw - M), r);
            }
        }
        dst[h * prec<HD>() + e] = r;
    }
    gsync();
}

// Stage space: KV head kh owns stages [pref[kh], pref[kh+1]).
struct StageMap {
    int64_t pref[65];
    int64_t cnt[64];   // union kept leaves per KV head (gather)
    int h_kv;
    __device__ void locate(int64_t i, int &kh, int64_t &st) const {
        kh = 0;
        while (kh + 1 < h_kv && i >= pref[kh + 1]) ++kh;
        st = i - pref[kh];
    }
    // CTAs [bf, bl] of a grid of nb cover some stage of KV head kh (bl < bf: none)
    __device__ void ctas(int kh, int nb, int &bf, int &bl) const {
        const int64_t U = pref[h_kv], p0 = pref[kh], p1 = pref[kh + 1];
        bf = 0;
        bl = -1;
        if (p1 > p0) {
            bf = (int)(((p0 + 1) * nb - 1) / U);
            bl = (int)((p1 * nb - 1) / U);
        }
    }
};

// Fill the stage map (thread 0) -- call before attn_stages, then sync the CTA.
template <bool DENSE>
__device__ void stage_map_init(const Decode &a, StageMap &map) {
    int64_t acc = 0;
    map.h_kv = a.t.h_kv;
    for (int kh = 0; kh < a.t.h_kv; ++kh) {
        map.pref[kh] = acc;
        map.cnt[kh] = DENSE ? 0 : __ldcg(a.kept_cnt + kh);
        const int64_t ntok = DENSE ? a.t.n_tokens : map.cnt[kh] * a.t.c;
        acc += (ntok + TT - 1) / TT;
    }
    map.pref[a.t.h_kv] = acc;
}

// This CTA's share of the attention: stages [U*b/nb, U*(b+1)/nb).  Leaves one
// partial per (head, KV head) in a.part[b] (-inf max for KV heads it did not
// touch).  All 9 warps of the CTA call it.
template <typename KT, int HD, int G, bool DENSE>
__device__ void attn_stages(const Decode &a, const StageMap &map, unsigned char *smem, int b, int nb) {
    using C = AttnCfg<KT, HD, G>;
    using SM = ASmem<KT, HD, G>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h_kv = a.t.h_kv, c = a.t.c;
    uint8_t *meta = smem + SM::off_meta;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::off_bar);
    uint64_t *empty = full + C::STAGES;
    volatile int *abort = reinterpret_cast<volatile int *>(smem + SM::off_abort);
    float *merge = reinterpret_cast<float *>(smem + SM::off_merge);
    float *pw = reinterpret_cast<float *>(smem + SM::off_pw) + warp * 32;
    const int64_t N = a.t.n_tokens;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], ACW);
        }
        *abort = 0;
        mbar_init_fence();
    }
    __syncthreads();
    const int64_t U = map.pref[h_kv];
    const int64_t u0 = U * b / nb, u1 = U * (b + 1) / nb;
    const int64_t n = u1 - u0;

    if (warp == ACW) {
        // ---------------- producer warp ----------------
        int32_t *win_ids = reinterpret_cast<int32_t *>(smem + SM::off_win);
        uint8_t *win_msk = smem + SM::off_win + (size_t)LEAF_WIN * 4;
        int win_kh = -1;
        int64_t win_k0 = 0;
        int64_t issued = 0;
        for (int64_t j = 0; j < n; ++j) {
            const int slot = (int)(j % C::STAGES);
            const uint32_t round = (uint32_t)(j / C::STAGES);
            if (round > 0 && !mbar_wait(&empty[slot], (round - 1) & 1u, abort)) {
                set_status(a.status, ZHA_TIMEOUT_CODE);
                *abort = 1;
                break;
            }
            int kh;
            int64_t st;
            map.locate(u0 + j, kh, st);
            const KT *Kh = reinterpret_cast<const KT *>(a.t.K) + (int64_t)kh * a.t.kv_cap * HD;
            const KT *Vh = reinterpret_cast<const KT *>(a.t.V) + (int64_t)kh * a.t.kv_cap * HD;
            unsigned char *sK = smem + (size_t)slot * C::STAGE_BYTES;
            unsigned char *sV = sK + TT * C::RB;
            uint8_t *mt = meta + slot * TT;
            const int64_t t0 = st * TT;
            // this lane's runs: rows of one leaf piece each (gather; a stage
            // touches at most TT/c + 2 <= 34 leaves, so at most 2 per lane),
            // or the whole stage (dense, lane 0)
            int64_t row0[2] = {0, 0};
            int dst0[2] = {0, 0}, nrows[2] = {0, 0};
            if (DENSE) {
                if (lane == 0) {
                    row0[0] = t0;
                    nrows[0] = (int)min((int64_t)TT, N - t0);
                }
                for (int t = lane; t < TT; t += 32) mt[t] = (t0 + t < N) ? 0xffu : 0u;
            } else {
                const int64_t L = map.cnt[kh];
                const int64_t kbase = (int64_t)kh * a.t.node_cap[0];
                const int64_t kf = t0 / c;
                const int64_t kl = min(L - 1, (t0 + TT - 1) / c);
                if (kh != win_kh || kl >= win_k0 + LEAF_WIN) {
                    // refill the window from leaf kf on: independent coalesced loads
                    win_kh = kh;
                    win_k0 = kf;
                    for (int i = lane; i < LEAF_WIN && kf + i < L; i += 32) {
                        win_ids[i] = __ldcg(a.kept_ids[0] + kbase + kf + i);
                        win_msk[i] = __ldcg(a.kept_mask[0] + kbase + kf + i);
                    }
                    __syncwarp();
                }
                int q = 0;
                for (int64_t k = kf + lane; k * c < t0 + TT && k < L && q < 2; k += 32, ++q) {
                    const int64_t a0 = max(t0, k * c), a1 = min(t0 + TT, (k + 1) * c);
                    const int64_t leaf = win_ids[k - win_k0];
                    const int64_t r0 = leaf * c + (a0 - k * c);
                    const int64_t r1 = min(leaf * c + (a1 - k * c), N);
                    const uint32_t mk = win_msk[k - win_k0];
                    for (int64_t t = a0; t < a1; ++t) mt[t - t0] = (leaf * c + (t - k * c) < N) ? (uint8_t)mk : 0;
                    row0[q] = r0;
                    dst0[q] = (int)(a0 - t0);
                    nrows[q] = (int)max((int64_t)0, r1 - r0);
                }
                // tokens past the end of the list
                const int64_t tend = L * c;
                for (int t = lane; t < TT; t += 32)
                    if (t0 + t >= tend) mt[t] = 0;
            }
            uint32_t bytes = (uint32_t)(nrows[0] + nrows[1]) * C::RB * 2;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) bytes += __shfl_xor_sync(FULL, bytes, off);
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                if (nrows[q] > 0) {
                    bulk_g2s(sK + (size_t)dst0[q] * C::RB, Kh + row0[q] * HD, (uint32_t)nrows[q] * C::RB, &full[slot]);
                    bulk_g2s(sV + (size_t)dst0[q] * C::RB, Vh + row0[q] * HD, (uint32_t)nrows[q] * C::RB, &full[slot]);
                }
            }
            issued = j + 1;
        }
        // on an abort, wait (bounded) for the copies already in flight
        if (*abort) {
            for (int64_t j = (issued > C::STAGES ? issued - C::STAGES : 0); j < issued; ++j)
                mbar_wait(&full[j % C::STAGES], (uint32_t)((j / C::STAGES) & 1), nullptr);
        }
    } else {
        // ---------------- consumer warps ----------------
        for (int idx = warp * 32 + lane; idx < h_kv * G; idx += ACW * 32)
            a.part[(((int64_t)b * h_kv + idx / G) * G + idx % G) * prec<HD>() + HD] = -INFINITY;
        gsync();
        WarpAttn<KT, HD, G> st;
        st.init();
        float qs[G][C::EPL];
        int kh_cur = -1;
        for (int64_t j = 0; j < n; ++j) {
            const int slot = (int)(j % C::STAGES);
            const uint32_t round = (uint32_t)(j / C::STAGES);
            // every consumer warp takes the same branches below whatever the
            // wait returned, so the named barriers inside the flushes match
            const bool ok = mbar_wait(&full[slot], round & 1u, abort);
            if (!ok) {
                set_status(a.status, ZHA_TIMEOUT_CODE);
                *abort = 1;
            }
            int kh;
            int64_t stage_in_kh;
            map.locate(u0 + j, kh, stage_in_kh);
            if (kh != kh_cur) {
                if (kh_cur >= 0)
                    flush_partial<KT, HD, G>(st, merge, a.part + ((int64_t)b * h_kv + kh_cur) * G * prec<HD>(), warp,
                                             lane);
                kh_cur = kh;
                st.init();
                const float qscale = a.t.scale * LOG2E;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float *qh = a.q + (int64_t)(kh * G + h) * HD + (lane % C::LPR) * C::EPL;
#pragma unroll
                    for (int e = 0; e < C::EPL; ++e) qs[h][e] = qh[e] * qscale;
                }
            }
            const KT *sK = reinterpret_cast<const KT *>(smem + (size_t)slot * C::STAGE_BYTES) + warp * TW * HD;
            const KT *sV = sK + TT * HD;
            if (ok) st.tokens(sK, sV, meta + slot * TT + warp * TW, qs, pw, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        if (kh_cur >= 0)
            flush_partial<KT, HD, G>(st, merge, a.part + ((int64_t)b * h_kv + kh_cur) * G * prec<HD>(), warp, lane);
    }
}

// Merge the partials of CTAs [b0, b1) for the G heads of KV head kh, add the
// sink token (gather: unless leaf 0 is in the head's set) and write the
// outputs.  Threads 0-255; every partial's (max, sum) is loaded at once, then
// each thread sweeps four output columns over the partials in a fixed order.
// `sm` holds 2*G*(b1-b0) + 4*G floats.
template <typename KT, int HD, int G>
__device__ __noinline__ void combine_kvh(const Decode &a, int kh, int b0, int b1, bool gather, float *sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = max(0, b1 - b0);
    float *wv = sm;              // [G][n]: max, then weight
    float *lv = sm + G * n;      // [G][n]: sums
    float *hd = lv + G * n;      // [G] L, [G] sink weight, [G] sink score
    const int h_kv = a.t.h_kv;
    for (int i = tid; i < n * G; i += GT) {
        const int bb = i / G, h = i % G;
        const float *pb = a.part + (((int64_t)(b0 + bb) * h_kv + kh) * G + h) * prec<HD>();
        wv[h * n + bb] = __ldcg(pb + HD);
        lv[h * n + bb] = __ldcg(pb + HD + 1);
    }
    const KT *Kh = reinterpret_cast<const KT *>(a.t.K) + (int64_t)kh * a.t.kv_cap * HD;
    const KT *Vh = reinterpret_cast<const KT *>(a.t.V) + (int64_t)kh * a.t.kv_cap * HD;
    const float qscale = a.t.scale * LOG2E;
    if (warp < G) {
        // sink score of head `warp` (-inf when it is not added)
        const int h = warp;
        bool add = false;
        if (gather) {
            const int64_t kbase = (int64_t)kh * a.t.node_cap[0];
            const bool has0 = __ldcg(a.kept_cnt + kh) > 0 && __ldcg(a.kept_ids[0] + kbase) == 0 &&
                              ((__ldcg(a.kept_mask[0] + kbase) >> h) & 1u);
            add = !has0;
        }
        float s0 = -INFINITY;
        if (add) {
            constexpr int CPL = HD / 32;
            float k0[CPL], qh[CPL];
#pragma unroll
            for (int e = 0; e < CPL; ++e) {
                qh[e] = a.q[(int64_t)(kh * G + h) * HD + lane * CPL + e] * qscale;
                if constexpr (sizeof(KT) == 2) k0[e] = __uint_as_float(((uint32_t)Kh[lane * CPL + e]) << 16);
                else k0[e] = Kh[lane * CPL + e];
            }
            s0 = warp_sum(lane_dot<CPL>(qh, k0));
        }
        if (lane == 0) hd[2 * G + h] = s0;
    }
    gsync();
    if (warp < G) {
        const int h = warp;
        const float s0 = hd[2 * G + h];
        float M = s0;
        for (int i = lane; i < n; i += 32) M = fmaxf(M, wv[h * n + i]);
        M = warp_max(M);
        __syncwarp();
        float L = 0.f;
        for (int i = lane; i < n; i += 32) {
            const float m = wv[h * n + i];
            const float w = (m == -INFINITY) ? 0.f : exp2f(m - M);
            wv[h * n + i] = w;
            L = fmaf(w, lv[h * n + i], L);
        }
        L = warp_sum(L);
        const float ws = (s0 == -INFINITY) ? 0.f : exp2f(s0 - M);
        if (lane == 0) {
            hd[h] = L + ws;
            hd[G + h] = ws;
        }
    }
    gsync();
    // outputs: thread -> (head, four columns)
    for (int idx = tid; idx < G * (HD / 4); idx += GT) {
        const int h = idx / (HD / 4), e4 = (idx % (HD / 4)) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int i = 0; i < n; ++i) {
            const float w = wv[h * n + i];
            if (w == 0.f) continue;
            const float4 o = __ldcg(reinterpret_cast<const float4 *>(
                a.part + (((int64_t)(b0 + i) * h_kv + kh) * G + h) * prec<HD>() + e4));
            acc.x = fmaf(w, o.x, acc.x);
            acc.y = fmaf(w, o.y, acc.y);
            acc.z = fmaf(w, o.z, acc.z);
            acc.w = fmaf(w, o.w, acc.w);
        }
        const float ws = hd[G + h];
        if (ws != 0.f) {
            float v0[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if constexpr (sizeof(KT) == 2) v0[e] = __uint_as_float(((uint32_t)Vh[e4 + e]) << 16);
                else v0[e] = Vh[e4 + e];
            }
            acc.x = fmaf(ws, v0[0], acc.x);
            acc.y = fmaf(ws, v0[1], acc.y);
            acc.z = fmaf(ws, v0[2], acc.z);
            acc.w = fmaf(ws, v0[3], acc.w);
        }
        const float inv = 1.f / hd[h];
        float4 r = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        *reinterpret_cast<float4 *>(a.out + (int64_t)(kh * G + h) * HD + e4) = r;
    }
}

}  // namespace zha
