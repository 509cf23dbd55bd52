// zha_attend.cuh -- exact attention over a token set, split over the CTAs of a
// grid, fed by a warp-specialised bulk-copy pipeline (sm_100a).
//
// Attention ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢":
// the first token is always kept as the attention sink; rit.work article,
// section "Дерево сокращает сам поиск нужных ключей": the main attention reads
// the raw keys of the found leaves):
//   o_h = sum_{i in T_h} softmax_i(q_h.k_i / sqrt(d)) v_i,
//   T_h = tokens of the leaf chunks head h kept  U  {0},  fp32 accumulation.
//
// The union leaf list of each KV head (every leaf any of its G query heads
// kept, with the head bitmask) is flattened into stages of TT tokens; the
// grid's CTAs take contiguous ranges of stages over all KV heads.  In each CTA
// one producer warp (warp 8) maps a stage's tokens to K/V rows a leaf at a
// time, writes the per-token head masks and issues one cp.async.bulk per run
// of consecutive K rows (and V rows) inside each group of the stage, into a
// ring of shared-memory stages guarded by mbarriers.  Rows land at a
// padded stride (16 bytes past the row for bf16) so that the consumers'
// 8-row matrix loads hit eight different bank groups.  Every K and V row
// crosses HBM once and serves all G heads of its group (GQA sharing).
//
// Consumers, warps 0-7, 16 tokens each (bf16: every stage to all 8 warps;
// fp32: stage j to warps 4(j%2)..+3):
//   bf16 K/V: tensor cores (mma.sync m16n8k16, fp32 accumulate).  The queries
//     and the probabilities are split into bf16 high and low parts (x = hi +
//     lo to ~2^-16 relative), rows h and 8+h of the A operand, so that the
//     fp32 accuracy of q.k and p.v is kept; K and V are exact in bf16.
//       S^T[16 x 8 tokens] = [q_hi; q_lo] x K^T, s_h = S[h] + S[8+h]
//       O[16 x d]         += [p_hi; p_lo] x V,  o_h = O[h] + O[8+h]
//   fp32 K/V: fp32 FMA (each lane a column slice of every row).
// Online softmax in the log2 domain.  Each CTA leaves one partial (max, sum,
// output) per head per KV head it touched; combine_kvh merges them.
#pragma once

#include <algorithm>

#include "zha_device.cuh"
#include "zha_internal.cuh"
#include "zha_mma.cuh"
#include "zha_tma.cuh"

namespace zha {

constexpr float LOG2E = 1.4426950408889634f;
constexpr int ACW = 8;                         // consumer warps
constexpr int A_THREADS = (ACW + 1) * 32;      // + one producer warp
constexpr int TW = 16;                         // tokens per consumer warp per stage
constexpr int LEAF_WIN = 1024;                 // leaf ids the producer keeps in shared memory
constexpr size_t STAGE_BUDGET = 200 * 1024;    // shared memory for the stage ring

// One partial record: o[HD], max, sum, two pads (16-byte aligned records).
template <int HD>
constexpr int prec() { return HD + 4; }

// A stage holds TT tokens as 8 groups of GR consecutive tokens (bf16: 128
// tokens, groups of 16 rows, 4 KB per copy at d = 128; fp32: 64 tokens, groups
// of 8).  Each group is filled by bulk copies of whole runs of rows; groups
// sit GS bytes apart, 16 bytes more than their rows, so that row w of the
// eight groups falls in eight different bank groups.  Token slot
// t = GR*group + w sits at row_off(t); K groups first, then V.  The stage goes
// to CW consumer warps (bf16: all 8; fp32: 4, the two halves alternating).
template <typename KT, int HD>
struct StageCfg {
    static constexpr int ES = (int)sizeof(KT);
    static constexpr int RB = HD * ES;                      // row bytes
    static constexpr int TT = ES == 2 ? 128 : 64;           // tokens per stage
    static constexpr int NG = 8;                            // groups per stage
    static constexpr int GR = TT / NG;                      // rows per group
    static constexpr int GLOG = ES == 2 ? 4 : 3;            // log2(GR)
    static constexpr int GS = GR * RB + 16;                 // group stride
    static constexpr int HALF = NG * GS;                    // K part (V part follows)
    static constexpr int STAGE_BYTES = 2 * HALF;
    static constexpr int CW = TT / TW;                      // consumer warps per stage
    static constexpr int HALVES = ACW / CW;                 // consumer halves alternating over stages
    static constexpr int S0 = (int)(STAGE_BUDGET / STAGE_BYTES);
    static constexpr int STAGES = S0 > 6 ? 6 : S0;
    static_assert(STAGES >= 2, "stage ring");
    static_assert(RB % 16 == 0 && GS % 16 == 0, "bulk copies need 16-byte aligned rows");
    static_assert((1 << GLOG) == GR && 2 * CW == GR, "each consumer warp takes two rows of every group");
    static_assert(HALVES * CW == ACW && TW * CW == TT, "consumer warps cover a stage");
    static __device__ __forceinline__ int row_off(int t) { return (t >> GLOG) * GS + (t & (GR - 1)) * RB; }
};

template <typename KT, int HD, int G>
struct ASmem {
    using C = StageCfg<KT, HD>;
    static constexpr size_t off_meta = (size_t)C::STAGES * C::STAGE_BYTES;
    static constexpr size_t off_bar = (off_meta + C::STAGES * C::TT + 15) / 16 * 16;  // full[ST], empty[ST]
    static constexpr size_t off_abort = off_bar + 2 * C::STAGES * 8;
    static constexpr size_t off_merge = (off_abort + 16 + 15) / 16 * 16;
    static constexpr size_t off_pw = off_merge + (size_t)ACW * G * (HD + 2) * 4;   // FMA consumers' p slots
    static constexpr size_t off_win = off_pw + (size_t)ACW * 32 * 4;                // producer's leaf-id window
    static constexpr size_t bytes = off_win + (size_t)LEAF_WIN * 5;
};

// ---- tensor-core consumer (bf16) ------------------------------------------

// Split (x0, x1) into bf16 high parts and bf16 low parts (x - hi).
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16(x0, x1);
    lo = pack_bf16(x0 - bf_lo(hi), x1 - bf_hi(hi));
}

template <int HD, int G>
struct MmaAttn {
    static constexpr int KS = HD / 16;  // k-steps of q.k
    static constexpr int NT = HD / 8;   // n-tiles of the output
    uint32_t qa[KS][4];                 // A fragments of [q_hi; q_lo] (scaled, log2 domain)
    float o[NT][4];                     // rows g (p_hi) and g+8 (p_lo), columns nt*8 + 2*c4 + {0,1}
    float m;                            // running max of head g (replicated over the quad)
    float l;                            // this thread's partial denominator

    __device__ void init() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
        m = -INFINITY;
        l = 0.f;
    }

    // q rows of KV head kh into A fragments; thread (g = lane/4, c4 = lane%4)
    // holds rows g (hi) and g+8 (lo) for g < G.
    __device__ void load_q(const float *q, int kh, float qscale, int lane) {
        const int g = lane >> 2, c4 = lane & 3;
        const float *qh = q + (int64_t)(kh * G + (g < G ? g : 0)) * HD;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int d0 = ks * 16 + 2 * c4;
            if (g < G) {
                const float2 x01 = *reinterpret_cast<const float2 *>(qh + d0);
                const float2 x89 = *reinterpret_cast<const float2 *>(qh + d0 + 8);
                split_bf16(x01.x * qscale, x01.y * qscale, qa[ks][0], qa[ks][1]);
                split_bf16(x89.x * qscale, x89.y * qscale, qa[ks][2], qa[ks][3]);
            } else {
                qa[ks][0] = qa[ks][1] = qa[ks][2] = qa[ks][3] = 0u;
            }
        }
    }

    // The 16 tokens of consumer slot wq of a stage: rows w1 = 2 wq and
    // w2 = 2 wq + 1 of each of the 8 groups.  Column n of the first score tile
    // is token GR n + w1, of the second GR n + w2; the same order is the k
    // order of p.v.  sK/sV: the stage's K and V parts, msk: its head masks.
    template <typename SC>
    __device__ void tokens(const unsigned char *sK, const unsigned char *sV, const uint8_t *msk, int wq, int lane) {
        const int g = lane >> 2, c4 = lane & 3;
        const int w1 = 2 * wq, w2 = 2 * wq + 1;
        const int mi = lane >> 3, r = lane & 7;  // this lane addresses row r of matrix mi
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        {
            // matrices: (w1, dims lo), (w1, dims hi), (w2, lo), (w2, hi) of a k-step
            const int w = (mi >> 1) ? w2 : w1;
            const uint32_t base = smem_addr(sK) + (uint32_t)(r * SC::GS + w * SC::RB + (mi & 1) * 16);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t kb[4];
                ldsm_x4(kb, base + ks * 32);
                mma_bf16(s0, qa[ks], kb[0], kb[1]);
                mma_bf16(s1, qa[ks], kb[2], kb[3]);
            }
        }
        const uint32_t hb = g < G ? (1u << g) : 0u;
        float x[4];
        constexpr int GR = SC::GR;
        x[0] = (msk[GR * (2 * c4) + w1] & hb) ? s0[0] + s0[2] : -INFINITY;
        x[1] = (msk[GR * (2 * c4 + 1) + w1] & hb) ? s0[1] + s0[3] : -INFINITY;
        x[2] = (msk[GR * (2 * c4) + w2] & hb) ? s1[0] + s1[2] : -INFINITY;
        x[3] = (msk[GR * (2 * c4 + 1) + w2] & hb) ? s1[1] + s1[3] : -INFINITY;
        float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 2));
        const float mn = fmaxf(m, mt);
        if (mn > m && m != -INFINITY) {
            const float alpha = exp2f(m - mn);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[nt][e] *= alpha;
            l *= alpha;
        }
        m = mn;
        float p[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) p[t] = (x[t] == -INFINITY) ? 0.f : exp2f(x[t] - mn);
        l += (p[0] + p[1]) + (p[2] + p[3]);
        uint32_t pa[4];
        split_bf16(p[0], p[1], pa[0], pa[1]);
        split_bf16(p[2], p[3], pa[2], pa[3]);
        {
            // matrices: (w1 tokens, dims lo), (w2, lo), (w1, hi), (w2, hi) of a column pair
            const int w = (mi & 1) ? w2 : w1;
            const uint32_t base = smem_addr(sV) + (uint32_t)(r * SC::GS + w * SC::RB + (mi >> 1) * 16);
#pragma unroll
            for (int i = 0; i < HD / 16; ++i) {
                uint32_t vb[4];
                ldsm_x4_t(vb, base + i * 32);
                mma_bf16(o[2 * i], pa, vb[0], vb[1]);
                mma_bf16(o[2 * i + 1], pa, vb[2], vb[3]);
            }
        }
    }

    // This warp's state into merge [G][HD+2] = (o, m, l).
    __device__ void store(float *wsm, int lane) {
        const int g = lane >> 2, c4 = lane & 3;
        float lt = l;
        lt += __shfl_xor_sync(FULL, lt, 1);
        lt += __shfl_xor_sync(FULL, lt, 2);
        if (g < G) {
            float *row = wsm + g * (HD + 2);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int d = nt * 8 + 2 * c4;
                row[d] = o[nt][0] + o[nt][2];
                row[d + 1] = o[nt][1] + o[nt][3];
            }
            if (c4 == 0) {
                row[HD] = m;
                row[HD + 1] = lt;
            }
        }
    }
};

// ---- fp32 FMA consumer -------------------------------------------------------

template <int HD, int G>
struct FmaCfg {
    static constexpr int RB = HD * 4;             // row bytes
    static constexpr int LPR = RB / 16;           // lanes per row (16-byte slices)
    static constexpr int RPL = 32 / LPR;          // rows per warp-wide access
    static constexpr int EPL = 4;                 // elements per lane per row
    // tokens per pass: one partial per lane after the reduce (RPB * G <= LPR)
    static constexpr int SUBT = (LPR / G) * RPL < TW ? (LPR / G) * RPL : TW;
    static constexpr int RPB = SUBT / RPL;        // rows per lane per pass
    static constexpr int NV = RPB * G;            // partial dots per lane
    static constexpr int NVP = NV > LPR ? NV : LPR;  // padded to the reduce width
    static_assert(LPR >= 1 && LPR <= 32 && RPB >= 1, "row layout");
    static_assert(LPR % G == 0, "row slices must cover the heads");
    static_assert(NV <= LPR && TW % SUBT == 0, "one partial per lane");
};

// Online-softmax state of one consumer warp for the G heads of one KV head.
template <int HD, int G>
struct FmaAttn {
    using C = FmaCfg<HD, G>;
    float m[G];          // running max (log2 domain), replicated over lanes
    float l;             // partial denominator of this lane's head (lane % G)
    float o[G][C::EPL];  // partial outputs of this lane's column slice
    float qs[G][C::EPL];

    __device__ void init() {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY;
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) o[h][e] = 0.f;
        }
        l = 0.f;
    }

    __device__ void load_q(const float *q, int kh, float qscale, int lane) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float *qh = q + (int64_t)(kh * G + h) * HD + (lane % C::LPR) * C::EPL;
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) qs[h][e] = qh[e] * qscale;
        }
    }

    // The warp's TW tokens (token i of consumer slot wq is stage slot
    // GR (i % 8) + 2 wq + i / 8), in passes of SUBT.
    template <typename SC>
    __device__ void tokens(const unsigned char *sK, const unsigned char *sV, const uint8_t *msk, int wq, float *pw,
                           int lane) {
#pragma unroll 1
        for (int i0 = 0; i0 < TW; i0 += C::SUBT) pass<SC>(sK, sV, msk, wq, i0, pw, lane);
    }

    template <typename SC>
    __device__ void pass(const unsigned char *sK, const unsigned char *sV, const uint8_t *msk, int wq, int i0, float *pw,
                         int lane) {
        const int grp = lane / C::LPR, col = (lane % C::LPR) * C::EPL;
        float v[C::NVP];
        uint32_t mr[C::RPB];
        int off[C::RPB];
#pragma unroll
        for (int r = 0; r < C::RPB; ++r) {
            const int i = i0 + r * C::RPL + grp;
            const int t = SC::GR * (i & 7) + 2 * wq + (i >> 3);
            off[r] = SC::row_off(t);
            mr[r] = msk[t];
            float k[C::EPL];
            Vec<float, C::EPL>::load(reinterpret_cast<const float *>(sK + off[r]) + col, k);
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
        for (int o2 = G; o2 < 32; o2 <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(FULL, bmax, o2));
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
            Vec<float, C::EPL>::load(reinterpret_cast<const float *>(sV + off[r]) + col, vv);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) o[h][e] = fmaf(pp[r * G + h], vv[e], o[h][e]);
        }
    }

    __device__ void store(float *wsm, int lane) {
#pragma unroll
        for (int off = C::LPR; off < 32; off <<= 1)
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) o[h][e] += __shfl_xor_sync(FULL, o[h][e], off);
        float lt = l;
#pragma unroll
        for (int off = G; off < 32; off <<= 1) lt += __shfl_xor_sync(FULL, lt, off);
        float lsum[G];
#pragma unroll
        for (int h = 0; h < G; ++h) lsum[h] = __shfl_sync(FULL, lt, h);
        if (lane < C::LPR) {
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) wsm[h * (HD + 2) + lane * C::EPL + e] = o[h][e];
        }
        if (lane == 0) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                wsm[h * (HD + 2) + HD] = m[h];
                wsm[h * (HD + 2) + HD + 1] = lsum[h];
            }
        }
    }
};

template <typename KT, int HD, int G>
struct Consumer;
template <int HD, int G>
struct Consumer<uint16_t, HD, G> {
    using T = MmaAttn<HD, G>;
};
template <int HD, int G>
struct Consumer<float, HD, G> {
    using T = FmaAttn<HD, G>;
};

// Merge the consumer warps' states (fixed order) into one partial per head
// at dst [G][HD+4] = (o[HD], m, l, pad).  Consumer warps only.
template <int HD, int G>
__device__ __noinline__ void merge_partials(const float *merge, float *dst, int warp, int lane) {
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

// Head masks of `n` consecutive stage rows: mk for the first `valid`, 0 after.
__device__ __forceinline__ void mask_rows(uint8_t *mt, uint32_t mk, int valid, int n) {
    if ((n & 3) == 0) {
        for (int w = 0; w < n; w += 4) {
            uint32_t v = 0u;
#pragma unroll
            for (int b = 0; b < 4; ++b) v |= (w + b < valid ? mk : 0u) << (8 * b);
            *reinterpret_cast<uint32_t *>(mt + w) = v;
        }
    } else {
        for (int w = 0; w < n; ++w) mt[w] = (uint8_t)(w < valid ? mk : 0u);
    }
}

// x / c for token positions (< 2^32): a shift when c is a power of two.
__device__ __forceinline__ uint32_t div_c(uint32_t x, int c, int clog) {
    return clog >= 0 ? (x >> clog) : x / (uint32_t)c;
}

// ---- the stage map -------------------------------------------------------------

// Stage space: KV head kh owns stages [pref[kh], pref[kh+1]).  For the routed
// attention, KV head kh's kept leaves are the level-1 segments: T1[kh] ranks,
// frontier S1[kh], per-rank kept counts with exclusive prefix
// spref[soff[kh] .. soff[kh] + T1[kh]].
struct StageMap {
    int64_t pref[65];
    int64_t cnt[64];   // union kept leaves per KV head (gather)
    int h_kv;
    int T1[64];
    int32_t S1[64];
    int soff[65];
    uint32_t spref[SEG_CAP + 65];
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
    // Position in kept_ids[0] (KV head kh's rows) of kept leaf rank k.
    __device__ int64_t leaf_at(int kh, int64_t k) const {
        const uint32_t *p = spref + soff[kh];
        const int T = T1[kh];
        int lo = 0, hi = T - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((int64_t)p[mid] <= k) lo = mid;
            else hi = mid - 1;
        }
        return (int64_t)S1[kh] * lo / T + (k - p[lo]);
    }
    // The same for a rank k not below the one `r` was found for: advance r
    // (the segment holding the last rank looked up) and return the position.
    __device__ int64_t leaf_at_from(int kh, int64_t k, int &r) const {
        const uint32_t *p = spref + soff[kh];
        const int T = T1[kh];
        while (r + 1 < T && (int64_t)p[r + 1] <= k) ++r;
        return (int64_t)S1[kh] * r / T + (k - p[r]);
    }
};

// Fill the stage map; all threads of the CTA call it, then it is valid after
// the __syncthreads inside.  Gather: the level-1 segments written by routing.
template <bool DENSE, int TT>
__device__ void stage_map_init(const Decode &a, StageMap &map) {
    const int h_kv = a.nvk;  // virtual KV heads
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if ((int)threadIdx.x < h_kv) {  // level 1's team and frontier sizes, in parallel
        const int kh = threadIdx.x;
        map.T1[kh] = DENSE ? 1 : __ldcg(a.lvl + (int64_t)kh * 2);
        map.S1[kh] = DENSE ? 0 : __ldcg(a.lvl + (int64_t)kh * 2 + 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        map.h_kv = h_kv;
        int off = 0;
#pragma unroll 1
        for (int kh = 0; kh < h_kv; ++kh) {
            map.soff[kh] = off;
            off += map.T1[kh] + 1;
        }
        map.soff[h_kv] = off;
    }
    __syncthreads();
    if (!DENSE) {
        // per KV head (one warp each): prefix of the level-1 per-rank counts
        for (int kh = warp; kh < h_kv; kh += A_THREADS / 32) {
            const int T = map.T1[kh];
            const uint32_t *sg = a.seg + (int64_t)kh * SEG_CAP;
            uint32_t carry = 0u;
            for (int r0 = 0; r0 < T; r0 += 32) {
                const uint32_t x = r0 + lane < T ? __ldcg(sg + r0 + lane) : 0u;
                uint32_t v = x;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t y = __shfl_up_sync(FULL, v, off);
                    if (lane >= off) v += y;
                }
                if (r0 + lane < T) map.spref[map.soff[kh] + r0 + lane + 1] = carry + v;
                carry += __shfl_sync(FULL, v, 31);
            }
            if (lane == 0) {
                map.spref[map.soff[kh]] = 0u;
                map.cnt[kh] = carry;
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int kh = 0; kh < h_kv; ++kh) {
            map.pref[kh] = acc;
            const int64_t ntok = DENSE ? a.t.n_tokens : map.cnt[kh] * a.t.c;
            acc += (ntok + TT - 1) / TT;
        }
        map.pref[h_kv] = acc;
    }
    __syncthreads();
}

// This CTA's share of the attention: stages [U*b/nb, U*(b+1)/nb).  Leaves one
// partial per (head, KV head) in a.part[b] (-inf max for KV heads it did not
// touch).  All 9 warps of the CTA call it.
template <typename KT, int HD, int G, bool DENSE>
__device__ void attn_stages(const Decode &a, const StageMap &map, unsigned char *smem, int b, int nb) {
    using C = StageCfg<KT, HD>;
    using SM = ASmem<KT, HD, G>;
    constexpr int ST = C::STAGES, RB = C::RB, GR = C::GR, TT = C::TT;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h_kv = a.nvk, c = a.t.c, clog = a.t.c_log2;  // virtual KV heads
    uint8_t *meta = smem + SM::off_meta;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::off_bar);
    uint64_t *empty = full + ST;
    volatile int *abort = reinterpret_cast<volatile int *>(smem + SM::off_abort);
    float *merge = reinterpret_cast<float *>(smem + SM::off_merge);
    const int N = (int)a.t.n_tokens;  // rows per KV head < 2^31
    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::CW);
        }
        *abort = 0;
        mbar_init_fence();
    }
    __syncthreads();
    const int64_t U = map.pref[h_kv];
    const int64_t u0 = U * b / nb, u1 = U * (b + 1) / nb;
    const int n = (int)(u1 - u0);

    if (warp == ACW) {
        // ---------------- producer warp ----------------
        // the kept leaves of the current KV head, ranks [., rhi) of them at
        // rank % LEAF_WIN: a ring refilled a chunk of RING_CHUNK ranks at a
        // time, each chunk's loads issued a chunk ahead of its use, so that
        // their latency hides behind the stages between
        int32_t *win_ids = reinterpret_cast<int32_t *>(smem + SM::off_win);
        uint8_t *win_msk = smem + SM::off_win + (size_t)LEAF_WIN * 4;
        constexpr int RING_CHUNK = 128, PERL = RING_CHUNK / 32;
        static_assert((LEAF_WIN & (LEAF_WIN - 1)) == 0 && RING_CHUNK <= LEAF_WIN / 2, "leaf ring");
        int win_kh = -1, rhi = 0, rend = 0, rseg = 0;
        bool pending = false;
        const int32_t *kid = nullptr;
        const uint8_t *kmk = nullptr;
        int32_t cid[PERL];
        uint32_t cmk[PERL];
        int issued = 0;
        const uint64_t pol = l2_evict_first();  // K/V rows are read once
        int kh;
        int64_t st64;
        map.locate(u0, kh, st64);
        int st = (int)st64;
        // lane gi < 8: K rows of group gi; lane 8 + gi: V rows of group gi
        // (fast = 0); fast = 1: a group never spans two leaves; fast = 2:
        // whole leaves tile each group (GR / c of them, a power of two) and
        // a stage holds at most 32 leaves
        const int fast = DENSE ? 0 : (c % GR == 0 ? 1 : (GR % c == 0 && TT / c <= 32 ? 2 : 0));
        const int lps = fast == 2 ? TT / c : 0;      // leaves per stage
        const int nlm = fast == 2 ? GR / c - 1 : 0;  // leaves per group - 1
        const int gi = lane & 7;
        const bool act = lane < 16;
        const bool isV = lane >= 8;
        // per KV head: its rows, kept leaves and last stage of this CTA
        int jnext = 0, L = 0;
        const unsigned char *Kh = nullptr, *Vh = nullptr;
        auto enter_head = [&]() {
            const int pk = kh % a.t.h_kv;  // physical KV head
            Kh = reinterpret_cast<const unsigned char *>(a.t.K) + (int64_t)pk * a.t.kv_cap * RB;
            Vh = reinterpret_cast<const unsigned char *>(a.t.V) + (int64_t)pk * a.t.kv_cap * RB;
            L = DENSE ? 0 : (int)map.cnt[kh];
            jnext = (int)(min(u1, map.pref[kh + 1]) - u0);
        };
        enter_head();
        int slot = 0;
        uint32_t round = 0u;
#pragma unroll 1
        for (int j = 0; j < n; ++j, ++st) {
            if (j >= jnext) {
                while (kh + 1 < h_kv && u0 + j >= map.pref[kh + 1]) ++kh;
                st = 0;
                enter_head();
            }
            if (round > 0 && !mbar_wait(&empty[slot], (round - 1) & 1u, abort)) {
                set_status(a.status, ZHA_TIMEOUT_CODE);
                *abort = 1;
                break;
            }
            unsigned char *sK = smem + (size_t)slot * C::STAGE_BYTES;
            uint8_t *mt = meta + slot * TT;
            const int t0 = st * TT;
            const int cur = slot;
            if (++slot == ST) {
                slot = 0;
                ++round;
            }
            int kf = 0;
            if (!DENSE) {
                kf = (int)div_c((uint32_t)t0, c, clog);
                const int kl = min(L - 1, (int)div_c((uint32_t)(t0 + TT - 1), c, clog));
                if (kh != win_kh) {
                    // a new KV head: its kept leaves from rank kf up to the last
                    // one this CTA needs
                    const int jl = (int)(min(u1, map.pref[kh + 1]) - 1 - map.pref[kh]);
                    win_kh = kh;
                    rend = min(L - 1, (int)div_c((uint32_t)(jl * TT + TT - 1), c, clog)) + 1;
                    rhi = kf;
                    rseg = 0;
                    pending = false;
                    kid = a.kept_ids[0] + (int64_t)kh * a.slot_cap[0];
                    kmk = a.kept_mask[0] + (int64_t)kh * a.slot_cap[0];
                }
                // ranks below kf are done with; a chunk goes out as soon as the
                // ring has room for it, and lands (its loads waited for) only
                // when a stage needs its ranks
#pragma unroll 1
                while (true) {
                    if (!pending && rhi < rend && rhi + RING_CHUNK - kf <= LEAF_WIN) {
                        // ranks rhi + lane + 32 t (the lane's segment only moves forward)
#pragma unroll
                        for (int t = 0; t < PERL; ++t) {
                            const int k = rhi + lane + 32 * t;
                            if (k < rend) {
                                const int at = (int)map.leaf_at_from(kh, k, rseg);
                                cid[t] = __ldcg(kid + at);
                                cmk[t] = __ldcg(kmk + at);
                            }
                        }
                        pending = true;
                    }
                    if (rhi > kl) break;
#pragma unroll
                    for (int t = 0; t < PERL; ++t) {
                        const int k = rhi + lane + 32 * t;
                        if (k < rend) {
                            win_ids[k & (LEAF_WIN - 1)] = cid[t];
                            win_msk[k & (LEAF_WIN - 1)] = (uint8_t)cmk[t];
                        }
                    }
                    __syncwarp();
                    rhi = min(rend, rhi + RING_CHUNK);
                    pending = false;
                }
            }
            if (fast) {
                // leaves that tile the groups: at most one run per lane, all
                // lanes at once (the generic path below walks leaves one by one)
                int rows = 0, row0 = 0, srow = 0;  // the lane's run: rows, first source row, first stage row
                int own = 0, valid = 0;            // stage rows the lane describes, and how many hold a token
                if (fast == 1) {
                    // every group lies inside one leaf: lane g < NG takes group g
                    if (lane < C::NG) {
                        const int ug = t0 + lane * GR;
                        uint32_t mk = 0u;
                        if (ug < L * c) {
                            const int k = (int)div_c((uint32_t)ug, c, clog);
                            mk = win_msk[k & (LEAF_WIN - 1)];
                            row0 = win_ids[k & (LEAF_WIN - 1)] * c + (ug - k * c);
                            rows = max(0, min(GR, N - row0));
                        }
                        srow = lane * GR;
                        own = GR;
                        valid = rows;
                        mask_rows(mt + srow, mk, valid, own);
                    }
                } else {
                    // lane q takes the stage's leaf q; a run starts at a
                    // group's first leaf or where the leaf ids stop following
                    // on (a leaf before another is always whole: only the
                    // sequence's last leaf can be partial)
                    const int k = kf + lane;
                    int id = 0;
                    uint32_t mk = 0u;
                    bool cont = false;
                    if (lane < lps && k < L) {
                        id = win_ids[k & (LEAF_WIN - 1)];
                        mk = win_msk[k & (LEAF_WIN - 1)];
                        valid = min(c, N - id * c);
                        if ((lane & nlm) != 0) cont = win_ids[(k - 1) & (LEAF_WIN - 1)] == id - 1;
                    }
                    const uint32_t cm = __ballot_sync(FULL, cont);
                    // leaves the run takes after its first: the continuing lanes just above
                    const int e = lane < 31 ? __ffs(~(cm >> (lane + 1))) - 1 : 0;
                    if (lane < lps) {
                        if (valid > 0 && !cont) {
                            row0 = id * c;
                            rows = min((e + 1) * c, N - row0);
                        }
                        srow = lane * c;
                        own = c;
                        mask_rows(mt + srow, mk, valid, own);
                    }
                }
                const uint32_t bytes = __reduce_add_sync(FULL, (uint32_t)rows) * (uint32_t)RB;
                // rows without a token: zeros (see below)
                if (valid < own) {
#pragma unroll 1
                    for (int w = srow + valid; w < srow + own; ++w) {
                        unsigned char *rk = sK + (w / GR) * C::GS + (w % GR) * RB;
                        for (int i = 0; i < RB / 16; ++i) {
                            reinterpret_cast<uint4 *>(rk)[i] = make_uint4(0u, 0u, 0u, 0u);
                            reinterpret_cast<uint4 *>(rk + C::HALF)[i] = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(&full[cur], 2u * bytes);
                __syncwarp();
                if (rows > 0) {
                    unsigned char *dk = sK + (srow / GR) * C::GS + (srow % GR) * RB;
                    bulk_g2s_hint(dk, Kh + (size_t)row0 * RB, (uint32_t)(rows * RB), &full[cur], pol);
                    bulk_g2s_hint(dk + C::HALF, Vh + (size_t)row0 * RB, (uint32_t)(rows * RB), &full[cur], pol);
                }
                issued = j + 1;
                continue;
            }
            // rows of this lane's group: flattened positions ug .. ug + GR - 1
            const int ug = t0 + gi * GR;
            const unsigned char *src = isV ? Vh : Kh;
            unsigned char *dst = sK + (isV ? C::HALF : 0) + gi * C::GS;
            uint32_t nvalid = 0u;  // the group's token slots that hold a row: a prefix of the group
            if (DENSE) {
                nvalid = act ? (uint32_t)max(0, min(GR, N - ug)) : 0u;
                if (act && !isV) {
#pragma unroll
                    for (int w = 0; w < GR; w += 4)
                        *reinterpret_cast<uint32_t *>(mt + gi * GR + w) =
                            (w + 0 < (int)nvalid ? 0xffu : 0u) | (w + 1 < (int)nvalid ? 0xff00u : 0u) |
                            (w + 2 < (int)nvalid ? 0xff0000u : 0u) | (w + 3 < (int)nvalid ? 0xff000000u : 0u);
                }
            } else if (act) {
                // the group's slots, one leaf at a time: leaf k covers slots
                // [k c, (k + 1) c) of the flattened list, rows id_k c + (0 .. c-1)
                int u = ug, k = (int)div_c((uint32_t)ug, c, clog), off = ug - k * c;
                while (u < ug + GR && k < L) {
                    const int id = win_ids[k & (LEAF_WIN - 1)];
                    const uint32_t mk = win_msk[k & (LEAF_WIN - 1)];
                    const int len = min(c - off, ug + GR - u);
                    const int vlen = max(0, min(len, N - (id * c + off)));
                    if (!isV) {
                        const int w0 = u - ug;
                        if (((w0 | vlen) & 3) == 0) {
                            const uint32_t m4 = mk * 0x01010101u;
                            for (int w = 0; w < vlen; w += 4) *reinterpret_cast<uint32_t *>(mt + gi * GR + w0 + w) = m4;
                        } else {
                            for (int w = 0; w < vlen; ++w) mt[gi * GR + w0 + w] = (uint8_t)mk;
                        }
                    }
                    nvalid += (uint32_t)vlen;
                    if (vlen < len) break;  // the sequence's last, partial leaf
                    u += len;
                    ++k;
                    off = 0;
                }
                if (!isV)
                    for (int w = (int)nvalid; w < GR; ++w) mt[gi * GR + w] = 0u;
            }
            uint32_t bytes = nvalid * RB;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) bytes += __shfl_xor_sync(FULL, bytes, o);
            // rows without a token: zeros, so that 0 * row stays 0 in the
            // products (the fence orders these generic stores before later
            // bulk copies into the same rows)
            if (act && nvalid < (uint32_t)GR) {
#pragma unroll 1
                for (int w = (int)nvalid; w < GR; ++w) {
                    uint4 *z = reinterpret_cast<uint4 *>(dst + w * RB);
                    for (int i = 0; i < RB / 16; ++i) z[i] = make_uint4(0u, 0u, 0u, 0u);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[cur], bytes);
            __syncwarp();
            if (act && nvalid > 0u) {
                if (DENSE) {
                    bulk_g2s_hint(dst, src + (size_t)ug * RB, nvalid * RB, &full[cur], pol);
                } else {
                    // one copy per run of consecutive rows: adjacent leaves merge
                    int u = ug, k = (int)div_c((uint32_t)ug, c, clog), off = ug - k * c;
                    int run_w = 0, run_row = -1, run_len = 0;
                    while (u < ug + (int)nvalid) {
                        const int r0 = win_ids[k & (LEAF_WIN - 1)] * c + off;
                        const int len = min(c - off, ug + (int)nvalid - u);
                        if (run_len > 0 && r0 == run_row + run_len) {
                            run_len += len;
                        } else {
                            if (run_len > 0)
                                bulk_g2s_hint(dst + run_w * RB, src + (size_t)run_row * RB, (uint32_t)(run_len * RB),
                                              &full[cur], pol);
                            run_w = u - ug;
                            run_row = r0;
                            run_len = len;
                        }
                        u += len;
                        ++k;
                        off = 0;
                    }
                    bulk_g2s_hint(dst + run_w * RB, src + (size_t)run_row * RB, (uint32_t)(run_len * RB), &full[cur],
                                  pol);
                }
            }
            issued = j + 1;
        }
        // on an abort, wait (bounded) for the copies already in flight
        if (*abort) {
            for (int j = (issued > ST ? issued - ST : 0); j < issued; ++j)
                mbar_wait(&full[j % ST], (uint32_t)((j / ST) & 1), nullptr);
        }
    } else {
        // ---------------- consumer warps ----------------
        for (int idx = warp * 32 + lane; idx < h_kv * G; idx += ACW * 32)
            a.part[(((int64_t)b * h_kv + idx / G) * G + idx % G) * prec<HD>() + HD] = -INFINITY;
        gsync();
        typename Consumer<KT, HD, G>::T st;
        st.init();
        const int half = warp / C::CW, wq = warp % C::CW;
        const float qscale = a.t.scale * LOG2E;
        int kh_cur = -1, kh = 0;
        while (kh + 1 < h_kv && u0 >= map.pref[kh + 1]) ++kh;
#pragma unroll 1
        for (int j = 0; j < n; ++j) {
            while (kh + 1 < h_kv && u0 + j >= map.pref[kh + 1]) ++kh;
            if (kh != kh_cur) {
                // every consumer warp sees every stage's KV head, so the
                // named barriers inside the flushes match
                if (kh_cur >= 0) {
                    st.store(merge + warp * G * (HD + 2), lane);
                    merge_partials<HD, G>(merge, a.part + ((int64_t)b * h_kv + kh_cur) * G * prec<HD>(), warp, lane);
                }
                kh_cur = kh;
                st.init();
                st.load_q(a.q, kh, qscale, lane);
            }
            if (j % C::HALVES != half) continue;
            const int slot = j % ST;
            const uint32_t round = (uint32_t)(j / ST);
            const bool ok = mbar_wait(&full[slot], round & 1u, abort);
            if (!ok) {
                set_status(a.status, ZHA_TIMEOUT_CODE);
                *abort = 1;
            }
            const unsigned char *sK = smem + (size_t)slot * C::STAGE_BYTES;
            const unsigned char *sV = sK + C::HALF;
            const uint8_t *msk = meta + slot * TT;
            if (ok) {
                if constexpr (sizeof(KT) == 2) {
                    st.template tokens<C>(sK, sV, msk, wq, lane);
                } else {
                    float *pws = reinterpret_cast<float *>(smem + SM::off_pw) + warp * 32;
                    st.template tokens<C>(sK, sV, msk, wq, pws, lane);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        if (kh_cur >= 0) {
            st.store(merge + warp * G * (HD + 2), lane);
            merge_partials<HD, G>(merge, a.part + ((int64_t)b * h_kv + kh_cur) * G * prec<HD>(), warp, lane);
        }
    }
}

// Merge the partials of CTAs [b0, b1) for the G heads of KV head kh, add the
// sink token (gather: unless leaf 0 is in the head's set) and write the
// outputs.  Threads 0-255, one gsync: thread t takes (head, four output
// columns) q = t % NQ and the contiguous part t / NQ of the partials, and
// merges its part online (running max, rescaled sum and columns), eight
// partials' loads in flight; meanwhile warps 0..G-1 compute the sink scores.
// Then threads q < NQ add the parts in order and the sink.  `sm` holds
// 6 * GT + G floats (part columns, maxima, sums, sink scores).
template <typename KT, int HD, int G>
__device__ __noinline__ void combine_kvh(const Decode &a, const StageMap &map, int kh, int b0, int b1, bool gather,
                                         float *sm) {
    constexpr int NQ = G * (HD / 4);  // (head, column quad) pairs
    constexpr int NS = GT / NQ;       // parts of the partial range
    static_assert(NS >= 1 && NS * NQ == GT, "threads cover (head, quad, part)");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = max(0, b1 - b0);
    float4 *racc = reinterpret_cast<float4 *>(sm);  // [GT] part columns
    float *rml = sm + 4 * GT;                          // [GT] part max, [GT] part sum
    float *hs0 = rml + 2 * GT;                         // [G] sink scores
    const int h_kv = a.nvk;
    const KT *Kh = reinterpret_cast<const KT *>(a.t.K) + (int64_t)(kh % a.t.h_kv) * a.t.kv_cap * HD;
    const KT *Vh = reinterpret_cast<const KT *>(a.t.V) + (int64_t)(kh % a.t.h_kv) * a.t.kv_cap * HD;
    if (warp < G) {
        // sink score of head `warp` (-inf when it is not added)
        const int h = warp;
        constexpr int CPL = HD / 32;
        const float qscale = a.t.scale * LOG2E;
        float k0[CPL], qh[CPL];
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
            qh[e] = a.q[(int64_t)(kh * G + h) * HD + lane * CPL + e] * qscale;
            if constexpr (sizeof(KT) == 2) k0[e] = __uint_as_float(((uint32_t)Kh[lane * CPL + e]) << 16);
            else k0[e] = Kh[lane * CPL + e];
        }
        bool add = false;
        if (gather) {
            bool has0 = false;
            if (map.cnt[kh] > 0) {
                const int64_t at = (int64_t)kh * a.slot_cap[0] + map.leaf_at(kh, 0);
                has0 = __ldcg(a.kept_ids[0] + at) == 0 && ((__ldcg(a.kept_mask[0] + at) >> h) & 1u);
            }
            add = !has0;
        }
        const float s0 = warp_sum(lane_dot<CPL>(qh, k0));
        if (lane == 0) hs0[h] = add ? s0 : -INFINITY;
    }
    {
        const int q = tid % NQ, sp = tid / NQ;
        const int h = q / (HD / 4), e4 = (q % (HD / 4)) * 4;
        const int i0 = n * sp / NS, i1 = n * (sp + 1) / NS;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float M = -INFINITY, L = 0.f;
        constexpr int CB = 8;  // partials loaded per batch
#pragma unroll 1
        for (int i = i0; i < i1; i += CB) {
            float m[CB], l[CB];
            float4 o[CB];
#pragma unroll
            for (int u = 0; u < CB; ++u) {
                if (i + u < i1) {
                    const float *pb = a.part + (((int64_t)(b0 + i + u) * h_kv + kh) * G + h) * prec<HD>();
                    m[u] = __ldcg(pb + HD);
                    l[u] = __ldcg(pb + HD + 1);
                    o[u] = __ldcg(reinterpret_cast<const float4 *>(pb + e4));
                } else {
                    m[u] = -INFINITY;
                    l[u] = 0.f;
                    o[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int u = 0; u < CB; ++u) {
                // a part with no token of head h has max -inf and is skipped
                if (m[u] == -INFINITY) continue;
                if (m[u] > M) {
                    const float r = exp2f(M - m[u]);
                    acc.x *= r;
                    acc.y *= r;
                    acc.z *= r;
                    acc.w *= r;
                    L *= r;
                    M = m[u];
                }
                const float w = exp2f(m[u] - M);
                acc.x = fmaf(w, o[u].x, acc.x);
                acc.y = fmaf(w, o[u].y, acc.y);
                acc.z = fmaf(w, o[u].z, acc.z);
                acc.w = fmaf(w, o[u].w, acc.w);
                L = fmaf(w, l[u], L);
            }
        }
        racc[tid] = acc;
        rml[tid] = M;
        rml[GT + tid] = L;
    }
    gsync();
    if (tid < NQ) {
        const int h = tid / (HD / 4), e4 = (tid % (HD / 4)) * 4;
        const float s0 = hs0[h];
        float M = s0;
#pragma unroll 1
        for (int sp = 0; sp < NS; ++sp) M = fmaxf(M, rml[sp * NQ + tid]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float L = 0.f;
#pragma unroll 1
        for (int sp = 0; sp < NS; ++sp) {
            const float m = rml[sp * NQ + tid];
            if (m == -INFINITY) continue;
            const float r = exp2f(m - M);
            const float4 x = racc[sp * NQ + tid];
            acc.x = fmaf(r, x.x, acc.x);
            acc.y = fmaf(r, x.y, acc.y);
            acc.z = fmaf(r, x.z, acc.z);
            acc.w = fmaf(r, x.w, acc.w);
            L = fmaf(r, rml[GT + sp * NQ + tid], L);
        }
        if (s0 != -INFINITY) {
            const float ws = exp2f(s0 - M);
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
            L += ws;
        }
        const float inv = 1.f / L;
        float4 r = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        *reinterpret_cast<float4 *>(a.out + (int64_t)(kh * G + h) * HD + e4) = r;
    }
}

}  // namespace zha
