// zha_route.cuh -- frontier scoring of one routing level (sm_100a).
//
// Routing ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢";
// "Zyphra 分层注意力（ZHA）…", section "机制拆解：树形索引如何高效筛选长上下文"): at
// each level the query scores every node of the frontier -- every top node,
// then the children of the nodes kept one level up -- with the tangent-plane
// estimate est(q) = max_j (b_j + q.g_j / sqrt(d)).
//
// The frontier of KV head kh is the union over its G query heads: the
// children of every node kept by any head, each carrying the bitmask of heads
// that kept its parent.  A node's summary is read from HBM once and scored for
// all G heads (a [R x d] x [d x G] product per node): lane l of a warp owns
// the d-slice [l*VEC, (l+1)*VEC) of every g row, forms the G*R partial dot
// products per node, and a reduce-scatter leaves each lane whole sums.
#pragma once

#include "zha_device.cuh"
#include "zha_internal.cuh"

namespace zha {

template <int HD, int R, int G>
struct RouteCfg {
    static constexpr int VEC = HD / 32;
    static constexpr int NPW = (G * R >= 32) ? 1 : 32 / (G * R);  // nodes per warp pass
    static constexpr int V = NPW * G * R;                          // partial dots per lane
    static constexpr int K = V / 32;                               // sums per lane after reduce-scatter
};

// Node id, validity and head mask of frontier slot s at level l of KV head kh.
template <int G>
__device__ __forceinline__ void slot_info(const Decode &a, int l, int kh, bool top, int64_t S, int64_t s,
                                          int32_t &node, bool &ok, uint32_t &msk) {
    if (s >= S) {
        node = 0; ok = false; msk = 0;
        return;
    }
    if (top) {
        node = (int32_t)s; ok = true; msk = (1u << G) - 1u;
        return;
    }
    const int c = a.t.c;
    const int64_t k = a.t.c_log2 >= 0 ? (s >> a.t.c_log2) : s / c;
    const int o = (int)(s - k * c);
    const int64_t pbase = (int64_t)kh * a.t.node_cap[l];
    const int32_t pid = __ldcg(a.kept_ids[l] + pbase + k);
    node = pid * c + o;
    ok = node < a.t.n_level[l - 1];
    msk = ok ? (uint32_t)__ldcg(a.kept_mask[l] + pbase + k) : 0u;
}

// Frontier size of KV head kh at level l (every top node, or c children per
// node kept one level up).
__device__ __forceinline__ int64_t frontier_size(const Decode &a, int l, int kh) {
    return (l == a.t.D) ? (int64_t)a.t.n_level[l - 1] : (int64_t)a.t.c * __ldcg(a.kept_cnt + l * a.t.h_kv + kh);
}

// Score the slots of KV head kh handled by this CTA (warp-strided over
// `nwarps` warps of `ncta` CTAs; this is CTA `bi`), write the scores (-inf
// where a head does not need the slot) and node ids, and the CTA's maximum
// per head to pmax[kh][bi].  Called by warps 0-7; `wsm` holds 256 floats.
template <int HD, int R, int G>
__device__ void route_score(const Decode &a, int l, int kh, int bi, int ncta, int64_t S, float *wsm) {
    using C = RouteCfg<HD, R, G>;
    constexpr int VEC = C::VEC, NPW = C::NPW, V = C::V, K = C::K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool top = (l == a.t.D);
    float qs[G][VEC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        Vec<float, VEC>::load(a.q + (int64_t)(kh * G + h) * HD + lane * VEC, qs[h]);
#pragma unroll
        for (int e = 0; e < VEC; ++e) qs[h][e] *= a.t.scale;
    }
    const int64_t cap = a.t.node_cap[l - 1];
    const float *gb = a.t.g[l - 1] + (int64_t)kh * cap * R * HD;
    const float *bb = a.t.b[l - 1] + (int64_t)kh * cap * R;
    float *scores = a.scores + (int64_t)kh * a.score_cap * G;
    int32_t *snode = a.slot_node + (int64_t)kh * a.score_cap;
    const int idx0 = lane * K;
    const int my_i = idx0 / (G * R), my_h = (idx0 / R) % G, my_j0 = idx0 % R;
    float lmax = -INFINITY;
    const int nwarps = GT / 32;
    for (int64_t grp = (int64_t)bi * nwarps + warp; grp * NPW < S; grp += (int64_t)ncta * nwarps) {
        float v[V];
#pragma unroll
        for (int i = 0; i < NPW; ++i) {
            int32_t node; bool ok; uint32_t msk;
            slot_info<G>(a, l, kh, top, S, grp * NPW + i, node, ok, msk);
#pragma unroll
            for (int j = 0; j < R; ++j) {
                float gs[VEC];
                if (ok) {
                    Vec<float, VEC>::load(gb + ((int64_t)node * R + j) * HD + lane * VEC, gs);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) gs[e] = 0.f;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) v[(i * G + h) * R + j] = lane_dot<VEC>(qs[h], gs);
            }
        }
        reduce_scatter<V>(v, lane);
        const int64_t s = grp * NPW + my_i;
        int32_t node; bool ok; uint32_t msk;
        slot_info<G>(a, l, kh, top, S, s, node, ok, msk);
        float est = -INFINITY;
        if (ok) {
#pragma unroll
            for (int t = 0; t < K; ++t) est = fmaxf(est, __ldg(bb + (int64_t)node * R + my_j0 + t) + v[t]);
        }
#pragma unroll
        for (int off = 1; off < R / K; off <<= 1) est = fmaxf(est, __shfl_xor_sync(FULL, est, off));
        if (my_j0 == 0 && s < S) {
            const bool need = ok && ((msk >> my_h) & 1u);
            scores[s * G + my_h] = need ? est : -INFINITY;
            if (need) lmax = fmaxf(lmax, est);
            if (my_h == 0) snode[s] = ok ? node : -1;
        }
    }
    // the CTA's maximum per head
    wsm[threadIdx.x] = (my_j0 == 0) ? lmax : -INFINITY;
    gsync();
    if (threadIdx.x < G) {
        float mx = -INFINITY;
        for (int t = 0; t < GT; ++t) {
            const int li0 = (t & 31) * K;
            if (((li0 / R) % G) == (int)threadIdx.x) mx = fmaxf(mx, wsm[t]);
        }
        a.pmax[((int64_t)kh * a.pmax_cap + bi) * G + threadIdx.x] = mx;
    }
    gsync();
}

}  // namespace zha
