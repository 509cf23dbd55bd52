// zha_build.cu -- summary-tree build and incremental append (sm_100a).
//
// Leaf summary ("ZHA 用树形稀疏注意力改造现有大模型", section
// "稀疏注意力为什么还会被索引拖慢": chunk summaries from reference queries, a
// tangent-plane estimate of the chunk's log attention mass, max over planes):
//   s_ij = r_j.k_i / sqrt(d),  m_j = logsumexp_i s_ij,
//   g_j  = sum_i exp(s_ij - m_j) k_i,  b_j = m_j - r_j.g_j / sqrt(d).
// Parent summary ("Zyphra 分层注意力（ZHA）…", section
// "机制拆解：树形索引如何高效筛选长上下文": summaries grouped and compressed
// recursively):
//   e_ch,j = max_j' (b_ch,j' + r_j.g_ch,j' / sqrt(d))   (child estimate at r_j)
//   m_j = logsumexp_ch e_ch,j,  g_j = sum_ch exp(e_ch,j - m_j) g_ch,j,
//   b_j = m_j - r_j.g_j / sqrt(d).
// Append (tree maintenance, rit.work article, section "Замеры подтверждают
// качество, а предельный выигрыш пока рассчитан"): the new row's leaf and its
// ancestors are recomputed by the same device functions as the build, so an
// appended tree is bit-identical to a tree built over the longer cache.
//
// Work layout: one warp per leaf tile / per parent node.  Lane l owns the
// d-slice [l*VEC, (l+1)*VEC) of every key, reference query and g row; dot
// products are per-lane fmaf chains followed by a 32-lane reduce-scatter.
// The kernels are bound by HBM for R = 1 and by fp32 FMA for R = 16.
#include <cuda_bf16.h>

#include <algorithm>

#include "zha_build_mma.cuh"
#include "zha_device.cuh"
#include "zha_internal.cuh"
#include "zha_tma.cuh"

namespace zha {

template <int HD, int R>
__device__ __forceinline__ void load_ref(const float *ref_h, float (&rj)[R][HD / 32], int lane) {
#pragma unroll
    for (int j = 0; j < R; ++j) Vec<float, HD / 32>::load(ref_h + j * HD + lane * (HD / 32), rj[j]);
}

// The router's bf16 copy of one plane (this lane's VEC elements of g_j) and
// its plane offset recomputed from that copy, b~_j = m_j - r_j.g~_j/sqrt(d),
// so that the rounded plane still passes through (r_j, m_j).  The dot
// product takes the same order as b_j's.  `writer` stores the offset.
template <int VEC>
__device__ __forceinline__ void router_plane(const float (&g)[VEC], const float (&r)[VEC], float m, float scale,
                                             uint16_t *g16dst, float *b16dst, int lane, int writer) {
    float gq[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        const __nv_bfloat16 h = __float2bfloat16_rn(g[e]);
        g16dst[e] = __bfloat16_as_ushort(h);
        gq[e] = __bfloat162float(h);
    }
    const float dot = warp_sum(lane_dot<VEC>(r, gq));
    if (lane == writer) *b16dst = m - scale * dot;
}

// Tokens per leaf tile processed by one warp: a whole number of leaves and at
// least one reduce-scatter batch (32 / R tokens).
__host__ __device__ inline int leaf_tile_tokens(int c, int R) {
    const int tpr = 32 / R;
    return ((tpr + c - 1) / c) * c;
}

template <typename KT, int HD, int R>
struct LeafOps {
    static constexpr int VEC = HD / 32;
    static constexpr int TPR = 32 / R;

    // Summaries of the leaves covering tokens [tok0, tok0 + ntok) of one head
    // (tok0 a multiple of c).  sh: warp-private shared scratch of
    // ntok*R + (ntok/c + 1)*R floats.
    // g16L / b16L: the router's bf16 copy and its offsets (null: none).
    static __device__ void tile(const KT *__restrict__ Kh, int64_t tok0, int ntok, int c,
                                const float (&rj)[R][VEC], float scale, float *__restrict__ gL,
                                float *__restrict__ bL, float *__restrict__ mL, float *sh, int lane,
                                uint16_t *__restrict__ g16L, float *__restrict__ b16L) {
        float *s_sh = sh;
        const int nleaf = (ntok + c - 1) / c;
        float *m_sh = sh + ntok * R;
        const int64_t leaf0 = tok0 / c;
        // pass 1: scaled scores of every (token, plane)
        for (int t0 = 0; t0 < ntok; t0 += TPR) {
            float v[32];
#pragma unroll
            for (int t = 0; t < TPR; ++t) {
                const int i = t0 + t;
                float k[VEC];
                if (i < ntok) {
                    Vec<KT, VEC>::load(Kh + (tok0 + i) * HD + lane * VEC, k);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) k[e] = 0.f;
                }
#pragma unroll
                for (int j = 0; j < R; ++j) v[t * R + j] = lane_dot<VEC>(rj[j], k);
            }
            reduce_scatter<32>(v, lane);
            const int i = t0 + lane / R;
            if (i < ntok) s_sh[i * R + (lane % R)] = v[0] * scale;
        }
        __syncwarp();
        // log mass per (leaf, plane) in token order; weights in place
        for (int pair = lane; pair < nleaf * R; pair += 32) {
            const int lf = pair / R, j = pair % R;
            const int i0 = lf * c, i1 = min(i0 + c, ntok);
            float mx = -INFINITY;
            for (int i = i0; i < i1; ++i) mx = fmaxf(mx, s_sh[i * R + j]);
            float sum = 0.f;
            for (int i = i0; i < i1; ++i) sum += expf(s_sh[i * R + j] - mx);
            const float m = mx + logf(sum);
            for (int i = i0; i < i1; ++i) s_sh[i * R + j] = expf(s_sh[i * R + j] - m);
            m_sh[pair] = m;
            mL[(leaf0 + lf) * R + j] = m;
        }
        __syncwarp();
        // g_j = sum_i w_ij k_i (token order), then the plane offsets
        for (int lf = 0; lf < nleaf; ++lf) {
            const int i0 = lf * c, i1 = min(i0 + c, ntok);
            float acc[R][VEC];
#pragma unroll
            for (int j = 0; j < R; ++j)
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[j][e] = 0.f;
            for (int i = i0; i < i1; ++i) {
                float k[VEC];
                Vec<KT, VEC>::load(Kh + (tok0 + i) * HD + lane * VEC, k);
#pragma unroll
                for (int j = 0; j < R; ++j) {
                    const float w = s_sh[i * R + j];
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[j][e] = fmaf(w, k[e], acc[j][e]);
                }
            }
            const int64_t node = leaf0 + lf;
#pragma unroll
            for (int j = 0; j < R; ++j) {
                float *dst = gL + (node * R + j) * HD + lane * VEC;
#pragma unroll
                for (int e = 0; e < VEC; ++e) dst[e] = acc[j][e];
                const float dot = warp_sum(lane_dot<VEC>(rj[j], acc[j]));
                if (lane == (j & 31)) bL[node * R + j] = m_sh[lf * R + j] - scale * dot;
                if (g16L)
                    router_plane<VEC>(acc[j], rj[j], m_sh[lf * R + j], scale,
                                      g16L + (node * R + j) * HD + lane * VEC, b16L + node * R + j, lane, j & 31);
            }
        }
        __syncwarp();
    }
};

template <int HD, int R>
struct ParentOps {
    static constexpr int VEC = HD / 32;

    // Summary of level-l node n from its nch children (rows ch0 .. ch0+nch-1
    // of level l-1; pointers for this head).  sh: warp-private shared scratch
    // of nch*R + R floats.
    static __device__ void node(const float *__restrict__ gC, const float *__restrict__ bC, int64_t ch0,
                                int nch, const float (&rj)[R][VEC], float scale, float *__restrict__ gP,
                                float *__restrict__ bP, float *__restrict__ mP, int64_t n, float *sh,
                                int lane, uint16_t *__restrict__ g16P, float *__restrict__ b16P) {
        float *e_sh = sh;
        float *m_sh = sh + nch * R;
        // child estimates at every reference query
        if constexpr (R == 1) {
            for (int c0 = 0; c0 < nch; c0 += 32) {
                float v[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const int ch = c0 + t;
                    if (ch < nch) {
                        float gs[VEC];
                        Vec<float, VEC>::load(gC + (ch0 + ch) * HD + lane * VEC, gs);
                        v[t] = lane_dot<VEC>(rj[0], gs);
                    } else {
                        v[t] = 0.f;
                    }
                }
                reduce_scatter<32>(v, lane);
                const int ch = c0 + lane;
                if (ch < nch) e_sh[ch] = bC[ch0 + ch] + scale * v[0];
            }
        } else {
            constexpr int JP = 32 / R;
            for (int ch = 0; ch < nch; ++ch) {
                float emax = -INFINITY;
                for (int jp0 = 0; jp0 < R; jp0 += JP) {
                    float v[32];
#pragma unroll
                    for (int t = 0; t < JP; ++t) {
                        float gs[VEC];
                        Vec<float, VEC>::load(gC + ((ch0 + ch) * R + jp0 + t) * HD + lane * VEC, gs);
#pragma unroll
                        for (int j = 0; j < R; ++j) v[t * R + j] = lane_dot<VEC>(rj[j], gs);
                    }
                    reduce_scatter<32>(v, lane);
                    const float val = bC[(ch0 + ch) * R + jp0 + lane / R] + scale * v[0];
                    emax = fmaxf(emax, val);
                }
#pragma unroll
                for (int off = R; off < 32; off <<= 1) emax = fmaxf(emax, __shfl_xor_sync(FULL, emax, off));
                if (lane < R) e_sh[ch * R + lane] = emax;
            }
        }
        __syncwarp();
        if (lane < R) {
            const int j = lane;
            float mx = -INFINITY;
            for (int ch = 0; ch < nch; ++ch) mx = fmaxf(mx, e_sh[ch * R + j]);
            float sum = 0.f;
            for (int ch = 0; ch < nch; ++ch) sum += expf(e_sh[ch * R + j] - mx);
            const float m = mx + logf(sum);
            for (int ch = 0; ch < nch; ++ch) e_sh[ch * R + j] = expf(e_sh[ch * R + j] - m);
            m_sh[j] = m;
            mP[n * R + j] = m;
        }
        __syncwarp();
        float acc[R][VEC];
#pragma unroll
        for (int j = 0; j < R; ++j)
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[j][e] = 0.f;
        for (int ch = 0; ch < nch; ++ch) {
#pragma unroll
            for (int j = 0; j < R; ++j) {
                float gs[VEC];
                Vec<float, VEC>::load(gC + ((ch0 + ch) * R + j) * HD + lane * VEC, gs);
                const float w = e_sh[ch * R + j];
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[j][e] = fmaf(w, gs[e], acc[j][e]);
            }
        }
#pragma unroll
        for (int j = 0; j < R; ++j) {
            float *dst = gP + (n * R + j) * HD + lane * VEC;
#pragma unroll
            for (int e = 0; e < VEC; ++e) dst[e] = acc[j][e];
            const float dot = warp_sum(lane_dot<VEC>(rj[j], acc[j]));
            if (lane == (j & 31)) bP[n * R + j] = m_sh[j] - scale * dot;
            if (g16P)
                router_plane<VEC>(acc[j], rj[j], m_sh[j], scale, g16P + (n * R + j) * HD + lane * VEC,
                                  b16P + n * R + j, lane, j & 31);
        }
        __syncwarp();
    }
};

// ---- kernels ---------------------------------------------------------------

template <typename KT, int HD, int R>
__global__ void __launch_bounds__(BUILD_THREADS) k_build_leaves(Tree t) {
    extern __shared__ __align__(16) float bsm[];
    constexpr int VEC = HD / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tt = leaf_tile_tokens(t.c, R);
    float *sh = bsm + warp * (tt * R + (tt / t.c + 1) * R);
    const int64_t tiles = (t.n_tokens + tt - 1) / tt;
    const int64_t total = tiles * t.h_kv;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    float rj[R][VEC];
    int cur_kh = -1;
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; w < total; w += nwarps) {
        const int kh = (int)(w / tiles);
        const int64_t tile = w % tiles;
        if (kh != cur_kh) {
            load_ref<HD, R>(t.ref + (int64_t)kh * R * HD, rj, lane);
            cur_kh = kh;
        }
        const int64_t tok0 = tile * tt;
        const int ntok = (int)min((int64_t)tt, t.n_tokens - tok0);
        const KT *Kh = reinterpret_cast<const KT *>(t.K) + (int64_t)kh * t.kv_cap * HD;
        const int64_t nc = t.node_cap[0];
        LeafOps<KT, HD, R>::tile(Kh, tok0, ntok, t.c, rj, t.scale, t.g[0] + (int64_t)kh * nc * R * HD,
                                 t.b[0] + (int64_t)kh * nc * R, t.m[0] + (int64_t)kh * nc * R, sh, lane,
                                 t.g16[0] ? t.g16[0] + (int64_t)kh * nc * R * HD : nullptr,
                                 t.g16[0] ? t.b16[0] + (int64_t)kh * nc * R : nullptr);
    }
}

template <int HD, int R>
__global__ void __launch_bounds__(BUILD_THREADS) k_build_parents(Tree t, int level) {
    extern __shared__ __align__(16) float bsm[];
    constexpr int VEC = HD / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float *sh = bsm + warp * (t.c * R + R);
    const int64_t nodes = t.n_level[level - 1];
    const int64_t nbelow = t.n_level[level - 2];
    const int64_t total = nodes * t.h_kv;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t capP = t.node_cap[level - 1], capC = t.node_cap[level - 2];
    float rj[R][VEC];
    int cur_kh = -1;
    for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; w < total; w += nwarps) {
        const int kh = (int)(w / nodes);
        const int64_t n = w % nodes;
        if (kh != cur_kh) {
            load_ref<HD, R>(t.ref + (int64_t)kh * R * HD, rj, lane);
            cur_kh = kh;
        }
        const int64_t ch0 = n * t.c;
        const int nch = (int)min((int64_t)t.c, nbelow - ch0);
        ParentOps<HD, R>::node(t.g[level - 2] + (int64_t)kh * capC * R * HD, t.b[level - 2] + (int64_t)kh * capC * R,
                               ch0, nch, rj, t.scale, t.g[level - 1] + (int64_t)kh * capP * R * HD,
                               t.b[level - 1] + (int64_t)kh * capP * R, t.m[level - 1] + (int64_t)kh * capP * R,
                               n, sh, lane, t.g16[level - 1] ? t.g16[level - 1] + (int64_t)kh * capP * R * HD : nullptr,
                               t.g16[level - 1] ? t.b16[level - 1] + (int64_t)kh * capP * R : nullptr);
    }
}

// Append, one plane at a time: warp j of the KV head's CTA recomputes plane
// j (reference query r_j) of the leaf holding the new row and of every
// ancestor.  Each plane of a node depends only on that plane's reference
// query and on the children's rows, so the planes are independent; every sum
// below takes the same order as in LeafOps / ParentOps (a dot product is a
// per-lane fmaf chain and a 32-lane butterfly, here as a reduce-scatter of 32
// dot products; log-sum-exp and weighted sums run over tokens / children in
// order), so the appended tree is bit-identical to a build.
template <typename KT, int HD, int R>
struct PlaneOps {
    static constexpr int VEC = HD / 32;

    // Leaf n of this head, plane j: tokens [tok0, tok0 + ntok).  sh: warp-
    // private shared scratch of ntok floats.
    // Kr: the leaf's rows, row i at Kr + i * HD (the cache, or a shared copy).
    static __device__ void leaf(const KT *Kr, int ntok, const float (&r)[VEC], int j,
                                float scale, float *__restrict__ gL, float *__restrict__ bL, float *__restrict__ mL,
                                int64_t n, float *sh, int lane, uint16_t *__restrict__ g16L,
                                float *__restrict__ b16L) {
        for (int i0 = 0; i0 < ntok; i0 += 32) {
            float v[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                float k[VEC];
                if (i0 + t < ntok) {
                    Vec<KT, VEC>::load(Kr + (int64_t)(i0 + t) * HD + lane * VEC, k);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) k[e] = 0.f;
                }
                v[t] = lane_dot<VEC>(r, k);
            }
            reduce_scatter<32>(v, lane);
            if (i0 + lane < ntok) sh[i0 + lane] = v[0] * scale;
        }
        __syncwarp();
        float m = 0.f;
        if (lane == 0) {
            float mx = -INFINITY;
            for (int i = 0; i < ntok; ++i) mx = fmaxf(mx, sh[i]);
            float sum = 0.f;
            for (int i = 0; i < ntok; ++i) sum += expf(sh[i] - mx);
            m = mx + logf(sum);
            mL[n * R + j] = m;
        }
        m = __shfl_sync(FULL, m, 0);
        __syncwarp();
        for (int i = lane; i < ntok; i += 32) sh[i] = expf(sh[i] - m);
        __syncwarp();
        float acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        for (int i = 0; i < ntok; ++i) {
            float k[VEC];
            Vec<KT, VEC>::load(Kr + (int64_t)i * HD + lane * VEC, k);
            const float w = sh[i];
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = fmaf(w, k[e], acc[e]);
        }
        float *dst = gL + (n * R + j) * HD + lane * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dst[e] = acc[e];
        const float dot = warp_sum(lane_dot<VEC>(r, acc));
        if (lane == 0) bL[n * R + j] = m - scale * dot;
        if (g16L) router_plane<VEC>(acc, r, m, scale, g16L + (n * R + j) * HD + lane * VEC, b16L + n * R + j, lane, 0);
        __syncwarp();
    }

    // Node n of this level, plane j, from its nch children (rows ch0 ..
    // ch0 + nch - 1 of the level below).  sh: warp-private scratch of nch floats.
    // gr / br: the children's g rows and plane offsets, child i's plane j' at
    // gr + (i * R + j') * HD and br[i * R + j'] (the store, or a shared copy).
    static __device__ void parent(const float *gr, const float *br, int nch,
                                  const float (&r)[VEC], int j, float scale, float *__restrict__ gP,
                                  float *__restrict__ bP, float *__restrict__ mP, int64_t n, float *sh, int lane,
                                  uint16_t *__restrict__ g16P, float *__restrict__ b16P) {
        // child estimates at r_j: max over the child's planes j'
        constexpr int CPB = 32 / R;  // children per batch of 32 dot products
        for (int c0 = 0; c0 < nch; c0 += CPB) {
            float v[32];
#pragma unroll
            for (int t = 0; t < CPB; ++t) {
#pragma unroll
                for (int jp = 0; jp < R; ++jp) {
                    float gs[VEC];
                    if (c0 + t < nch) {
                        Vec<float, VEC>::load(gr + ((int64_t)(c0 + t) * R + jp) * HD + lane * VEC, gs);
                    } else {
#pragma unroll
                        for (int e = 0; e < VEC; ++e) gs[e] = 0.f;
                    }
                    v[t * R + jp] = lane_dot<VEC>(r, gs);
                }
            }
            reduce_scatter<32>(v, lane);
            const int t = lane / R, jp = lane % R;
            float val = -INFINITY;
            if (c0 + t < nch) val = br[(c0 + t) * R + jp] + scale * v[0];
#pragma unroll
            for (int off = 1; off < R; off <<= 1) val = fmaxf(val, __shfl_xor_sync(FULL, val, off));
            if (jp == 0 && c0 + t < nch) sh[c0 + t] = val;
        }
        __syncwarp();
        float m = 0.f;
        if (lane == 0) {
            float mx = -INFINITY;
            for (int ch = 0; ch < nch; ++ch) mx = fmaxf(mx, sh[ch]);
            float sum = 0.f;
            for (int ch = 0; ch < nch; ++ch) sum += expf(sh[ch] - mx);
            m = mx + logf(sum);
            for (int ch = 0; ch < nch; ++ch) sh[ch] = expf(sh[ch] - m);
            mP[n * R + j] = m;
        }
        m = __shfl_sync(FULL, m, 0);
        __syncwarp();
        float acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
        for (int ch = 0; ch < nch; ++ch) {
            float gs[VEC];
            Vec<float, VEC>::load(gr + ((int64_t)ch * R + j) * HD + lane * VEC, gs);
            const float w = sh[ch];
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = fmaf(w, gs[e], acc[e]);
        }
        float *dst = gP + (n * R + j) * HD + lane * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dst[e] = acc[e];
        const float dot = warp_sum(lane_dot<VEC>(r, acc));
        if (lane == 0) bP[n * R + j] = m - scale * dot;
        if (g16P) router_plane<VEC>(acc, r, m, scale, g16P + (n * R + j) * HD + lane * VEC, b16P + n * R + j, lane, 0);
        __syncwarp();
    }
};

constexpr int64_t APPEND_STAGE = 64 * 1024;  // shared copy of the rows every plane reads

// Bytes of that copy for a tree (0: planes read the rows from global memory):
// a full leaf's keys or a full node's children, whichever is larger, each
// only when it fits APPEND_STAGE.  The kernel stages a level's rows when they
// fit this size.
template <typename KT, int HD, int R>
__host__ __device__ __forceinline__ int64_t append_stage_bytes(int c, int D) {
    if (R == 1) return 0;
    const int64_t leaf_bytes = (int64_t)c * HD * (int64_t)sizeof(KT);
    const int64_t child_bytes = D > 1 ? (int64_t)c * R * (HD + 1) * 4 : 0;  // g rows, then plane offsets
    int64_t need = 0;
    if (leaf_bytes <= APPEND_STAGE) need = leaf_bytes;
    if (child_bytes <= APPEND_STAGE && child_bytes > need) need = child_bytes;
    return need;
}

// Copy `bytes` (a multiple of 16, both ends 16-byte aligned) from global to
// shared memory with every thread of the CTA, all loads of a thread in flight
// at once.  Coherent loads: the rows may have been written by this CTA.
__device__ __forceinline__ void stage_copy(void *dst, const void *src, int64_t bytes) {
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    const int64_t n = bytes / 16;
#pragma unroll 8
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) d[i] = __ldcg(s + i);
}

// One CTA per KV head, one warp per plane: store the new row, prefetch every
// ancestor's children into L2, then recompute the leaf holding the row and
// every ancestor, a level at a time.  t.n_tokens and t.n_level already count
// the new token.
template <typename KT, int HD, int R>
__global__ void __launch_bounds__(32 * R) k_append(Tree t, const KT *__restrict__ knew, const KT *__restrict__ vnew) {
    extern __shared__ __align__(16) float bsm[];
    constexpr int VEC = HD / 32;
    const int lane = threadIdx.x & 31, j = threadIdx.x >> 5;
    const int kh = blockIdx.x;
    const int64_t pos = t.n_tokens - 1;
    // a decode launched next may start its launch now (it waits for this grid)
    griddep_launch_dependents();
    KT *Kh = const_cast<KT *>(reinterpret_cast<const KT *>(t.K)) + (int64_t)kh * t.kv_cap * HD;
    KT *Vh = const_cast<KT *>(reinterpret_cast<const KT *>(t.V)) + (int64_t)kh * t.kv_cap * HD;
    if (j == 0) {
        for (int e = lane; e < HD; e += 32) {
            Kh[pos * HD + e] = knew[kh * HD + e];
            Vh[pos * HD + e] = vnew[kh * HD + e];
        }
    }
    // the children of every ancestor: 128-byte lines into L2
    {
        int64_t n = pos / t.c;
        for (int level = 2; level <= t.D; ++level) {
            n /= t.c;
            const int64_t ch0 = n * t.c;
            const int nch = (int)min((int64_t)t.c, (int64_t)t.n_level[level - 2] - ch0);
            const float *g = t.g[level - 2] + ((int64_t)kh * t.node_cap[level - 2] + ch0) * R * HD;
            const int64_t lines = ((int64_t)nch * R * HD * 4 + 127) / 128;
            for (int64_t i = threadIdx.x; i < lines; i += blockDim.x)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char *>(g) + i * 128));
        }
    }
    __syncthreads();
    float r[VEC];
    Vec<float, VEC>::load(t.ref + ((int64_t)kh * R + j) * HD + lane * VEC, r);
    float *sh = bsm + j * (t.c > 32 ? t.c : 32);
    // rows every plane's warp reads (the leaf's keys, then each level's
    // children) go to shared memory once when they fit the staged copy
    unsigned char *stg = reinterpret_cast<unsigned char *>(bsm + R * (t.c > 32 ? t.c : 32));
    const int64_t stage_cap = append_stage_bytes<KT, HD, R>(t.c, t.D);
    int64_t n = pos / t.c;
    bool leaf_done = false;
    if constexpr (sizeof(KT) == 2 && R == LM_R) {
        if (leaf_mma_applies(t.kv_dtype, HD, R, t.c)) {
            // the leaf's unit, recomputed as the tensor-core build does it
            unsigned char *lm = stg + stage_cap;
            const int passes = leaf_mma_load_ref<HD>(t.ref + (int64_t)kh * R * HD, lm);
            if (j == 0) {
                const int U = leaf_mma_unit_tokens(t.c);
                const int64_t u = pos / U;
                const uint16_t *Kb = reinterpret_cast<const uint16_t *>(Kh);
                TileRegs<HD> nxt;
                tile_load<HD>(Kb, u * U, t.n_tokens, nxt, lane);
                leaf_mma_unit<HD>(t, kh, u, lm, reinterpret_cast<uint16_t *>(lm + LeafMma<HD>::off_k), passes, nxt,
                                  -1, lane);
            }
            leaf_done = true;
        }
    }
    if (!leaf_done) {
        const int64_t tok0 = n * t.c;
        const int ntok = (int)(t.n_tokens - tok0);
        const int64_t nc = t.node_cap[0];
        const KT *Kr = Kh + tok0 * HD;
        const int64_t bytes = (int64_t)ntok * HD * sizeof(KT);
        if (bytes <= stage_cap) {
            stage_copy(stg, Kr, bytes);
            __syncthreads();
            Kr = reinterpret_cast<const KT *>(stg);
        }
        PlaneOps<KT, HD, R>::leaf(Kr, ntok, r, j, t.scale, t.g[0] + (int64_t)kh * nc * R * HD,
                                  t.b[0] + (int64_t)kh * nc * R, t.m[0] + (int64_t)kh * nc * R, n, sh, lane,
                                  t.g16[0] ? t.g16[0] + (int64_t)kh * nc * R * HD : nullptr,
                                  t.g16[0] ? t.b16[0] + (int64_t)kh * nc * R : nullptr);
    }
    __syncthreads();
    for (int level = 2; level <= t.D; ++level) {
        n /= t.c;
        const int64_t ch0 = n * t.c;
        const int nch = (int)min((int64_t)t.c, (int64_t)t.n_level[level - 2] - ch0);
        const int64_t capP = t.node_cap[level - 1], capC = t.node_cap[level - 2];
        const float *gr = t.g[level - 2] + ((int64_t)kh * capC + ch0) * R * HD;
        const float *br = t.b[level - 2] + ((int64_t)kh * capC + ch0) * R;
        const int64_t bytes = (int64_t)nch * R * HD * 4, bbytes = (int64_t)nch * R * 4;
        if (bytes + bbytes <= stage_cap && bbytes % 16 == 0) {
            stage_copy(stg, gr, bytes);
            stage_copy(stg + bytes, br, bbytes);
            __syncthreads();
            gr = reinterpret_cast<const float *>(stg);
            br = reinterpret_cast<const float *>(stg + bytes);
        }
        PlaneOps<KT, HD, R>::parent(gr, br, nch, r, j, t.scale,
                                    t.g[level - 1] + (int64_t)kh * capP * R * HD, t.b[level - 1] + (int64_t)kh * capP * R,
                                    t.m[level - 1] + (int64_t)kh * capP * R, n, sh, lane,
                                    t.g16[level - 1] ? t.g16[level - 1] + (int64_t)kh * capP * R * HD : nullptr,
                                    t.g16[level - 1] ? t.b16[level - 1] + (int64_t)kh * capP * R : nullptr);
        __syncthreads();
    }
}

// ---- dispatch ----------------------------------------------------------------

template <typename KT, int HD, int R>
static cudaError_t build_impl(const Tree &t, cudaStream_t s, int n_sm) {
    const int warps = BUILD_THREADS / 32;
    static PerDeviceMax<> leaf_attr, parent_attr;
    cudaError_t err;
    bool leaves_done = false;
    if constexpr (sizeof(KT) == 2 && R == LM_R) {
        if (leaf_mma_applies(t.kv_dtype, HD, R, t.c)) {
            // bf16 cache, 16 reference queries: leaves on the tensor cores
            static PerDeviceMax<> mma_attr;
            const size_t smem = LeafMma<HD>::bytes(LM_WARPS);
            err = allow_smem(k_build_leaves_mma<HD>, smem, mma_attr);
            if (err != cudaSuccess) return err;
            const int U = leaf_mma_unit_tokens(t.c);
            const int64_t units = (t.n_tokens + U - 1) / U;
            const int gx = (int)std::max<int64_t>(
                1, std::min<int64_t>((units + LM_WARPS - 1) / LM_WARPS, std::max(1, n_sm * 4 / t.h_kv)));
            k_build_leaves_mma<HD><<<dim3(gx, t.h_kv), LM_WARPS * 32, smem, s>>>(t);
            err = cudaGetLastError();
            if (err != cudaSuccess) return err;
            leaves_done = true;
        }
    }
    if (!leaves_done) {
        const int tt = leaf_tile_tokens(t.c, R);
        size_t smem = (size_t)warps * (tt * R + (tt / t.c + 1) * R) * sizeof(float);
        err = allow_smem(k_build_leaves<KT, HD, R>, smem, leaf_attr);
        if (err != cudaSuccess) return err;
        const int64_t tiles = ((t.n_tokens + tt - 1) / tt) * t.h_kv;
        int grid = (int)std::min<int64_t>((tiles + warps - 1) / warps, (int64_t)n_sm * 8);
        k_build_leaves<KT, HD, R><<<grid, BUILD_THREADS, smem, s>>>(t);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    size_t psmem = (size_t)warps * (t.c * R + R) * sizeof(float);
    err = allow_smem(k_build_parents<HD, R>, psmem, parent_attr);
    if (err != cudaSuccess) return err;
    for (int level = 2; level <= t.D; ++level) {
        const int64_t work = (int64_t)t.n_level[level - 1] * t.h_kv;
        int pgrid = (int)std::min<int64_t>((work + warps - 1) / warps, (int64_t)n_sm * 8);
        k_build_parents<HD, R><<<pgrid, BUILD_THREADS, psmem, s>>>(t, level);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

// Parent levels [from, to] over the current tree (a tree growing a new top
// level after an append).
template <typename KT, int HD, int R>
static cudaError_t build_levels_impl(const Tree &t, int from, int to, cudaStream_t s, int n_sm) {
    const int warps = BUILD_THREADS / 32;
    const size_t psmem = (size_t)warps * (t.c * R + R) * sizeof(float);
    static PerDeviceMax<> parent_attr;
    cudaError_t err = allow_smem(k_build_parents<HD, R>, psmem, parent_attr);
    if (err != cudaSuccess) return err;
    for (int level = from; level <= to; ++level) {
        const int64_t work = (int64_t)t.n_level[level - 1] * t.h_kv;
        const int pgrid = (int)std::min<int64_t>((work + warps - 1) / warps, (int64_t)n_sm * 8);
        k_build_parents<HD, R><<<pgrid, BUILD_THREADS, psmem, s>>>(t, level);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
}

template <typename KT, int HD, int R>
static cudaError_t append_impl(const Tree &t, const void *k, const void *v, cudaStream_t s) {
    // per plane warp: one score per token of a leaf, or one estimate per child
    size_t smem = (size_t)R * (t.c > 32 ? t.c : 32) * sizeof(float);
    smem += (size_t)append_stage_bytes<KT, HD, R>(t.c, t.D);  // the shared copy of the rows every plane reads
    if (sizeof(KT) == 2 && R == LM_R && leaf_mma_applies(t.kv_dtype, HD, R, t.c))
        smem += LeafMma<HD>::bytes(1);  // the tensor-core leaf of one warp
    static PerDeviceMax<> attr;
    const cudaError_t err = allow_smem(k_append<KT, HD, R>, smem, attr);
    if (err != cudaSuccess) return err;
    k_append<KT, HD, R><<<t.h_kv, 32 * R, smem, s>>>(t, reinterpret_cast<const KT *>(k), reinterpret_cast<const KT *>(v));
    return cudaGetLastError();
}

#define ZHA_BUILD_DISPATCH(FN, ...)                                                           \
    do {                                                                                      \
        if (t.kv_dtype == 1) {                                                                \
            if (t.d == 128 && t.R == 16) return FN<uint16_t, 128, 16>(__VA_ARGS__);           \
            if (t.d == 128 && t.R == 1) return FN<uint16_t, 128, 1>(__VA_ARGS__);             \
            if (t.d == 64 && t.R == 16) return FN<uint16_t, 64, 16>(__VA_ARGS__);             \
            if (t.d == 64 && t.R == 1) return FN<uint16_t, 64, 1>(__VA_ARGS__);               \
        } else {                                                                              \
            if (t.d == 128 && t.R == 16) return FN<float, 128, 16>(__VA_ARGS__);              \
            if (t.d == 128 && t.R == 1) return FN<float, 128, 1>(__VA_ARGS__);                \
            if (t.d == 64 && t.R == 16) return FN<float, 64, 16>(__VA_ARGS__);                \
            if (t.d == 64 && t.R == 1) return FN<float, 64, 1>(__VA_ARGS__);                  \
        }                                                                                     \
        return cudaErrorInvalidValue;                                                         \
    } while (0)

cudaError_t launch_build(const Tree &t, cudaStream_t s, int n_sm) { ZHA_BUILD_DISPATCH(build_impl, t, s, n_sm); }

cudaError_t launch_append(const Tree &t, const void *k, const void *v, cudaStream_t s) {
    ZHA_BUILD_DISPATCH(append_impl, t, k, v, s);
}

cudaError_t launch_build_levels(const Tree &t, int from, int to, cudaStream_t s, int n_sm) {
    if (from < 2 || to > t.D || from > to) return cudaErrorInvalidValue;
    ZHA_BUILD_DISPATCH(build_levels_impl, t, from, to, s, n_sm);
}

}  // namespace zha
