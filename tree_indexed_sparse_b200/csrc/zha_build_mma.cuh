// zha_build_mma.cuh -- leaf summaries of a bf16 cache with 16 reference
// queries on the tensor cores (mma.sync m16n8k16, bf16 operands, fp32
// accumulation), sm_100a.
//
// Leaf summary ("ZHA 用树形稀疏注意力改造现有大模型", section
// "稀疏注意力为什么还会被索引拖慢": chunk summaries from reference queries):
//   s_ij = r_j.k_i / sqrt(d),  m_j = logsumexp_i s_ij,
//   g_j  = sum_i softmax_i(s_.j) k_i,  b_j = m_j - r_j.g_j / sqrt(d).
// Both contractions are dense over a tile of 16 tokens:
//   S^T (16 planes x 16 tokens) = R (16 x d) . K_tile^T (d x 16)
//   G   (16 planes x d)         = P (16 x 16 tokens) . K_tile (16 x d)
// K is bf16, so every product is exact when its other factor is bf16: the
// reference queries are split r = r_hi + r_mid + r_lo into three bf16 parts
// (exact for any fp32 r; the parts that are zero everywhere are skipped, so
// bf16-representable queries cost one pass) and so are the weights
// p = p_hi + p_mid + p_lo; the accumulation is fp32.  S's accumulator
// fragments are P's operand fragments (the same register layout), so the
// weights never leave registers.
//
// A work unit is one tile of 16 tokens when a leaf has c <= 16 tokens (c a
// power of two: 16 / c leaves per tile, the softmax reduced over the lanes
// that hold a leaf's tokens), or one leaf of c = 16 k tokens (k tiles, an
// online softmax: running maximum and sum, accumulators rescaled).  One warp
// per unit; the tile is staged in shared memory (rows padded by 16 bytes, so
// that the 8x8 matrix loads hit eight bank groups) and read by ldmatrix.
//
// The append recomputes the leaf holding a new token with the same unit
// function, so an appended tree stays bit-identical to a build.
#pragma once

#include <cuda_bf16.h>

#include "zha_device.cuh"
#include "zha_internal.cuh"
#include "zha_mma.cuh"
#include "zha_tma.cuh"

namespace zha {

constexpr int LM_WARPS = 8;  // warps (units in flight) per CTA of the build
constexpr int LM_R = 16;     // reference queries: the MMA's m extent

// Shared memory of the tensor-core leaf build: the reference queries (three
// bf16 parts, padded rows; and fp32) and one 16-token K tile per warp.
template <int HD>
struct LeafMma {
    static constexpr int RS = HD + 8;  // padded row, bf16 elements (a 16-byte shift per row)
    static constexpr int NB = HD / 8;  // n-blocks of the g accumulators
    static constexpr int KS = HD / 16; // k-steps of s
    static constexpr size_t off_r = 0;                                     // [3][16][RS] bf16
    static constexpr size_t off_rf = off_r + (size_t)3 * LM_R * RS * 2;    // [16][HD] fp32
    static constexpr size_t off_k = off_rf + (size_t)LM_R * HD * 4;        // [warps][16][RS] bf16
    static constexpr size_t tile_bytes = (size_t)16 * RS * 2;
    static size_t __host__ __device__ bytes(int warps) { return off_k + (size_t)warps * tile_bytes; }
    static_assert(off_rf % 16 == 0 && off_k % 16 == 0 && tile_bytes % 16 == 0, "16-byte aligned rows");
};

// Whether a tree's leaves are built on the tensor cores.
__host__ __device__ inline bool leaf_mma_applies(int kv_dtype, int d, int R, int c) {
    const bool pow2_small = c >= 2 && c <= 16 && (c & (c - 1)) == 0;
    return kv_dtype == 1 && R == LM_R && (d == 64 || d == 128) && (pow2_small || c % 16 == 0);
}

// Tokens of one work unit.
__host__ __device__ inline int leaf_mma_unit_tokens(int c) { return c <= 16 ? 16 : c; }

// Load reference queries of KV head kh into shared memory: fp32 rows and
// the three bf16 parts.  Returns the number of parts with a nonzero element
// (1 to 3).  All threads of the block call it.
template <int HD>
__device__ int leaf_mma_load_ref(const float *ref_h, unsigned char *smem) {
    using L = LeafMma<HD>;
    __nv_bfloat16 *rs = reinterpret_cast<__nv_bfloat16 *>(smem + L::off_r);
    float *rf = reinterpret_cast<float *>(smem + L::off_rf);
    int mid = 0, lo = 0;
    for (int i = threadIdx.x; i < LM_R * HD; i += blockDim.x) {
        const int j = i / HD, e = i % HD;
        const float x = ref_h[i];
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        const float r1 = x - __bfloat162float(h);
        const __nv_bfloat16 m = __float2bfloat16_rn(r1);
        const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
        rf[i] = x;
        rs[(0 * LM_R + j) * L::RS + e] = h;
        rs[(1 * LM_R + j) * L::RS + e] = m;
        rs[(2 * LM_R + j) * L::RS + e] = l;
        mid |= __bfloat162float(m) != 0.f;
        lo |= __bfloat162float(l) != 0.f;
    }
    mid = __syncthreads_or(mid);
    lo = __syncthreads_or(lo);
    return lo ? 3 : (mid ? 2 : 1);
}

// Three bf16 parts of a fragment pair (x0, x1): x = hi + mid + lo exactly.
__device__ __forceinline__ void split3(float x0, float x1, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
    hi = pack_bf16(x0, x1);
    const float y0 = x0 - bf_lo(hi), y1 = x1 - bf_hi(hi);
    mid = pack_bf16(y0, y1);
    lo = pack_bf16(y0 - bf_lo(mid), y1 - bf_hi(mid));
}

// 16-byte chunks of one 16-token tile each lane moves.
template <int HD>
struct TileRegs {
    static constexpr int CPR = HD / 8;         // 16-byte chunks per row
    static constexpr int PER = 16 * CPR / 32;  // chunks per lane
    uint4 v[PER];
};

// Load tokens [tok0, tok0 + 16) of K (rows of this head; rows at or past n,
// and every row when tok0 < 0, are zero) into registers, through L2 (the
// append reads a row its own kernel just wrote).  The loads stay in flight
// until tile_store uses them, so a warp can load its next tile while it
// computes on the current one.
template <int HD>
__device__ __forceinline__ void tile_load(const uint16_t *Kh, int64_t tok0, int64_t n, TileRegs<HD> &r, int lane) {
    using T = TileRegs<HD>;
#pragma unroll
    for (int k = 0; k < T::PER; ++k) {
        const int idx = lane + 32 * k, row = idx / T::CPR, ch = idx % T::CPR;
        r.v[k] = (tok0 >= 0 && tok0 + row < n) ? __ldcg(reinterpret_cast<const uint4 *>(Kh + (tok0 + row) * HD) + ch)
                                               : make_uint4(0u, 0u, 0u, 0u);
    }
}

// The loaded tile into the warp's staging tile (padded rows).
template <int HD>
__device__ __forceinline__ void tile_store(uint16_t *tile, const TileRegs<HD> &r, int lane) {
    using L = LeafMma<HD>;
    using T = TileRegs<HD>;
    __syncwarp();  // the previous tile's reads are done
#pragma unroll
    for (int k = 0; k < T::PER; ++k) {
        const int idx = lane + 32 * k, row = idx / T::CPR, ch = idx % T::CPR;
        *reinterpret_cast<uint4 *>(tile + row * L::RS + ch * 8) = r.v[k];
    }
    __syncwarp();
}

// S^T of the staged tile: s[j][*] holds (plane g, tokens 8j + 2t, +1) and
// (plane g + 8, the same tokens), g = lane / 4, t = lane % 4; scaled by
// 1/sqrt(d); tokens at or past n are -inf.
template <int HD>
__device__ __forceinline__ void leaf_mma_scores(const unsigned char *smem, const uint16_t *tile, int passes,
                                                int64_t tok0, int64_t n, float scale, float (&s)[2][4], int lane) {
    using L = LeafMma<HD>;
    const uint16_t *rs = reinterpret_cast<const uint16_t *>(smem + L::off_r);
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[j][e] = 0.f;
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll 1
    for (int p = 0; p < passes; ++p) {
#pragma unroll
        for (int kk = 0; kk < L::KS; ++kk) {
            uint32_t a[4], b[4];
            // A: planes (mi & 1) * 8 + ri, dims kk * 16 + (mi >> 1) * 8
            ldsm_x4(a, smem_addr(rs + ((p * LM_R) + (mi & 1) * 8 + ri) * L::RS + kk * 16 + (mi >> 1) * 8));
            // B: tokens (mi >> 1) * 8 + ri, dims kk * 16 + (mi & 1) * 8
            ldsm_x4(b, smem_addr(tile + ((mi >> 1) * 8 + ri) * L::RS + kk * 16 + (mi & 1) * 8));
            mma_bf16(s[0], a, b[0], b[1]);
            mma_bf16(s[1], a, b[2], b[3]);
        }
    }
    const int t = lane & 3;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t tok = tok0 + 8 * j + 2 * t + (e & 1);
            s[j][e] = tok < n ? s[j][e] * scale : -INFINITY;
        }
}

// G += P . tile for the weights p[j][*] (the layout of s), all n-blocks;
// bk: the tile's B fragments (trans loads), three weight parts.
template <int HD>
__device__ __forceinline__ void leaf_mma_gacc(const float (&p)[2][4], const uint32_t (&bk)[HD / 8][2],
                                              float (&acc)[HD / 8][4]) {
    uint32_t ah[4], am[4], al[4];
    split3(p[0][0], p[0][1], ah[0], am[0], al[0]);
    split3(p[0][2], p[0][3], ah[1], am[1], al[1]);
    split3(p[1][0], p[1][1], ah[2], am[2], al[2]);
    split3(p[1][2], p[1][3], ah[3], am[3], al[3]);
#pragma unroll
    for (int nb = 0; nb < HD / 8; ++nb) {
        mma_bf16(acc[nb], ah, bk[nb][0], bk[nb][1]);
        mma_bf16(acc[nb], am, bk[nb][0], bk[nb][1]);
        mma_bf16(acc[nb], al, bk[nb][0], bk[nb][1]);
    }
}

// B fragments of the staged tile for G = P . K: b0 = (tokens 2t, 2t+1;
// dim 8 nb + g), b1 = (tokens 8 + 2t, 9 + 2t; the same dim).
template <int HD>
__device__ __forceinline__ void leaf_mma_kfrag(const uint16_t *tile, uint32_t (&bk)[HD / 8][2], int lane) {
    using L = LeafMma<HD>;
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int nb = 0; nb < HD / 8; nb += 2) {
        uint32_t r[4];
        // matrices: (tokens 0-7 | 8-15) x (dims 8 nb | 8 (nb + 1)), transposed
        ldsm_x4_t(r, smem_addr(tile + ((mi & 1) * 8 + ri) * L::RS + 8 * (nb + (mi >> 1))));
        bk[nb][0] = r[0];
        bk[nb][1] = r[1];
        bk[nb + 1][0] = r[2];
        bk[nb + 1][1] = r[3];
    }
}

// Store one leaf's summaries from the accumulators (planes g, g + 8; dims
// 8 nb + 2t, +1), divided by `div` per plane row: g rows, m, b = m - r.g
// scale (the lane `writer` of each group of four stores m and b), and the
// router copy when asked.
template <int HD>
__device__ __forceinline__ void leaf_mma_store(const Tree &t, int kh, int64_t leaf, const float (&acc)[HD / 8][4],
                                               const float (&div)[2], const float (&m)[2], bool writer,
                                               const unsigned char *smem, int lane) {
    using L = LeafMma<HD>;
    const float *rf = reinterpret_cast<const float *>(smem + L::off_rf);
    const int g = lane >> 2, tq = lane & 3;
    const int64_t nc = t.node_cap[0];
    float *gL = t.g[0] + ((int64_t)kh * nc + leaf) * LM_R * HD;
    uint16_t *g16 = t.g16[0] ? t.g16[0] + ((int64_t)kh * nc + leaf) * LM_R * HD : nullptr;
    float dot[2] = {0.f, 0.f}, dot16[2] = {0.f, 0.f};
#pragma unroll
    for (int nb = 0; nb < HD / 8; ++nb) {
        const int e = 8 * nb + 2 * tq;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int plane = g + 8 * rr;
            const float x0 = acc[nb][2 * rr] / div[rr], x1 = acc[nb][2 * rr + 1] / div[rr];
            *reinterpret_cast<float2 *>(gL + plane * HD + e) = make_float2(x0, x1);
            dot[rr] = fmaf(rf[plane * HD + e + 1], x1, fmaf(rf[plane * HD + e], x0, dot[rr]));
            if (g16) {
                const uint32_t q = pack_bf16(x0, x1);
                *reinterpret_cast<uint32_t *>(g16 + plane * HD + e) = q;
                dot16[rr] = fmaf(rf[plane * HD + e + 1], bf_hi(q), fmaf(rf[plane * HD + e], bf_lo(q), dot16[rr]));
            }
        }
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        dot[rr] += __shfl_xor_sync(FULL, dot[rr], 1);
        dot[rr] += __shfl_xor_sync(FULL, dot[rr], 2);
        dot16[rr] += __shfl_xor_sync(FULL, dot16[rr], 1);
        dot16[rr] += __shfl_xor_sync(FULL, dot16[rr], 2);
    }
    if (writer) {
        const int64_t row = ((int64_t)kh * nc + leaf) * LM_R;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int plane = g + 8 * rr;
            t.m[0][row + plane] = m[rr];
            t.b[0][row + plane] = m[rr] - t.scale * dot[rr];
            if (g16) t.b16[0][row + plane] = m[rr] - t.scale * dot16[rr];
        }
    }
}

// One work unit (see the top of the file) of KV head kh: unit u covers
// tokens [u U, (u + 1) U), U = max(c, 16).  `tile`: this warp's staging
// tile; `passes`: bf16 parts of the reference queries.  On entry `nxt`
// holds the unit's first tile (tile_load); each tile's successor -- the
// unit's next tile, else the first tile at token next_tok0 (< 0: none) --
// is loaded while the tile is computed, and is in `nxt` on return.
template <int HD>
__device__ __forceinline__ void leaf_mma_unit(const Tree &t, int kh, int64_t u, const unsigned char *smem,
                                              uint16_t *tile, int passes, TileRegs<HD> &nxt, int64_t next_tok0,
                                              int lane) {
    const int c = t.c;
    const int64_t n = t.n_tokens;
    const uint16_t *Kh = reinterpret_cast<const uint16_t *>(t.K) + (int64_t)kh * t.kv_cap * HD;
    const int tq = lane & 3;
    float s[2][4];
    float acc[HD / 8][4];
    uint32_t bk[HD / 8][2];
    if (c <= 16) {
        const int64_t tok0 = u * 16;
        tile_store<HD>(tile, nxt, lane);
        tile_load<HD>(Kh, next_tok0, n, nxt, lane);
        leaf_mma_scores<HD>(smem, tile, passes, tok0, n, t.scale, s, lane);
        leaf_mma_kfrag<HD>(tile, bk, lane);
        // per (plane row rr, n-block j): the leaf's maximum and sum over the
        // lanes holding its tokens (pairs in a lane, then t bits, then j)
        float mx[2][2], sm[2][2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float v = fmaxf(s[j][2 * rr], s[j][2 * rr + 1]);
                if (c >= 4) v = fmaxf(v, __shfl_xor_sync(FULL, v, 1));
                if (c >= 8) v = fmaxf(v, __shfl_xor_sync(FULL, v, 2));
                mx[rr][j] = v;
            }
        if (c == 16)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) mx[rr][0] = mx[rr][1] = fmaxf(mx[rr][0], mx[rr][1]);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float M = mx[rr][j];
                float v = M == -INFINITY ? 0.f : expf(s[j][2 * rr] - M) + expf(s[j][2 * rr + 1] - M);
                if (c >= 4) v += __shfl_xor_sync(FULL, v, 1);
                if (c >= 8) v += __shfl_xor_sync(FULL, v, 2);
                sm[rr][j] = v;
            }
        if (c == 16)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) sm[rr][0] = sm[rr][1] = sm[rr][0] + sm[rr][1];
        float m[2][2];  // log mass per (rr, j)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int j = 0; j < 2; ++j) m[rr][j] = mx[rr][j] + logf(sm[rr][j]);
        // every leaf of the tile: weights masked to its tokens, then G
        const int nleaf = 16 / c;
#pragma unroll 1
        for (int lf = 0; lf < nleaf; ++lf) {
            const int64_t leaf = (tok0 >> 4) * nleaf + lf;
            if (leaf * c >= n) break;
            float p[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tk = 8 * j + 2 * tq + (e & 1);
                    const int rr = e >> 1;
                    p[j][e] = (tk / c == lf && s[j][e] != -INFINITY) ? expf(s[j][e] - m[rr][j]) : 0.f;
                }
#pragma unroll
            for (int nb = 0; nb < HD / 8; ++nb)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nb][e] = 0.f;
            leaf_mma_gacc<HD>(p, bk, acc);
            // the lane holding the leaf's first token writes m and b
            const int first = lf * c;
            const int jf = first / 8;
            const bool writer = tq == (first % 8) / 2;
            const float mm[2] = {jf ? m[0][1] : m[0][0], jf ? m[1][1] : m[1][0]};
            const float one[2] = {1.f, 1.f};
            leaf_mma_store<HD>(t, kh, leaf, acc, one, mm, writer, smem, lane);
        }
    } else {
        // one leaf of c / 16 tiles, online softmax per plane
        const int64_t leaf = u;
        float M[2] = {-INFINITY, -INFINITY}, Lsum[2] = {0.f, 0.f};
#pragma unroll
        for (int nb = 0; nb < HD / 8; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nb][e] = 0.f;
#pragma unroll 1
        for (int i = 0; i < c / 16; ++i) {
            const int64_t tok0 = leaf * c + 16 * i;
            if (tok0 >= n) break;
            tile_store<HD>(tile, nxt, lane);
            const int64_t tn = tok0 + 16;
            tile_load<HD>(Kh, (i + 1 < c / 16 && tn < n) ? tn : next_tok0, n, nxt, lane);
            leaf_mma_scores<HD>(smem, tile, passes, tok0, n, t.scale, s, lane);
            leaf_mma_kfrag<HD>(tile, bk, lane);
            float p[2][4];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                float v = fmaxf(fmaxf(s[0][2 * rr], s[0][2 * rr + 1]), fmaxf(s[1][2 * rr], s[1][2 * rr + 1]));
                v = fmaxf(v, __shfl_xor_sync(FULL, v, 1));
                v = fmaxf(v, __shfl_xor_sync(FULL, v, 2));
                const float Mn = fmaxf(M[rr], v);
                const float alpha = M[rr] == -INFINITY ? 0.f : expf(M[rr] - Mn);
                float sum = 0.f;
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float x = s[j][2 * rr + e];
                        p[j][2 * rr + e] = x == -INFINITY ? 0.f : expf(x - Mn);
                        sum += p[j][2 * rr + e];
                    }
                sum += __shfl_xor_sync(FULL, sum, 1);
                sum += __shfl_xor_sync(FULL, sum, 2);
                Lsum[rr] = Lsum[rr] * alpha + sum;
#pragma unroll
                for (int nb = 0; nb < HD / 8; ++nb) {
                    acc[nb][2 * rr] *= alpha;
                    acc[nb][2 * rr + 1] *= alpha;
                }
                M[rr] = Mn;
            }
            leaf_mma_gacc<HD>(p, bk, acc);
        }
        const float mm[2] = {M[0] + logf(Lsum[0]), M[1] + logf(Lsum[1])};
        leaf_mma_store<HD>(t, kh, leaf, acc, Lsum, mm, tq == 0, smem, lane);
    }
    __syncwarp();
}

// The leaf level of every KV head: blockIdx.y is the KV head, each warp
// takes units blockIdx.x * LM_WARPS + warp, + gridDim.x * LM_WARPS, ...
template <int HD>
__global__ void __launch_bounds__(LM_WARPS * 32) k_build_leaves_mma(Tree t) {
    extern __shared__ __align__(16) unsigned char lsm[];
    using L = LeafMma<HD>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int kh = blockIdx.y;
    const int passes = leaf_mma_load_ref<HD>(t.ref + (int64_t)kh * LM_R * HD, lsm);
    uint16_t *tile = reinterpret_cast<uint16_t *>(lsm + L::off_k + (size_t)warp * L::tile_bytes);
    const int U = leaf_mma_unit_tokens(t.c);
    const int64_t units = (t.n_tokens + U - 1) / U;
    const int64_t stride = (int64_t)gridDim.x * LM_WARPS;
    const uint16_t *Kh = reinterpret_cast<const uint16_t *>(t.K) + (int64_t)kh * t.kv_cap * HD;
    int64_t u = (int64_t)blockIdx.x * LM_WARPS + warp;
    TileRegs<HD> nxt;
    tile_load<HD>(Kh, u < units ? u * U : -1, t.n_tokens, nxt, lane);
    for (; u < units; u += stride)
        leaf_mma_unit<HD>(t, kh, u, lsm, tile, passes, nxt, u + stride < units ? (u + stride) * U : -1, lane);
}

}  // namespace zha
