// zha_route.cu -- one routing level of zha_decode (sm_100a).
//
// Routing ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢";
// "階層型疎Attention「ZHA」…", section "【技術的ディープダイブ】": top-p, not a
// fixed top-k): the query scores every node of the frontier, softmax-normalises
// the estimates within the frontier, keeps the smallest set in descending order
// (ties to the lower node id) whose cumulative mass reaches p, and expands only
// the kept nodes' children at the next level.
//
// One launch per level.  The frontier of KV head kh is the union over its G
// query heads: the children of every node kept by any head, each carrying the
// bitmask of heads that kept its parent.  A node's summary is read from HBM
// once and scored for all G heads (a [R x d] x [d x G] product per node).
//
// Phase 1 (every CTA; the CTAs of the grid are split evenly over KV heads):
//   est(q_h) = max_j (b_j + q_h.g_j / sqrt(d)) for every frontier slot, written
//   to the score buffer, plus a per-CTA max per query head.
// Phase 2 (the last CTA of each KV head to finish phase 1, found with a
// fence + ticket counter): exact top-p per query head, then the ordered union
// compaction that becomes the next level's frontier.
//
// Exact, deterministic top-p: masses are exp(est - max) in 2^-40 fixed point,
// summed with integer atomics (order independent).  A 1024-bucket histogram
// over (max - est) finds the bucket holding the cut; the bucket is refined by
// value until at most 256 candidates remain (or all tie exactly), and those
// are ranked by (est descending, node id ascending).  The kept set of head h
// is every eligible slot whose key (desc(est), slot) is <= the cut key.
#include <algorithm>

#include "zha_device.cuh"
#include "zha_internal.cuh"

namespace zha {

template <int HD, int R, int G>
struct RouteCfg {
    static constexpr int VEC = HD / 32;
    static constexpr int NPW = (G * R >= 32) ? 1 : 32 / (G * R);  // nodes per warp pass
    static constexpr int V = NPW * G * R;                          // partial dots per lane
    static constexpr int K = V / 32;                               // sums per lane after reduce-scatter
    static constexpr int STAGE_SLOTS = STAGE_BYTES / (4 * G);
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

__device__ __forceinline__ int coarse_bucket(float M, float e) {
    const float x = (M - e) * BUCKETS_PER_UNIT;
    return x < (float)(NB - 1) ? (int)x : NB - 1;
}

// Shared-memory carve of the select phase.
template <int G>
struct SelectSmem {
    static constexpr int STAGE_SLOTS = STAGE_BYTES / (4 * G);
    static constexpr size_t off_el = STAGE_BYTES;
    static constexpr size_t off_hm = (off_el + STAGE_SLOTS + 255) / 256 * 256;
    static constexpr size_t off_hc = off_hm + NB * 8;
    static constexpr size_t off_ck = off_hc + NB * 4;
    static constexpr size_t off_cm = off_ck + CAND_MAX * 8;
    static constexpr size_t off_cut = off_cm + CAND_MAX * 8;
    static constexpr size_t off_misc = off_cut + 8 * 8;
    static constexpr size_t bytes = off_misc + 1024;
};

size_t route_smem_bytes(int G) {
    switch (G) {
        case 1: return SelectSmem<1>::bytes;
        case 2: return SelectSmem<2>::bytes;
        case 4: return SelectSmem<4>::bytes;
        default: return SelectSmem<8>::bytes;
    }
}

// Bucket holding the cut: the first bucket whose inclusive cumulative mass
// reaches target.  Returns the bucket and writes the mass strictly before it.
__device__ int find_cut_bucket(const unsigned long long *hm, unsigned long long target,
                               unsigned long long *mass_before, unsigned long long *sh64, uint32_t *sh32,
                               unsigned long long *bcast) {
    const int tid = threadIdx.x, NT = blockDim.x;
    const int per = NB / NT;
    unsigned long long local = 0;
    for (int q = 0; q < per; ++q) local += hm[tid * per + q];
    unsigned long long tot;
    const unsigned long long incl = block_scan_u64(local, sh64, &tot);
    unsigned long long run = incl - local;
    uint32_t mine = 0xffffffffu;
    unsigned long long above = 0;
    for (int q = 0; q < per; ++q) {
        const unsigned long long m = hm[tid * per + q];
        if (run + m >= target && mine == 0xffffffffu) {
            mine = tid * per + q;
            above = run;
        }
        run += m;
    }
    uint32_t B = block_min_u32(mine, sh32);
    if (mine == B && B != 0xffffffffu) *bcast = above;
    if (B == 0xffffffffu) {
        // unreachable when target <= total mass; keep every index in range anyway
        B = NB - 1;
        if (tid == 0) *bcast = tot - hm[NB - 1];
    }
    __syncthreads();
    *mass_before = *bcast;
    __syncthreads();
    return (int)B;
}

template <int HD, int R, int G>
__device__ void select_kvh(const Decode &a, int l, int kh, int64_t S, int nb, unsigned char *smem) {
    using SM = SelectSmem<G>;
    const int tid = threadIdx.x, NT = blockDim.x;
    const int lane = tid & 31, wid = tid >> 5, nw = NT >> 5;
    const bool top = (l == a.t.D);
    float *sc = reinterpret_cast<float *>(smem);
    uint8_t *el = smem + SM::off_el;
    unsigned long long *hm = reinterpret_cast<unsigned long long *>(smem + SM::off_hm);
    uint32_t *hc = reinterpret_cast<uint32_t *>(smem + SM::off_hc);
    unsigned long long *ck = reinterpret_cast<unsigned long long *>(smem + SM::off_ck);
    unsigned long long *cmass = reinterpret_cast<unsigned long long *>(smem + SM::off_cm);
    unsigned long long *cut = reinterpret_cast<unsigned long long *>(smem + SM::off_cut);
    unsigned char *misc = smem + SM::off_misc;
    unsigned long long *sh64 = reinterpret_cast<unsigned long long *>(misc);          // 32 x u64
    uint32_t *sh32 = reinterpret_cast<uint32_t *>(misc + 256);                         // 32 x u32
    float *shf = reinterpret_cast<float *>(misc + 384);                                // 32 x f32
    unsigned long long *bc64 = reinterpret_cast<unsigned long long *>(misc + 512);     // broadcasts
    uint32_t *bc32 = reinterpret_cast<uint32_t *>(misc + 576);
    uint32_t *wcnt = reinterpret_cast<uint32_t *>(misc + 640);                         // [nw][G+1]
    uint32_t *run_off = reinterpret_cast<uint32_t *>(misc + 960);                      // [G+1]

    const int64_t sbase = (int64_t)kh * a.score_cap * G;
    const bool staged = S <= SM::STAGE_SLOTS;
    if (staged) {
        for (int64_t s = tid; s < S; s += NT) {
            int32_t node; bool ok; uint32_t msk;
            slot_info<G>(a, l, kh, top, S, s, node, ok, msk);
            el[s] = (uint8_t)msk;
#pragma unroll
            for (int h = 0; h < G; ++h) sc[s * G + h] = __ldcg(a.scores + sbase + s * G + h);
        }
        __syncthreads();
    }
    auto elig = [&](int64_t s) -> uint32_t {
        if (staged) return el[s];
        int32_t node; bool ok; uint32_t msk;
        slot_info<G>(a, l, kh, top, S, s, node, ok, msk);
        return msk;
    };
    auto score = [&](int64_t s, int h) -> float {
        return staged ? sc[s * G + h] : __ldcg(a.scores + sbase + s * G + h);
    };

    uint32_t Fh[G];
    const float p = a.p;
    for (int h = 0; h < G; ++h) {
        // frontier max of head h from the per-CTA maxima
        float M = -INFINITY;
        for (int i = tid; i < nb; i += NT) M = fmaxf(M, __ldcg(a.pmax + ((int64_t)kh * a.pmax_cap + i) * G + h));
        M = block_max(M, shf);
        for (int i = tid; i < NB; i += NT) { hm[i] = 0ull; hc[i] = 0u; }
        __syncthreads();
        uint32_t f = 0;
        unsigned long long z = 0;
        for (int64_t s = tid; s < S; s += NT) {
            if ((elig(s) >> h) & 1u) {
                const float e = score(s, h);
                const unsigned long long wf = mass_fx(expf(e - M));
                const int bk = coarse_bucket(M, e);
                atomicAdd(&hm[bk], wf);
                atomicAdd(&hc[bk], 1u);
                ++f;
                z += wf;
            }
        }
        __syncthreads();
        Fh[h] = block_sum_int<uint32_t>(f, sh32);
        const unsigned long long Z = block_sum_int<unsigned long long>(z, sh64);
        if (!(p < 1.0f)) {
            if (tid == 0) cut[h] = ~0ull;
            __syncthreads();
            continue;
        }
        unsigned long long target = (unsigned long long)ceil((double)p * (double)Z);
        if (target > Z) target = Z;
        if (target == 0ull) target = 1ull;
        unsigned long long above;
        const int B = find_cut_bucket(hm, target, &above, sh64, sh32, bc64);
        uint32_t count = hc[B];
        // candidate set: slots of bucket B, narrowed by value while too many
        bool refined = false;
        uint32_t dlo = 0u, dhi = 0xffffffffu;
        auto member = [&](int64_t s, float &e, uint32_t &dk) -> bool {
            if (!((elig(s) >> h) & 1u)) return false;
            e = score(s, h);
            dk = desc_key(e);
            if (!refined) return coarse_bucket(M, e) == B;
            return dk >= dlo && dk <= dhi;
        };
        if (count > (uint32_t)CAND_MAX) {
            uint32_t lo = 0xffffffffu, hi = 0u;
            for (int64_t s = tid; s < S; s += NT) {
                float e; uint32_t dk;
                if (member(s, e, dk)) { lo = min(lo, dk); hi = max(hi, dk); }
            }
            dlo = block_min_u32(lo, sh32);
            dhi = block_max_u32(hi, sh32);
            refined = true;
            while (count > (uint32_t)CAND_MAX && dlo < dhi) {
                for (int i = tid; i < NB; i += NT) { hm[i] = 0ull; hc[i] = 0u; }
                __syncthreads();
                const unsigned long long span = (unsigned long long)(dhi - dlo) + 1ull;
                for (int64_t s = tid; s < S; s += NT) {
                    float e; uint32_t dk;
                    if (member(s, e, dk)) {
                        const int sb = (int)(((unsigned long long)(dk - dlo) * NB) / span);
                        atomicAdd(&hm[sb], mass_fx(expf(e - M)));
                        atomicAdd(&hc[sb], 1u);
                    }
                }
                __syncthreads();
                unsigned long long need_left = target - above;
                unsigned long long sub_above;
                const int SB = find_cut_bucket(hm, need_left, &sub_above, sh64, sh32, bc64);
                above += sub_above;
                count = hc[SB];
                lo = 0xffffffffu; hi = 0u;
                for (int64_t s = tid; s < S; s += NT) {
                    float e; uint32_t dk;
                    if (member(s, e, dk)) {
                        const int sb = (int)(((unsigned long long)(dk - dlo) * NB) / span);
                        if (sb == SB) { lo = min(lo, dk); hi = max(hi, dk); }
                    }
                }
                const uint32_t nlo = block_min_u32(lo, sh32);
                const uint32_t nhi = block_max_u32(hi, sh32);
                dlo = nlo;
                dhi = nhi;
            }
        }
        if (count <= (uint32_t)CAND_MAX) {
            if (tid == 0) bc32[0] = 0u;
            __syncthreads();
            for (int64_t s = tid; s < S; s += NT) {
                float e; uint32_t dk;
                if (member(s, e, dk)) {
                    const uint32_t idx = atomicAdd(&bc32[0], 1u);
                    if (idx < (uint32_t)CAND_MAX) {
                        ck[idx] = ((unsigned long long)dk << 32) | (unsigned long long)s;
                        cmass[idx] = mass_fx(expf(e - M));
                    }
                }
            }
            __syncthreads();
            const int n = (int)min(bc32[0], (uint32_t)CAND_MAX);
            if (tid == 0) {
                unsigned long long mx = 0ull;
                for (int i = 0; i < n; ++i) mx = max(mx, ck[i]);
                cut[h] = mx;  // safe default: keep every candidate
            }
            __syncthreads();
            for (int i = tid; i < n; i += NT) {
                const unsigned long long key = ck[i];
                unsigned long long before = 0ull;
                for (int j = 0; j < n; ++j)
                    if (ck[j] < key) before += cmass[j];
                const unsigned long long lo_m = above + before;
                if (lo_m < target && lo_m + cmass[i] >= target) cut[h] = key;
            }
            __syncthreads();
        } else {
            // exact tie of more than CAND_MAX slots: equal masses, the first t
            // of them in slot (= node id) order are kept
            unsigned long long wtie = 0ull;
            {
                float e = desc_key_to_float(dlo);
                wtie = mass_fx(expf(e - M));
            }
            const unsigned long long need_left = target - above;
            const unsigned long long t_need = wtie ? (need_left + wtie - 1ull) / wtie : (unsigned long long)count;
            if (tid == 0) { cut[h] = ((unsigned long long)dlo << 32) | 0xffffffffull; bc32[1] = 0u; }
            __syncthreads();
            for (int64_t base = 0; base < S; base += NT) {
                const int64_t s = base + tid;
                float e; uint32_t dk;
                const uint32_t fl = (s < S && member(s, e, dk)) ? 1u : 0u;
                uint32_t tot;
                const uint32_t incl = block_scan_u32(fl, sh32, &tot);
                const unsigned long long rank = (unsigned long long)bc32[1] + incl;
                if (fl && rank == t_need) cut[h] = ((unsigned long long)dlo << 32) | (unsigned long long)s;
                __syncthreads();
                if (tid == 0) bc32[1] += tot;
                __syncthreads();
            }
        }
    }

    // ordered compaction: union list (next frontier) and per-head lists
    const bool per_head = (l == 1) || (a.trace_ids != nullptr);
    if (tid <= G) run_off[tid] = 0u;
    __syncthreads();
    const int64_t kbase = (int64_t)kh * a.t.node_cap[l - 1];
    for (int64_t base = 0; base < S; base += NT) {
        const int64_t s = base + tid;
        int32_t node = 0;
        bool ok = false;
        uint32_t msk = 0;
        slot_info<G>(a, l, kh, top, S, s, node, ok, msk);
        uint32_t kb = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            if ((msk >> h) & 1u) {
                const float e = score(s, h);
                const unsigned long long key = ((unsigned long long)desc_key(e) << 32) | (unsigned long long)s;
                if (key <= cut[h]) kb |= 1u << h;
            }
        }
        const unsigned lt = (1u << lane) - 1u;
        const unsigned bu = __ballot_sync(FULL, kb != 0u);
        if (lane == 0) wcnt[wid * (G + 1)] = __popc(bu);
        unsigned bh[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            bh[h] = __ballot_sync(FULL, (kb >> h) & 1u);
            if (lane == 0) wcnt[wid * (G + 1) + 1 + h] = __popc(bh[h]);
        }
        __syncthreads();
        if (tid <= G) {
            // exclusive scan over warps for list `tid`, in place; totals added to run_off
            uint32_t acc = run_off[tid];
            for (int w = 0; w < nw; ++w) {
                const uint32_t c = wcnt[w * (G + 1) + tid];
                wcnt[w * (G + 1) + tid] = acc;
                acc += c;
            }
            run_off[tid] = acc;
        }
        __syncthreads();
        if (kb) {
            const uint32_t pos = wcnt[wid * (G + 1)] + __popc(bu & lt);
            a.kept_ids[l - 1][kbase + pos] = node;
            a.kept_mask[l - 1][kbase + pos] = (uint8_t)kb;
        }
        if (per_head) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                if ((kb >> h) & 1u) {
                    const uint32_t pos = wcnt[wid * (G + 1) + 1 + h] + __popc(bh[h] & lt);
                    const int hq = kh * G + h;
                    if (l == 1 && a.leaf_idx) {
                        if (pos < (uint32_t)a.leaf_cap) a.leaf_idx[(int64_t)hq * a.leaf_cap + pos] = node;
                    }
                    if (a.trace_ids && pos < (uint32_t)a.trace_cap)
                        a.trace_ids[((int64_t)(l - 1) * a.t.h_q + hq) * a.trace_cap + pos] = node;
                }
            }
        }
        __syncthreads();
    }
    if (tid == 0) {
        a.kept_cnt[(l - 1) * a.t.h_kv + kh] = (int32_t)run_off[0];
        for (int h = 0; h < G; ++h) {
            const int hq = kh * G + h;
            const uint32_t nk = run_off[1 + h];
            const int64_t prev = (l == a.t.D) ? 0 : a.vis_acc[hq];
            const int64_t vis = prev + (int64_t)Fh[h];
            a.vis_acc[hq] = vis;
            if (a.trace_cnt) a.trace_cnt[(l - 1) * a.t.h_q + hq] = (int32_t)nk;
            if (a.trace_ids && nk > (uint32_t)a.trace_cap) set_status(a.status, -2);
            if (l == 1) {
                if (a.n_leaf) a.n_leaf[hq] = (int32_t)nk;
                if (a.visited) a.visited[hq] = vis;
                if (a.leaf_idx && nk > (uint32_t)a.leaf_cap) set_status(a.status, -2);
            }
        }
    }
}

template <int HD, int R, int G>
__global__ void __launch_bounds__(ROUTE_THREADS, 1) k_route_level(Decode a, int l) {
    extern __shared__ __align__(16) unsigned char rsm[];
    using C = RouteCfg<HD, R, G>;
    constexpr int VEC = C::VEC, NPW = C::NPW, V = C::V, K = C::K;
    const int h_kv = a.t.h_kv;
    const int kh = blockIdx.x % h_kv, bi = blockIdx.x / h_kv, nb = gridDim.x / h_kv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    const bool top = (l == a.t.D);
    const int64_t S = top ? (int64_t)a.t.n_level[l - 1]
                          : (int64_t)a.t.c * __ldcg(a.kept_cnt + l * h_kv + kh);

    // scaled query slices of the G heads sharing this KV head
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

    // head and plane of this lane's sums after the reduce-scatter
    const int idx0 = lane * K;
    const int my_i = idx0 / (G * R), my_h = (idx0 / R) % G, my_j0 = idx0 % R;
    float lmax = -INFINITY;

    for (int64_t grp = (int64_t)bi * nwarp + warp; grp * NPW < S; grp += (int64_t)nb * nwarp) {
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
            scores[s * G + my_h] = ok ? est : -INFINITY;
            if (ok && ((msk >> my_h) & 1u)) lmax = fmaxf(lmax, est);
        }
    }

    // per-CTA max per head
    float *wmax = reinterpret_cast<float *>(rsm);
    wmax[threadIdx.x] = (my_j0 == 0) ? lmax : -INFINITY;
    __syncthreads();
    if (threadIdx.x < G) {
        float mx = -INFINITY;
        for (int t = 0; t < (int)blockDim.x; ++t) {
            const int ln = t & 31;
            const int li0 = ln * K;
            if (((li0 / R) % G) == (int)threadIdx.x) mx = fmaxf(mx, wmax[t]);
        }
        a.pmax[((int64_t)kh * a.pmax_cap + bi) * G + threadIdx.x] = mx;
    }
    __threadfence();
    __syncthreads();
    __shared__ int s_last;
    if (threadIdx.x == 0) {
        const unsigned tk = atomicAdd(a.done + (l - 1) * h_kv + kh, 1u);
        s_last = (tk == (unsigned)(nb - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    select_kvh<HD, R, G>(a, l, kh, S, nb, rsm);
    if (threadIdx.x == 0) a.done[(l - 1) * h_kv + kh] = 0u;
}

template <int HD, int R, int G>
static cudaError_t route_impl(const Decode &dc, int level, int n_cta, size_t smem, cudaStream_t s) {
    cudaError_t err = cudaFuncSetAttribute(k_route_level<HD, R, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    k_route_level<HD, R, G><<<n_cta, ROUTE_THREADS, smem, s>>>(dc, level);
    return cudaGetLastError();
}

cudaError_t launch_route_level(const Decode &dc, int level, int n_cta, size_t smem, cudaStream_t s) {
    const Tree &t = dc.t;
    if (t.G == 4) {
        if (t.d == 128 && t.R == 16) return route_impl<128, 16, 4>(dc, level, n_cta, smem, s);
        if (t.d == 128 && t.R == 1) return route_impl<128, 1, 4>(dc, level, n_cta, smem, s);
        if (t.d == 64 && t.R == 16) return route_impl<64, 16, 4>(dc, level, n_cta, smem, s);
        if (t.d == 64 && t.R == 1) return route_impl<64, 1, 4>(dc, level, n_cta, smem, s);
    } else if (t.G == 1) {
        if (t.d == 128 && t.R == 16) return route_impl<128, 16, 1>(dc, level, n_cta, smem, s);
        if (t.d == 128 && t.R == 1) return route_impl<128, 1, 1>(dc, level, n_cta, smem, s);
        if (t.d == 64 && t.R == 16) return route_impl<64, 16, 1>(dc, level, n_cta, smem, s);
        if (t.d == 64 && t.R == 1) return route_impl<64, 1, 1>(dc, level, n_cta, smem, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace zha
