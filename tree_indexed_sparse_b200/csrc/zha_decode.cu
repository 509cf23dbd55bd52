// zha_decode.cu -- one decoded token for every query head, in one persistent
// cooperative kernel (sm_100a): every routing level, then the routed
// attention.
//
// Routing ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢":
// score the top nodes, keep the smallest set whose estimated mass reaches p,
// expand only their children, repeat down to the raw entries; "Zyphra
// 分层注意力（ZHA）…", section "机制拆解：树形索引如何高效筛选长上下文"):
//   the grid's CTAs are split into h_kv teams of nbk = gridDim / h_kv CTAs,
//   one per KV head, which route independently, level D .. 1: a small
//   frontier is scored and cut by every CTA of the team on its own (no
//   inter-CTA wait), a mid-size one is scored in slices and cut by every CTA
//   after one team barrier, and a large one is scored and cut in slices
//   against the team's histograms (zha_route.cuh, LevelMode).
//   a grid barrier ends the routing; every CTA then writes the leaf lists and
//   traces of its own segments while the attention over the kept leaves plus
//   the sink token runs split over every CTA (zha_attend.cuh); the last CTA
//   to finish a KV head's stages merges its partials (ticket).
// The grid is one CTA per SM, launched cooperatively so that the barriers
// cannot deadlock; every barrier wait is bounded by a clock budget, after
// which the kernel records ZHA_ERR_TIMEOUT, raises the abort word and leaves.
#include "zha_attend.cuh"
#include "zha_route.cuh"
#include "zha_sync.cuh"

namespace zha {

__device__ __forceinline__ void stamp(const Decode &a, int i) {
    if (a.phase_ns && blockIdx.x == 0 && threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        a.phase_ns[i] = (int64_t)t;
    }
}

// Per-head lists of one CTA's segments: level-1 leaf ids (leaf_idx, n_leaf)
// and, when requested, every level's kept ids (trace).  Positions come from
// the lower ranks' per-head counts.  Warps 0-7.
template <int G>
__device__ __noinline__ void write_lists(const Decode &a, int kh, int tr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int D = a.t.D;
    for (int task = warp; task < D * G; task += GT / 32) {
        const int l = 1 + task / G, h = task % G;
        const bool leaf = (l == 1);
        const bool tr_on = a.trace_ids != nullptr;
        if (!leaf && !tr_on) continue;
        const int32_t *lv = lvl_ptr(a, l, kh);
        const int T = __ldcg(lv);
        const int64_t S = __ldcg(lv + 1);
        const int hq = kh * G + h;
        const uint32_t *hs = hseg_ptr(a, l, kh);
        // lower ranks' counts and the total of head h
        uint32_t before = 0u, total = 0u;
        for (int r = lane; r < T; r += 32) {
            const uint32_t x = __ldcg(hs + (int64_t)r * G + h);
            total += x;
            if (r < tr) before += x;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            before += __shfl_xor_sync(FULL, before, off);
            total += __shfl_xor_sync(FULL, total, off);
        }
        if (tr == 0 && lane == 0) {
            if (leaf && a.n_leaf) a.n_leaf[hq] = (int32_t)total;
            if (leaf && a.leaf_idx && total > (uint32_t)a.leaf_cap) set_status(a.status, ZHA_CAPACITY_CODE);
            if (tr_on) {
                a.trace_cnt[(int64_t)(l - 1) * a.nvk * G + hq] = (int32_t)total;
                if (total > (uint32_t)a.trace_cap) set_status(a.status, ZHA_CAPACITY_CODE);
            }
        }
        if (tr >= T) continue;
        const uint32_t n = __ldcg(seg_ptr(a, l, kh) + tr);
        const int64_t src = (int64_t)kh * a.slot_cap[l - 1] + seg_start(S, T, tr);
        const int32_t *ids = a.kept_ids[l - 1] + src;
        const uint8_t *msk = a.kept_mask[l - 1] + src;
        uint32_t pos = before;
        for (uint32_t i0 = 0; i0 < n; i0 += 32) {
            const uint32_t i = i0 + lane;
            const bool mine = i < n && ((__ldcg(msk + i) >> h) & 1u);
            const unsigned bal = __ballot_sync(FULL, mine);
            if (mine) {
                const uint32_t p = pos + __popc(bal & ((1u << lane) - 1u));
                const int32_t id = __ldcg(ids + i);
                if (leaf && a.leaf_idx && p < (uint32_t)a.leaf_cap) a.leaf_idx[(int64_t)hq * a.leaf_cap + p] = id;
                if (tr_on && p < (uint32_t)a.trace_cap)
                    a.trace_ids[((int64_t)(l - 1) * a.nvk * G + hq) * a.trace_cap + p] = id;
            }
            pos += __popc(bal);
        }
    }
}

// All routing levels of KV head kh as rank tr of a team of T CTAs, level D
// down to 1, each in the way level_mode picks from its frontier size.  The
// parents of a level are either the kept list every CTA holds in shared
// memory (after an LV_ALL or LV_SPLIT level) or the segments of an LV_TEAM
// level in global memory; a level routed by every CTA after an LV_TEAM level
// first copies those segments in.  Warps 0-7.
template <int HD, int R, int G, typename RT>
__device__ __noinline__ bool route_kvh(const Decode &a, int kh, int tr, int T, unsigned char *smem, TeamSync &ts) {
    using SM = RouteSmem<G>;
    uint32_t *pref = reinterpret_cast<uint32_t *>(smem + SM::off_pref);
    uint32_t *scratch = reinterpret_cast<uint32_t *>(smem + SM::off_misc) + 8;
    int32_t *pid = reinterpret_cast<int32_t *>(smem + SM::off_pid);
    uint8_t *pmk = smem + SM::off_pmk;
    const int D = a.t.D;
    int64_t vis[G];
#pragma unroll
    for (int h = 0; h < G; ++h) vis[h] = 0;
    int Tp = 1;            // team size and frontier size of level l + 1 (its segments)
    int64_t Sp = 0;
    int64_t S = a.t.n_level[D - 1];
    bool par_local = true;  // level l's parents are the kept list in pid / pmk
    int buf = 0;           // team score buffer of the next LV_SPLIT level
    stages_init<G>(smem);
#pragma unroll 1
    for (int l = D; l >= 1; --l) {
        const int mode = level_mode<HD, R, RT>(S, T);
        uint32_t F[G];
        int64_t Snext = 0;
        if (mode != LV_TEAM) {
            if (!par_local) {
                // the whole kept list of level l + 1 from its segments
                Level P;
                P.l = l;
                P.kh = kh;
                P.Tp = Tp;
                P.Sp = Sp;
                int64_t k0 = 0;
                load_parents(a, P, 0, S, pref, pid, pmk, k0);
                gsync();
                par_local = true;
            }
            int64_t nk = 0;
            if (!route_level_rd<HD, R, G, RT>(a, l, kh, T, tr, S, mode, buf, smem, ts, F, nk)) return false;
            if (mode == LV_SPLIT) buf ^= 1;
            Tp = 1;
            Sp = S;
            Snext = nk * a.t.c;
        } else {
            int Tout;
            if (!route_level<HD, R, G, RT>(a, l, kh, T, tr, S, Tp, Sp, par_local, smem, ts, F, Tout)) return false;
            par_local = false;
            Tp = Tout;
            Sp = S;
            if (l > 1) Snext = load_segments(a, l, kh, Tp, pref, scratch) * a.t.c;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) vis[h] += F[h];
        if (l > 1) stamp(a, D - l + 1);
        S = Snext;
    }
    stages_inval<G>(smem);
    if (tr == 0 && threadIdx.x < G && a.visited) {
#pragma unroll
        for (int h = 0; h < G; ++h)
            if (h == (int)threadIdx.x) a.visited[kh * G + h] = vis[h];
    }
    return true;
}

template <typename KT, int HD, int R, int G, typename RT>
__global__ void __launch_bounds__(A_THREADS, 1) k_decode(const __grid_constant__ Decode a) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ StageMap map;
    __shared__ int s_flag;
    __shared__ int s_last[64];
    const int warp = threadIdx.x >> 5;
    const int nb = gridDim.x, b = blockIdx.x;
    const int h_kv = a.nvk;     // virtual KV heads: one team each
    const int nbk = nb / h_kv;  // CTAs per KV head team
    unsigned *words = a.sync;
    unsigned *abortw = words + h_kv + 2;
    // launched as a programmatic dependent of the previous kernel on the
    // stream (an append, typically): nothing is read before it completes
    griddep_wait();
    stamp(a, 0);
    const bool router = b < nbk * h_kv;
    const int kh = router ? b / nbk : 0, tr = router ? b % nbk : 0;
    bool ok = true;
    if (router && warp < ACW) {
        TeamSync ts{words + kh, abortw, a.status, &s_flag, nbk, 0u, a.wait_budget};
        ok = route_kvh<HD, R, G, RT>(a, kh, tr, nbk, smem, ts);
    }
    __shared__ int s_ok;
    if (threadIdx.x == 0) s_ok = 1;
    __syncthreads();
    if (!ok && threadIdx.x == 0) s_ok = 0;
    __syncthreads();
    unsigned gepoch = 0;
    if (s_ok && grid_barrier(words + h_kv, nb, gepoch, abortw, a.status, &s_flag, a.wait_budget)) {
        stamp(a, a.t.D);
        stage_map_init<false, StageCfg<KT, HD>::TT>(a, map);
        if (router && warp < ACW) write_lists<G>(a, kh, tr);
        attn_stages<KT, HD, G, false>(a, map, smem, b, nb);
        stamp(a, a.t.D + 1);
        // the last CTA to finish a KV head's stages merges its partials
        __threadfence();
        __syncthreads();
        if (threadIdx.x < h_kv) {
            const int k = threadIdx.x;
            int bf, bl;
            map.ctas(k, nb, bf, bl);
            int last = 0;
            if (bl >= 0 && b >= bf && b <= bl) {
                const unsigned tk = atomicAdd(a.ticket + k, 1u);
                last = (tk == (unsigned)(bl - bf));
                if (last) a.ticket[k] = 0u;
            }
            s_last[k] = last;
        }
        __syncthreads();
        for (int k = 0; k < h_kv; ++k) {
            if (!s_last[k]) continue;
            __threadfence();
            int bf, bl;
            map.ctas(k, nb, bf, bl);
            if (warp < ACW) combine_kvh<KT, HD, G>(a, map, k, bf, bl + 1, true, reinterpret_cast<float *>(smem));
            __syncthreads();
        }
        stamp(a, a.t.D + 2);
    }
    kernel_exit(words, h_kv + 3, h_kv + 1);
}

template <typename KT, int HD, int R, int G, typename RT>
static size_t decode_smem() {
    return std::max(RouteSmem<G>::bytes, ASmem<KT, HD, G>::bytes);
}

template <typename KT, int HD, int R, int G, typename RT>
static cudaError_t decode_impl(const Decode &dc, int n_cta, cudaStream_t s) {
    const size_t smem = decode_smem<KT, HD, R, G, RT>();
    static PerDeviceMax<> attr;
    const cudaError_t err = allow_smem(k_decode<KT, HD, R, G, RT>, smem, attr);
    if (err != cudaSuccess) return err;
    // cooperative (the CTAs meet at barriers), and a programmatic dependent
    // of the previous kernel so that its launch overlaps that kernel's tail
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n_cta);
    cfg.blockDim = dim3(A_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k_decode<KT, HD, R, G, RT>, dc);
}

template <typename KT, int HD, int R, int G, typename RT>
static int decode_occupancy() {
    const size_t smem = decode_smem<KT, HD, R, G, RT>();
    static PerDeviceMax<> attr;
    if (allow_smem(k_decode<KT, HD, R, G, RT>, smem, attr) != cudaSuccess) return 0;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, k_decode<KT, HD, R, G, RT>, A_THREADS, smem) != cudaSuccess)
        return 0;
    return blocks;
}

#define ZHA_DECODE_DISPATCH(FN, ...)                                                                      \
    do {                                                                                                  \
        const Tree &t = dc.t;                                                                             \
        if (t.g16[0]) {                                                                                   \
            if (t.kv_dtype == 1 && t.d == 128) {                                                          \
                if (t.R == 16 && t.G == 4) return FN<uint16_t, 128, 16, 4, uint16_t>(__VA_ARGS__);        \
                if (t.R == 1 && t.G == 4) return FN<uint16_t, 128, 1, 4, uint16_t>(__VA_ARGS__);          \
                if (t.R == 16 && t.G == 1) return FN<uint16_t, 128, 16, 1, uint16_t>(__VA_ARGS__);        \
                if (t.R == 1 && t.G == 1) return FN<uint16_t, 128, 1, 1, uint16_t>(__VA_ARGS__);          \
            }                                                                                             \
        } else if (t.kv_dtype == 1) {                                                                     \
            if (t.d == 128 && t.R == 16 && t.G == 4) return FN<uint16_t, 128, 16, 4, float>(__VA_ARGS__); \
            if (t.d == 128 && t.R == 1 && t.G == 4) return FN<uint16_t, 128, 1, 4, float>(__VA_ARGS__);   \
            if (t.d == 128 && t.R == 16 && t.G == 1) return FN<uint16_t, 128, 16, 1, float>(__VA_ARGS__); \
            if (t.d == 128 && t.R == 1 && t.G == 1) return FN<uint16_t, 128, 1, 1, float>(__VA_ARGS__);   \
            if (t.d == 64 && t.R == 16 && t.G == 4) return FN<uint16_t, 64, 16, 4, float>(__VA_ARGS__);   \
            if (t.d == 64 && t.R == 1 && t.G == 4) return FN<uint16_t, 64, 1, 4, float>(__VA_ARGS__);     \
            if (t.d == 64 && t.R == 16 && t.G == 1) return FN<uint16_t, 64, 16, 1, float>(__VA_ARGS__);   \
            if (t.d == 64 && t.R == 1 && t.G == 1) return FN<uint16_t, 64, 1, 1, float>(__VA_ARGS__);     \
        } else {                                                                                          \
            if (t.d == 128 && t.R == 16 && t.G == 4) return FN<float, 128, 16, 4, float>(__VA_ARGS__);    \
            if (t.d == 128 && t.R == 1 && t.G == 4) return FN<float, 128, 1, 4, float>(__VA_ARGS__);      \
            if (t.d == 128 && t.R == 16 && t.G == 1) return FN<float, 128, 16, 1, float>(__VA_ARGS__);    \
            if (t.d == 128 && t.R == 1 && t.G == 1) return FN<float, 128, 1, 1, float>(__VA_ARGS__);      \
            if (t.d == 64 && t.R == 16 && t.G == 4) return FN<float, 64, 16, 4, float>(__VA_ARGS__);      \
            if (t.d == 64 && t.R == 1 && t.G == 4) return FN<float, 64, 1, 4, float>(__VA_ARGS__);        \
            if (t.d == 64 && t.R == 16 && t.G == 1) return FN<float, 64, 16, 1, float>(__VA_ARGS__);      \
            if (t.d == 64 && t.R == 1 && t.G == 1) return FN<float, 64, 1, 1, float>(__VA_ARGS__);        \
        }                                                                                                 \
    } while (0)

cudaError_t launch_decode(const Decode &dc, int n_cta, cudaStream_t s) {
    ZHA_DECODE_DISPATCH(decode_impl, dc, n_cta, s);
    return cudaErrorInvalidValue;
}

int decode_blocks_per_sm(const Decode &dc) {
    ZHA_DECODE_DISPATCH(decode_occupancy);
    return 0;
}

}  // namespace zha
