// zha_route.cuh -- one routing level of one KV head, cut by a team of CTAs.
//
// Routing ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢":
// the query scores the top nodes, keeps the smallest set whose estimated mass
// reaches p and expands only their children, down to the raw entries;
// "Zyphra 分层注意力（ZHA）…", section "机制拆解：树形索引如何高效筛选长上下文").
// For query head h with frontier F_h at a level: est_n = max_j (b_j + q.g_j/√d)
// (the tangent-plane estimate), P_n = softmax over F_h, order by P descending
// with ties to the lower node id, keep the shortest prefix whose cumulative P
// reaches p; p >= 1 keeps every node.
//
// The frontier of KV head kh is the union over its G query heads: the
// children of every node any head kept one level up, each with the bitmask of
// the heads that kept its parent.  A team of T CTAs routes it, in one of
// three ways (LevelMode), chosen by the frontier size alone:
//   LV_ALL (small frontiers): every CTA scores every slot itself and cuts
//   the whole frontier, so every CTA knows the kept list without waiting for
//   another (the summaries come from L2 after the first CTA's read);
//   LV_SPLIT (up to RDS_MAX slots): each CTA scores a contiguous slice of
//   the slots into a team buffer, one team barrier, then every CTA copies all
//   the scores in and cuts the whole frontier itself;
//   LV_TEAM (larger): each CTA scores and cuts its own slice against the
//   team's histograms (below) and writes its kept nodes as a segment.
// Every CTA of a team computes the same integers in the same order, so the
// cuts of the first two ways agree on every CTA.
// Scoring streams each node's summary rows once (bulk copies into per-warp
// shared-memory stages) and scores each node for all G heads.  Masses are
// w = exp(est - M_h) in 2^-40 fixed point (integer sums are exact and do not
// depend on the order of addition), M_h the maximum over the frontier, and
// the target is ceil(p * Z_h) of the total Z_h.  Every decision is
// deterministic:
//   one CTA, at most SOLO_MAX slots: each head's slots are ordered by
//   (estimate descending, node id ascending) -- ranked slot against slot up
//   to RANK_MAX slots, sorted above -- and kept while the mass before each is
//   below the target;
//   otherwise, round 0 histograms mass and count over buckets of width 1/32
//   of a log-mass unit below M_h; the bucket where the cumulative mass first
//   reaches the target holds the cut: every node of a lower bucket is kept,
//   none of a higher one; when that bucket holds more than CAND_MAX nodes,
//   rounds 1 and 2 split it 1024-fold again (widths 1/32768 and 1/2^25); the
//   nodes of the final bucket are ranked exactly as above; a final bucket
//   still larger than CAND_MAX holds estimates within 2^-25 of each other and
//   is taken in node-id order.
// On an LV_TEAM level, team barriers separate: the maxima (A), each
// histogram round (B), the boundary lists (C) and the written segments (D).
//
// Code size matters here as much as arithmetic: every function runs once per
// level on little data, so cold instruction fetch dominates unless the code is
// short.  Loops that are not hot are kept rolled.
//
// `kh` below is a virtual KV head (Decode::nvk): a query of the batch paired
// with a KV head.  Scratch, teams and lists are indexed by it; summaries are
// read from its physical KV head, kh % h_kv.
//
// Every function here is called by threads 0-255 of a CTA (warps 0-7) and
// synchronises them with the named barrier of gsync().
#pragma once

#include "zha_device.cuh"
#include "zha_internal.cuh"
#include "zha_sync.cuh"

namespace zha {

constexpr int PAR_CAP = LOC_CAP;        // parents held in shared memory: a whole kept list, or the
                                        // window of LOC_CAP consecutive slots (c >= 2)
constexpr int SOLO_MAX = GT;           // one-CTA cuts up to this many slots are sorted (one warp per head)
constexpr int RANK_MAX = 32;           // ... ranked slot against slot up to this many (shorter code)
constexpr int RDA_SLOTS = SOLO_MAX;     // every CTA scores every slot itself up to this many slots
constexpr int64_t RDA_BYTES = 160 * 1024;  // ... and this many summary bytes
constexpr int RDS_MAX = 1000;           // scored in slices and cut by every CTA up to this many slots (a
                                        // larger frontier is cut faster in slices against team histograms)

// How a level is routed (the same choice on every CTA of the team):
//   LV_ALL   every CTA scores and cuts the whole frontier (no inter-CTA wait);
//   LV_SPLIT each CTA scores a slice, one team barrier, every CTA cuts the
//            whole frontier from all the scores;
//   LV_TEAM  each CTA scores and cuts a slice against the team's histograms
//            (barriers A-D), and writes its slice's kept nodes as a segment.
enum LevelMode : int { LV_ALL = 0, LV_SPLIT = 1, LV_TEAM = 2 };

enum CutMode : int { CUT_OPEN = 0, CUT_RANK = 1, CUT_ORDER = 2, CUT_ALL = 3, CUT_NONE = 4 };

struct HeadCut {
    unsigned long long Z, target, C;  // total mass, target, mass strictly above the bucket path
    float M;                          // maximum estimate
    uint32_t F;                       // frontier nodes of this head
    uint32_t nfin;                    // nodes in the last fixed bucket
    int32_t path[HIST_ROUNDS];        // bucket fixed in each round
    int rounds;                       // rounds fixed so far
    int mode;
};

constexpr int SW_STAGES = 2;            // scoring stages per warp
constexpr int SW_BYTES = 8 * 1024;      // one stage of summary rows
constexpr int SW_ROWS_MAX = 32;         // summary rows (and slots) in a stage at most
constexpr int SW_N = (GT / 32) * SW_STAGES;  // stages of the CTA

// Shared memory of the routing.  The two scoring chunks share their space
// with the histogram and boundary lists, which are used only after scoring.
template <int G>
struct RouteSmem {
    // [LOC_CAP][G] f32 scores: this CTA's slots of a team level, or every
    // slot of a level cut by every CTA (at most RDS_MAX slots)
    static constexpr size_t off_sc = 0;
    static_assert(RDS_MAX <= LOC_CAP, "a level cut by every CTA fits the local score array");
    static constexpr size_t off_node = off_sc + (size_t)LOC_CAP * G * 4;  // [LOC_CAP] i32
    static constexpr size_t off_keep = off_node + (size_t)LOC_CAP * 4;    // [LOC_CAP] u8
    static constexpr size_t off_u = off_keep + LOC_CAP;                   // union: chunks | cut scratch
    static constexpr size_t off_chunk = off_u;                            // [8 warps][SW_STAGES][SW_BYTES]
    // the cut scratch closes the union: the histograms during the rounds,
    // then the boundary lists in the same bytes (the rounds are over by then)
    static constexpr size_t hist_bytes = (size_t)G * NB * 12;
    static constexpr size_t cand_bytes = (size_t)G * CAND_MAX * 16;
    static constexpr size_t scr_bytes = hist_bytes > cand_bytes ? hist_bytes : cand_bytes;
    static constexpr size_t u_end = off_u + ((size_t)SW_N * SW_BYTES > scr_bytes ? (size_t)SW_N * SW_BYTES : scr_bytes);
    static constexpr size_t off_scr = u_end - scr_bytes;
    static constexpr size_t off_hc = off_scr;                             // [G][NB] u32
    static constexpr size_t off_hm = off_hc + (size_t)G * NB * 4;         // [G][NB] u64 (solo: [SOLO_MAX][G] masses)
    static constexpr size_t off_cw = off_scr;                             // [G][CAND_MAX] u64
    static constexpr size_t off_cs = off_cw + (size_t)G * CAND_MAX * 8;   // [G][CAND_MAX] u32
    static constexpr size_t off_own = off_cs + (size_t)G * CAND_MAX * 4;  // [G*CAND_MAX] u32
    // A slice that spills (more than LOC_CAP slots) comes back on chip for
    // its cut when its scores fit below the scratch: the local arrays and
    // the scoring stages are idle then (its node ids and keep bits stay in
    // global memory)
    static constexpr int64_t SPILL_CAP = (int64_t)(off_scr / (G * 4));
    static constexpr size_t off_pid = u_end;                              // [PAR_CAP] i32 parents
    static constexpr size_t off_pmk = off_pid + (size_t)PAR_CAP * 4;      // [PAR_CAP] u8 their head masks
    static constexpr size_t off_pref = (off_pmk + PAR_CAP + 15) / 16 * 16;  // [SEG_CAP + 1] u32
    static constexpr size_t off_cut = (off_pref + (SEG_CAP + 1) * 4 + 15) / 16 * 16;  // [G] HeadCut
    static constexpr size_t off_wm = (off_cut + G * sizeof(HeadCut) + 15) / 16 * 16;  // [8][G] f32 warp maxima
    static constexpr size_t off_wc = off_wm + 8 * G * 4;                  // [8][G] u32 warp counts
    static constexpr size_t off_red = (off_wc + 8 * G * 4 + 15) / 16 * 16; // [GT] u64
    static constexpr size_t off_bar = off_red + GT * 8;                   // [SW_N] u64 stage barriers
    static constexpr size_t off_uses = off_bar + SW_N * 8;               // [SW_N] u32 completed phases
    static constexpr size_t off_cnode = off_uses + SW_N * 4;              // [SW_N][SW_ROWS_MAX] i32
    static constexpr size_t off_cmask = off_cnode + (size_t)SW_N * SW_ROWS_MAX * 4;  // [SW_N][SW_ROWS_MAX] u8
    static constexpr size_t off_cb = (off_cmask + (size_t)SW_N * SW_ROWS_MAX + 15) / 16 * 16;  // [SW_N][SW_ROWS_MAX] f32
    static constexpr size_t off_misc = off_cb + (size_t)SW_N * SW_ROWS_MAX * 4;  // u32 counters
    static constexpr size_t off_cbar = off_misc + 64;                     // u64: barrier of the scores' return
    static constexpr size_t off_cuse = off_cbar + 8;                      // u32: its completed phases
    static constexpr size_t bytes = off_cuse + 8;
    static_assert(SOLO_MAX * G * 8 <= G * NB * 8, "solo masses fit the histogram area");
    static_assert(off_u % 16 == 0, "bulk copies land on 16-byte boundaries");
};

// One level of one KV head as seen by one CTA of its team.
struct Level {
    int l, kh, T, tr;
    bool top;
    int64_t S, s0, n;       // frontier slots, first local slot, local slots
    int Tp;                 // team size of the parent level
    int64_t Sp;             // frontier size of the parent level
    float *sc;              // [n][G] local scores (shared memory, or global when n > LOC_CAP)
    bool sc_local;          // sc is in shared memory
    int32_t *node;          // [n] node of each local slot (-1: no such child)
    uint8_t *keep;          // [n] heads that keep the slot
};

struct TeamSync {
    unsigned *ctr;
    unsigned *abortw;
    int32_t *status;
    int *flag;
    int T;
    unsigned epoch;
    long long budget;  // clock cycles one barrier wait may take
    __device__ __forceinline__ bool sync() {
        if (T == 1) {
            gsync();
            return true;
        }
        return team_barrier(ctr, T, epoch, abortw, status, flag, budget);
    }
};

// ---- level bookkeeping ---------------------------------------------------

__device__ __forceinline__ uint32_t *seg_ptr(const Decode &a, int l, int kh) {
    return a.seg + ((int64_t)(l - 1) * a.nvk + kh) * SEG_CAP;
}
__device__ __forceinline__ uint32_t *hseg_ptr(const Decode &a, int l, int kh) {
    return a.hseg + ((int64_t)(l - 1) * a.nvk + kh) * SEG_CAP * a.t.G;
}
__device__ __forceinline__ int32_t *lvl_ptr(const Decode &a, int l, int kh) {
    return a.lvl + ((int64_t)(l - 1) * a.nvk + kh) * 2;
}
// First slot of team rank r's range of a level with S slots and T ranks.
__device__ __forceinline__ int64_t seg_start(int64_t S, int T, int r) { return S * r / T; }

// Exclusive prefix of level l's per-rank kept counts (T ranks, known to the
// caller) into pref[0..T] (shared); returns the total.  `scratch`: 8 shared
// uint32.
__device__ __noinline__ int64_t load_segments(const Decode &a, int l, int kh, int T, uint32_t *pref,
                                              uint32_t *scratch) {
    const uint32_t *sg = seg_ptr(a, l, kh);
    const uint32_t x = (int)threadIdx.x < T ? __ldcg(sg + threadIdx.x) : 0u;
    uint32_t total;
    const uint32_t incl = g_scan_u32(x, scratch, &total);
    if ((int)threadIdx.x < T) pref[threadIdx.x + 1] = incl;
    if (threadIdx.x == 0) pref[0] = 0u;
    gsync();
    return total;
}

// Team rank holding kept rank k of a level (pref: exclusive prefix, T ranks).
__device__ __forceinline__ int seg_find(const uint32_t *pref, int T, int64_t k) {
    int lo = 0, hi = T - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)pref[mid] <= k) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Parents of slots [c0, c1) of level L (ranks [k0, k1]) into the window.
__device__ __noinline__ void load_parents(const Decode &a, const Level &L, int64_t c0, int64_t c1, const uint32_t *pref,
                                          int32_t *pid, uint8_t *pmk, int64_t &k0) {
    const int c = a.t.c, clog = a.t.c_log2;
    k0 = clog >= 0 ? (c0 >> clog) : c0 / c;
    const int64_t k1 = clog >= 0 ? ((c1 - 1) >> clog) : (c1 - 1) / c;
    const int lp = L.l + 1;
    const int64_t pbase = (int64_t)L.kh * a.slot_cap[lp - 1];
#pragma unroll 1
    for (int64_t k = k0 + threadIdx.x; k <= k1; k += GT) {
        const int r = seg_find(pref, L.Tp, k);
        const int64_t at = pbase + seg_start(L.Sp, L.Tp, r) + (k - pref[r]);
        pid[k - k0] = __ldcg(a.kept_ids[lp - 1] + at);
        pmk[k - k0] = __ldcg(a.kept_mask[lp - 1] + at);
    }
}

// ---- scoring ----------------------------------------------------------------

// Sums of the G per-lane partial dots over the warp.  G = 4: a reduce-scatter
// (xor 16, 8) then a butterfly (xor 4, 2, 1) leaves lane l with the sum of
// head (l >> 3) & 3.  G = 1: a butterfly.  One fixed order each.
template <int G>
__device__ __forceinline__ float head_sum(const float (&v)[G], int lane) {
    if constexpr (G == 4) {
        const bool up = (lane & 16) != 0;
        float s0 = up ? v[2] : v[0], s1 = up ? v[3] : v[1];
        const float t0 = up ? v[0] : v[2], t1 = up ? v[1] : v[3];
        s0 += __shfl_xor_sync(FULL, t0, 16);
        s1 += __shfl_xor_sync(FULL, t1, 16);
        const bool up8 = (lane & 8) != 0;
        float k = up8 ? s1 : s0;
        k += __shfl_xor_sync(FULL, up8 ? s0 : s1, 8);
        k += __shfl_xor_sync(FULL, k, 4);
        k += __shfl_xor_sync(FULL, k, 2);
        k += __shfl_xor_sync(FULL, k, 1);
        return k;
    } else {
        float k = v[0];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) k += __shfl_xor_sync(FULL, k, off);
        return k;
    }
}

// The g rows and plane offsets the router reads: fp32 (RT = float) or the
// bf16 copy (RT = uint16_t) with its own offsets.
template <typename RT>
__device__ __forceinline__ const RT *router_g(const Tree &t, int l);
template <>
__device__ __forceinline__ const float *router_g<float>(const Tree &t, int l) { return t.g[l - 1]; }
template <>
__device__ __forceinline__ const uint16_t *router_g<uint16_t>(const Tree &t, int l) { return t.g16[l - 1]; }
template <typename RT>
__device__ __forceinline__ const float *router_b(const Tree &t, int l) {
    return sizeof(RT) == 2 ? t.b16[l - 1] : t.b[l - 1];
}

template <int HD, int R, typename RT>
struct ScoreStage {
    static constexpr int NODE_BYTES = R * HD * (int)sizeof(RT);      // g rows of one node (fp32 or the bf16 copy)
    static constexpr int SLOTS = SW_BYTES / NODE_BYTES < SW_ROWS_MAX / R ? SW_BYTES / NODE_BYTES
                                                                          : SW_ROWS_MAX / R;  // slots per stage
    static constexpr int ROWS = SLOTS * R;                           // summary rows per stage
    static_assert(SLOTS >= 1 && ROWS % 8 == 0 && ROWS <= SW_ROWS_MAX, "stage shape");
};

// One warp: node ids of the slots of unit u (SLOTS consecutive local slots
// from c0), bulk copies of their g rows (one copy per run of consecutive
// nodes) into this warp's stage buffer `dst`, and the plane offset of each
// row (slot r / R, plane r % R) into cb[r] by 4-byte asynchronous copies, all
// completing on the stage barrier `bar` (each copying lane adds one pending
// arrival that its copy's completion clears, before the expect-tx arrive).
template <int HD, int R, int G, typename RT>
__device__ __forceinline__ void stage_issue(const Level &L, int64_t c0, int64_t c1, int64_t k0, int64_t u,
                                            const int32_t *pid, const uint8_t *pmk, const RT *gb, const float *bb,
                                            int c, int clog, int32_t nl, unsigned char *dst, uint64_t *bar,
                                            int32_t *cn, uint8_t *cm, float *cb, int lane) {
    using C = ScoreStage<HD, R, RT>;
    const int64_t sb = c0 + u * C::SLOTS;
    const int ns = (int)min((int64_t)C::SLOTS, c1 - sb);
    int nd = -1;
    if (lane < ns) {
        const int s = (int)(sb + lane);
        nd = s;
        uint32_t mk = (1u << G) - 1u;
        if (!L.top) {
            const int kk = clog >= 0 ? (s >> clog) : (int)((uint32_t)s / (uint32_t)c);
            nd = pid[kk - (int)k0] * c + (s - kk * c);
            mk = pmk[kk - (int)k0];
        }
        if (nd >= nl) nd = -1;
        cn[lane] = nd;
        cm[lane] = nd >= 0 ? (uint8_t)mk : 0;
    }
    const uint32_t nvalid = __popc(__ballot_sync(FULL, nd >= 0));
    const int ndr = __shfl_sync(FULL, nd, (lane / R) & 31);
    if (lane < C::ROWS && ndr >= 0) {
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(cb + lane)),
                     "l"(bb + (size_t)ndr * R + lane % R)
                     : "memory");
        asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
    }
    __syncwarp();
    // (the stage's earlier contents were only read, and those reads completed
    // before the warp got here: a bulk copy may overwrite it without a fence)
    if (lane == 0) mbar_arrive_expect_tx(bar, nvalid * (uint32_t)C::NODE_BYTES);
    __syncwarp();
    // a run starts where the node does not follow its left neighbour's
    const int left = __shfl_up_sync(FULL, nd, 1);
    const bool start = nd >= 0 && (lane == 0 || left < 0 || left + 1 != nd);
    const unsigned brk = __ballot_sync(FULL, start || nd < 0);
    if (start) {
        const unsigned after = lane == 31 ? 0u : (brk >> (lane + 1));
        const int len = after ? __ffs(after) : 32 - lane;
        bulk_g2s_hint(dst + (size_t)lane * C::NODE_BYTES, gb + (size_t)nd * R * HD, (uint32_t)(len * C::NODE_BYTES),
                      bar, l2_evict_first());
    }
}

// Sums over the warp of 8 rows x G heads of per-lane partial dots, v[row*G + h].
// Afterwards lane l holds the sum of (row (l / G) % 8, head l % G): G = 4 is a
// reduce-scatter of 32 values; G = 1 reduce-scatters 8 values over 8 lanes and
// finishes with a butterfly over the groups of 8.  One fixed order each.
template <int G>
__device__ __forceinline__ float batch_sum(float (&v)[8 * G], int lane) {
    if constexpr (G == 4) {
        reduce_scatter<32>(v, lane);
        return v[0];
    } else {
        reduce_scatter<8, 8>(v, lane);
        float k = v[0];
        k += __shfl_xor_sync(FULL, k, 8);
        k += __shfl_xor_sync(FULL, k, 16);
        return k;
    }
}

// The scoring stage barriers of every warp: initialised once before the
// first level (one arrival per phase: the expect-tx arrive of the issuing
// lane) with their phase counts, and invalidated after the last level, so
// that the memory can serve other purposes.  Warps 0-7, each its own.
template <int G>
__device__ __forceinline__ void stages_init(unsigned char *smem) {
    using SM = RouteSmem<G>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::off_bar) + warp * SW_STAGES;
        uint32_t *uses = reinterpret_cast<uint32_t *>(smem + SM::off_uses) + warp * SW_STAGES;
#pragma unroll
        for (int st = 0; st < SW_STAGES; ++st) {
            mbar_init(&bars[st], 1);
            uses[st] = 0u;
        }
        if (warp == 0) {
            mbar_init(reinterpret_cast<uint64_t *>(smem + SM::off_cbar), 1);
            *reinterpret_cast<uint32_t *>(smem + SM::off_cuse) = 0u;
        }
        mbar_init_fence();
    }
    __syncwarp();
}

template <int G>
__device__ __forceinline__ void stages_inval(unsigned char *smem) {
    using SM = RouteSmem<G>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncwarp();
    if (lane == 0) {
        uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::off_bar) + warp * SW_STAGES;
#pragma unroll
        for (int st = 0; st < SW_STAGES; ++st) mbar_inval(&bars[st]);
        if (warp == 0) mbar_inval(reinterpret_cast<uint64_t *>(smem + SM::off_cbar));
    }
    __syncwarp();
}

// Score local slots [c0, c1) (global slot ids) of level L.  The slots go in
// units of ScoreStage::SLOTS consecutive slots, unit u to warp u % 8; each
// warp streams its own units through SW_STAGES shared-memory stages with
// their own barriers (bulk copies of unit j + SW_STAGES are issued as soon as
// the warp has scored unit j), so no warp waits for another while scoring.
// A warp scores 8 summary rows at a time (one reduce-scatter per 8 rows) and
// keeps each node's maximum over its planes in registers.  Parent window:
// ranks [k0, ...) in pid/pmk.  Writes L.sc / L.node at (s - L.s0) and folds
// the maxima and counts per head into wm/wc[warp][h].
template <int HD, int R, int G, typename RT>
__device__ __noinline__ void score_chunks(const Decode &a, const Level &L, int64_t c0, int64_t c1, int64_t k0,
                                          const int32_t *pid, const uint8_t *pmk, unsigned char *smem, float *wm,
                                          uint32_t *wc) {
    static_assert(G == 1 || G == 4, "query heads per KV head");
    static_assert(R == 1 || R % 8 == 0, "planes per node: 1 or a multiple of 8");
    using C = ScoreStage<HD, R, RT>;
    using SM = RouteSmem<G>;
    constexpr int VEC = HD / 32;
    constexpr int NW = GT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kh = L.kh, l = L.l;
    unsigned char *bufs = smem + SM::off_chunk + (size_t)warp * SW_STAGES * SW_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::off_bar) + warp * SW_STAGES;
    int32_t *cnode = reinterpret_cast<int32_t *>(smem + SM::off_cnode) + warp * SW_STAGES * SW_ROWS_MAX;
    uint8_t *cmask = smem + SM::off_cmask + warp * SW_STAGES * SW_ROWS_MAX;
    float *cbs = reinterpret_cast<float *>(smem + SM::off_cb) + warp * SW_STAGES * SW_ROWS_MAX;
    float qs[G][VEC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        Vec<float, VEC>::load(a.q + (int64_t)(kh * G + h) * HD + lane * VEC, qs[h]);
#pragma unroll
        for (int e = 0; e < VEC; ++e) qs[h][e] *= a.t.scale;
    }
    const int64_t cap = a.t.node_cap[l - 1];
    const int pk = kh % a.t.h_kv;  // the physical KV head of virtual head kh
    const RT *gb = router_g<RT>(a.t, l) + (int64_t)pk * cap * R * HD;
    const float *bb = router_b<RT>(a.t, l) + (int64_t)pk * cap * R;
    const int c = a.t.c, clog = a.t.c_log2;
    const int32_t nl = a.t.n_level[l - 1];
    const int64_t nu = (c1 - c0 + C::SLOTS - 1) / C::SLOTS;  // units
    const int nmine = nu > warp ? (int)((nu - 1 - warp) / NW + 1) : 0;
    static_assert(SW_STAGES == 2, "two stages: units 0 and 1 go out before the loop");
    // phases each stage barrier has completed before this call
    uint32_t *uses = reinterpret_cast<uint32_t *>(smem + SM::off_uses) + warp * SW_STAGES;
    const uint32_t u0 = uses[0], u1 = uses[1];
    // the stages' bytes were last written through the generic proxy (the
    // previous level's cut scratch): fenced once here, before any copy lands
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    gsync();
    if (nmine > 0)
        stage_issue<HD, R, G, RT>(L, c0, c1, k0, warp, pid, pmk, gb, bb, c, clog, nl, bufs, &bars[0], cnode, cmask,
                                  cbs, lane);
    if (nmine > 1)
        stage_issue<HD, R, G, RT>(L, c0, c1, k0, warp + NW, pid, pmk, gb, bb, c, clog, nl, bufs + SW_BYTES, &bars[1],
                                  cnode + SW_ROWS_MAX, cmask + SW_ROWS_MAX, cbs + SW_ROWS_MAX, lane);
    const int hl = lane % G;             // head of this lane's sum
    const int rl = (lane / G) % 8;       // row of this lane's sum within the batch
    float mymax = -INFINITY;             // this lane's head's maximum (lanes < G report)
    uint32_t mycnt = 0u;
#pragma unroll 1
    for (int j = 0; j < nmine; ++j) {
        const int st = j % SW_STAGES;
        const int64_t u = warp + (int64_t)j * NW;
        const int64_t sb = c0 + u * C::SLOTS;
        const int ns = (int)min((int64_t)C::SLOTS, c1 - sb);
        const int32_t *cn = cnode + st * SW_ROWS_MAX;
        const uint8_t *cm = cmask + st * SW_ROWS_MAX;
        if (!mbar_wait(&bars[st], ((st ? u1 : u0) + (uint32_t)(j / SW_STAGES)) & 1u, nullptr))
            set_status(a.status, ZHA_TIMEOUT_CODE);
        const float *cbr = cbs + st * SW_ROWS_MAX;  // plane offsets of the stage's rows
        const RT *cb = reinterpret_cast<const RT *>(bufs + (size_t)st * SW_BYTES);
        float est = -INFINITY;
#pragma unroll 2
        for (int r0 = 0; r0 < C::ROWS; r0 += 8) {
            // rows r0 .. r0 + 7: slot r / R, plane r % R
            float v[8 * G];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int r = r0 + q;
                float gs[VEC];
                if (r / R < ns) {
                    Vec<RT, VEC>::load(cb + (size_t)r * HD + lane * VEC, gs);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) gs[e] = 0.f;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) v[q * G + h] = lane_dot<VEC>(qs[h], gs);
            }
            const float sum = batch_sum<G>(v, lane);
            const int r = r0 + rl;
            const float e = cbr[r] + sum;
            if constexpr (R == 1) {
                // every row is its own slot
                const int i = r;
                if (i < ns && (G == 4 || lane < 8)) {
                    const int nd = cn[i];
                    const bool need = nd >= 0 && ((cm[i] >> hl) & 1u);
                    const int64_t s = sb + i - L.s0;
                    L.sc[s * G + hl] = need ? e : -INFINITY;
                    if (hl == 0) L.node[s] = nd;
                    if (need) {
                        mymax = fmaxf(mymax, e);
                        mycnt += 1u;
                    }
                }
            } else {
                // the 8 rows belong to one slot: max over them, then over batches
                float m8 = e;
#pragma unroll
                for (int off = G; off < 8 * G; off <<= 1) m8 = fmaxf(m8, __shfl_xor_sync(FULL, m8, off));
                est = fmaxf(est, m8);
                if ((r0 + 8) % R == 0) {
                    const int i = r0 / R;
                    if (i < ns && lane < G) {
                        const int nd = cn[i];
                        const bool need = nd >= 0 && ((cm[i] >> hl) & 1u);
                        const int64_t s = sb + i - L.s0;
                        L.sc[s * G + hl] = need ? est : -INFINITY;
                        if (hl == 0) L.node[s] = nd;
                        if (need) {
                            mymax = fmaxf(mymax, est);
                            mycnt += 1u;
                        }
                    }
                    est = -INFINITY;
                }
            }
        }
        __syncwarp();  // stage st is free
        if (j + SW_STAGES < nmine)
            stage_issue<HD, R, G, RT>(L, c0, c1, k0, u + (int64_t)SW_STAGES * NW, pid, pmk, gb, bb, c, clog, nl,
                                      bufs + (size_t)st * SW_BYTES, &bars[st], cnode + st * SW_ROWS_MAX,
                                      cmask + st * SW_ROWS_MAX, cbs + st * SW_ROWS_MAX, lane);
    }
    __syncwarp();
    if (lane == 0) {
        uses[0] = u0 + (uint32_t)(nmine + 1) / 2;
        uses[1] = u1 + (uint32_t)nmine / 2;
    }
    // per-warp maxima and counts of each head: lanes with equal head
#pragma unroll
    for (int off = G; off < 32; off <<= 1) {
        mymax = fmaxf(mymax, __shfl_xor_sync(FULL, mymax, off));
        mycnt += __shfl_xor_sync(FULL, mycnt, off);
    }
    if (lane < G) {
        wm[warp * G + lane] = fmaxf(wm[warp * G + lane], mymax);
        wc[warp * G + lane] += mycnt;
    }
    gsync();
}

// ---- the cut ------------------------------------------------------------------

__device__ __forceinline__ int round_bucket(const HeadCut &H, float e, int r) {
    const float x = H.M - e;
    float f;
    if (r == 0) {
        f = x * 32.f;
    } else if (r == 1) {
        f = x * 32768.f - 1024.f * (float)H.path[0];
    } else {
        f = x * 33554432.f - 1024.f * (1024.f * (float)H.path[0] + (float)H.path[1]);
    }
    if (!(f >= 0.f)) return 0;
    return f < (float)(NB - 1) ? (int)f : NB - 1;
}

// A head's cut state in registers: the passes over every slot (histogram,
// classification) read these fields for every score, and shared-memory
// loads of them would sit on each score's dependency chain.
struct PathReg {
    float M;
    int p0, p1, p2, rounds, mode;
    PathReg() = default;
    __device__ __forceinline__ explicit PathReg(const HeadCut &H)
        : M(H.M), p0(H.path[0]), p1(H.path[1]), p2(H.path[2]), rounds(H.rounds), mode(H.mode) {}
    // round_bucket of score e in round r (the same arithmetic)
    __device__ __forceinline__ int bucket(float e, int r) const {
        const float x = M - e;
        float f;
        if (r == 0) {
            f = x * 32.f;
        } else if (r == 1) {
            f = x * 32768.f - 1024.f * (float)p0;
        } else {
            f = x * 33554432.f - 1024.f * (1024.f * (float)p0 + (float)p1);
        }
        if (!(f >= 0.f)) return 0;
        return f < (float)(NB - 1) ? (int)f : NB - 1;
    }
    // path_cmp over the first n rounds (n <= HIST_ROUNDS)
    __device__ __forceinline__ int cmp(float e, int n) const {
        static_assert(HIST_ROUNDS == 3, "three rounds");
        if (n > 0) {
            const int b = bucket(e, 0);
            if (b != p0) return b < p0 ? -1 : 1;
        }
        if (n > 1) {
            const int b = bucket(e, 1);
            if (b != p1) return b < p1 ? -1 : 1;
        }
        if (n > 2) {
            const int b = bucket(e, 2);
            if (b != p2) return b < p2 ? -1 : 1;
        }
        return 0;
    }
};

// -1: above the fixed path (kept), 1: below (dropped), 0: on it.
__device__ __forceinline__ int path_cmp(const HeadCut &H, float e, int rounds) {
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {
        const int b = round_bucket(H, e, r);
        if (b < H.path[r]) return -1;
        if (b > H.path[r]) return 1;
    }
    return 0;
}

__device__ __forceinline__ unsigned long long target_of(unsigned long long Z, float p) {
    unsigned long long tg = (unsigned long long)ceil((double)p * (double)Z);
    if (tg > Z) tg = Z;
    return tg ? tg : 1ull;
}

// Set head bit `bit` of keep[i] (byte array, any alignment) atomically.
__device__ __forceinline__ void keep_or(uint8_t *keep, int64_t i, uint32_t bit) {
    const uintptr_t at = reinterpret_cast<uintptr_t>(keep + i);
    atomicOr(reinterpret_cast<uint32_t *>(at & ~(uintptr_t)3), bit << (8 * (at & 3)));
}

// Exact cut of a one-CTA level with n <= RANK_MAX slots: thread i ranks slot
// i against every other slot of each head by (estimate descending, node id
// ascending) -- the order of the masses, which are monotone in the estimate --
// and sums the masses before it.  w: shared [SOLO_MAX][G] masses.
template <int G>
__device__ __noinline__ void solo_cut(const Level &L, HeadCut *cut, unsigned long long *w, float p) {
    static_assert(RANK_MAX * G <= GT, "one thread per (slot, head)");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = (int)L.n;
    // thread idx = slot * G + head: its mass, then the head's total over the
    // warps (lanes with equal idx % G; integer sums, any order)
    unsigned long long *wz = w + RANK_MAX * G;  // [GT / 32][G] per-warp totals
    const int h = tid % G;
    float ei = -INFINITY;
    unsigned long long wi = 0ull;
    if (tid < n * G) {
        ei = L.sc[tid];
        if (ei != -INFINITY) wi = mass_fx(expf(ei - cut[h].M));
        w[tid] = wi;
    }
    unsigned long long z = wi;
#pragma unroll
    for (int off = G; off < 32; off <<= 1) z += __shfl_xor_sync(FULL, z, off);
    if (lane < G) wz[warp * G + lane] = z;
    gsync();
    if (tid < G) {
        unsigned long long Z = 0ull;
#pragma unroll
        for (int v = 0; v < GT / 32; ++v) Z += wz[v * G + tid];
        cut[tid].Z = Z;
        cut[tid].target = target_of(Z, p);
    }
    gsync();
    // rank (slot, head) against the head's other slots: (estimate descending, slot ascending)
    bool kept = false;
    if (tid < n * G && ei != -INFINITY) {
        const int i = tid / G;
        unsigned long long pre = 0ull;
#pragma unroll 4
        for (int j = 0; j < n; ++j) {
            const float ej = L.sc[j * G + h];
            if (ej > ei || (ej == ei && j < i)) pre += w[j * G + h];
        }
        kept = pre < cut[h].target;
    }
    // the slot's keep bits: lanes i * G .. i * G + G - 1 of one warp (G divides 32)
    uint32_t kb = kept ? 1u << h : 0u;
#pragma unroll
    for (int off = 1; off < G; off <<= 1) kb |= __shfl_xor_sync(FULL, kb, off);
    if (tid < n * G && h == 0) L.keep[tid / G] = (uint8_t)kb;
    gsync();
}

// Exact cut of a one-CTA level with RANK_MAX < n <= SOLO_MAX slots.  Warp h sorts head
// h's slots by (estimate descending, slot ascending) -- the order of the
// masses, which are monotone in the estimate; slots follow node ids -- with a
// bitonic network over the warp (SOLO_MAX / 32 keys per lane: the float's
// order-preserving bits above the complemented slot), then sums the masses in
// that order and keeps each slot while the mass before it is below the
// target.  Slots a head does not score (-inf) sort last and are not kept.
template <int G>
__device__ __noinline__ void sort_cut(const Level &L, const HeadCut *cut, float p) {
    constexpr int E = SOLO_MAX / 32;  // keys per lane; key i = lane * E + k
    static_assert(SOLO_MAX % 32 == 0 && (E & (E - 1)) == 0 && G <= GT / 32, "sort shape");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n = (int)L.n;
#pragma unroll 1
    for (int i = threadIdx.x; i < n; i += GT) L.keep[i] = 0;
    gsync();
    if (warp < G) {
        const int h = warp;
        unsigned long long key[E];
#pragma unroll
        for (int k = 0; k < E; ++k) {
            const int i = lane * E + k;
            const float e = i < n ? L.sc[i * G + h] : -INFINITY;
            const uint32_t u = __float_as_uint(e);
            const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
            key[k] = e == -INFINITY ? 0ull : ((unsigned long long)ord << 32) | (0xFFFFFFFFu - (uint32_t)i);
        }
        // bitonic network, descending overall, over the first nsort keys (a
        // power of two >= n; the rest are 0 and already last); rolled loops
        // keep the code short, the per-lane keys stay in registers
        int nsort = 2;
        while (nsort < n) nsort <<= 1;
#pragma unroll 1
        for (int size = 2; size <= nsort; size <<= 1) {
#pragma unroll 1
            for (int j = size >> 1; j >= E; j >>= 1) {
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    const int i = lane * E + k;
                    const unsigned long long o = __shfl_xor_sync(FULL, key[k], j / E);
                    const bool take_max = ((i & j) == 0) == ((i & size) == 0);
                    key[k] = take_max ? (key[k] > o ? key[k] : o) : (key[k] < o ? key[k] : o);
                }
            }
            // in-lane stages j = E/2 .. 1 (those below size)
#pragma unroll
            for (int j = E >> 1; j > 0; j >>= 1) {
                if (j < size) {
#pragma unroll
                    for (int k = 0; k < E; ++k) {
                        if (k & j) continue;
                        const int i = lane * E + k;
                        const unsigned long long a = key[k], b = key[k | j];
                        const bool desc = (i & size) == 0;
                        const unsigned long long hi = a > b ? a : b, lo = a > b ? b : a;
                        key[k] = desc ? hi : lo;
                        key[k | j] = desc ? lo : hi;
                    }
                }
            }
        }
        // masses in sorted order, then the exclusive prefix over the warp
        const float M = cut[h].M;
        unsigned long long w[E], mine = 0ull;
#pragma unroll
        for (int k = 0; k < E; ++k) {
            w[k] = 0ull;
            if (key[k]) {
                const int i = (int)(0xFFFFFFFFu - (uint32_t)key[k]);
                w[k] = mass_fx(expf(L.sc[i * G + h] - M));
            }
            mine += w[k];
        }
        unsigned long long incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned long long y = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += y;
        }
        const unsigned long long Z = __shfl_sync(FULL, incl, 31);
        const unsigned long long target = target_of(Z, p);
        unsigned long long run = incl - mine;
#pragma unroll
        for (int k = 0; k < E; ++k) {
            if (key[k]) {
                const int i = (int)(0xFFFFFFFFu - (uint32_t)key[k]);
                if (run < target) keep_or(L.keep, i, 1u << h);
                run += w[k];
            }
        }
    }
    gsync();
}

// Local histogram of round r over this CTA's slots on the path of every open
// head: counts into hc, masses into hw.  A mass (at most 2^40 in units of
// 2^-40) is added as its low 20 bits and the rest into two 32-bit words, the
// bucket's pair in hw (the 8 bytes of its 64-bit mass): 64-bit atomics on
// shared memory cost about ten times as much as 32-bit ones.  Both sums stay
// below 2^31 for up to HIST_WIN slots, after which fold_window() or
// fold_local() must take them.  Slots of heads whose mass is 0 add nothing.
constexpr int HIST_WIN = 2048;
template <int G>
__device__ __noinline__ void local_hist(const Level &L, const HeadCut *cut, int r, uint32_t *hc, uint32_t *hw) {
    // GT is a multiple of G: every entry this thread visits belongs to head tid % G
    const int h = (int)(threadIdx.x % G);
    const PathReg H(cut[h]);
    if (H.mode == CUT_OPEN && H.rounds == r) {
        const int64_t total = L.n * G;
#pragma unroll 1
        for (int64_t i0 = threadIdx.x; i0 < total; i0 += 4 * GT) {
            float e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) e[u] = i0 + u * GT < total ? L.sc[i0 + u * GT] : -INFINITY;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (e[u] == -INFINITY || H.cmp(e[u], r) != 0) continue;
                const int b = h * NB + H.bucket(e[u], r);
                const unsigned long long m = mass_fx(expf(e[u] - H.M));
                const uint32_t lo = (uint32_t)(m & 0xfffffull), hi = (uint32_t)(m >> 20);
                atomicAdd(&hc[b], 1u);
                if (lo) atomicAdd(&hw[2 * b], lo);
                if (hi) atomicAdd(&hw[2 * b + 1], hi);
            }
        }
    }
    gsync();
}

// A window's counts and masses into the team's histogram of the round
// (global, exact integer sums); the shared words are left cleared.
template <int G>
__device__ __forceinline__ void fold_window(uint32_t *hc, uint32_t *hw, uint32_t *gc, unsigned long long *gm) {
#pragma unroll 1
    for (int i = threadIdx.x; i < G * NB; i += GT) {
        const uint32_t n = hc[i];
        if (n) {
            atomicAdd(gc + i, n);
            atomicAdd(gm + i, (unsigned long long)hw[2 * i] + ((unsigned long long)hw[2 * i + 1] << 20));
            hc[i] = 0u;
            hw[2 * i] = 0u;
            hw[2 * i + 1] = 0u;
        }
    }
    gsync();
}

// One window's mass words turned, in place, into the 64-bit masses find_cut reads.
template <int G>
__device__ __forceinline__ void fold_local(uint32_t *hw) {
#pragma unroll 1
    for (int i = threadIdx.x; i < G * NB; i += GT) {
        const unsigned long long m = (unsigned long long)hw[2 * i] + ((unsigned long long)hw[2 * i + 1] << 20);
        reinterpret_cast<unsigned long long *>(hw)[i] = m;
    }
    gsync();
}

// Fix the bucket of round r for every open head from the histogram (masses
// in shared memory; counts in shared memory, or the team's global counts
// `gcnt` read through L2 when not null: only the chosen bucket's is read).
template <int G>
__device__ __noinline__ void find_cut(HeadCut *cut, int r, const uint32_t *cnt, const uint32_t *gcnt,
                                      const unsigned long long *mass, float p, unsigned long long *red) {
    constexpr int TPH = GT / G, BPT = NB / TPH;
    static_assert((BPT & (BPT - 1)) == 0, "buckets per thread: a power of two");
    const int tid = threadIdx.x, h = tid / TPH, j = tid % TPH, lane = tid & 31;
    const bool act = cut[h].mode == CUT_OPEN && cut[h].rounds == r;
    unsigned long long sum = 0ull;
    // each thread sums its run of BPT buckets starting at a lane-dependent
    // offset, so that the lanes of a warp read different banks
#pragma unroll 4
    for (int i = 0; i < BPT; ++i) {
        const int b = j * BPT + ((i + lane) & (BPT - 1));
        sum += act ? mass[h * NB + b] : 0ull;
    }
    // inclusive scan of the per-thread sums within each head's TPH threads
    unsigned long long incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) red[tid >> 5] = incl;
    gsync();
    unsigned long long base = 0ull, tot = 0ull;
    const int w0 = (h * TPH) >> 5, w1 = ((h + 1) * TPH) >> 5;
#pragma unroll 1
    for (int w = w0; w < w1; ++w) {
        const unsigned long long s = red[w];
        if (w < (tid >> 5)) base += s;
        tot += s;
    }
    const unsigned long long excl = base + incl - sum;
    if (r == 0 && act && j == 0) {
        HeadCut &H = cut[h];
        H.Z = tot;
        H.target = target_of(tot, p);
        H.C = 0ull;
    }
    gsync();
    if (act) {
        const HeadCut &H = cut[h];
        const unsigned long long C = H.C, target = H.target;
        if (C + excl < target && C + excl + sum >= target) {
            unsigned long long run = C + excl;
            int b = j * BPT;
#pragma unroll 1
            for (int i = 0; i < BPT; ++i) {
                const int bi = j * BPT + i;
                const unsigned long long m = mass[h * NB + bi];
                if (run + m >= target) {
                    b = bi;
                    break;
                }
                run += m;
            }
            const uint32_t n = gcnt ? __ldcg(gcnt + h * NB + b) : cnt[h * NB + b];
            HeadCut &Hw = cut[h];
            Hw.path[r] = b;
            Hw.C = run;
            Hw.nfin = n;
            Hw.rounds = r + 1;
            Hw.mode = (n <= (uint32_t)CAND_MAX) ? CUT_RANK : (r + 1 == HIST_ROUNDS ? CUT_ORDER : CUT_OPEN);
        }
    }
    gsync();
}


// Classify every local slot for every head: kept above the path, dropped
// below it, boundary candidate on it.  Writes keep[], appends candidates
// (CUT_RANK) to the list (global team list or shared list) and to own[],
// and sums boundary masses (CUT_ORDER) into osum[h] (shared).
template <int G>
__device__ __noinline__ void classify(const Level &L, const HeadCut *cut, unsigned long long *lw, uint32_t *ls,
                                      uint32_t *lcnt, uint32_t *own, uint32_t *own_cnt, unsigned long long *osum,
                                      int64_t ibase = 0) {
    const int lane = threadIdx.x & 31;
    const int64_t iters = (L.n + GT - 1) / GT;
    // every head's cut state in registers (see PathReg)
    PathReg Hr[G];
    unsigned long long osum_t[G];  // this thread's boundary masses of CUT_ORDER heads
#pragma unroll
    for (int h = 0; h < G; ++h) {
        Hr[h] = PathReg(cut[h]);
        osum_t[h] = 0ull;
    }
#pragma unroll 1
    for (int64_t it = 0; it < iters; ++it) {
        const int64_t i = it * GT + threadIdx.x;
        uint32_t kbits = 0u;
        float ev[G];
#pragma unroll
        for (int h = 0; h < G; ++h) ev[h] = i < L.n ? L.sc[i * G + h] : -INFINITY;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const PathReg &H = Hr[h];
            const float e = ev[h];
            bool cand = false;
            unsigned long long w = 0ull;
            if (e != -INFINITY) {
                if (H.mode == CUT_ALL) {
                    kbits |= 1u << h;
                } else if (H.mode == CUT_RANK || H.mode == CUT_ORDER) {
                    const int pc = H.cmp(e, H.rounds);
                    if (pc < 0) kbits |= 1u << h;
                    else if (pc == 0) {
                        w = mass_fx(expf(e - H.M));
                        if (H.mode == CUT_RANK) cand = true;
                        else osum_t[h] += w;
                    }
                }
            }
            const unsigned bal = __ballot_sync(FULL, cand);
            if (bal) {
                const int leader = __ffs(bal) - 1;
                uint32_t base = 0, obase = 0;
                if (lane == leader) {
                    base = atomicAdd(&lcnt[h], (uint32_t)__popc(bal));
                    obase = atomicAdd(own_cnt, (uint32_t)__popc(bal));
                }
                base = __shfl_sync(FULL, base, leader);
                obase = __shfl_sync(FULL, obase, leader);
                if (cand) {
                    const uint32_t rank = __popc(bal & ((1u << lane) - 1u));
                    const uint32_t at = base + rank;
                    if (at < (uint32_t)CAND_MAX) {
                        lw[h * CAND_MAX + at] = w;
                        ls[h * CAND_MAX + at] = (uint32_t)(L.s0 + i);
                    }
                    if (obase + rank < (uint32_t)(G * CAND_MAX))
                        own[obase + rank] = ((uint32_t)(ibase + i) << 3) | (uint32_t)h;
                }
            }
        }
        if (i < L.n) L.keep[i] = (uint8_t)kbits;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
        unsigned long long x = osum_t[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        if (lane == 0 && x) atomicAdd(&osum[h], x);
    }
    gsync();
}

// Rank this CTA's boundary candidates against the whole list (shared cw/cs,
// counts from cut[h].nfin) and keep those the target still needs.
template <int G>
__device__ __noinline__ void rank_own(const Level &L, const HeadCut *cut, const unsigned long long *cw,
                                      const uint32_t *cs, const uint32_t *own, uint32_t n_own) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
    for (uint32_t o = warp; o < n_own; o += GT / 32) {
        const uint32_t code = own[o];
        const int h = (int)(code & 7u);
        const int64_t i = (int64_t)(code >> 3);
        const HeadCut &H = cut[h];
        const uint32_t nc = H.nfin;
        const uint32_t slot = (uint32_t)(L.s0 + i);
        const unsigned long long wi = mass_fx(expf(L.sc[i * G + h] - H.M));
        unsigned long long pre = 0ull;
#pragma unroll 1
        for (uint32_t jj = lane; jj < nc; jj += 32) {
            const unsigned long long wj = cw[h * CAND_MAX + jj];
            const uint32_t sj = cs[h * CAND_MAX + jj];
            if (wj > wi || (wj == wi && sj < slot)) pre += wj;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) pre += __shfl_xor_sync(FULL, pre, off);
        if (lane == 0 && H.C + pre < H.target) keep_or(L.keep, i, 1u << h);
    }
    gsync();
}

// Slot-order cut of the boundary for CUT_ORDER heads: `base[h]` is the mass
// before this CTA's first slot (cut.C plus lower ranks' boundary masses).
template <int G>
__device__ __noinline__ void order_own(const Level &L, const HeadCut *cut, const unsigned long long *base,
                                       unsigned long long *red) {
    const int64_t per = (L.n + GT - 1) / GT;
    const int64_t i0 = min(L.n, per * threadIdx.x), i1 = min(L.n, i0 + per);
#pragma unroll 1
    for (int h = 0; h < G; ++h) {
        const HeadCut &H = cut[h];
        if (H.mode != CUT_ORDER) continue;
        unsigned long long mine = 0ull;
#pragma unroll 4
        for (int64_t i = i0; i < i1; ++i) {
            const float e = L.sc[i * G + h];
            if (e != -INFINITY && path_cmp(H, e, H.rounds) == 0) mine += mass_fx(expf(e - H.M));
        }
        unsigned long long tot;
        unsigned long long run = g_scan_u64(mine, red, &tot) - mine + base[h];
#pragma unroll 1
        for (int64_t i = i0; i < i1; ++i) {
            const float e = L.sc[i * G + h];
            if (e != -INFINITY && path_cmp(H, e, H.rounds) == 0) {
                if (run < H.target) keep_or(L.keep, i, 1u << h);
                run += mass_fx(expf(e - H.M));
            }
        }
    }
    gsync();
}

// Keep bits of local slot i.  Bits set by atomics live at L2 when the slots
// overflow shared memory, so global keep bits are read around L1.
__device__ __forceinline__ uint32_t keep_at(const Level &L, int64_t i) {
    return L.n > LOC_CAP ? (uint32_t)__ldcg(L.keep + i) : (uint32_t)L.keep[i];
}

// Write this CTA's kept slots (ascending) at the start of its slot range,
// with per-rank counts.
template <int G>
__device__ __noinline__ void write_segment(const Decode &a, const Level &L, uint32_t *red32) {
    const int64_t per = (L.n + GT - 1) / GT;
    const int64_t i0 = min(L.n, per * threadIdx.x), i1 = min(L.n, i0 + per);
    uint32_t mine = 0u;
    uint32_t hc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) hc[h] = 0u;
#pragma unroll 4
    for (int64_t i = i0; i < i1; ++i) {
        const uint32_t k = keep_at(L, i);
        mine += k != 0u;
#pragma unroll
        for (int h = 0; h < G; ++h) hc[h] += (k >> h) & 1u;
    }
    uint32_t tot;
    uint32_t at = g_scan_u32(mine, red32, &tot) - mine;
    const int64_t dst = (int64_t)L.kh * a.slot_cap[L.l - 1] + L.s0;
    int32_t *ids = a.kept_ids[L.l - 1] + dst;
    uint8_t *msk = a.kept_mask[L.l - 1] + dst;
#pragma unroll 4
    for (int64_t i = i0; i < i1; ++i) {
        const uint32_t k = keep_at(L, i);
        if (k) {
            ids[at] = L.node[i];
            msk[at] = (uint8_t)k;
            ++at;
        }
    }
    // per-head counts: warp sums, then one atomic per warp into shared
    uint32_t *hs = red32 + 16;
    if (threadIdx.x < G) hs[threadIdx.x] = 0u;
    gsync();
#pragma unroll
    for (int h = 0; h < G; ++h) {
        uint32_t x = hc[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        if ((threadIdx.x & 31) == 0 && x) atomicAdd(&hs[h], x);
    }
    gsync();
    if (threadIdx.x == 0) {
        seg_ptr(a, L.l, L.kh)[L.tr] = tot;
        if (L.tr == 0) {
            int32_t *lv = lvl_ptr(a, L.l, L.kh);
            lv[0] = L.T;
            lv[1] = (int32_t)L.S;
        }
    }
    if (threadIdx.x < G) hseg_ptr(a, L.l, L.kh)[(int64_t)L.tr * G + threadIdx.x] = hs[threadIdx.x];
}

// ---- levels whose slots spill to global memory --------------------------------

// Copy local slots [c0, c0 + n) (n <= LOC_CAP) of a spilled level's scores
// into the shared score array: every thread's loads are issued together, so
// a chunk costs one round trip to L2 instead of one per few slots.
template <int G>
__device__ __forceinline__ void chunk_scores_in(const Level &L, int64_t c0, int64_t n, float *ssc) {
    if constexpr (G == 4) {
        const float4 *src = reinterpret_cast<const float4 *>(L.sc + c0 * G);
        float4 *dst = reinterpret_cast<float4 *>(ssc);
        constexpr int PER = LOC_CAP / GT;
        float4 v[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * GT;
            if (i < n) v[k] = __ldcg(src + i);
        }
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * GT;
            if (i < n) dst[i] = v[k];
        }
    } else {
        constexpr int PER = LOC_CAP * G / GT;
        float v[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * GT;
            if (i < n * G) v[k] = __ldcg(L.sc + c0 * G + i);
        }
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int64_t i = threadIdx.x + (int64_t)k * GT;
            if (i < n * G) ssc[i] = v[k];
        }
    }
}

// The local slots [c0, c0 + n) of a spilled level as a level of their own
// whose scores are the shared copy `ssc` (keep bits stay in global memory).
__device__ __forceinline__ Level chunk_level(const Level &L, int64_t c0, int64_t n, float *ssc) {
    Level C = L;
    C.s0 = L.s0 + c0;
    C.n = n;
    C.sc = ssc;
    C.sc_local = true;
    C.node = L.node + c0;
    C.keep = L.keep + c0;
    return C;
}

// write_segment for a spilled level: the keep bits and node ids come in by
// chunks of LOC_CAP slots into the shared arrays, each chunk compacted in
// slot order after the chunks before it.
template <int G>
__device__ __noinline__ void write_segment_spilled(const Decode &a, const Level &L, int32_t *snode, uint8_t *skeep,
                                                   uint32_t *red32) {
    const int64_t dst = (int64_t)L.kh * a.slot_cap[L.l - 1] + L.s0;
    int32_t *ids = a.kept_ids[L.l - 1] + dst;
    uint8_t *msk = a.kept_mask[L.l - 1] + dst;
    uint32_t hc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) hc[h] = 0u;
    uint32_t base = 0u;
    constexpr int PER = LOC_CAP / GT;
#pragma unroll 1
    for (int64_t c0 = 0; c0 < L.n; c0 += LOC_CAP) {
        const int64_t n = min((int64_t)LOC_CAP, L.n - c0);
        {
            uint32_t kv[PER];
            int32_t nv[PER];
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                const int64_t i = threadIdx.x + (int64_t)k * GT;
                kv[k] = i < n ? (uint32_t)__ldcg(L.keep + c0 + i) : 0u;
                nv[k] = i < n ? __ldcg(L.node + c0 + i) : -1;
            }
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                const int64_t i = threadIdx.x + (int64_t)k * GT;
                if (i < n) {
                    skeep[i] = (uint8_t)kv[k];
                    snode[i] = nv[k];
                }
            }
        }
        gsync();
        const int64_t per = (n + GT - 1) / GT;
        const int64_t i0 = min(n, per * threadIdx.x), i1 = min(n, i0 + per);
        uint32_t mine = 0u;
#pragma unroll 4
        for (int64_t i = i0; i < i1; ++i) {
            const uint32_t k = skeep[i];
            mine += k != 0u;
#pragma unroll
            for (int h = 0; h < G; ++h) hc[h] += (k >> h) & 1u;
        }
        uint32_t tot;
        uint32_t at = base + g_scan_u32(mine, red32, &tot) - mine;
#pragma unroll 4
        for (int64_t i = i0; i < i1; ++i) {
            const uint32_t k = skeep[i];
            if (k) {
                ids[at] = snode[i];
                msk[at] = (uint8_t)k;
                ++at;
            }
        }
        base += tot;
        gsync();
    }
    uint32_t *hs = red32 + 16;
    if (threadIdx.x < G) hs[threadIdx.x] = 0u;
    gsync();
#pragma unroll
    for (int h = 0; h < G; ++h) {
        uint32_t x = hc[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        if ((threadIdx.x & 31) == 0 && x) atomicAdd(&hs[h], x);
    }
    gsync();
    if (threadIdx.x == 0) {
        seg_ptr(a, L.l, L.kh)[L.tr] = base;
        if (L.tr == 0) {
            int32_t *lv = lvl_ptr(a, L.l, L.kh);
            lv[0] = L.T;
            lv[1] = (int32_t)L.S;
        }
    }
    if (threadIdx.x < G) hseg_ptr(a, L.l, L.kh)[(int64_t)L.tr * G + threadIdx.x] = hs[threadIdx.x];
}

// ---- one level ------------------------------------------------------------------

// The histogram path of the cut (team, or one CTA with more than SOLO_MAX
// slots): rounds, classification, boundary lists.  false: a barrier gave up.
template <int G>
__device__ __noinline__ bool hist_cut(const Decode &a, const Level &L, unsigned char *smem, TeamSync &ts) {
    using SM = RouteSmem<G>;
    HeadCut *cut = reinterpret_cast<HeadCut *>(smem + SM::off_cut);
    unsigned long long *red = reinterpret_cast<unsigned long long *>(smem + SM::off_red);
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + SM::off_misc);
    uint32_t *hc = reinterpret_cast<uint32_t *>(smem + SM::off_hc);
    unsigned long long *hm = reinterpret_cast<unsigned long long *>(smem + SM::off_hm);
    unsigned long long *cw = reinterpret_cast<unsigned long long *>(smem + SM::off_cw);
    uint32_t *cs = reinterpret_cast<uint32_t *>(smem + SM::off_cs);
    uint32_t *own = reinterpret_cast<uint32_t *>(smem + SM::off_own);
    const int tid = threadIdx.x, kh = L.kh, T = L.T, tr = L.tr;
    const bool team = T > 1;
    const int64_t hbase = (int64_t)kh * HIST_ROUNDS * G * NB;
    int rounds_used = 0;
#pragma unroll 1
    for (int r = 0; r < HIST_ROUNDS; ++r) {
        bool open = false;
#pragma unroll 1
        for (int h = 0; h < G; ++h) open |= cut[h].mode == CUT_OPEN;
        if (!open) break;
        // windows of HIST_WIN slots (the spilled ones by chunks through the
        // shared score array); a team folds each into its global histogram,
        // a lone CTA (at most HIST_WIN slots: teams take larger slices) in place
        uint32_t *gc = a.hist_cnt + hbase + (int64_t)r * G * NB;
        unsigned long long *gm = a.hist_mass + hbase + (int64_t)r * G * NB;
        uint32_t *hw = reinterpret_cast<uint32_t *>(hm);
#pragma unroll 1
        for (int i = tid; i < G * NB; i += GT) {
            hc[i] = 0u;
            hm[i] = 0ull;
        }
        gsync();
        static_assert(HIST_WIN == LOC_CAP, "a spilled chunk is one histogram window");
        float *ssc = reinterpret_cast<float *>(smem + SM::off_sc);
#pragma unroll 1
        for (int64_t w0 = 0; w0 < L.n; w0 += HIST_WIN) {
            const int64_t n = min((int64_t)HIST_WIN, L.n - w0);
            if (!L.sc_local) {
                chunk_scores_in<G>(L, w0, n, ssc);
                gsync();
            }
            local_hist<G>(chunk_level(L, w0, n, L.sc_local ? L.sc + w0 * G : ssc), cut, r, hc, hw);
            if (team || L.n > HIST_WIN) fold_window<G>(hc, hw, gc, gm);
        }
        rounds_used = r + 1;
        if (!team && L.n > HIST_WIN) {
            // (a lone CTA with more slots: the sums went through the global histogram)
#pragma unroll 16
            for (int i = tid; i < G * NB; i += GT) {
                hm[i] = __ldcg(gm + i);
                hc[i] = __ldcg(gc + i);
                gm[i] = 0ull;
                gc[i] = 0u;
            }
            gsync();
            find_cut<G>(cut, r, hc, nullptr, hm, a.p, red);
        } else if (team) {
            if (!ts.sync()) return false;  // B
            // the team's bucket masses into shared memory: independent loads
#pragma unroll 16
            for (int i = tid; i < G * NB; i += GT) hm[i] = __ldcg(gm + i);
            gsync();
            find_cut<G>(cut, r, hc, gc, hm, a.p, red);
        } else {
            fold_local<G>(hw);
            find_cut<G>(cut, r, hc, nullptr, hm, a.p, red);
        }
    }
    // classify, boundary lists
    unsigned long long *osum = red + 64;
    if (tid < 8) misc[tid] = 0u;  // [0]: own count, [4 + h]: shared list counters
    if (tid < G) osum[tid] = 0ull;
    gsync();
    // candidates go to shared lists first (shared counters); a team then
    // reserves room in its global lists with one atomic per head
    if (L.sc_local) {
        classify<G>(L, cut, cw, cs, misc + 4, own, misc, osum);
    } else {
        float *ssc = reinterpret_cast<float *>(smem + SM::off_sc);
#pragma unroll 1
        for (int64_t c0 = 0; c0 < L.n; c0 += LOC_CAP) {
            const int64_t n = min((int64_t)LOC_CAP, L.n - c0);
            chunk_scores_in<G>(L, c0, n, ssc);
            gsync();
            classify<G>(chunk_level(L, c0, n, ssc), cut, cw, cs, misc + 4, own, misc, osum, c0);
        }
    }
    unsigned long long *lw = team ? a.cand_w + (int64_t)kh * G * CAND_MAX : cw;
    uint32_t *ls = team ? a.cand_slot + (int64_t)kh * G * CAND_MAX : cs;
    if (team) {
        uint32_t *gbase = misc + 8;
        if (tid < G) {
            const uint32_t nh = min(misc[4 + tid], (uint32_t)CAND_MAX);
            gbase[tid] = nh ? atomicAdd(a.cand_cnt + (int64_t)kh * G + tid, nh) : 0u;
        }
        gsync();
#pragma unroll 1
        for (int h = 0; h < G; ++h) {
            const uint32_t nh = min(misc[4 + h], (uint32_t)CAND_MAX), base = gbase[h];
            for (uint32_t j = tid; j < nh; j += GT) {
                if (base + j < (uint32_t)CAND_MAX) {
                    lw[h * CAND_MAX + base + j] = cw[h * CAND_MAX + j];
                    ls[h * CAND_MAX + base + j] = cs[h * CAND_MAX + j];
                }
            }
        }
    }
    bool any_order = false, any_rank = false;
#pragma unroll 1
    for (int h = 0; h < G; ++h) {
        any_order |= cut[h].mode == CUT_ORDER;
        any_rank |= cut[h].mode == CUT_RANK;
    }
    if (team && any_order && tid < G) a.tsum[((int64_t)kh * SEG_CAP + tr) * G + tid] = osum[tid];
    if (team) {
        if (!ts.sync()) return false;  // C
        // the histograms are consumed: clear this rank's share for the next level
#pragma unroll 1
        for (int r = 0; r < rounds_used; ++r) {
            uint32_t *gc = a.hist_cnt + hbase + (int64_t)r * G * NB;
            unsigned long long *gm = a.hist_mass + hbase + (int64_t)r * G * NB;
            const int64_t lo = (int64_t)G * NB * tr / T, hi = (int64_t)G * NB * (tr + 1) / T;
#pragma unroll 1
            for (int64_t i = lo + tid; i < hi; i += GT) {
                gc[i] = 0u;
                gm[i] = 0ull;
            }
        }
    }
    const uint32_t n_own = min(misc[0], (uint32_t)(G * CAND_MAX));
    if (any_rank && n_own > 0) {
        if (team) {
            // bring the team's lists into shared memory
#pragma unroll 1
            for (int h = 0; h < G; ++h) {
                if (cut[h].mode != CUT_RANK) continue;
#pragma unroll 1
                for (uint32_t j = tid; j < cut[h].nfin; j += GT) {
                    cw[h * CAND_MAX + j] = __ldcg(lw + h * CAND_MAX + j);
                    cs[h * CAND_MAX + j] = __ldcg(ls + h * CAND_MAX + j);
                }
            }
            gsync();
        }
        rank_own<G>(L, cut, cw, cs, own, n_own);
    }
    if (any_order) {
        unsigned long long *base = red + 72;
        // mass of the boundary before this rank: lower ranks' sums (parallel
        // loads, reduced per head in a fixed order)
        unsigned long long x = 0ull;
        if (team) {
#pragma unroll 1
            for (int t = tid; t < tr * G; t += GT) x += __ldcg(a.tsum + (int64_t)kh * SEG_CAP * G + t);
        }
#pragma unroll
        for (int off = G; off < 32; off <<= 1) x += __shfl_xor_sync(FULL, x, off);
        if ((tid & 31) < G) red[128 + (tid >> 5) * G + (tid & 31)] = x;
        gsync();
        if (tid < G) {
            unsigned long long bsum = cut[tid].C;
            if (cut[tid].mode == CUT_ORDER) {
#pragma unroll 1
                for (int w = 0; w < GT / 32; ++w) bsum += red[128 + w * G + tid];
            }
            base[tid] = bsum;
        }
        gsync();
        order_own<G>(L, cut, base, red);
    }
    return true;
}

// Score and cut level l of KV head kh as rank tr of a team of T CTAs (T = 1:
// this CTA alone).  `S` is the frontier size, `pref`/Tp/Sp the parent level's
// segments (loaded by the caller).  F[h] receives the frontier counts.
// Returns false when a team barrier gave up.
template <int HD, int R, int G, typename RT>
__device__ __noinline__ bool route_level(const Decode &a, int l, int kh, int T, int tr, int64_t S, int Tp, int64_t Sp,
                                         bool par_local, unsigned char *smem, TeamSync &ts, uint32_t (&F)[G],
                                         int &Tout) {
    using SM = RouteSmem<G>;
    HeadCut *cut = reinterpret_cast<HeadCut *>(smem + SM::off_cut);
    uint32_t *pref = reinterpret_cast<uint32_t *>(smem + SM::off_pref);
    float *wm = reinterpret_cast<float *>(smem + SM::off_wm);
    uint32_t *wc = reinterpret_cast<uint32_t *>(smem + SM::off_wc);
    const int tid = threadIdx.x;
    Level L;
    L.l = l;
    L.kh = kh;
    L.T = T;
    L.tr = tr;
    L.top = (l == a.t.D);
    L.S = S;
    L.s0 = seg_start(S, T, tr);
    L.n = seg_start(S, T, tr + 1) - L.s0;
    L.Tp = Tp;
    L.Sp = Sp;
    Tout = T;
    const bool team = T > 1;
    L.sc_local = L.n <= LOC_CAP;
    if (!L.sc_local) {
        const int64_t base = (int64_t)kh * a.score_cap + L.s0;
        L.sc = a.scores + base * G;
        L.node = a.slot_node + base;
        L.keep = a.slot_keep + base;
    } else {
        L.sc = reinterpret_cast<float *>(smem + SM::off_sc);
        L.node = reinterpret_cast<int32_t *>(smem + SM::off_node);
        L.keep = smem + SM::off_keep;
    }
    // ---- score
    if (tid < 8 * G) {
        wm[tid] = -INFINITY;
        wc[tid] = 0u;
    }
    int32_t *pid = reinterpret_cast<int32_t *>(smem + SM::off_pid);
    uint8_t *pmk = smem + SM::off_pmk;
    // slots scored per pipeline run: the local arrays' capacity, or, when
    // they spill to global memory anyway, as many as one parent window covers
    // (the whole slice when the parents are the local kept list): fewer runs
    // drain the copy pipeline fewer times
    const int64_t chunk = L.n <= LOC_CAP ? (int64_t)LOC_CAP
                          : (par_local || L.top) ? L.n
                                                 : max((int64_t)LOC_CAP, (int64_t)(PAR_CAP - 2) * a.t.c);
#pragma unroll 1
    for (int64_t c0 = L.s0; c0 < L.s0 + L.n; c0 += chunk) {
        const int64_t c1 = min(L.s0 + L.n, c0 + chunk);
        int64_t k0 = 0;  // parents already local: the whole kept list from rank 0
        if (!L.top && !par_local) load_parents(a, L, c0, c1, pref, pid, pmk, k0);
        gsync();
        score_chunks<HD, R, G, RT>(a, L, c0, c1, k0, pid, pmk, smem, wm, wc);
        gsync();
    }
    // a spilled slice that fits below the cut scratch comes back on chip in
    // one bulk copy, whose latency the maxima's barrier hides
    uint64_t *cbar = reinterpret_cast<uint64_t *>(smem + SM::off_cbar);
    const bool back = G == 4 && !L.sc_local && L.n <= SM::SPILL_CAP;
    if (back) {
        // this thread's score stores (global) and earlier writes to the
        // destination (shared), ordered before the copy
        asm volatile("fence.proxy.async;" ::: "memory");
        gsync();
        if (tid == 0) {
            const uint32_t nbytes = (uint32_t)(L.n * G * 4);
            mbar_arrive_expect_tx(cbar, nbytes);
            bulk_g2s(smem + SM::off_sc, L.sc, nbytes, cbar);
        }
    }
    if (tid < G) {
        float m = -INFINITY;
        uint32_t c = 0u;
#pragma unroll 1
        for (int w = 0; w < GT / 32; ++w) {
            m = fmaxf(m, wm[w * G + tid]);
            c += wc[w * G + tid];
        }
        if (team) {
            a.tmax[((int64_t)kh * SEG_CAP + tr) * G + tid] = m;
            a.tcnt[((int64_t)kh * SEG_CAP + tr) * G + tid] = c;
        } else {
            cut[tid].M = m;
            cut[tid].F = c;
        }
    }
    if (team && !ts.sync()) return false;  // A
    if (team) {
        // thread t < T*G loads rank t/G's (max, count) of head t%G; then a
        // reduction over threads with equal t%G (fixed order)
        float m = -INFINITY;
        uint32_t c = 0u;
#pragma unroll 1
        for (int t = tid; t < T * G; t += GT) {  // GT is a multiple of G: t % G == tid % G
            m = fmaxf(m, __ldcg(a.tmax + (int64_t)kh * SEG_CAP * G + t));
            c += __ldcg(a.tcnt + (int64_t)kh * SEG_CAP * G + t);
        }
#pragma unroll
        for (int off = G; off < 32; off <<= 1) {
            m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
            c += __shfl_xor_sync(FULL, c, off);
        }
        if ((tid & 31) < G) {
            wm[(tid >> 5) * G + (tid & 31)] = m;
            wc[(tid >> 5) * G + (tid & 31)] = c;
        }
        gsync();
        if (tid < G) {
            float mm = -INFINITY;
            uint32_t cc = 0u;
#pragma unroll 1
            for (int w = 0; w < GT / 32; ++w) {
                mm = fmaxf(mm, wm[w * G + tid]);
                cc += wc[w * G + tid];
            }
            cut[tid].M = mm;
            cut[tid].F = cc;
        }
    }
    if (back) {
        uint32_t *cuse = reinterpret_cast<uint32_t *>(smem + SM::off_cuse);
        if (!mbar_wait(cbar, *cuse & 1u, nullptr)) set_status(a.status, ZHA_TIMEOUT_CODE);
        gsync();
        if (tid == 0) *cuse += 1u;
        L.sc = reinterpret_cast<float *>(smem + SM::off_sc);
        L.sc_local = true;
    }
    const bool keep_all = !(a.p < 1.f);
    const bool solo = L.T == 1;
    gsync();
    if (tid < G) {
        HeadCut &H = cut[tid];
        H.rounds = 0;
        H.nfin = 0u;
        H.mode = H.F == 0u ? CUT_NONE : (keep_all ? CUT_ALL : CUT_OPEN);
    }
    gsync();
#pragma unroll
    for (int h = 0; h < G; ++h) F[h] = cut[h].F;
    // ---- cut
    if (keep_all) {
#pragma unroll 1
        for (int64_t i = tid; i < L.n; i += GT) {
            uint32_t kb = 0u;
#pragma unroll 1
            for (int h = 0; h < G; ++h) kb |= (L.sc[i * G + h] != -INFINITY ? 1u : 0u) << h;
            L.keep[i] = (uint8_t)kb;
        }
        gsync();
    } else if (solo && L.n <= RANK_MAX) {
        solo_cut<G>(L, cut, reinterpret_cast<unsigned long long *>(smem + SM::off_hm), a.p);
    } else if (solo && L.n <= SOLO_MAX) {
        sort_cut<G>(L, cut, a.p);
    } else {
        if (!hist_cut<G>(a, L, smem, ts)) return false;
    }
    if (L.n <= LOC_CAP)
        write_segment<G>(a, L, reinterpret_cast<uint32_t *>(smem + SM::off_red));
    else
        write_segment_spilled<G>(a, L, reinterpret_cast<int32_t *>(smem + SM::off_node), smem + SM::off_keep,
                                 reinterpret_cast<uint32_t *>(smem + SM::off_red));
    if (team) {
        if (!ts.sync()) return false;  // D
        // the boundary lists are consumed: rank 0 clears the counters
        if (tr == 0 && tid < G) a.cand_cnt[(int64_t)kh * G + tid] = 0u;
    } else {
        gsync();
    }
    return true;
}

// ---- levels cut by every CTA over the whole frontier ------------------------------

// The way level l is routed by a team of T CTAs, from its frontier size S
// (the same on every CTA).
template <int HD, int R, typename RT>
__device__ __forceinline__ int level_mode(int64_t S, int T) {
    constexpr int64_t node_bytes = (int64_t)R * (HD * (int64_t)sizeof(RT) + 4);
    if (S <= LOC_CAP && (T == 1 || (S <= RDA_SLOTS && S * node_bytes <= RDA_BYTES))) return LV_ALL;
    if (S <= RDS_MAX) return LV_SPLIT;
    return LV_TEAM;
}

// Node of frontier slot s of level l whose parents are the kept list in
// pid (none at the top level): child s % c of parent s / c; -1 past the
// level's last node.
__device__ __forceinline__ int32_t slot_node(const Decode &a, int l, bool top, const int32_t *pid, int64_t s) {
    const int c = a.t.c, clog = a.t.c_log2;
    int64_t nd = s;
    if (!top) {
        const int64_t k = clog >= 0 ? (s >> clog) : s / c;
        nd = (int64_t)pid[k] * c + (s - k * c);
    }
    return nd < a.t.n_level[l - 1] ? (int32_t)nd : -1;
}

// Score and cut level l of KV head kh (frontier of S <= LOC_CAP slots) so
// that every CTA of the team ends with the same kept list, ascending, in
// pid / pmk (*nk entries) -- the parents of the next level -- without
// waiting for another CTA to write it.  On entry pid / pmk hold the kept
// list of level l + 1 (unused at the top level).
//   LV_ALL: this CTA scores every slot.
//   LV_SPLIT: this CTA scores its slice [S r / T, S (r + 1) / T) into the
//   team's score buffer `buf` (global); after one team barrier it copies
//   every slot's scores in.  Consecutive LV_SPLIT levels use the two
//   buffers in turn: a CTA writes a buffer again only after the barrier of
//   the LV_SPLIT level in between, which every CTA reaches after reading it.
// Then every CTA cuts the whole frontier alone (one-CTA rank, sort or
// histogram path; the same integers on every CTA) and compacts the kept
// slots.  Rank 0 also writes the kept list as the level's single segment
// (team size 1), which the leaf lists, the trace and the attention read
// after the grid barrier.  F[h]: frontier counts.  false: the barrier gave
// up.
template <int HD, int R, int G, typename RT>
__device__ __noinline__ bool route_level_rd(const Decode &a, int l, int kh, int T, int tr, int64_t S, int mode,
                                            int buf, unsigned char *smem, TeamSync &ts, uint32_t (&F)[G],
                                            int64_t &nk) {
    using SM = RouteSmem<G>;
    HeadCut *cut = reinterpret_cast<HeadCut *>(smem + SM::off_cut);
    float *wm = reinterpret_cast<float *>(smem + SM::off_wm);
    uint32_t *wc = reinterpret_cast<uint32_t *>(smem + SM::off_wc);
    int32_t *pid = reinterpret_cast<int32_t *>(smem + SM::off_pid);
    uint8_t *pmk = smem + SM::off_pmk;
    float *sc = reinterpret_cast<float *>(smem + SM::off_sc);
    int32_t *node = reinterpret_cast<int32_t *>(smem + SM::off_node);
    uint8_t *keep = smem + SM::off_keep;
    uint32_t *red32 = reinterpret_cast<uint32_t *>(smem + SM::off_red);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool top = (l == a.t.D);
    float *gsc = a.rd_scores + (int64_t)(kh * 2 + buf) * LOC_CAP * G;
    Level L;
    L.l = l;
    L.kh = kh;
    L.T = 1;
    L.tr = 0;
    L.top = top;
    L.S = S;
    L.Tp = 1;
    L.Sp = 0;
    L.keep = keep;
    L.sc_local = mode == LV_ALL;
    if (mode == LV_ALL) {
        L.s0 = 0;
        L.n = S;
        L.sc = sc;
        L.node = node;
    } else {
        L.s0 = seg_start(S, T, tr);
        L.n = seg_start(S, T, tr + 1) - L.s0;
        L.sc = gsc + L.s0 * G;   // indexed by slot - s0
        L.node = node + L.s0;
    }
    // ---- score (the parents' kept list is the whole window: k0 = 0)
    if (tid < 8 * G) {
        wm[tid] = -INFINITY;
        wc[tid] = 0u;
    }
    gsync();
    if (L.n > 0) score_chunks<HD, R, G, RT>(a, L, L.s0, L.s0 + L.n, 0, pid, pmk, smem, wm, wc);
    if (mode == LV_SPLIT) {
        if (!ts.sync()) return false;
        // every slot's scores (written before the barrier) and node
        if constexpr (G == 4) {
            const float4 *s4 = reinterpret_cast<const float4 *>(gsc);
            float4 *d4 = reinterpret_cast<float4 *>(sc);
#pragma unroll 8
            for (int64_t i = tid; i < S; i += GT) d4[i] = __ldcg(s4 + i);
        } else {
#pragma unroll 8
            for (int64_t i = tid; i < S * G; i += GT) sc[i] = __ldcg(gsc + i);
        }
#pragma unroll 4
        for (int64_t i = tid; i < S; i += GT) node[i] = slot_node(a, l, top, pid, i);
        gsync();
    }
    // ---- maxima and frontier counts of every head over the whole frontier
    {
        // GT is a multiple of G: every entry this thread visits is head tid % G
        float m = -INFINITY;
        uint32_t cnt = 0u;
#pragma unroll 4
        for (int64_t i = tid; i < S * G; i += GT) {
            const float e = sc[i];
            m = fmaxf(m, e);
            cnt += e != -INFINITY;
        }
#pragma unroll
        for (int off = G; off < 32; off <<= 1) {
            m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
            cnt += __shfl_xor_sync(FULL, cnt, off);
        }
        if (lane < G) {
            wm[warp * G + lane] = m;
            wc[warp * G + lane] = cnt;
        }
        gsync();
        if (tid < G) {
            float mm = -INFINITY;
            uint32_t cc = 0u;
#pragma unroll 1
            for (int w = 0; w < GT / 32; ++w) {
                mm = fmaxf(mm, wm[w * G + tid]);
                cc += wc[w * G + tid];
            }
            HeadCut &H = cut[tid];
            H.M = mm;
            H.F = cc;
            H.rounds = 0;
            H.nfin = 0u;
            H.mode = cc == 0u ? CUT_NONE : (!(a.p < 1.f) ? CUT_ALL : CUT_OPEN);
        }
        gsync();
    }
#pragma unroll
    for (int h = 0; h < G; ++h) F[h] = cut[h].F;
    // ---- the cut of the whole frontier, by this CTA alone
    Level LA = L;
    LA.s0 = 0;
    LA.n = S;
    LA.sc = sc;
    LA.sc_local = true;
    LA.node = node;
    if (!(a.p < 1.f)) {
#pragma unroll 1
        for (int64_t i = tid; i < S; i += GT) {
            uint32_t kb = 0u;
#pragma unroll
            for (int h = 0; h < G; ++h) kb |= (sc[i * G + h] != -INFINITY ? 1u : 0u) << h;
            keep[i] = (uint8_t)kb;
        }
        gsync();
    } else if (S <= RANK_MAX) {
        solo_cut<G>(LA, cut, reinterpret_cast<unsigned long long *>(smem + SM::off_hm), a.p);
    } else if (S <= SOLO_MAX) {
        sort_cut<G>(LA, cut, a.p);
    } else {
        TeamSync solo = ts;
        solo.T = 1;
        hist_cut<G>(a, LA, smem, solo);  // no inter-CTA barrier with a team of one
        gsync();
    }
    // ---- compaction: the kept list, ascending, into pid / pmk (the node ids
    // of every slot are in node[], so the old list is no longer needed)
    const int64_t per = (S + GT - 1) / GT;
    const int64_t i0 = min(S, per * tid), i1 = min(S, i0 + per);
    uint32_t mine = 0u;
    uint32_t hc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) hc[h] = 0u;
#pragma unroll 4
    for (int64_t i = i0; i < i1; ++i) {
        const uint32_t k = keep[i];
        mine += k != 0u;
#pragma unroll
        for (int h = 0; h < G; ++h) hc[h] += (k >> h) & 1u;
    }
    uint32_t tot;
    uint32_t at = g_scan_u32(mine, red32, &tot) - mine;
#pragma unroll 4
    for (int64_t i = i0; i < i1; ++i) {
        const uint32_t k = keep[i];
        if (k) {
            pid[at] = node[i];
            pmk[at] = (uint8_t)k;
            ++at;
        }
    }
    uint32_t *hs = red32 + 16;
    if (tid < G) hs[tid] = 0u;
    gsync();
#pragma unroll
    for (int h = 0; h < G; ++h) {
        uint32_t x = hc[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
        if (lane == 0 && x) atomicAdd(&hs[h], x);
    }
    gsync();
    nk = tot;
    if (tr == 0) {
        // the level's single segment: team size 1, all tot kept nodes
        const int64_t dst = (int64_t)kh * a.slot_cap[l - 1];
        int32_t *ids = a.kept_ids[l - 1] + dst;
        uint8_t *msk = a.kept_mask[l - 1] + dst;
#pragma unroll 4
        for (uint32_t i = tid; i < tot; i += GT) {
            ids[i] = pid[i];
            msk[i] = pmk[i];
        }
        if (tid == 0) {
            seg_ptr(a, l, kh)[0] = tot;
            int32_t *lv = lvl_ptr(a, l, kh);
            lv[0] = 1;
            lv[1] = (int32_t)S;
        }
        if (tid < G) hseg_ptr(a, l, kh)[tid] = hs[tid];
    }
    gsync();
    return true;
}

}  // namespace zha
