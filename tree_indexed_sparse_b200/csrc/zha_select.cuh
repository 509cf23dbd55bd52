// zha_select.cuh -- exact top-p cut and ordered compaction of one routing
// frontier, for every query head of one KV head, by warps 0-7 of one CTA.
//
// Top-p ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢": keep
// the smallest node set whose cumulative estimated mass reaches p; "階層型疎
// Attention「ZHA」…", section "【技術的ディープダイブ】": top-p, not top-k).  For
// head h with frontier F_h: P_n = softmax over F_h of est_n; order by P
// descending, ties to the lower node id; keep the shortest prefix whose
// cumulative P reaches p (p >= 1 keeps every node).
//
// Deterministic and exact for the fp32 estimates.  Masses are
// w = exp(est - max) in 2^-40 fixed point, summed as integers (order
// independent) in per-thread registers and combined by tree reductions.  All
// G heads share each pass over the frontier:
//   1. counts per bucket of (max - est) * 32 (32-bit shared atomics), the
//      total mass Z_h and the frontier size;
//   2. every node of bucket b weighs between exp(-(b+1)/32) and exp(-b/32),
//      so cumulative count x weight bounds bracket the bucket holding the cut
//      between B_lo and B_hi (usually one or two buckets);
//   3. a second pass sums exactly the mass of every node above B_lo and
//      gathers the nodes of [B_lo, B_hi] as candidates (warp-aggregated);
//   4. candidates are ranked exactly by (est descending, slot ascending); the
//      cut is the candidate where the cumulative mass first reaches
//      ceil(p * Z_h), and a slot is kept when its key is <= the cut key.
// A bracket holding more than SEL_CAND nodes is narrowed by value (the same
// bracketing on a finer grid of the key range); an exact tie wider than the
// candidate list keeps the first nodes of the tie in slot (= node id) order.
//
// Every function here is called by threads 0-255 only and synchronises them
// with the named barrier of gsync().
#pragma once

#include "zha_device.cuh"
#include "zha_internal.cuh"

namespace zha {

constexpr int SEL_CAND = 512;  // candidates ranked exactly per head

struct HeadSel {
    unsigned long long Z, target, above, cut;
    float M;
    uint32_t F, Blo, Bhi, count, ncand;
    uint32_t klo, khi;  // candidate key range (desc keys) when refined
    int refined;        // 0: members are buckets [Blo, Bhi]; 1: keys in [klo, khi]
    int mode;           // 0: keep all; 1: rank candidates; 2: exact tie wider than the list
};

// Scores of one KV head's frontier, [slot][G], -inf where a head does not
// need the slot; staged in shared memory when they fit.
struct ScoreView {
    const float *sc;
    int G;
    bool staged;
    __device__ __forceinline__ float operator()(int64_t s, int h) const {
        return staged ? sc[s * G + h] : __ldcg(sc + s * G + h);
    }
};

template <int G>
struct SelectSmem {
    static constexpr int STAGE_SLOTS = STAGE_BYTES / (4 * G);
    static constexpr size_t off_hc = STAGE_BYTES;                                  // [G][NB] u32
    static constexpr size_t off_ck = off_hc + (size_t)G * NB * 4;                 // [G][SEL_CAND] u64
    static constexpr size_t off_cm = off_ck + (size_t)G * SEL_CAND * 8;           // [G][SEL_CAND] u64
    static constexpr size_t off_hs = off_cm + (size_t)G * SEL_CAND * 8;           // [G] HeadSel
    static constexpr size_t off_red = (off_hs + G * sizeof(HeadSel) + 15) / 16 * 16;  // [8][2G] u64
    static constexpr size_t off_scan = off_red + 8 * (2 * G) * 8;                  // [GT] u64
    static constexpr size_t off_misc = off_scan + GT * 8;
    static constexpr size_t bytes = off_misc + 512;
};

__device__ __forceinline__ int coarse_bucket(float M, float e) {
    const float x = (M - e) * BUCKETS_PER_UNIT;
    return x < (float)(NB - 1) ? (int)x : NB - 1;
}

// Bounds of one node's fixed-point mass in coarse bucket b (generous by a
// hundredth of a bucket and two units of the last place, to cover rounding).
__device__ __forceinline__ unsigned long long bucket_w_hi(int b) {
    return mass_fx(expf(-((float)b - 0.01f) / BUCKETS_PER_UNIT)) + 2ull;
}
__device__ __forceinline__ unsigned long long bucket_w_lo(int b) {
    if (b >= NB - 1) return 0ull;
    const unsigned long long w = mass_fx(expf(-((float)b + 1.01f) / BUCKETS_PER_UNIT));
    return w > 2ull ? w - 2ull : 0ull;
}
// Bounds of a node's mass for an estimate given by its descending key.
__device__ __forceinline__ unsigned long long key_w_hi(uint32_t k, float M) {
    return mass_fx(expf(desc_key_to_float(k) - M)) + 2ull;
}
__device__ __forceinline__ unsigned long long key_w_lo(uint32_t k, float M) {
    const unsigned long long w = mass_fx(expf(desc_key_to_float(k) - M));
    return w > 2ull ? w - 2ull : 0ull;
}

// One pass over the frontier for the heads in ranking mode (or only head
// `only` when only >= 0): the mass strictly above each head's candidate
// range goes to hs[h].above, the range's slots are appended as candidates.
template <int G>
__device__ __noinline__ void gather_pass(HeadSel *hs, int64_t S, ScoreView score, unsigned long long *ck,
                                         unsigned long long *cm, unsigned long long *red, int only) {
    const int tid = threadIdx.x, lane = tid & 31;
    unsigned long long above[G];
#pragma unroll
    for (int h = 0; h < G; ++h) above[h] = 0ull;
    const int64_t iters = (S + GT - 1) / GT;
#pragma unroll 1
    for (int64_t it = 0; it < iters; ++it) {
        const int64_t s = it * GT + tid;
#pragma unroll 1
        for (int h = 0; h < G; ++h) {
            const HeadSel &H = hs[h];
            const bool act = (only < 0 || h == only) && H.mode == 1;
            const float e = (act && s < S) ? score(s, h) : -INFINITY;
            bool member = false;
            unsigned long long wf = 0ull;
            uint32_t dk = 0u;
            if (e != -INFINITY) {
                wf = mass_fx(expf(e - H.M));
                dk = desc_key(e);
                bool is_above;
                if (H.refined) {
                    is_above = dk < H.klo;
                    member = !is_above && dk <= H.khi;
                } else {
                    const int b = coarse_bucket(H.M, e);
                    is_above = b < (int)H.Blo;
                    member = !is_above && b <= (int)H.Bhi;
                }
#pragma unroll
                for (int hh = 0; hh < G; ++hh)
                    if (hh == h && is_above) above[hh] += wf;
            }
            const unsigned bal = __ballot_sync(FULL, member);
            if (bal) {
                const int leader = __ffs(bal) - 1;
                uint32_t base = 0;
                if (lane == leader) base = atomicAdd(&hs[h].ncand, (uint32_t)__popc(bal));
                base = __shfl_sync(FULL, base, leader);
                if (member) {
                    const uint32_t idx = base + __popc(bal & ((1u << lane) - 1u));
                    if (idx < (uint32_t)SEL_CAND) {
                        ck[h * SEL_CAND + idx] = ((unsigned long long)dk << 32) | (unsigned long long)s;
                        cm[h * SEL_CAND + idx] = wf;
                    }
                }
            }
        }
    }
    g_sum_u64<G>(above, red);
    if (tid < G && (only < 0 || tid == only) && hs[tid].mode == 1) {
#pragma unroll
        for (int h = 0; h < G; ++h)
            if (h == tid) hs[tid].above = above[h];
    }
    gsync();
}

// Narrow the candidate range of head hh, whose bracket holds more than
// SEL_CAND nodes, by histograms over its key range.  Leaves hs[hh] with
// refined = 1, the key range, its count, and mode 1 (ranking) or 2 (an exact
// tie wider than the list).
template <int G>
__device__ __noinline__ void refine_head(HeadSel *hs, int hh, int64_t S, ScoreView score, uint32_t *cnt,
                                        unsigned long long *ck, unsigned long long *cm, unsigned long long *red,
                                        uint32_t *sh32, unsigned long long *sh64) {
    const int tid = threadIdx.x;
    gather_pass<G>(hs, S, score, ck, cm, red, hh);  // mass above the coarse bracket
    const float M = hs[hh].M;
    uint32_t lo = 0xffffffffu, hi = 0u;
    {
        const int B0 = (int)hs[hh].Blo, B1 = (int)hs[hh].Bhi;
        for (int64_t s = tid; s < S; s += GT) {
            const float e = score(s, hh);
            if (e == -INFINITY) continue;
            const int b = coarse_bucket(M, e);
            if (b >= B0 && b <= B1) {
                const uint32_t dk = desc_key(e);
                lo = min(lo, dk);
                hi = max(hi, dk);
            }
        }
    }
    uint32_t klo = g_min_u32(lo, sh32), khi = g_max_u32(hi, sh32);
    uint32_t count = hs[hh].count;
    const unsigned long long target = hs[hh].target;
    while (count > (uint32_t)SEL_CAND && klo < khi) {
        const unsigned long long above = hs[hh].above;
        for (int i = tid; i < NB; i += GT) cnt[i] = 0u;
        gsync();
        const unsigned long long span = (unsigned long long)(khi - klo) + 1ull;
        for (int64_t s = tid; s < S; s += GT) {
            const float e = score(s, hh);
            if (e == -INFINITY) continue;
            const uint32_t dk = desc_key(e);
            if (dk >= klo && dk <= khi) atomicAdd(&cnt[(int)(((unsigned long long)(dk - klo) * NB) / span)], 1u);
        }
        gsync();
        // sub-bucket sb holds keys [klo + ceil(sb*span/NB), klo + ceil((sb+1)*span/NB) - 1];
        // the smaller key is the larger estimate and weight
        const int per = NB / GT;
        unsigned long long ub = 0, lb = 0;
        for (int q = 0; q < per; ++q) {
            const int sb = tid * per + q;
            const unsigned long long n = cnt[sb];
            if (!n) continue;
            const uint32_t k0 = klo + (uint32_t)(((unsigned long long)sb * span + NB - 1) / NB);
            const uint32_t k1 = klo + (uint32_t)(((unsigned long long)(sb + 1) * span + NB - 1) / NB) - 1u;
            ub += n * key_w_hi(k0, M);
            lb += n * key_w_lo(k1, M);
        }
        unsigned long long tot;
        const unsigned long long iu = g_scan_u64(ub, sh64, &tot);
        const unsigned long long il = g_scan_u64(lb, sh64, &tot);
        unsigned long long ru = above + iu - ub, rl = above + il - lb;
        uint32_t slo = 0xffffffffu, shi = 0xffffffffu;
        for (int q = 0; q < per; ++q) {
            const int sb = tid * per + q;
            const unsigned long long n = cnt[sb];
            if (n) {
                const uint32_t k0 = klo + (uint32_t)(((unsigned long long)sb * span + NB - 1) / NB);
                const uint32_t k1 = klo + (uint32_t)(((unsigned long long)(sb + 1) * span + NB - 1) / NB) - 1u;
                ru += n * key_w_hi(k0, M);
                rl += n * key_w_lo(k1, M);
            }
            if (ru >= target && slo == 0xffffffffu) slo = sb;
            if (rl >= target && shi == 0xffffffffu) shi = sb;
        }
        const uint32_t SBlo = g_min_u32(slo, sh32);
        uint32_t SBhi = g_min_u32(shi, sh32);
        if (SBhi == 0xffffffffu) SBhi = NB - 1;
        const uint32_t SB0 = SBlo > SBhi ? 0u : SBlo;
        const uint32_t nklo = klo + (uint32_t)(((unsigned long long)SB0 * span + NB - 1) / NB);
        const unsigned long long e1 = klo + ((unsigned long long)(SBhi + 1) * span + NB - 1) / NB;
        const uint32_t nkhi = (uint32_t)min((unsigned long long)khi, e1 - 1ull);
        uint32_t nloc = 0;
        for (uint32_t b = SB0 + tid; b <= SBhi; b += GT) nloc += cnt[b];
        uint32_t n;
        g_scan_u32(nloc, sh32, &n);
        if (tid == 0) {
            hs[hh].refined = 1;
            hs[hh].klo = nklo;
            hs[hh].khi = nkhi;
        }
        gsync();
        gather_pass<G>(hs, S, score, ck, cm, red, hh);  // exact mass above the new range
        klo = nklo;
        khi = nkhi;
        count = n;
    }
    if (tid == 0) {
        HeadSel &H = hs[hh];
        H.refined = 1;
        H.klo = klo;
        H.khi = khi;
        H.count = count;
        H.mode = (count > (uint32_t)SEL_CAND) ? 2 : 1;
        H.ncand = 0;
    }
    gsync();
}

// Head hh's cut falls inside an exact tie of more than SEL_CAND equal
// estimates (key klo): the first t of them in slot order are kept.
template <int G>
__device__ __noinline__ void tie_head(HeadSel *hs, int hh, int64_t S, ScoreView score, unsigned long long *ck,
                                     unsigned long long *cm, unsigned long long *red, uint32_t *sh32,
                                     uint32_t *bc32) {
    const int tid = threadIdx.x;
    const uint32_t dlo = hs[hh].klo;
    const unsigned long long wtie = mass_fx(expf(desc_key_to_float(dlo) - hs[hh].M));
    if (tid == 0) { hs[hh].mode = 1; hs[hh].refined = 1; hs[hh].khi = dlo; }
    gsync();
    gather_pass<G>(hs, S, score, ck, cm, red, hh);  // mass strictly above the tie
    const unsigned long long need = hs[hh].target - hs[hh].above;
    const unsigned long long t_need = wtie ? (need + wtie - 1ull) / wtie : (unsigned long long)hs[hh].count;
    if (tid == 0) {
        hs[hh].mode = 2;
        hs[hh].cut = ((unsigned long long)dlo << 32) | 0xffffffffull;
        bc32[0] = 0u;
    }
    gsync();
    for (int64_t base = 0; base < S; base += GT) {
        const int64_t s = base + tid;
        const float e = s < S ? score(s, hh) : -INFINITY;
        const uint32_t fl = (e != -INFINITY && desc_key(e) == dlo) ? 1u : 0u;
        uint32_t tot;
        const uint32_t incl = g_scan_u32(fl, sh32, &tot);
        if (fl && (unsigned long long)bc32[0] + incl == t_need)
            hs[hh].cut = ((unsigned long long)dlo << 32) | (unsigned long long)s;
        gsync();
        if (tid == 0) bc32[0] += tot;
        gsync();
    }
}

// Ordered compaction: the union kept list (the next frontier, with head
// masks) and the per-head lists (leaf outputs at level 1, traces).  Each
// thread takes SPT consecutive slots of a tile (their node ids loaded up
// front); one group scan of G+1 packed 12-bit counters per tile gives every
// write position.
template <int G>
__device__ __noinline__ void compact(const Decode &a, int l, int kh, int64_t S, ScoreView score,
                                     const unsigned long long *cut_sm, uint32_t *tot_out,
                                     unsigned long long *sh64) {
    constexpr int SPT = 8;
    static_assert(G * SPT <= 32 && G <= 4, "packed kept bits and 12-bit counters");
    const int tid = threadIdx.x;
    const bool per_head = (l == 1) || (a.trace_ids != nullptr);
    const int64_t kbase = (int64_t)kh * a.t.node_cap[l - 1];
    const int32_t *snode = a.slot_node + (int64_t)kh * a.score_cap;
    uint32_t tot_list[G + 1];
#pragma unroll
    for (int i = 0; i <= G; ++i) tot_list[i] = 0u;
#pragma unroll 1
    for (int64_t base = 0; base < S; base += (int64_t)GT * SPT) {
        const int64_t s0 = base + (int64_t)tid * SPT;
        int32_t nd[SPT];
#pragma unroll
        for (int i = 0; i < SPT; ++i) nd[i] = (s0 + i < S) ? __ldcg(snode + s0 + i) : -1;
        uint32_t bits = 0u;  // G bits per slot
        unsigned long long packed = 0ull;
#pragma unroll
        for (int i = 0; i < SPT; ++i) {
            const int64_t s = s0 + i;
            uint32_t kb = 0u;
            if (s < S) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float e = score(s, h);
                    if (e != -INFINITY &&
                        (((unsigned long long)desc_key(e) << 32) | (unsigned long long)s) <= cut_sm[h])
                        kb |= 1u << h;
                }
            }
            bits |= kb << (G * i);
            if (kb) {
                packed += 1ull;
#pragma unroll
                for (int h = 0; h < G; ++h) packed += (unsigned long long)((kb >> h) & 1u) << (12 * (h + 1));
            }
        }
        unsigned long long tile_tot;
        const unsigned long long incl = g_scan_u64(packed, sh64, &tile_tot);
        const unsigned long long excl = incl - packed;
        uint32_t pos[G + 1];
#pragma unroll
        for (int i = 0; i <= G; ++i) pos[i] = tot_list[i] + (uint32_t)((excl >> (12 * i)) & 0xfffull);
#pragma unroll
        for (int i = 0; i < SPT; ++i) {
            const uint32_t kb = (bits >> (G * i)) & ((1u << G) - 1u);
            if (!kb) continue;
            a.kept_ids[l - 1][kbase + pos[0]] = nd[i];
            a.kept_mask[l - 1][kbase + pos[0]] = (uint8_t)kb;
            ++pos[0];
            if (!per_head) continue;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                if (!((kb >> h) & 1u)) continue;
                const int hq = kh * G + h;
                const uint32_t ph = pos[1 + h]++;
                if (l == 1 && a.leaf_idx && ph < (uint32_t)a.leaf_cap) a.leaf_idx[(int64_t)hq * a.leaf_cap + ph] = nd[i];
                if (a.trace_ids && ph < (uint32_t)a.trace_cap)
                    a.trace_ids[((int64_t)(l - 1) * a.t.h_q + hq) * a.trace_cap + ph] = nd[i];
            }
        }
#pragma unroll
        for (int i = 0; i <= G; ++i) tot_list[i] += (uint32_t)((tile_tot >> (12 * i)) & 0xfffull);
    }
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i <= G; ++i) tot_out[i] = tot_list[i];
    }
}

// Top-p cut and compaction of level l for KV head kh.  `S` is the frontier
// size, `nb` the number of per-CTA maxima written for this KV head.
template <int HD, int R, int G>
__device__ __noinline__ void select_kvh(const Decode &a, int l, int kh, int64_t S, int nb, unsigned char *smem) {
    using SM = SelectSmem<G>;
    const int tid = threadIdx.x;
    const int lane = tid & 31, wid = tid >> 5;
    float *sc = reinterpret_cast<float *>(smem);
    uint32_t *hc = reinterpret_cast<uint32_t *>(smem + SM::off_hc);
    unsigned long long *ck = reinterpret_cast<unsigned long long *>(smem + SM::off_ck);
    unsigned long long *cm = reinterpret_cast<unsigned long long *>(smem + SM::off_cm);
    HeadSel *hs = reinterpret_cast<HeadSel *>(smem + SM::off_hs);
    unsigned long long *red = reinterpret_cast<unsigned long long *>(smem + SM::off_red);
    unsigned long long *scan = reinterpret_cast<unsigned long long *>(smem + SM::off_scan);
    unsigned char *misc = smem + SM::off_misc;
    uint32_t *sh32 = reinterpret_cast<uint32_t *>(misc);                            // 8 x u32
    unsigned long long *sh64 = reinterpret_cast<unsigned long long *>(misc + 128);  // 8 x u64
    uint32_t *bc32 = reinterpret_cast<uint32_t *>(misc + 384);
    unsigned long long *cuts = reinterpret_cast<unsigned long long *>(misc + 416);   // [G]
    uint32_t *tot = reinterpret_cast<uint32_t *>(misc + 480);                        // [G+1]

    const int64_t sbase = (int64_t)kh * a.score_cap * G;
    const bool staged = S <= SM::STAGE_SLOTS;
    if (staged) {
        if constexpr (G % 4 == 0) {  // whole 16-byte rows, 16-byte aligned per KV head
            const float4 *src = reinterpret_cast<const float4 *>(a.scores + sbase);
            float4 *dst = reinterpret_cast<float4 *>(sc);
            for (int64_t i = tid; i < S * G / 4; i += GT) dst[i] = __ldcg(src + i);
        } else {
            for (int64_t i = tid; i < S * G; i += GT) sc[i] = __ldcg(a.scores + sbase + i);
        }
    }
    const ScoreView score{staged ? sc : a.scores + sbase, G, staged};
    const float p = a.p;
    const bool keep_all = !(p < 1.0f);

    // frontier max per head from the per-CTA maxima; clear the counts
    {
        float mx[G];
#pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
        for (int i = tid; i < nb; i += GT) {
#pragma unroll
            for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], __ldcg(a.pmax + ((int64_t)kh * a.pmax_cap + i) * G + h));
        }
        float *redf = reinterpret_cast<float *>(red);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float v = warp_max(mx[h]);
            if (lane == 0) redf[wid * G + h] = v;
        }
        for (int i = tid; i < G * NB; i += GT) hc[i] = 0u;
        gsync();
        if (tid < G) {
            float M = -INFINITY;
            for (int w = 0; w < GT / 32; ++w) M = fmaxf(M, redf[w * G + tid]);
            HeadSel &H = hs[tid];
            H.M = M; H.Z = 0; H.F = 0; H.Blo = 0xffffffffu; H.Bhi = 0xffffffffu; H.count = 0; H.ncand = 0;
            H.refined = 0; H.mode = keep_all ? 0 : 1; H.cut = ~0ull; H.above = 0; H.klo = 0; H.khi = 0;
        }
        gsync();
    }

    // 1. counts per bucket, total mass and frontier size of every head
    {
        unsigned long long w[2 * G];  // [0, G): masses; [G, 2G): frontier sizes
#pragma unroll
        for (int h = 0; h < 2 * G; ++h) w[h] = 0ull;
        float M[G];
#pragma unroll
        for (int h = 0; h < G; ++h) M[h] = hs[h].M;
#pragma unroll 1
        for (int64_t s = tid; s < S; s += GT) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float e = score(s, h);
                if (e != -INFINITY) {
                    w[G + h] += 1ull;
                    if (!keep_all) {
                        w[h] += mass_fx(expf(e - M[h]));
                        atomicAdd(&hc[h * NB + coarse_bucket(M[h], e)], 1u);
                    }
                }
            }
        }
        g_sum_u64<2 * G>(w, red);
        if (tid < G) {
            unsigned long long zt = 0, ft = 0;
#pragma unroll
            for (int h = 0; h < G; ++h)
                if (h == tid) { zt = w[h]; ft = w[G + h]; }
            hs[tid].F = (uint32_t)ft;
            hs[tid].Z = zt;
            unsigned long long tg = (unsigned long long)ceil((double)p * (double)zt);
            if (tg > zt) tg = zt;
            hs[tid].target = tg ? tg : 1ull;
        }
        gsync();
    }

    if (!keep_all) {
        // 2. bracket the cut bucket of every head from count x weight bounds
        {
            constexpr int TPG = GT / G, per = NB / TPG;
            const int h = tid / TPG, gl = tid % TPG;
            unsigned long long ub = 0, lb = 0;
            for (int q = 0; q < per; ++q) {
                const int b = gl * per + q;
                const unsigned long long n = hc[h * NB + b];
                if (n) {
                    ub += n * bucket_w_hi(b);
                    lb += n * bucket_w_lo(b);
                }
            }
            unsigned long long t2;
            const unsigned long long iu = g_scan_u64(ub, sh64, &t2);
            scan[tid] = iu;
            gsync();
            const unsigned long long base_u = (h > 0) ? scan[h * TPG - 1] : 0ull;
            gsync();
            const unsigned long long il = g_scan_u64(lb, sh64, &t2);
            scan[tid] = il;
            gsync();
            const unsigned long long base_l = (h > 0) ? scan[h * TPG - 1] : 0ull;
            const unsigned long long target = hs[h].target;
            unsigned long long ru = iu - ub - base_u, rl = il - lb - base_l;
            uint32_t blo = 0xffffffffu, bhi = 0xffffffffu;
            for (int q = 0; q < per; ++q) {
                const int b = gl * per + q;
                const unsigned long long n = hc[h * NB + b];
                if (n) {
                    ru += n * bucket_w_hi(b);
                    rl += n * bucket_w_lo(b);
                }
                if (ru >= target && blo == 0xffffffffu) blo = b;
                if (rl >= target && bhi == 0xffffffffu) bhi = b;
            }
            if (blo != 0xffffffffu) atomicMin(&hs[h].Blo, blo);
            if (bhi != 0xffffffffu) atomicMin(&hs[h].Bhi, bhi);
            gsync();
            if (tid < G) {
                HeadSel &H = hs[tid];
                if (H.Bhi == 0xffffffffu) H.Bhi = NB - 1;
                if (H.Blo == 0xffffffffu || H.Blo > H.Bhi) H.Blo = 0;
                uint32_t n = 0;
                for (uint32_t b = H.Blo; b <= H.Bhi; ++b) n += hc[tid * NB + b];
                H.count = n;
            }
            gsync();
        }
        // 3. narrow crowded brackets by value (rare)
#pragma unroll 1
        for (int hh = 0; hh < G; ++hh)
            if (hs[hh].count > (uint32_t)SEL_CAND) refine_head<G>(hs, hh, S, score, hc + hh * NB, ck, cm, red, sh32, sh64);
        // 4. one pass: exact mass above each bracket and its candidates
        if (tid < G) hs[tid].ncand = 0;
        gsync();
        gather_pass<G>(hs, S, score, ck, cm, red, -1);
        if (tid < G && hs[tid].mode == 1) {
            unsigned long long mx = 0ull;
            const int n = (int)min(hs[tid].ncand, (uint32_t)SEL_CAND);
            for (int i = 0; i < n; ++i) mx = max(mx, ck[tid * SEL_CAND + i]);
            hs[tid].cut = mx;  // safe default: keep every candidate
        }
        gsync();
#pragma unroll 1
        for (int i = tid; i < G * SEL_CAND; i += GT) {
            const int hh = i / SEL_CAND, ci = i % SEL_CAND;
            if (hs[hh].mode != 1) continue;
            const int n = (int)min(hs[hh].ncand, (uint32_t)SEL_CAND);
            if (ci >= n) continue;
            const unsigned long long key = ck[hh * SEL_CAND + ci];
            unsigned long long before = 0ull;
            for (int j = 0; j < n; ++j)
                if (ck[hh * SEL_CAND + j] < key) before += cm[hh * SEL_CAND + j];
            const unsigned long long lo_m = hs[hh].above + before;
            if (lo_m < hs[hh].target && lo_m + cm[hh * SEL_CAND + ci] >= hs[hh].target) hs[hh].cut = key;
        }
        gsync();
        // exact ties wider than the candidate list (rare)
#pragma unroll 1
        for (int hh = 0; hh < G; ++hh)
            if (hs[hh].mode == 2) tie_head<G>(hs, hh, S, score, ck, cm, red, sh32, bc32);
    }

    if (tid < G) cuts[tid] = hs[tid].cut;
    gsync();
    compact<G>(a, l, kh, S, score, cuts, tot, sh64);
    gsync();
    if (tid < G) {
        const int h = tid;
        const int hq = kh * G + h;
        const uint32_t nk = tot[1 + h];
        const int64_t prev = (l == a.t.D) ? 0 : a.vis_acc[hq];
        const int64_t vis = prev + (int64_t)hs[h].F;
        a.vis_acc[hq] = vis;
        if (a.trace_cnt) a.trace_cnt[(l - 1) * a.t.h_q + hq] = (int32_t)nk;
        if (a.trace_ids && nk > (uint32_t)a.trace_cap) set_status(a.status, ZHA_CAPACITY_CODE);
        if (l == 1) {
            if (a.n_leaf) a.n_leaf[hq] = (int32_t)nk;
            if (a.visited) a.visited[hq] = vis;
            if (a.leaf_idx && nk > (uint32_t)a.leaf_cap) set_status(a.status, ZHA_CAPACITY_CODE);
        }
    }
    if (tid == 0) a.kept_cnt[(l - 1) * a.t.h_kv + kh] = (int32_t)tot[0];
}

template <int G>
constexpr size_t route_select_smem() {
    return SelectSmem<G>::bytes;
}

}  // namespace zha
