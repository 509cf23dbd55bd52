// zha_api.cu -- the extern "C" boundary of libzha.so (declared in include/zha.h).
//
// Host-side only: argument checks, the workspace layout, and the launch
// sequence of each call.  The library allocates no device memory; every
// buffer belongs to the caller.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>

#include "../../include/zha.h"
#include "zha_internal.cuh"
#include "zha_tma.cuh"

using namespace zha;

struct zha_ctx {
    zha_config cfg;
    Tree t;                   // pointers into the workspace; K, V, ref set by zha_build
    bool built;
    unsigned char *ws;
    int64_t ws_bytes;
    Decode scratch;           // decode scratch pointers (inside the workspace); t and outputs unset
    unsigned char *scratch_begin;
    int64_t scratch_bytes;
    int64_t *phase_ns;        // caller's device buffer for phase stamps, or null
    long long wait_budget;    // clock cycles one inter-CTA barrier wait of the decode may take
    int decode_cta;
    int n_sm;
    int attn_cta;
    int D0, Dmax;             // least and greatest depth (equal unless the depth grows)
};

namespace {

constexpr int PART_CAP = SEG_CAP;  // attention partial records per KV head (one per CTA)

int64_t align256(int64_t x) { return (x + 255) / 256 * 256; }

// ceil(n / c^level), saturating at 1 once c^level exceeds n.
int64_t level_nodes(int64_t n, int c, int level) {
    int64_t span = 1;
    for (int l = 0; l < level; ++l) {
        if (span > n) return n > 0 ? 1 : 0;
        span *= c;
    }
    return (n + span - 1) / span;
}

int check_config(const zha_config *cfg) {
    if (!cfg) return ZHA_ERR_BAD_ARG;
    if (cfg->h_kv < 1 || cfg->h_kv > 64 || cfg->h_q < cfg->h_kv || cfg->h_q % cfg->h_kv) return ZHA_ERR_BAD_ARG;
    if (cfg->d <= 0 || cfg->R <= 0 || cfg->c < 2 || cfg->D < 1 || cfg->D > MAXD) return ZHA_ERR_BAD_ARG;
    if (cfg->kv_dtype != ZHA_F32 && cfg->kv_dtype != ZHA_BF16) return ZHA_ERR_BAD_ARG;
    if (cfg->capacity_tokens < 1 || cfg->capacity_tokens > (int64_t)0x7fffffff) return ZHA_ERR_BAD_ARG;
    if (cfg->max_depth != 0 && (cfg->max_depth <= cfg->D || cfg->max_depth > MAXD)) return ZHA_ERR_BAD_ARG;
    if (cfg->router_dtype != ZHA_F32 && cfg->router_dtype != ZHA_BF16) return ZHA_ERR_BAD_ARG;
    if (cfg->max_batch < 0 || (int64_t)cfg->h_kv * (cfg->max_batch > 1 ? cfg->max_batch : 1) > 64)
        return ZHA_ERR_BAD_ARG;
    const int G = cfg->h_q / cfg->h_kv;
    if (!compiled_combo(cfg->kv_dtype, cfg->d, cfg->R, G, cfg->router_dtype)) return ZHA_ERR_UNSUPPORTED;
    return ZHA_OK;
}

// Byte layout of the workspace.  Each region starts 256-byte aligned.
struct Layout {
    int64_t node_cap[MAXD], slot_cap[MAXD];
    int64_t g_off[MAXD], b_off[MAXD], m_off[MAXD], g16_off[MAXD], b16_off[MAXD];
    int64_t kid_off[MAXD], kmask_off[MAXD];
    int64_t seg_off, hseg_off, lvl_off, rdsc_off, scores_off, snode_off, skeep_off, tmax_off, tcnt_off, tsum_off;
    int64_t hcnt_off, hmass_off, cw_off, cs_off, ccnt_off, ticket_off, part_off, sync_off, status_off;
    int64_t scratch_off, total;
    int64_t score_cap;
};

// Levels the workspace holds: the greatest depth.
int max_levels(const zha_config *cfg) { return cfg->max_depth > cfg->D ? cfg->max_depth : cfg->D; }

// Depth over n tokens: the least depth in [D0, Dmax] whose top level holds
// at most c nodes, or Dmax (D0 when the depth does not grow).
int depth_for(int64_t n, int c, int D0, int Dmax) {
    int D = D0;
    while (D < Dmax && level_nodes(n, c, D) > c) ++D;
    return D;
}

// Queries one decode call may carry (zha_decode_batch).
int max_batch(const zha_config *cfg) { return cfg->max_batch > 1 ? cfg->max_batch : 1; }

void make_layout(const zha_config *cfg, Layout *L) {
    const int G = cfg->h_q / cfg->h_kv;
    const int64_t H = cfg->h_kv;                        // summary store: per KV head
    const int64_t HV = (int64_t)cfg->h_kv * max_batch(cfg);  // decode scratch: per (query, KV head)
    const int DL = max_levels(cfg);
    int64_t off = 0;
    for (int l = 1; l <= DL; ++l) {
        const int64_t nc = level_nodes(cfg->capacity_tokens, cfg->c, l);
        L->node_cap[l - 1] = nc;
        L->g_off[l - 1] = off;
        off = align256(off + H * nc * cfg->R * cfg->d * 4);
        L->b_off[l - 1] = off;
        off = align256(off + H * nc * cfg->R * 4);
        L->m_off[l - 1] = off;
        off = align256(off + H * nc * cfg->R * 4);
        L->g16_off[l - 1] = L->b16_off[l - 1] = -1;
        if (cfg->router_dtype == ZHA_BF16) {
            L->g16_off[l - 1] = off;
            off = align256(off + H * nc * cfg->R * cfg->d * 2);
            L->b16_off[l - 1] = off;
            off = align256(off + H * nc * cfg->R * 4);
        }
    }
    // frontier slots of level l: every top node, or c children of each node
    // of level l + 1
    int64_t sc = 0;
    for (int l = 1; l <= DL; ++l) {
        L->slot_cap[l - 1] = (l == DL) ? L->node_cap[l - 1] : (int64_t)cfg->c * L->node_cap[l];
        sc = std::max(sc, L->slot_cap[l - 1]);
    }
    L->score_cap = sc;
    L->scratch_off = off;
    for (int l = 1; l <= DL; ++l) {
        L->kid_off[l - 1] = off;
        off = align256(off + HV * L->slot_cap[l - 1] * 4);
        L->kmask_off[l - 1] = off;
        off = align256(off + HV * L->slot_cap[l - 1]);
    }
    auto take = [&](int64_t &at, int64_t bytes) {
        at = off;
        off = align256(off + bytes);
    };
    take(L->seg_off, (int64_t)MAXD * HV * SEG_CAP * 4);
    take(L->hseg_off, (int64_t)MAXD * HV * SEG_CAP * G * 4);
    take(L->lvl_off, (int64_t)MAXD * HV * 2 * 4);
    take(L->rdsc_off, HV * 2 * LOC_CAP * G * 4);
    take(L->scores_off, HV * sc * G * 4);
    take(L->snode_off, HV * sc * 4);
    take(L->skeep_off, HV * sc + 4);
    take(L->tmax_off, HV * SEG_CAP * G * 4);
    take(L->tcnt_off, HV * SEG_CAP * G * 4);
    take(L->tsum_off, HV * SEG_CAP * G * 8);
    take(L->hcnt_off, HV * HIST_ROUNDS * G * NB * 4);
    take(L->hmass_off, HV * HIST_ROUNDS * G * NB * 8);
    take(L->cw_off, HV * G * CAND_MAX * 8);
    take(L->cs_off, HV * G * CAND_MAX * 4);
    take(L->ccnt_off, HV * G * 4);
    take(L->ticket_off, HV * 4);
    take(L->part_off, (int64_t)PART_CAP * HV * G * (cfg->d + 4) * 4);
    take(L->sync_off, (HV + 3) * 4);
    take(L->status_off, 4);
    L->total = off;
}

bool fault_injected(const char *what) {
    const char *f = std::getenv("ZHA_FAULT");
    return f && std::strcmp(f, what) == 0;
}

void fill_tree_levels(zha_ctx *ctx) {
    Tree &t = ctx->t;
    for (int l = 1; l <= t.D; ++l) t.n_level[l - 1] = (int32_t)level_nodes(t.n_tokens, t.c, l);
}

Decode make_decode(zha_ctx *ctx) {
    Decode dc = ctx->scratch;
    dc.t = ctx->t;
    dc.nvk = ctx->t.h_kv;
    dc.phase_ns = ctx->phase_ns;
    dc.wait_budget = ctx->wait_budget;
    return dc;
}

}  // namespace

extern "C" {

int64_t zha_workspace_bytes(const zha_config *cfg) {
    const int rc = check_config(cfg);
    if (rc != ZHA_OK) return rc;
    Layout L;
    make_layout(cfg, &L);
    return L.total;
}

int zha_create(const zha_config *cfg, void *d_workspace, int64_t ws_bytes, zha_ctx **out) {
    if (!out) return ZHA_ERR_BAD_ARG;
    *out = nullptr;
    const int rc = check_config(cfg);
    if (rc != ZHA_OK) return rc;
    Layout L;
    make_layout(cfg, &L);
    if (!d_workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(d_workspace) & 255u))
        return ZHA_ERR_BAD_ARG;
    zha_ctx *ctx = new (std::nothrow) zha_ctx;
    if (!ctx) return ZHA_ERR_BAD_ARG;
    std::memset(ctx, 0, sizeof *ctx);
    ctx->cfg = *cfg;
    ctx->wait_budget = WAIT_BUDGET_CYCLES;
    unsigned char *ws = static_cast<unsigned char *>(d_workspace);
    ctx->ws = ws;
    ctx->ws_bytes = ws_bytes;
    Tree &t = ctx->t;
    t.h_kv = cfg->h_kv;
    t.h_q = cfg->h_q;
    t.G = cfg->h_q / cfg->h_kv;
    t.d = cfg->d;
    t.R = cfg->R;
    t.c = cfg->c;
    t.D = cfg->D;
    t.kv_dtype = cfg->kv_dtype;
    t.c_log2 = -1;
    for (int s = 0; s < 31; ++s)
        if ((1 << s) == cfg->c) t.c_log2 = s;
    t.kv_cap = cfg->capacity_tokens;
    t.scale = (float)(1.0 / std::sqrt((double)cfg->d));
    ctx->D0 = cfg->D;
    ctx->Dmax = max_levels(cfg);
    Decode &d = ctx->scratch;
    std::memset(&d, 0, sizeof d);
    for (int l = 1; l <= ctx->Dmax; ++l) {
        t.node_cap[l - 1] = L.node_cap[l - 1];
        t.g[l - 1] = reinterpret_cast<float *>(ws + L.g_off[l - 1]);
        t.b[l - 1] = reinterpret_cast<float *>(ws + L.b_off[l - 1]);
        t.m[l - 1] = reinterpret_cast<float *>(ws + L.m_off[l - 1]);
        t.g16[l - 1] = L.g16_off[l - 1] >= 0 ? reinterpret_cast<uint16_t *>(ws + L.g16_off[l - 1]) : nullptr;
        t.b16[l - 1] = L.b16_off[l - 1] >= 0 ? reinterpret_cast<float *>(ws + L.b16_off[l - 1]) : nullptr;
        d.kept_ids[l - 1] = reinterpret_cast<int32_t *>(ws + L.kid_off[l - 1]);
        d.kept_mask[l - 1] = reinterpret_cast<uint8_t *>(ws + L.kmask_off[l - 1]);
        d.slot_cap[l - 1] = L.slot_cap[l - 1];
    }
    d.seg = reinterpret_cast<uint32_t *>(ws + L.seg_off);
    d.hseg = reinterpret_cast<uint32_t *>(ws + L.hseg_off);
    d.lvl = reinterpret_cast<int32_t *>(ws + L.lvl_off);
    d.rd_scores = reinterpret_cast<float *>(ws + L.rdsc_off);
    d.scores = reinterpret_cast<float *>(ws + L.scores_off);
    d.slot_node = reinterpret_cast<int32_t *>(ws + L.snode_off);
    d.slot_keep = reinterpret_cast<uint8_t *>(ws + L.skeep_off);
    d.score_cap = L.score_cap;
    d.tmax = reinterpret_cast<float *>(ws + L.tmax_off);
    d.tcnt = reinterpret_cast<uint32_t *>(ws + L.tcnt_off);
    d.tsum = reinterpret_cast<unsigned long long *>(ws + L.tsum_off);
    d.hist_cnt = reinterpret_cast<uint32_t *>(ws + L.hcnt_off);
    d.hist_mass = reinterpret_cast<unsigned long long *>(ws + L.hmass_off);
    d.cand_w = reinterpret_cast<unsigned long long *>(ws + L.cw_off);
    d.cand_slot = reinterpret_cast<uint32_t *>(ws + L.cs_off);
    d.cand_cnt = reinterpret_cast<uint32_t *>(ws + L.ccnt_off);
    d.ticket = reinterpret_cast<uint32_t *>(ws + L.ticket_off);
    d.part = reinterpret_cast<float *>(ws + L.part_off);
    d.part_cap = PART_CAP;
    d.sync = reinterpret_cast<unsigned *>(ws + L.sync_off);
    d.status = reinterpret_cast<int32_t *>(ws + L.status_off);
    ctx->scratch_begin = ws + L.scratch_off;
    ctx->scratch_bytes = L.total - L.scratch_off;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&ctx->n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        delete ctx;
        return ZHA_ERR_CUDA;
    }
    ctx->attn_cta = std::min(PART_CAP, ctx->n_sm);  // one CTA per SM, one wave
    // the decode kernel: one resident CTA per SM (cooperative launch), a
    // multiple of h_kv so that every KV head gets a team of the same size
    {
        Decode probe = make_decode(ctx);
        const int per_sm = decode_blocks_per_sm(probe);
        if (per_sm < 1) {
            delete ctx;
            return ZHA_ERR_CUDA;
        }
        ctx->decode_cta = std::min(ctx->n_sm, PART_CAP);  // rounded to a multiple of the teams per call
    }
    if (cudaMemset(ctx->scratch_begin, 0, (size_t)ctx->scratch_bytes) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
        delete ctx;
        return ZHA_ERR_CUDA;
    }
    *out = ctx;
    return ZHA_OK;
}

void zha_destroy(zha_ctx *ctx) { delete ctx; }

int zha_build(zha_ctx *ctx, void *d_K, void *d_V, int64_t n_tokens, const float *d_ref_q, int32_t c, int32_t D,
              void *stream) {
    if (!ctx || !d_K || !d_V || !d_ref_q) return ZHA_ERR_BAD_ARG;
    if (c != ctx->cfg.c || D != ctx->cfg.D) return ZHA_ERR_BAD_ARG;
    if (n_tokens < 1) return ZHA_ERR_BAD_ARG;
    if (n_tokens > ctx->cfg.capacity_tokens) return ZHA_ERR_CAPACITY;
    if (((reinterpret_cast<uintptr_t>(d_K) | reinterpret_cast<uintptr_t>(d_V)) & 15u) ||
        (reinterpret_cast<uintptr_t>(d_ref_q) & 15u))
        return ZHA_ERR_BAD_ARG;
    Tree &t = ctx->t;
    t.K = d_K;
    t.V = d_V;
    t.ref = d_ref_q;
    t.n_tokens = n_tokens;
    t.D = depth_for(n_tokens, t.c, ctx->D0, ctx->Dmax);
    fill_tree_levels(ctx);
    if (fault_injected("cuda_launch")) return ZHA_ERR_CUDA;
    if (launch_build(t, static_cast<cudaStream_t>(stream), ctx->n_sm) != cudaSuccess) return ZHA_ERR_CUDA;
    ctx->built = true;
    return ZHA_OK;
}

int zha_append(zha_ctx *ctx, const void *d_k, const void *d_v, void *stream) {
    if (!ctx || !d_k || !d_v) return ZHA_ERR_BAD_ARG;
    if (!ctx->built) return ZHA_ERR_NOT_BUILT;
    if (ctx->t.n_tokens >= ctx->cfg.capacity_tokens || fault_injected("capacity")) return ZHA_ERR_CAPACITY;
    Tree t = ctx->t;
    t.n_tokens += 1;
    for (int l = 1; l <= t.D; ++l) t.n_level[l - 1] = (int32_t)level_nodes(t.n_tokens, t.c, l);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_append(t, d_k, d_v, s) != cudaSuccess) return ZHA_ERR_CUDA;
    // a growing tree whose top level now holds c + 1 nodes: a new top level
    const int D_new = depth_for(t.n_tokens, t.c, ctx->D0, ctx->Dmax);
    if (D_new > t.D) {
        const int D_old = t.D;
        t.D = D_new;
        for (int l = 1; l <= t.D; ++l) t.n_level[l - 1] = (int32_t)level_nodes(t.n_tokens, t.c, l);
        if (launch_build_levels(t, D_old + 1, D_new, s, ctx->n_sm) != cudaSuccess) return ZHA_ERR_CUDA;
    }
    ctx->t = t;
    return ZHA_OK;
}

int zha_decode(zha_ctx *ctx, const float *d_q, float p, float *d_out, int32_t *d_leaf_idx, int32_t leaf_cap,
               int32_t *d_n_leaf, int64_t *d_nodes_visited, int32_t *d_trace_ids, int32_t *d_trace_counts,
               int32_t trace_cap, void *stream) {
    return zha_decode_batch(ctx, d_q, 1, p, d_out, d_leaf_idx, leaf_cap, d_n_leaf, d_nodes_visited, d_trace_ids,
                            d_trace_counts, trace_cap, stream);
}

int zha_decode_batch(zha_ctx *ctx, const float *d_q, int32_t n_q, float p, float *d_out, int32_t *d_leaf_idx,
                     int32_t leaf_cap, int32_t *d_n_leaf, int64_t *d_nodes_visited, int32_t *d_trace_ids,
                     int32_t *d_trace_counts, int32_t trace_cap, void *stream) {
    if (!ctx || !d_q || !d_out) return ZHA_ERR_BAD_ARG;
    if (n_q < 1 || n_q > max_batch(&ctx->cfg)) return ZHA_ERR_BAD_ARG;
    if (!ctx->built) return ZHA_ERR_NOT_BUILT;
    if (!(p > 0.f) || std::isnan(p)) return ZHA_ERR_BAD_ARG;
    if ((d_leaf_idx && leaf_cap < 0) || (d_trace_ids && (!d_trace_counts || trace_cap < 0))) return ZHA_ERR_BAD_ARG;
    if ((reinterpret_cast<uintptr_t>(d_q) | reinterpret_cast<uintptr_t>(d_out)) & 15u) return ZHA_ERR_BAD_ARG;
    Decode dc = make_decode(ctx);
    dc.nvk = n_q * ctx->t.h_kv;
    dc.q = d_q;
    dc.p = p;
    dc.out = d_out;
    dc.leaf_idx = d_leaf_idx;
    dc.leaf_cap = d_leaf_idx ? leaf_cap : 0;
    dc.n_leaf = d_n_leaf;
    dc.visited = d_nodes_visited;
    dc.trace_ids = d_trace_ids;
    dc.trace_cnt = d_trace_ids ? d_trace_counts : nullptr;
    dc.trace_cap = d_trace_ids ? trace_cap : 0;
    // one team of CTAs per (query, KV head): the grid is the largest
    // multiple of that count within one CTA per SM
    const int n_cta = std::max(1, ctx->decode_cta / dc.nvk) * dc.nvk;
    if (n_cta > std::min(ctx->n_sm, PART_CAP)) return ZHA_ERR_UNSUPPORTED;
    if (launch_decode(dc, n_cta, static_cast<cudaStream_t>(stream)) != cudaSuccess) return ZHA_ERR_CUDA;
    return ZHA_OK;
}

int zha_dense_decode(zha_ctx *ctx, const float *d_q, float *d_out, void *stream) {
    if (!ctx || !d_q || !d_out) return ZHA_ERR_BAD_ARG;
    if (!ctx->built) return ZHA_ERR_NOT_BUILT;
    if ((reinterpret_cast<uintptr_t>(d_q) | reinterpret_cast<uintptr_t>(d_out)) & 15u) return ZHA_ERR_BAD_ARG;
    Decode dc = make_decode(ctx);
    dc.q = d_q;
    dc.out = d_out;
    if (launch_dense(dc, ctx->attn_cta, static_cast<cudaStream_t>(stream)) != cudaSuccess) return ZHA_ERR_CUDA;
    return ZHA_OK;
}

int zha_device_status(zha_ctx *ctx, int32_t *out_status, void *stream) {
    if (!ctx || !out_status) return ZHA_ERR_BAD_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t host = 0;
    if (cudaMemcpyAsync(&host, ctx->scratch.status, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(ctx->scratch.status, 0, sizeof host, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return ZHA_ERR_CUDA;
    // after a timed-out wait the barrier words, tickets and boundary lists may
    // be left raised: clear the decode scratch for the next call
    if (host == ZHA_ERR_TIMEOUT &&
        (cudaMemsetAsync(ctx->scratch_begin, 0, (size_t)ctx->scratch_bytes, s) != cudaSuccess ||
         cudaStreamSynchronize(s) != cudaSuccess))
        return ZHA_ERR_CUDA;
    *out_status = host;
    return ZHA_OK;
}

int zha_set_phase_timer(zha_ctx *ctx, int64_t *d_ns) {
    if (!ctx) return ZHA_ERR_BAD_ARG;
    if (d_ns && (reinterpret_cast<uintptr_t>(d_ns) & 7u)) return ZHA_ERR_BAD_ARG;
    ctx->phase_ns = d_ns;
    return ZHA_OK;
}

int zha_set_wait_budget(zha_ctx *ctx, int64_t cycles) {
    if (!ctx || cycles < 0) return ZHA_ERR_BAD_ARG;
    ctx->wait_budget = cycles > 0 ? (long long)cycles : 0;
    return ZHA_OK;
}

int32_t zha_depth(const zha_ctx *ctx) { return ctx && ctx->built ? ctx->t.D : 0; }

int64_t zha_n_tokens(const zha_ctx *ctx) { return ctx && ctx->built ? ctx->t.n_tokens : 0; }

int zha_summary_layout(const zha_ctx *ctx, int32_t level, int64_t *g_offset, int64_t *b_offset, int64_t *m_offset,
                       int64_t *node_cap) {
    if (!ctx || level < 1 || level > ctx->Dmax) return ZHA_ERR_BAD_ARG;
    const unsigned char *ws = ctx->ws;
    if (g_offset) *g_offset = reinterpret_cast<const unsigned char *>(ctx->t.g[level - 1]) - ws;
    if (b_offset) *b_offset = reinterpret_cast<const unsigned char *>(ctx->t.b[level - 1]) - ws;
    if (m_offset) *m_offset = reinterpret_cast<const unsigned char *>(ctx->t.m[level - 1]) - ws;
    if (node_cap) *node_cap = ctx->t.node_cap[level - 1];
    return ZHA_OK;
}

int zha_router_layout(const zha_ctx *ctx, int32_t level, int64_t *g_offset, int64_t *b_offset, int64_t *node_cap) {
    if (!ctx || level < 1 || level > ctx->Dmax || !ctx->t.g16[level - 1]) return ZHA_ERR_BAD_ARG;
    const unsigned char *ws = ctx->ws;
    if (g_offset) *g_offset = reinterpret_cast<const unsigned char *>(ctx->t.g16[level - 1]) - ws;
    if (b_offset) *b_offset = reinterpret_cast<const unsigned char *>(ctx->t.b16[level - 1]) - ws;
    if (node_cap) *node_cap = ctx->t.node_cap[level - 1];
    return ZHA_OK;
}

const char *zha_strerror(int code) {
    switch (code) {
        case ZHA_OK: return "ok";
        case ZHA_ERR_BAD_ARG: return "invalid argument";
        case ZHA_ERR_CAPACITY: return "capacity exceeded";
        case ZHA_ERR_NOT_BUILT: return "tree not built";
        case ZHA_ERR_CUDA: return "CUDA runtime error";
        case ZHA_ERR_TIMEOUT: return "device wait timed out";
        case ZHA_ERR_UNSUPPORTED: return "configuration not compiled";
        default: return "unknown status";
    }
}

}  // extern "C"
