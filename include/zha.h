/*
 * zha.h -- C ABI of libzha.so: single-layer decode attention over a full KV
 * cache, routed through the Zyphra Hierarchical Attention (ZHA) tree indexer,
 * on one NVIDIA B200 (sm_100a).
 *
 * What the method computes (pages cited by title and section):
 *  - "ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢":
 *    contiguous keys are split into chunks, each chunk gets a summary, the
 *    summaries are grouped and compressed again into a tree (chunk 4 and 6
 *    levels cover 4,096 tokens); a few reference queries give tangent-plane
 *    estimates of each chunk's log attention mass and the estimate is the max
 *    over several planes; at decode time the query scores the top nodes, keeps
 *    the smallest set whose estimated mass reaches p, expands only their
 *    children down to the raw KV entries, and token 0 is always kept as the
 *    attention sink.
 *  - "Zyphra 分层注意力（ZHA）：通向真次二次注意力的新路径，挑战长上下文瓶颈",
 *    section "机制拆解：树形索引如何高效筛选长上下文": recursive summary tree,
 *    reference queries, top-p routing repeated level by level.
 *  - rit.work "ZHA tree indexer" article, section "Дерево сокращает сам поиск
 *    нужных ключей": the main attention reads the raw keys of the found
 *    leaves, not their summaries; the full KV cache is kept.
 *  - same article, section "Замеры подтверждают качество, а предельный выигрыш
 *    пока рассчитан": tree maintenance is part of the per-token cost.
 *
 * Conventions for every entry point:
 *  - All pointers named d_* are DEVICE pointers on the current CUDA device;
 *    the library never allocates, frees or copies host memory for them and
 *    never takes ownership.  The caller keeps every buffer alive until the
 *    work enqueued on `stream` has finished.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls only enqueue work; they do not synchronise, except
 *    zha_device_status.
 *  - Return value: ZHA_OK (0) or a negative ZHA_ERR_* code found on the host
 *    (bad argument, capacity, CUDA launch error).  Errors that only the device
 *    can see (output capacity, an exhausted bounded wait) are recorded in a
 *    device status word read by zha_device_status; outputs count as valid only
 *    when that word is ZHA_OK.  Nothing traps on the device.
 *  - Layouts are row-major.  K and V hold `capacity_tokens` rows per KV head:
 *    element (head h, token t, dim e) is at index (h*capacity_tokens + t)*d + e.
 *    Query heads are grouped: query head i reads KV head i / (h_q / h_kv).
 */
#ifndef ZHA_H
#define ZHA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define ZHA_OK 0
#define ZHA_ERR_BAD_ARG (-1)     /* invalid argument or configuration */
#define ZHA_ERR_CAPACITY (-2)    /* cache, leaf list or trace list is full */
#define ZHA_ERR_NOT_BUILT (-3)   /* zha_build has not run on this context */
#define ZHA_ERR_CUDA (-4)        /* a CUDA runtime call failed */
#define ZHA_ERR_TIMEOUT (-5)     /* a bounded device-side wait gave up */
#define ZHA_ERR_UNSUPPORTED (-6) /* valid but not compiled (see zha_config) */

/* key/value storage types */
#define ZHA_F32 0
#define ZHA_BF16 1

/*
 * Static shape of one cache and its tree.
 *   h_kv, h_q        KV heads and query heads (h_q a multiple of h_kv;
 *                    compiled group sizes h_q/h_kv: 1 and 4)
 *   d                head dimension (compiled: 64, 128)
 *   R                reference queries per KV head (compiled: 1, 16)
 *   c                chunk size = children per node (>= 2)
 *   D                depth: routing levels; a top node covers c^D tokens
 *                    (1 <= D <= 16); with max_depth > D, the least depth
 *   kv_dtype         ZHA_F32 or ZHA_BF16
 *   max_depth        0: the depth stays D.  D < max_depth <= 16: the depth
 *                    grows with the context (rit.work "ZHA tree indexer",
 *                    section "Дерево сокращает сам поиск нужных ключей",
 *                    last paragraph): it is always the least depth >= D
 *                    whose top level holds at most c nodes (at most
 *                    max_depth), so zha_build starts there and an append
 *                    that leaves c + 1 top nodes adds a new top level over
 *                    them; zha_depth gives the current depth
 *   capacity_tokens  rows per KV head in K and V (room for appends)
 *   router_dtype     ZHA_F32: the routing reads the fp32 g rows.  ZHA_BF16:
 *                    the build and every append also store a bf16 copy of
 *                    each node's g rows (round to nearest even) with plane
 *                    offsets recomputed from that copy, m_j - r_j.g~_j/sqrt(d)
 *                    (so each rounded plane still passes through (r_j, m_j)),
 *                    and the routing reads those: half the router's bytes
 *                    ("ZHA 用树形稀疏注意力改造现有大模型", section
 *                    "几百倍加速，离实际部署还有多远": a reduced-precision
 *                    router).  Compiled for bf16 caches with d = 128.
 *   max_batch        most queries one zha_decode_batch call may carry (0 or
 *                    1: one); h_kv * max_batch <= 64.  The decode scratch
 *                    is sized for it.
 */
typedef struct {
    int32_t h_kv, h_q, d, R, c, D;
    int32_t kv_dtype;
    int32_t max_depth;
    int64_t capacity_tokens;
    int32_t router_dtype;
    int32_t max_batch;
} zha_config;

typedef struct zha_ctx zha_ctx; /* opaque host-side state: pointers and sizes only */

/*
 * Bytes of device workspace one context needs: the summary store of every
 * level at full capacity plus the decode scratch.  Returns a negative
 * ZHA_ERR_* code for an invalid configuration.
 */
int64_t zha_workspace_bytes(const zha_config *cfg);

/*
 * Create a context over a caller-allocated device workspace of ws_bytes
 * (>= zha_workspace_bytes(cfg), 256-byte aligned).  The context records the
 * pointer; the caller owns and frees the workspace after zha_destroy.
 * Enqueues nothing on the GPU except a clear of the decode scratch on the
 * legacy default stream, which it waits for.
 */
int zha_create(const zha_config *cfg, void *d_workspace, int64_t ws_bytes, zha_ctx **out);

/* Destroy the host-side context (the workspace is the caller's). */
void zha_destroy(zha_ctx *ctx);

/*
 * Build the summary tree over the first n_tokens rows of every KV head.
 * Source: leaf summaries and recursive parents, "ZHA 用树形稀疏注意力改造现有大模型",
 * section "稀疏注意力为什么还会被索引拖慢"; "Zyphra 分层注意力（ZHA）…", section
 * "机制拆解：树形索引如何高效筛选长上下文".
 *   d_K, d_V   [h_kv][capacity_tokens][d] kv_dtype; read in place, and the
 *              context keeps both pointers: later appends write row n into
 *              them and decodes read them.  The caller must not free them
 *              while the context is in use.
 *   n_tokens   1 <= n_tokens <= capacity_tokens
 *   d_ref_q    [h_kv][R][d] fp32 reference queries
 *   c, D       must equal the configuration's (checked)
 * Leaf chunk n covers tokens [n c, min((n+1) c, n_tokens)); for reference
 * query r_j it stores m_j = logsumexp_i(r_j.k_i/sqrt(d)), the softmax-weighted
 * mean key g_j, and the plane offset b_j = m_j - r_j.g_j/sqrt(d).  A level-l
 * node n (l >= 2) has the children [n c, min((n+1) c, n_{l-1})) and stores
 * m_j = logsumexp over children of the child's estimate at r_j, and g_j =
 * the children's g_j weighted by softmax of those estimates.  The estimate of
 * a node for query q is max_j (b_j + q.g_j/sqrt(d)).
 */
int zha_build(zha_ctx *ctx, void *d_K, void *d_V, int64_t n_tokens, const float *d_ref_q,
              int32_t c, int32_t D, void *stream);

/*
 * Append one token to every KV head and maintain the tree.
 * Source: tree maintenance, rit.work article section "Замеры подтверждают
 * качество, а предельный выигрыш пока рассчитан".
 *   d_k, d_v   [h_kv][d] kv_dtype: the new row of each KV head
 * Writes row n_tokens of the built K and V, recomputes the leaf holding it and
 * every ancestor (creating a node, or a new top node, at a boundary), then
 * n_tokens += 1.  With a growing depth (zha_config.max_depth), when the top
 * level then holds c + 1 nodes a new top level is built over it (a second
 * launch on `stream`) and the depth grows by one.  Returns ZHA_ERR_CAPACITY
 * when the cache is full and ZHA_ERR_NOT_BUILT before zha_build.
 */
int zha_append(zha_ctx *ctx, const void *d_k, const void *d_v, void *stream);

/*
 * Decode one token for all h_q query heads (batch 1, one layer).
 * Source: routing and attention, "ZHA 用树形稀疏注意力改造现有大模型", section
 * "稀疏注意力为什么还会被索引拖慢"; rit.work article section "Дерево сокращает сам
 * поиск нужных ключей".
 *   d_q              [h_q][d] fp32 queries
 *   p                top-p mass in (0, 1]; p >= 1 keeps every node
 *   d_out            [h_q][d] fp32 attention outputs
 *   d_leaf_idx       [h_q][leaf_cap] int32: ascending ids of the leaf chunks
 *                    head i kept at the last routing level (the sink token is
 *                    attended but not listed)
 *   d_n_leaf         [h_q] int32: number of kept leaf chunks per head
 *   d_nodes_visited  [h_q] int64: nodes scored over all levels per head
 *   d_trace_ids      nullable; [D][h_q][trace_cap] int32, D the current
 *                    depth (zha_depth): ascending kept node ids of level l
 *                    (1-based) at ((l-1)*h_q+i)*trace_cap
 *   d_trace_counts   nullable together with d_trace_ids; [D][h_q] int32
 * Routing per query head, level D down to 1: the frontier is every top node,
 * then the children of the nodes kept one level up; estimates are
 * softmax-normalised within the frontier, ordered by probability descending
 * with ties to the lower node id, and the shortest prefix whose cumulative
 * probability reaches p is kept.  Attention is exact softmax(q.k/sqrt(d))
 * over every token of the kept leaf chunks plus token 0, in fp32.
 * A list longer than its capacity is cut to the capacity and the device
 * status becomes ZHA_ERR_CAPACITY.
 * Launch: one cooperative kernel, a programmatic dependent of the kernel
 * before it on `stream` (its launch overlaps that kernel's tail); it reads no
 * input before that kernel has completed, so stream order is kept.
 */
int zha_decode(zha_ctx *ctx, const float *d_q, float p, float *d_out, int32_t *d_leaf_idx,
               int32_t leaf_cap, int32_t *d_n_leaf, int64_t *d_nodes_visited,
               int32_t *d_trace_ids, int32_t *d_trace_counts, int32_t trace_cap, void *stream);

/*
 * Decode n_q query tokens against the same cache in one launch: each query
 * is routed and attended exactly as zha_decode does it for one (every query
 * sees the whole cache as it is; none sees another).  Multi-query routing:
 * "Дерево сокращает сам поиск нужных ключей" (rit.work article) counts the
 * routing of every query of a sequence against the tree.  The grid gives
 * each (query, KV head) pair its own team of CTAs, so the queries route in
 * parallel; the G query heads of a pair share its summary and K/V reads.
 *   n_q              1 <= n_q <= zha_config.max_batch (or 1)
 *   d_q, d_out       [n_q][h_q][d] fp32
 *   d_leaf_idx       [n_q][h_q][leaf_cap]; d_n_leaf, d_nodes_visited [n_q][h_q]
 *   d_trace_ids      nullable; [D][n_q * h_q][trace_cap], d_trace_counts [D][n_q * h_q]
 * Returns ZHA_ERR_BAD_ARG for n_q outside [1, max_batch] and
 * ZHA_ERR_UNSUPPORTED when n_q * h_kv exceeds the CTAs of one wave.
 */
int zha_decode_batch(zha_ctx *ctx, const float *d_q, int32_t n_q, float p, float *d_out, int32_t *d_leaf_idx,
                     int32_t leaf_cap, int32_t *d_n_leaf, int64_t *d_nodes_visited, int32_t *d_trace_ids,
                     int32_t *d_trace_counts, int32_t trace_cap, void *stream);

/*
 * Dense flash-decode over the same cache (the comparison kernel): exact
 * softmax attention of every query head over all n_tokens rows.
 *   d_q [h_q][d] fp32, d_out [h_q][d] fp32.  Uses the context's scratch.
 */
int zha_dense_decode(zha_ctx *ctx, const float *d_q, float *d_out, void *stream);

/*
 * Dense flash-decode straight from a KV cache, with no context and no
 * workspace.  The pages have no counterpart: this serves layers that keep
 * plain dense attention inside an engine that reserves all of its device
 * memory up front and may not allocate while it serves, so it has no
 * workspace to hand over.  The split partials and merge tickets live in a
 * fixed scratch array of ZHA_STATIC_SCRATCH_BYTES inside the library's device
 * image; the call allocates nothing.
 *   cfg              h_kv, h_q, d, kv_dtype, capacity_tokens as for a context
 *                    (R, c, D are ignored)
 *   d_K, d_V         [h_kv][capacity_tokens][d] kv_dtype, 16-byte aligned
 *   n_tokens         rows attended per KV head, 1 <= n_tokens <= capacity
 *   d_q, d_out       [h_q][d] fp32, 16-byte aligned
 *   d_status         caller's device int32; a device-side failure (an
 *                    exhausted bounded wait) writes ZHA_ERR_TIMEOUT there if
 *                    it holds ZHA_OK; the caller reads and clears it
 * Same arithmetic and grid as zha_dense_decode.  Returns ZHA_ERR_CAPACITY
 * when the partials, h_q * (d + 4) * 4 bytes per SM (one CTA per SM, at most
 * 256), plus h_kv * 4 bytes of tickets, exceed ZHA_STATIC_SCRATCH_BYTES
 * (for d = 128 on 148 SMs: h_q <= 107).
 * The first call on each device looks up the scratch's device address
 * (cudaGetSymbolAddress, with that device current).  Under CUDA's default
 * lazy module loading, that first call (or any earlier use of this library's
 * kernels on the device) also loads the library's device module, which
 * reserves the fixed scratch and the kernel code in device memory.  So make
 * the first call during engine set-up (warm-up), before serving starts and
 * before any stream capture begins; later calls allocate nothing.  Every
 * call clears the tickets on `stream` first.
 * One call at a time per device: calls in flight together, on any streams or
 * host threads, share the scratch and corrupt each other's outputs.
 */
#define ZHA_STATIC_SCRATCH_BYTES (8 * 1024 * 1024)
int zha_dense_decode_static(const zha_config *cfg, const void *d_K, const void *d_V, int64_t n_tokens,
                            const float *d_q, float *d_out, int32_t *d_status, void *stream);

/*
 * Copy the device status word to *out_status and clear it.  Synchronises
 * `stream` first.  ZHA_OK means every decode since the last read was valid.
 */
int zha_device_status(zha_ctx *ctx, int32_t *out_status, void *stream);

/*
 * Profiling hook: zha_decode runs as one kernel; when a buffer is set, the
 * kernel writes the GPU global timer (nanoseconds) at its phase boundaries:
 *   d_ns  caller-owned device buffer of D + 3 int64 (8-byte aligned), kept
 *         alive while set; NULL clears.  d_ns[0] = start (after the wait
 *         for the kernel before it on the stream), d_ns[i] for
 *         i = 1 .. D-1 = end of routing level D - i + 1 as seen by the first
 *         CTA of KV head 0, d_ns[D] = end of the routing (every level, every
 *         KV head), d_ns[D + 1] = end of that CTA's share of the attention
 *         over the kept tokens, d_ns[D + 2] = end of the merge.
 * No effect on results.
 */
int zha_set_phase_timer(zha_ctx *ctx, int64_t *d_ns);

/*
 * Testing hook: the clock-cycle budget of each wait of zha_decode on other
 * CTAs (its team and grid barriers; default 2e9 cycles, about one second).
 * When a wait runs out, that CTA records ZHA_ERR_TIMEOUT in the device status
 * word and raises an abort flag, every CTA of the decode leaves at its next
 * wait without attending, and the call's outputs are invalid;
 * zha_device_status then reports ZHA_ERR_TIMEOUT and clears the decode
 * scratch, so the next decode starts clean.  0 makes every wait that is not
 * already satisfied give up at once.  Waits for the decode's own bulk copies
 * keep the default budget.  Returns ZHA_ERR_BAD_ARG for a negative budget.
 */
int zha_set_wait_budget(zha_ctx *ctx, int64_t cycles);

/* Current depth of the tree (routing levels; 0 before zha_build).  Equals
 * the configuration's D unless its max_depth lets the tree grow. */
int32_t zha_depth(const zha_ctx *ctx);

/* Tokens currently in the cache (host-side count; 0 before zha_build). */
int64_t zha_n_tokens(const zha_ctx *ctx);

/*
 * Where level `level` (1..max(D, max_depth)) of the summary store lives inside the workspace,
 * for inspection: byte offsets of g [h_kv][node_cap][R][d] fp32, b
 * [h_kv][node_cap][R] fp32 and m [h_kv][node_cap][R] fp32, and node_cap (the
 * node rows per KV head).  Returns ZHA_ERR_BAD_ARG for an invalid level.
 */
int zha_summary_layout(const zha_ctx *ctx, int32_t level, int64_t *g_offset, int64_t *b_offset,
                       int64_t *m_offset, int64_t *node_cap);

/*
 * Where the bf16 router copy of level `level` lives inside the workspace
 * (router_dtype ZHA_BF16): byte offsets of g~ [h_kv][node_cap][R][d] bf16
 * and of its plane offsets [h_kv][node_cap][R] fp32, and node_cap.
 * ZHA_ERR_BAD_ARG for an invalid level or a context without the copy.
 */
int zha_router_layout(const zha_ctx *ctx, int32_t level, int64_t *g_offset, int64_t *b_offset, int64_t *node_cap);

/* Static description of a status code. */
const char *zha_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* ZHA_H */
