/*
 * zha_oracle.c -- plain, slow, fp64 CPU statement of the ZHA decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker that the CUDA library
 * is compared against.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load it.  It shares no code, header,
 * table or helper with the CUDA library, and the library never calls it.
 *
 * Every quantity is computed in double precision from the exact stored
 * inputs: bf16 keys/values are widened bit-exactly (bf16 -> fp32 -> fp64),
 * fp32 inputs are widened to fp64.  No blocking, fusion or reordering is
 * done beyond what each definition states; loops follow the definitions.
 *
 * Sources (web pages on Zyphra Hierarchical Attention, cited by title and
 * section):
 *   [ZH-CN1] "Zyphra 分层注意力（ZHA）：通向真次二次注意力的新路径，挑战长上下文瓶颈",
 *            section "机制拆解：树形索引如何高效筛选长上下文"
 *   [ZH-CN2] "ZHA 用树形稀疏注意力改造现有大模型",
 *            section "稀疏注意力为什么还会被索引拖慢"
 *   [ZH-RU]  rit.work "ZHA tree indexer" article,
 *            section "Дерево сокращает сам поиск нужных ключей"
 *   [ZH-JA]  "階層型疎Attention「ZHA」──長文LLMの探索コストを削る新設計",
 *            section "【技術的ディープダイブ】"
 *   [ZH-ID]  "Zyphra Luncurkan ZHA: Attention Sparse Tree-based yang Beneran
 *            Subquadratic?", opening section (how ZHA works)
 *
 * Readings taken where the pages are vague (each is also listed with the
 * design notes of the repository):
 *   - Leaf summary: for reference query r_j the chunk's log attention mass
 *     m_j = logsumexp_i(r_j.k_i/sqrt(d)) and its gradient g_j (the
 *     softmax-weighted mean key); the chunk's estimated log mass for a query
 *     q is the max over the tangent planes m_j + (q - r_j).g_j/sqrt(d)
 *     ([ZH-CN2]: each reference query gives one linear estimate of the
 *     chunk's log mass, and the chunk's estimate is the largest of them).
 *   - Parent summary: m_j = logsumexp over children of the child's estimate
 *     at q = r_j; g_j = children's g_j weighted by softmax of those
 *     estimates ([ZH-CN1]: summaries grouped and compressed recursively).
 *   - Depth D: a top node covers c^D tokens and there are D routing levels
 *     ([ZH-CN2]/[ZH-JA]: chunk 4 and 6 levels cover 4,096 tokens).
 *   - Top-p: softmax over the current frontier, order by probability
 *     descending with ties to the lower node id, keep the shortest prefix
 *     whose cumulative probability reaches p; p >= 1 keeps every node
 *     ([ZH-CN2]: the kept set is the fewest nodes whose mass adds up to p;
 *     [ZH-JA]: top-p, not a fixed top-k).
 *   - Attention: exact softmax attention over the raw keys of the kept leaf
 *     chunks plus token 0, the attention sink ([ZH-RU]: attention uses the
 *     raw keys of the found leaves; [ZH-CN2]/[ZH-ID]: the first token is
 *     always kept).
 *   - Append: the new row joins its leaf chunk; that leaf and every ancestor
 *     is recomputed from its definition (tree maintenance, [ZH-RU] section
 *     "Замеры подтверждают качество, а предельный выигрыш пока рассчитан").
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_F32 0
#define ORC_BF16 1

/* Widen one stored element to double.  bf16 is the upper half of an IEEE
 * fp32 word, so the widening is exact. */
static double widen(const void *base, int dtype, int64_t idx)
{
    if (dtype == ORC_F32)
        return (double)((const float *)base)[idx];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double dotd(const double *a, const double *b, int n)
{
    double acc = 0.0;
    for (int k = 0; k < n; ++k)
        acc += a[k] * b[k];
    return acc;
}

/* Number of nodes at level `level` (1 = leaf chunks) for n_tokens tokens:
 * ceil(n_tokens / c^level). */
int64_t orc_level_nodes(int64_t n_tokens, int c, int level)
{
    int64_t span = 1;
    for (int l = 0; l < level; ++l)
        span *= c;
    return (n_tokens + span - 1) / span;
}

/*
 * Leaf summary of the chunk holding tokens [t0, t1) of one head's key
 * matrix K[n][d] ([ZH-CN1], [ZH-CN2]).  For every reference query r_j:
 *   s_i = r_j . k_i / sqrt(d)
 *   m_j = max_i s_i + log sum_i exp(s_i - max)
 *   g_j = sum_i exp(s_i - m_j) k_i          (softmax-weighted mean key)
 *   b_j = m_j - r_j . g_j / sqrt(d)         (plane offset; est = max_j b_j + q.g_j/sqrt(d))
 * Outputs m[R], g[R*d], b[R].
 */
void orc_leaf_summary(const void *K, int dtype, int64_t t0, int64_t t1, int d,
                      const double *ref, int R, double *m, double *g, double *b)
{
    const double scale = 1.0 / sqrt((double)d);
    const int64_t n = t1 - t0;
    double *s = (double *)malloc((size_t)n * sizeof(double));
    double *k = (double *)malloc((size_t)d * sizeof(double));
    for (int j = 0; j < R; ++j) {
        const double *rj = ref + (size_t)j * d;
        double mx = -INFINITY;
        for (int64_t i = 0; i < n; ++i) {
            for (int e = 0; e < d; ++e)
                k[e] = widen(K, dtype, (t0 + i) * d + e);
            s[i] = scale * dotd(rj, k, d);
            if (s[i] > mx)
                mx = s[i];
        }
        double sum = 0.0;
        for (int64_t i = 0; i < n; ++i)
            sum += exp(s[i] - mx);
        m[j] = mx + log(sum);
        double *gj = g + (size_t)j * d;
        for (int e = 0; e < d; ++e)
            gj[e] = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            const double w = exp(s[i] - m[j]);
            for (int e = 0; e < d; ++e)
                gj[e] += w * widen(K, dtype, (t0 + i) * d + e);
        }
        b[j] = m[j] - scale * dotd(rj, gj, d);
    }
    free(k);
    free(s);
}

/*
 * Estimated log attention mass of one node for query q: the max over its R
 * tangent planes, est(q) = max_j [ m_j + (q - r_j) . g_j / sqrt(d) ]
 * ([ZH-CN2]: several estimate planes, take the maximum).
 */
double orc_estimate(const double *m, const double *g, int R, int d,
                    const double *ref, const double *q)
{
    const double scale = 1.0 / sqrt((double)d);
    double best = -INFINITY;
    for (int j = 0; j < R; ++j) {
        const double *rj = ref + (size_t)j * d;
        const double *gj = g + (size_t)j * d;
        double acc = 0.0;
        for (int e = 0; e < d; ++e)
            acc += (q[e] - rj[e]) * gj[e];
        const double v = m[j] + scale * acc;
        if (v > best)
            best = v;
    }
    return best;
}

/*
 * Parent summary from nch children ([ZH-CN1]: summaries are grouped and
 * compressed recursively).  Children's m are cm[nch*R], g are cg[nch*R*d].
 * For every reference query r_j:
 *   e_ch = est_child(r_j)                    (the child's estimate at q = r_j)
 *   m_j  = logsumexp_ch e_ch
 *   g_j  = sum_ch exp(e_ch - m_j) g_{ch,j}   (mass-weighted mean of the children's g_j)
 *   b_j  = m_j - r_j . g_j / sqrt(d)
 */
void orc_parent_summary(const double *cm, const double *cg, int nch, int d,
                        const double *ref, int R, double *m, double *g, double *b)
{
    const double scale = 1.0 / sqrt((double)d);
    double *e = (double *)malloc((size_t)nch * sizeof(double));
    for (int j = 0; j < R; ++j) {
        const double *rj = ref + (size_t)j * d;
        double mx = -INFINITY;
        for (int ch = 0; ch < nch; ++ch) {
            e[ch] = orc_estimate(cm + (size_t)ch * R, cg + (size_t)ch * R * d, R, d, ref, rj);
            if (e[ch] > mx)
                mx = e[ch];
        }
        double sum = 0.0;
        for (int ch = 0; ch < nch; ++ch)
            sum += exp(e[ch] - mx);
        m[j] = mx + log(sum);
        double *gj = g + (size_t)j * d;
        for (int k = 0; k < d; ++k)
            gj[k] = 0.0;
        for (int ch = 0; ch < nch; ++ch) {
            const double w = exp(e[ch] - m[j]);
            const double *cgj = cg + ((size_t)ch * R + j) * d;
            for (int k = 0; k < d; ++k)
                gj[k] += w * cgj[k];
        }
        b[j] = m[j] - scale * dotd(rj, gj, d);
    }
    free(e);
}

/*
 * Summary store of one head: node (level l, id n) lives at row
 * level_off[l-1] + n of m[.,R], g[.,R,d], b[.,R].  Level l has
 * ceil(N / c^l) nodes; leaf n covers tokens [n c, min((n+1) c, N)); the
 * children of level-l node n are the level-(l-1) ids
 * [n c, min((n+1) c, n_{l-1})).
 */
static void node_recompute(const void *K, int dtype, int64_t N, int d, const double *ref,
                           int R, int c, int level, int64_t n, double *m, double *g,
                           double *b, const int64_t *level_off)
{
    const int64_t row = level_off[level - 1] + n;
    if (level == 1) {
        const int64_t t0 = n * c;
        int64_t t1 = t0 + c;
        if (t1 > N)
            t1 = N;
        orc_leaf_summary(K, dtype, t0, t1, d, ref, R, m + row * R, g + row * R * d, b + row * R);
    } else {
        const int64_t nbelow = orc_level_nodes(N, c, level - 1);
        const int64_t c0 = n * c;
        int64_t c1 = c0 + c;
        if (c1 > nbelow)
            c1 = nbelow;
        const int64_t crow = level_off[level - 2] + c0;
        orc_parent_summary(m + crow * R, g + crow * R * d, (int)(c1 - c0), d, ref, R,
                           m + row * R, g + row * R * d, b + row * R);
    }
}

/* Whole tree of one head over its first N tokens: leaves, then each parent
 * level in turn. */
void orc_build(const void *K, int dtype, int64_t N, int d, const double *ref, int R, int c,
               int D, double *m, double *g, double *b, const int64_t *level_off)
{
    for (int level = 1; level <= D; ++level) {
        const int64_t nl = orc_level_nodes(N, c, level);
        for (int64_t n = 0; n < nl; ++n)
            node_recompute(K, dtype, N, d, ref, R, c, level, n, m, g, b, level_off);
    }
}

/*
 * Depth of a tree whose depth grows with the context ([ZH-RU] section
 * "Дерево сокращает сам поиск нужных ключей", last paragraph: levels are
 * added as the context grows; the reading taken: a level is added on top
 * whenever the top level would hold more than c nodes): the smallest depth
 * D in [D0, Dmax] whose top level holds at most c nodes for N tokens, or
 * Dmax when none does.  Dmax <= D0 keeps the depth fixed at D0.
 */
int orc_depth_for(int64_t N, int c, int D0, int Dmax)
{
    if (Dmax <= D0)
        return D0;
    for (int D = D0; D < Dmax; ++D)
        if (orc_level_nodes(N, c, D) <= c)
            return D;
    return Dmax;
}

/* Every node of one level, from the raw keys (level 1) or from the level
 * below (the parent summary of each node's children). */
void orc_build_level(const void *K, int dtype, int64_t N, int d, const double *ref, int R, int c, int level,
                     double *m, double *g, double *b, const int64_t *level_off)
{
    const int64_t nl = orc_level_nodes(N, c, level);
    for (int64_t n = 0; n < nl; ++n)
        node_recompute(K, dtype, N, d, ref, R, c, level, n, m, g, b, level_off);
}

/*
 * Tree maintenance for one appended token.  The caller has stored the new
 * key as row N-1 (N already counts it).  The leaf holding it is recomputed
 * from its tokens, then each ancestor from its children; a node that did not
 * exist before (a new chunk, or a new top node) is created the same way.
 */
void orc_append_update(const void *K, int dtype, int64_t N, int d, const double *ref, int R,
                       int c, int D, double *m, double *g, double *b, const int64_t *level_off)
{
    int64_t n = (N - 1) / c;
    for (int level = 1; level <= D; ++level) {
        node_recompute(K, dtype, N, d, ref, R, c, level, n, m, g, b, level_off);
        n /= c;
    }
}

/* ---- top-p over one frontier ------------------------------------------ */

typedef struct {
    double p;
    int64_t id;
    int64_t pos;
} orc_item;

static int item_cmp(const void *a, const void *b)
{
    const orc_item *x = (const orc_item *)a, *y = (const orc_item *)b;
    if (x->p > y->p)
        return -1;
    if (x->p < y->p)
        return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id) ? 1 : 0;
}

/*
 * Adaptive top-p cut over a frontier of F nodes with estimates est[F] and
 * node ids ids[F] ([ZH-CN1], [ZH-CN2], [ZH-JA]):
 *   P_i = softmax over the frontier of est_i;
 *   order the nodes by P descending, ties by lower id;
 *   keep the shortest prefix whose cumulative P reaches p (p >= 1: keep all).
 * Outputs (each indexed like the input): kept[i] in {0,1}, prob[i] = P_i,
 * cum_before[i] = cumulative P of the nodes ordered before node i,
 * rank[i] = position of node i in that order.  Returns the number kept.
 */
int64_t orc_topp(const double *est, const int64_t *ids, int64_t F, double p, uint8_t *kept,
                 double *prob, double *cum_before, int64_t *rank)
{
    if (F <= 0)
        return 0;
    double mx = -INFINITY;
    for (int64_t i = 0; i < F; ++i)
        if (est[i] > mx)
            mx = est[i];
    double Z = 0.0;
    for (int64_t i = 0; i < F; ++i)
        Z += exp(est[i] - mx);
    orc_item *it = (orc_item *)malloc((size_t)F * sizeof(orc_item));
    for (int64_t i = 0; i < F; ++i) {
        prob[i] = exp(est[i] - mx) / Z;
        it[i].p = prob[i];
        it[i].id = ids[i];
        it[i].pos = i;
        kept[i] = 0;
    }
    qsort(it, (size_t)F, sizeof(orc_item), item_cmp);
    double cum = 0.0;
    int64_t nkept = 0;
    int done = 0;
    for (int64_t r = 0; r < F; ++r) {
        const int64_t i = it[r].pos;
        cum_before[i] = cum;
        rank[i] = r;
        if (!done) {
            kept[i] = 1;
            ++nkept;
        }
        cum += it[r].p;
        if (p < 1.0 && cum >= p)
            done = 1;
    }
    free(it);
    return nkept;
}

/* ---- routing ------------------------------------------------------------ */

/*
 * Route one query down the tree of one head ([ZH-CN1]: score the top-level
 * nodes, keep a top-p set, expand only the kept nodes' children, repeat
 * until the raw entries).  The frontier at level D is every top node.
 * Outputs: kept ids of level l in kept[l-1][0 .. kept_count[l-1]) (ascending
 * id), each list with room for ceil(N / c^l) ids; *visited = total number of
 * nodes scored.  Returns 0.
 */
int orc_route(const double *m, const double *g, const int64_t *level_off, int64_t N, int R,
              int d, int c, int D, const double *ref, const double *q, double p,
              int64_t **kept, int64_t *kept_count, int64_t *visited)
{
    const int64_t ntop = orc_level_nodes(N, c, D);
    int64_t *front = (int64_t *)malloc((size_t)(orc_level_nodes(N, c, 1) + c) * sizeof(int64_t));
    int64_t nf = ntop;
    for (int64_t n = 0; n < ntop; ++n)
        front[n] = n;
    *visited = 0;
    for (int level = D; level >= 1; --level) {
        double *est = (double *)malloc((size_t)nf * sizeof(double));
        double *prob = (double *)malloc((size_t)nf * sizeof(double));
        double *cb = (double *)malloc((size_t)nf * sizeof(double));
        int64_t *rk = (int64_t *)malloc((size_t)nf * sizeof(int64_t));
        uint8_t *kf = (uint8_t *)malloc((size_t)nf);
        for (int64_t i = 0; i < nf; ++i) {
            const int64_t row = level_off[level - 1] + front[i];
            est[i] = orc_estimate(m + row * R, g + row * R * d, R, d, ref, q);
        }
        *visited += nf;
        orc_topp(est, front, nf, p, kf, prob, cb, rk);
        int64_t nk = 0;
        for (int64_t i = 0; i < nf; ++i)
            if (kf[i])
                kept[level - 1][nk++] = front[i];
        kept_count[level - 1] = nk;
        if (level > 1) {
            const int64_t nbelow = orc_level_nodes(N, c, level - 1);
            int64_t nn = 0;
            for (int64_t k = 0; k < nk; ++k)
                for (int64_t ch = kept[level - 1][k] * c; ch < (kept[level - 1][k] + 1) * c; ++ch)
                    if (ch < nbelow)
                        front[nn++] = ch;
            nf = nn;
        }
        free(est);
        free(prob);
        free(cb);
        free(rk);
        free(kf);
    }
    free(front);
    return 0;
}

/* ---- exact attention ---------------------------------------------------- */

/*
 * Exact softmax attention of query q over the listed tokens of one head
 * ([ZH-RU]: the main attention uses the raw keys of the found leaves):
 *   s_i = q . k_i / sqrt(d);  out = sum_i softmax(s)_i v_i.
 */
void orc_attend(const void *K, const void *V, int dtype, int d, const int64_t *tok, int64_t T,
                const double *q, double *out)
{
    const double scale = 1.0 / sqrt((double)d);
    double *s = (double *)malloc((size_t)T * sizeof(double));
    double mx = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
        double acc = 0.0;
        for (int e = 0; e < d; ++e)
            acc += q[e] * widen(K, dtype, tok[t] * d + e);
        s[t] = scale * acc;
        if (s[t] > mx)
            mx = s[t];
    }
    double den = 0.0;
    for (int e = 0; e < d; ++e)
        out[e] = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        const double w = exp(s[t] - mx);
        den += w;
        for (int e = 0; e < d; ++e)
            out[e] += w * widen(V, dtype, tok[t] * d + e);
    }
    for (int e = 0; e < d; ++e)
        out[e] /= den;
    free(s);
}

/*
 * Attended token set of one query: every token of the kept leaf chunks,
 * plus token 0 (the attention sink, [ZH-CN2], [ZH-ID]) when it is not
 * already among them.  Leaves are given ascending; tokens come out
 * ascending.  Returns the count.
 */
int64_t orc_token_set(const int64_t *leaves, int64_t nleaf, int64_t N, int c, int64_t *tok)
{
    int64_t T = 0;
    if (nleaf == 0 || leaves[0] != 0)
        tok[T++] = 0;
    for (int64_t k = 0; k < nleaf; ++k)
        for (int64_t t = leaves[k] * c; t < (leaves[k] + 1) * c && t < N; ++t)
            tok[T++] = t;
    return T;
}

/*
 * One decoded token for one query head: route, gather the token set and
 * attend.  Outputs out[d], the kept leaf ids (ascending) in leaf_out, their
 * count, and the number of nodes scored.  kept_buf must hold
 * sum_l ceil(N / c^l) ids.  Returns the leaf count.
 */
int64_t orc_decode_one(const void *K, const void *V, int dtype, int64_t N, int d,
                       const double *m, const double *g, const int64_t *level_off, int R, int c,
                       int D, const double *ref, const double *q, double p, double *out,
                       int64_t *leaf_out, int64_t *visited, int64_t *kept_buf)
{
    int64_t **kept = (int64_t **)malloc((size_t)D * sizeof(int64_t *));
    int64_t *kcount = (int64_t *)malloc((size_t)D * sizeof(int64_t));
    int64_t off = 0;
    for (int l = 1; l <= D; ++l) {
        kept[l - 1] = kept_buf + off;
        off += orc_level_nodes(N, c, l);
    }
    orc_route(m, g, level_off, N, R, d, c, D, ref, q, p, kept, kcount, visited);
    const int64_t nleaf = kcount[0];
    memcpy(leaf_out, kept[0], (size_t)nleaf * sizeof(int64_t));
    int64_t *tok = (int64_t *)malloc((size_t)(nleaf * c + 1) * sizeof(int64_t));
    const int64_t T = orc_token_set(kept[0], nleaf, N, c, tok);
    orc_attend(K, V, dtype, d, tok, T, q, out);
    free(tok);
    free(kcount);
    free(kept);
    return nleaf;
}

/*
 * Decode of several query heads of one step, query head h reading KV head
 * h / G.  Heads run in parallel when built with OpenMP; each head's work is
 * exactly orc_decode_one.  K, V are [H_kv][kv_stride][d]; m, g are the
 * per-KV-head stores (m_stride, g_stride doubles apart); q is [H_q][d];
 * ref is [H_kv][R][d]; kept_buf needs H_q * kept_stride ids.
 */
void orc_decode_heads(const void *K, const void *V, int dtype, int64_t kv_stride, int64_t N,
                      int d, int H_kv, int H_q, const double *m, int64_t m_stride,
                      const double *g, int64_t g_stride, const int64_t *level_off, int R, int c,
                      int D, const double *ref, const double *q, double p, double *out,
                      int64_t *leaf_out, int64_t leaf_stride, int64_t *nleaf, int64_t *visited,
                      int64_t *kept_buf, int64_t kept_stride)
{
    const int G = H_q / H_kv;
    const size_t esize = dtype == ORC_F32 ? 4 : 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H_q; ++h) {
        const int kh = h / G;
        const char *Kh = (const char *)K + (size_t)kh * kv_stride * d * esize;
        const char *Vh = (const char *)V + (size_t)kh * kv_stride * d * esize;
        nleaf[h] = orc_decode_one(Kh, Vh, dtype, N, d, m + kh * m_stride, g + kh * g_stride,
                                  level_off, R, c, D, ref + (size_t)kh * R * d,
                                  q + (size_t)h * d, p, out + (size_t)h * d,
                                  leaf_out + h * leaf_stride, visited + h,
                                  kept_buf + h * kept_stride);
    }
}

/* Build the trees of several KV heads (OpenMP over heads). */
void orc_build_heads(const void *K, int dtype, int64_t kv_stride, int64_t N, int d, int H_kv,
                     const double *ref, int R, int c, int D, double *m, int64_t m_stride,
                     double *g, int64_t g_stride, double *b, const int64_t *level_off)
{
    const size_t esize = dtype == ORC_F32 ? 4 : 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (int kh = 0; kh < H_kv; ++kh)
        orc_build((const char *)K + (size_t)kh * kv_stride * d * esize, dtype, N, d,
                  ref + (size_t)kh * R * d, R, c, D, m + kh * m_stride, g + kh * g_stride,
                  b + kh * m_stride, level_off);
}

/* ---- batch helpers for the checks (loops over the definitions above) ---- */

/* est[i] = orc_estimate of node ids[i] of one level (rows level_row0 + id). */
void orc_estimate_many(const double *m, const double *g, int64_t level_row0, const int64_t *ids,
                       int64_t n, int R, int d, const double *ref, const double *q, double *est)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const int64_t row = level_row0 + ids[i];
        est[i] = orc_estimate(m + row * R, g + row * R * d, R, d, ref, q);
    }
}

/*
 * Summary of one node (level, n) computed from the raw keys of its subtree
 * alone: a leaf by orc_leaf_summary, a parent by orc_parent_summary over its
 * children, each child computed the same way (recursion).  Used to check
 * sampled nodes of trees too large to build on the host.
 */
void orc_node_summary(const void *K, int dtype, int64_t N, int d, const double *ref, int R, int c,
                      int level, int64_t n, double *m, double *g, double *b)
{
    if (level == 1) {
        const int64_t t0 = n * c;
        int64_t t1 = t0 + c;
        if (t1 > N)
            t1 = N;
        orc_leaf_summary(K, dtype, t0, t1, d, ref, R, m, g, b);
        return;
    }
    const int64_t nbelow = orc_level_nodes(N, c, level - 1);
    const int64_t c0 = n * c;
    int64_t c1 = c0 + c;
    if (c1 > nbelow)
        c1 = nbelow;
    const int nch = (int)(c1 - c0);
    double *cm = (double *)malloc((size_t)nch * R * sizeof(double));
    double *cg = (double *)malloc((size_t)nch * R * d * sizeof(double));
    double *cb = (double *)malloc((size_t)nch * R * sizeof(double));
    for (int ch = 0; ch < nch; ++ch)
        orc_node_summary(K, dtype, N, d, ref, R, c, level - 1, c0 + ch, cm + (size_t)ch * R,
                         cg + (size_t)ch * R * d, cb + (size_t)ch * R);
    orc_parent_summary(cm, cg, nch, d, ref, R, m, g, b);
    free(cm);
    free(cg);
    free(cb);
}

/* Threads the multi-head drivers use (OpenMP builds); no arithmetic. */
void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
