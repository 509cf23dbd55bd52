"""Pins of the fp64 oracle to facts outside itself.

Each ``pin_*`` function takes an oracle library handle (``oracle.load()`` or a
deliberately broken build of it) and raises AssertionError when the oracle
disagrees with mathematics or with the pages.  The independent side is
written with numpy / scipy only (log-sum-exp, softmax, sorting, subset
enumeration), never with the oracle's own routines.

Facts used (page citations by title and section):
  * a top node of a tree with chunk 4 and 6 levels covers 4,096 tokens
    ("ZHA 用树形稀疏注意力改造现有大模型", section "稀疏注意力为什么还会被索引拖慢";
    "階層型疎Attention「ZHA」…", section "【技術的ディープダイブ】");
  * the estimate is a max over tangent planes of the chunk's log attention
    mass (same section of the first page), so by convexity of log-sum-exp
    it is a lower bound of the exact subtree log mass, tight at every
    reference query, with the exact gradient there;
  * top-p keeps the smallest node set whose mass reaches p (same section);
  * attention reads the raw keys of the kept leaves plus token 0 (rit.work
    article, section "Дерево сокращает сам поиск нужных ключей"; first page:
    the first token is always kept), so p = 1 gives dense attention.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
from scipy.special import logsumexp, softmax

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _tree_cases():
    # (N, c, D, R, d) -- ragged tails, several depths and plane counts
    return [(37, 2, 3, 3, 4), (64, 4, 2, 5, 8), (100, 3, 3, 1, 6), (256, 4, 3, 4, 8), (19, 4, 1, 2, 4),
            (50, 2, 4, 1, 4)]


def _subtree(N, c, level, n):
    span = c ** level
    return n * span, min((n + 1) * span, N)


def pin_closed_form_subtree(lib):
    """Every node's (m_j, g_j) equals log-sum-exp and softmax-weighted mean key
    of r_j.k/sqrt(d) over ALL raw keys of its subtree, and est(r_j) = m_j."""
    for case_i, (N, c, D, R, d) in enumerate(_tree_cases()):
        rng = _rng(100 + case_i)
        K = rng.standard_normal((N, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        tree = oracle.build(K, N, ref, c, D, lib=lib)
        K64 = K.astype(np.float64)
        for level in range(1, D + 1):
            m, g, b = tree.level(level)
            for n in range(m.shape[0]):
                t0, t1 = _subtree(N, c, level, n)
                for j in range(R):
                    s = K64[t0:t1] @ ref[j] / math.sqrt(d)
                    m_ref = logsumexp(s)
                    g_ref = softmax(s) @ K64[t0:t1]
                    assert abs(m[n, j] - m_ref) <= 1e-10 * max(1.0, abs(m_ref)), (level, n, j, m[n, j], m_ref)
                    assert np.max(np.abs(g[n, j] - g_ref)) <= 1e-10 * max(1.0, np.max(np.abs(g_ref))), (level, n, j)
                    est = oracle.estimate(m[n], g[n], ref, ref[j], lib=lib)
                    assert abs(est - m_ref) <= 1e-10 * max(1.0, abs(m_ref)), (level, n, j, est, m_ref)


def pin_lower_bound_and_tangent(lib):
    """est(q) <= exact subtree log mass for any q (tangent planes of a convex
    function), with equality to first order around each r_j."""
    for case_i, (N, c, D, R, d) in enumerate(_tree_cases()):
        rng = _rng(200 + case_i)
        K = rng.standard_normal((N, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        tree = oracle.build(K, N, ref, c, D, lib=lib)
        K64 = K.astype(np.float64)
        qs = [rng.standard_normal(d) * s for s in (0.5, 1.0, 3.0)] + [ref[0] * 2.0, -ref[-1]]
        for level in range(1, D + 1):
            m, g, b = tree.level(level)
            for n in range(m.shape[0]):
                t0, t1 = _subtree(N, c, level, n)
                for q in qs:
                    exact = logsumexp(K64[t0:t1] @ q / math.sqrt(d))
                    est = oracle.estimate(m[n], g[n], ref, q, lib=lib)
                    assert est <= exact + 1e-9, (level, n, est, exact)
                for j in range(R):
                    delta = rng.standard_normal(d)
                    delta *= 1e-4 / np.linalg.norm(delta)
                    q = ref[j] + delta
                    exact = logsumexp(K64[t0:t1] @ q / math.sqrt(d))
                    est = oracle.estimate(m[n], g[n], ref, q, lib=lib)
                    # second-order gap only: a wrong gradient shows at first order (~1e-4)
                    assert exact - est <= 1e-6, (level, n, j, exact - est)


def pin_single_plane_affine(lib):
    """With one reference query the estimate is affine in q, est(0) = b and
    est(r) = m."""
    rng = _rng(300)
    N, c, D, d = 90, 3, 3, 8
    K = rng.standard_normal((N, d)).astype(np.float32)
    ref = rng.standard_normal((1, d))
    tree = oracle.build(K, N, ref, c, D, lib=lib)
    for level in range(1, D + 1):
        m, g, b = tree.level(level)
        for n in range(m.shape[0]):
            q1, q2 = rng.standard_normal(d), rng.standard_normal(d)
            e1 = oracle.estimate(m[n], g[n], ref, q1, lib=lib)
            e2 = oracle.estimate(m[n], g[n], ref, q2, lib=lib)
            e3 = oracle.estimate(m[n], g[n], ref, 0.3 * q1 + 0.7 * q2, lib=lib)
            assert abs(e3 - (0.3 * e1 + 0.7 * e2)) <= 1e-10 * (1 + abs(e3))
            e0 = oracle.estimate(m[n], g[n], ref, np.zeros(d), lib=lib)
            assert abs(e0 - b[n, 0]) <= 1e-10 * (1 + abs(e0))
            assert abs(oracle.estimate(m[n], g[n], ref, ref[0], lib=lib) - m[n, 0]) <= 1e-10 * (1 + abs(m[n, 0]))


def _flat_topp(P, ids, p):
    """Independent top-p: sort by (P desc, id asc), shortest prefix reaching p."""
    order = sorted(range(len(P)), key=lambda i: (-P[i], ids[i]))
    kept, cum = [], 0.0
    for i in order:
        kept.append(ids[i])
        cum += P[i]
        if p < 1.0 and cum >= p:
            break
    return sorted(kept)


def pin_exact_leaves_token_topp(lib):
    """Chunk size 1: every leaf holds one token, the estimate is the exact
    score q.k/sqrt(d), and one routing level is exact token-level top-p."""
    rng = _rng(400)
    N, d = 40, 8
    K = rng.standard_normal((N, d)).astype(np.float32)
    ref = rng.standard_normal((3, d))
    tree = oracle.build(K, N, ref, 1, 1, lib=lib)
    m, g, b = tree.level(1)
    for trial in range(5):
        q = rng.standard_normal(d) * 2.0
        scores = K.astype(np.float64) @ q / math.sqrt(d)
        for n in range(N):
            est = oracle.estimate(m[n], g[n], ref, q, lib=lib)
            assert abs(est - scores[n]) <= 1e-10 * (1 + abs(scores[n]))
        P = softmax(scores)
        for p in (0.3, 0.75, 0.95):
            kept, _ = oracle.route(tree, ref, q, p, lib=lib)
            assert list(kept[0]) == _flat_topp(P, list(range(N)), p), (p,)


def pin_dense_at_p1(lib):
    """p = 1 keeps every node, so decode is dense softmax attention."""
    rng = _rng(500)
    for (N, c, D, R, d) in [(77, 4, 2, 3, 8), (130, 2, 4, 1, 4)]:
        K = rng.standard_normal((N, d)).astype(np.float32)
        V = rng.standard_normal((N, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        tree = oracle.build(K, N, ref, c, D, lib=lib)
        q = rng.standard_normal(d)
        out, leaves, visited = oracle.decode_one(K, V, tree, ref, q, 1.0, lib=lib)
        w = softmax(K.astype(np.float64) @ q / math.sqrt(d))
        assert np.max(np.abs(out - w @ V.astype(np.float64))) <= 1e-12
        assert list(leaves) == list(range(-(-N // c)))
        assert visited == sum(-(-N // c ** l) for l in range(1, D + 1))


def pin_flat_chunk_topp(lib):
    """Depth 1 is flat top-p over the chunk estimates (the wide tree)."""
    rng = _rng(600)
    N, c, R, d = 200, 8, 4, 8
    K = rng.standard_normal((N, d)).astype(np.float32)
    ref = rng.standard_normal((R, d))
    tree = oracle.build(K, N, ref, c, 1, lib=lib)
    m, g, b = tree.level(1)
    nl = m.shape[0]
    for trial in range(6):
        q = rng.standard_normal(d) * (1 + trial)
        est = np.array([oracle.estimate(m[n], g[n], ref, q, lib=lib) for n in range(nl)])
        P = softmax(est)
        for p in (0.5, 0.9, 0.99):
            kept, visited = oracle.route(tree, ref, q, p, lib=lib)
            assert list(kept[0]) == _flat_topp(P, list(range(nl)), p)
            assert visited == nl


def pin_routing_invariants(lib):
    """At every level: the frontier is exactly the children of the nodes kept
    one level up; the kept set reaches p, is minimal, and is a prefix in
    (P desc, id asc) order; nodes visited = sum of frontier sizes."""
    rng = _rng(700)
    for (N, c, D, R, d) in [(300, 3, 3, 4, 8), (512, 4, 3, 2, 8), (257, 2, 5, 1, 4)]:
        K = rng.standard_normal((N, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        tree = oracle.build(K, N, ref, c, D, lib=lib)
        for trial in range(4):
            q = rng.standard_normal(d) * (0.5 + trial)
            p = (0.6, 0.8, 0.9, 0.97)[trial]
            kept, visited = oracle.route(tree, ref, q, p, lib=lib)
            nvis = 0
            front = list(range(-(-N // c ** D)))
            for level in range(D, 0, -1):
                m, g, b = tree.level(level)
                est = np.array([oracle.estimate(m[n], g[n], ref, q, lib=lib) for n in front])
                P = softmax(est)
                ks = set(int(x) for x in kept[level - 1])
                assert ks <= set(front)
                mass = sum(P[i] for i, n in enumerate(front) if n in ks)
                assert mass >= p - 1e-12
                pk = [P[i] for i, n in enumerate(front) if n in ks]
                assert mass - min(pk) < p + 1e-12
                order = sorted(range(len(front)), key=lambda i: (-P[i], front[i]))
                assert set(front[i] for i in order[:len(ks)]) == ks
                nvis += len(front)
                nb = -(-N // c ** (level - 1))
                front = [ch for n in sorted(ks) for ch in range(n * c, (n + 1) * c) if ch < nb]
            assert visited == nvis


def pin_ties_lower_id(lib):
    """Two chunks with identical keys get identical estimates; with a small p
    only one is kept, and it is the lower id."""
    rng = _rng(800)
    N, c, R, d = 64, 4, 3, 8
    K = rng.standard_normal((N, d)).astype(np.float32) * 0.1
    q = rng.standard_normal(d)
    needle = (4.0 * math.sqrt(d) * q / np.linalg.norm(q)).astype(np.float32)
    K[9] = needle            # chunk 2
    K[4 * 11:4 * 12] = K[8:12]  # chunk 11 duplicates chunk 2
    ref = rng.standard_normal((R, d))
    ref[0] = q  # tangent at q: both duplicated chunks get their exact, dominant log mass
    tree = oracle.build(K, N, ref, c, 1, lib=lib)
    kept, _ = oracle.route(tree, ref, q, 0.3, lib=lib)
    assert list(kept[0]) == [2], kept[0]
    kept, _ = oracle.route(tree, ref, q, 0.6, lib=lib)
    assert list(kept[0]) == [2, 11], kept[0]


def pin_topp_brute_force(lib):
    """Exhaustive subset search on tiny frontiers: the kept set has the
    minimum size among all sets reaching p, the maximum mass among sets of
    that size, and the lowest ids among those (ties)."""
    rng = _rng(900)
    for trial in range(60):
        F = int(rng.integers(1, 9))
        est = rng.standard_normal(F) * 2
        if trial % 3 == 0 and F > 2:
            est[1] = est[0]
        ids = np.sort(rng.choice(1000, size=F, replace=False))
        p = float(rng.choice([0.2, 0.5, 0.75, 0.9, 0.95, 1.0]))
        kept, prob, cb, rank = oracle.topp(est, ids, p, lib=lib)
        P = softmax(est)
        assert np.allclose(prob, P, rtol=0, atol=1e-14)
        best = None
        for k in range(1, F + 1):
            for sub in itertools.combinations(range(F), k):
                mass = sum(P[i] for i in sub)
                if p >= 1.0 and k < F:
                    continue
                if p < 1.0 and mass < p:
                    continue
                key = (-mass, [ids[i] for i in sorted(sub, key=lambda i: (-P[i], ids[i]))])
                if best is None or key < best[0]:
                    best = (key, set(sub))
            if best is not None:
                break
        assert set(np.nonzero(kept)[0]) == best[1], (est, p, kept, best)
    # p = 1 keeps every node even when the cumulative mass reaches 1.0 early
    for est in ([0.0, -1000.0, -2000.0], [5.0, 5.0, -900.0, 4.0]):
        kept, _, _, _ = oracle.topp(np.array(est), np.arange(len(est)), 1.0, lib=lib)
        assert kept.all(), (est, kept)


def pin_attention_and_sink(lib):
    """Exact attention over a token list matches softmax attention; the
    token set is every token of the kept leaves plus token 0."""
    rng = _rng(1000)
    N, d, c = 50, 8, 4
    K = rng.standard_normal((N, d)).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    q = rng.standard_normal(d)
    toks = np.array([0, 3, 7, 8, 20, 49])
    out = oracle.attend(K, V, toks, q, lib=lib)
    w = softmax(K[toks].astype(np.float64) @ q / math.sqrt(d))
    assert np.max(np.abs(out - w @ V[toks].astype(np.float64))) <= 1e-13
    assert list(oracle.token_set([2, 12], N, c, lib=lib)) == [0, 8, 9, 10, 11, 48, 49]
    assert list(oracle.token_set([0, 3], N, c, lib=lib)) == [0, 1, 2, 3, 12, 13, 14, 15]


def pin_bf16_widening(lib):
    """bf16 keys are widened exactly: a bf16 cache gives the same tree as
    the fp32 cache holding the same values."""
    rng = _rng(1100)
    N, c, D, R, d = 40, 4, 2, 2, 8
    Kf = rng.standard_normal((N, d)).astype(np.float32)
    bits = (Kf.view(np.uint32) >> 16).astype(np.uint16)
    Kr = (bits.astype(np.uint32) << 16).view(np.float32)
    ref = rng.standard_normal((R, d))
    t_bf = oracle.build(bits, N, ref, c, D, lib=lib)
    t_f = oracle.build(Kr, N, ref, c, D, lib=lib)
    assert np.array_equal(t_bf.m, t_f.m) and np.array_equal(t_bf.g, t_f.g)


def pin_append_equivalence(lib):
    """Building over N tokens then appending a tokens one by one gives the
    tree built over N + a tokens (new chunks and a new top node included)."""
    rng = _rng(1200)
    for (N, a, c, D, R, d) in [(30, 7, 2, 3, 2, 4), (60, 5, 4, 2, 3, 8), (16, 1, 4, 2, 1, 4)]:
        K = rng.standard_normal((N + a, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        t_inc = oracle.build(K, N, ref, c, D, capacity=N + a, lib=lib)
        for _ in range(a):
            oracle.append_update(t_inc, K, ref, lib=lib)
        t_full = oracle.build(K, N + a, ref, c, D, lib=lib)
        for level in range(1, D + 1):
            mi, gi, bi = t_inc.level(level)
            mf, gf, bf = t_full.level(level)
            assert mi.shape == mf.shape
            assert np.max(np.abs(mi - mf)) <= 1e-12 and np.max(np.abs(gi - gf)) <= 1e-12


def pin_golden_geometry(lib):
    """Geometry facts stated by the pages (tests/golden/tree_geometry.txt):
    tokens covered by one top node, checked through the subtree closed form
    on a cache spanning several top nodes."""
    rows = []
    with open(os.path.join(GOLDEN, "tree_geometry.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                c, D, span = (int(x) for x in line.split()[:3])
                rows.append((c, D, span))
    assert rows
    rng = _rng(1300)
    for c, D, span in rows:
        N = 2 * span + 5
        d = 4
        K = (rng.standard_normal((N, d)) * 0.5).astype(np.float32)
        ref = rng.standard_normal((1, d))
        tree = oracle.build(K, N, ref, c, D, lib=lib)
        m, g, b = tree.level(D)
        assert m.shape[0] == 3
        s = K.astype(np.float64) @ ref[0] / math.sqrt(d)
        assert abs(m[0, 0] - logsumexp(s[:span])) <= 1e-10 * abs(m[0, 0])
        assert abs(m[1, 0] - logsumexp(s[span:2 * span])) <= 1e-10 * abs(m[1, 0])
        assert abs(m[2, 0] - logsumexp(s[2 * span:])) <= 1e-10 * max(1.0, abs(m[2, 0]))


def pin_node_summary_subtree(lib):
    """orc_node_summary, which recomputes one node from its own subtree's raw
    keys, equals the log-sum-exp and softmax-weighted mean key of r_j.k/sqrt(d)
    over exactly that subtree (ragged tails included), its plane offset is the
    tangent plane's value at q = 0, and it equals the row the whole-tree build
    stores for the same node."""
    for case_i, (N, c, D, R, d) in enumerate(_tree_cases()):
        rng = _rng(1400 + case_i)
        K = rng.standard_normal((N, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        K64 = K.astype(np.float64)
        tree = oracle.build(K, N, ref, c, D, lib=lib)
        for level in range(1, D + 1):
            n_l = -(-N // c ** level)
            tm, tg, tb = tree.level(level)
            assert tm.shape[0] == n_l
            for n in range(n_l):
                m, g, b = oracle.node_summary(K, N, ref, c, level, n, lib=lib)
                t0, t1 = _subtree(N, c, level, n)
                for j in range(R):
                    s = K64[t0:t1] @ ref[j] / math.sqrt(d)
                    m_ref = logsumexp(s)
                    g_ref = softmax(s) @ K64[t0:t1]
                    # tangent plane of lse(q.k/sqrt(d)) at r_j, evaluated at q = 0
                    b_ref = m_ref - ref[j] @ g_ref / math.sqrt(d)
                    assert abs(m[j] - m_ref) <= 1e-10 * max(1.0, abs(m_ref)), (case_i, level, n, j)
                    assert np.max(np.abs(g[j] - g_ref)) <= 1e-10 * max(1.0, np.max(np.abs(g_ref))), (level, n, j)
                    assert abs(b[j] - b_ref) <= 1e-10 * max(1.0, abs(m_ref), abs(b_ref)), (level, n, j)
                assert np.max(np.abs(m - tm[n])) <= 1e-12 * max(1.0, np.max(np.abs(m)))
                assert np.max(np.abs(g - tg[n])) <= 1e-12 * max(1.0, np.max(np.abs(g)))


def pin_estimate_many_rows(lib):
    """The batch estimate of listed node ids of one level (rows offset by the
    level's first row) is, at q = r_j, the exact log mass of each listed
    node's subtree, and below it for any other q."""
    for case_i, (N, c, D, R, d) in enumerate(_tree_cases()):
        rng = _rng(1500 + case_i)
        K = rng.standard_normal((N, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        K64 = K.astype(np.float64)
        tree = oracle.build(K, N, ref, c, D, lib=lib)
        for level in range(1, D + 1):
            n_l = -(-N // c ** level)
            ids = rng.permutation(n_l)[: max(1, (2 * n_l) // 3)]
            exact_at = {}
            for j in range(R):
                est = oracle.estimate_many(tree.m, tree.g, int(tree.level_off[level - 1]), ids, ref, ref[j],
                                           lib=lib)
                for i, n in enumerate(ids):
                    t0, t1 = _subtree(N, c, level, int(n))
                    m_ref = logsumexp(K64[t0:t1] @ ref[j] / math.sqrt(d))
                    assert abs(est[i] - m_ref) <= 1e-10 * max(1.0, abs(m_ref)), (case_i, level, int(n), j)
            q = rng.standard_normal(d) * 1.5
            est = oracle.estimate_many(tree.m, tree.g, int(tree.level_off[level - 1]), ids, ref, q, lib=lib)
            for i, n in enumerate(ids):
                t0, t1 = _subtree(N, c, level, int(n))
                assert est[i] <= logsumexp(K64[t0:t1] @ q / math.sqrt(d)) + 1e-9, (case_i, level, int(n))


def pin_heads_drivers(lib):
    """The multi-head drivers (several KV heads in one strided store, G query
    heads per KV head) give, per KV head, the subtree closed form of every
    node of that head's own keys, and per query head, exactly the single-head
    decode with that head's own keys, values and reference queries; at p = 1
    every query head's output is dense softmax attention over its KV head."""
    rng = _rng(1600)
    H_kv, G, cap, N, c, D, R, d = 2, 2, 160, 151, 3, 3, 2, 8
    H_q = H_kv * G
    K = np.zeros((H_kv, cap, d), dtype=np.float32)
    V = np.zeros((H_kv, cap, d), dtype=np.float32)
    K[:, :N] = rng.standard_normal((H_kv, N, d))
    V[:, :N] = rng.standard_normal((H_kv, N, d))
    K[:, N:] = 7.0  # rows past N must never be read
    V[:, N:] = -7.0
    ref = rng.standard_normal((H_kv, R, d))
    ht = oracle.build_heads(K, N, ref, c, D, capacity=cap, lib=lib)
    for kh in range(H_kv):
        K64 = K[kh, :N].astype(np.float64)
        tree = ht.head(kh)
        single = oracle.build(K[kh], N, ref[kh], c, D, capacity=cap, lib=lib)
        for level in range(1, D + 1):
            m, g, b = tree.level(level)
            sm, sg, sb = single.level(level)
            assert np.array_equal(m, sm) and np.array_equal(g, sg) and np.array_equal(b, sb), (kh, level)
            for n in range(m.shape[0]):
                t0, t1 = _subtree(N, c, level, n)
                for j in range(R):
                    s = K64[t0:t1] @ ref[kh, j] / math.sqrt(d)
                    assert abs(m[n, j] - logsumexp(s)) <= 1e-10 * max(1.0, abs(m[n, j])), (kh, level, n, j)
                    b_ref = logsumexp(s) - ref[kh, j] @ (softmax(s) @ K64[t0:t1]) / math.sqrt(d)
                    assert abs(b[n, j] - b_ref) <= 1e-10 * max(1.0, abs(b_ref), abs(m[n, j])), (kh, level, n, j)
    for p in (0.5, 0.8, 1.0):
        Q = rng.standard_normal((H_q, d)) * 2.0
        out, leaves, vis = oracle.decode_heads(K, V, ht, ref, Q, p, lib=lib)
        for h in range(H_q):
            kh = h // G
            o1, l1, v1 = oracle.decode_one(K[kh], V[kh], ht.head(kh), ref[kh], Q[h], p, lib=lib)
            assert np.array_equal(out[h], o1) and list(leaves[h]) == list(l1) and int(vis[h]) == v1, (p, h)
            if p >= 1.0:
                w = softmax(K[kh, :N].astype(np.float64) @ Q[h] / math.sqrt(d))
                assert np.max(np.abs(out[h] - w @ V[kh, :N].astype(np.float64))) <= 1e-12, h


def pin_depth_growth(lib):
    """A tree whose depth grows with the context: the depth is the least one
    (from the given minimum) whose top level holds at most c nodes -- chunk
    4 and 6 levels cover 4,096 tokens per top node, so 16,384 tokens fit
    depth 6 and one more token needs depth 7 -- and appending tokens across
    a growth step gives exactly the tree built over all of them, whose new
    top level holds the log mass of its whole subtree (closed form)."""
    assert oracle.depth_for(16384, 4, 6, 8, lib=lib) == 6
    assert oracle.depth_for(16385, 4, 6, 8, lib=lib) == 7
    assert oracle.depth_for(16385, 4, 6, 0, lib=lib) == 6      # no growth without room
    assert oracle.depth_for(4 ** 9, 4, 6, 8, lib=lib) == 8      # capped at the maximum
    rng = _rng(1700)
    # the first case grows at its last append (nothing after it rebuilds the new level)
    for (N, a, c, D0, Dm, R, d) in [(16, 1, 4, 1, 3, 2, 4), (16, 3, 4, 1, 3, 2, 4), (60, 8, 2, 2, 6, 1, 4),
                                    (250, 10, 4, 2, 4, 3, 6)]:
        K = rng.standard_normal((N + a, d)).astype(np.float32)
        ref = rng.standard_normal((R, d))
        t_inc = oracle.build(K, N, ref, c, D0, capacity=N + a, max_depth=Dm, lib=lib)
        D_start = t_inc.D
        for _ in range(a):
            oracle.append_update(t_inc, K, ref, lib=lib)
        t_full = oracle.build(K, N + a, ref, c, D0, max_depth=Dm, lib=lib)
        assert t_inc.D == t_full.D > D_start, (N, a, D_start, t_inc.D, t_full.D)
        K64 = K.astype(np.float64)
        for level in range(1, t_full.D + 1):
            mi, gi, bi = t_inc.level(level)
            mf, gf, bf = t_full.level(level)
            assert mi.shape == mf.shape
            assert np.max(np.abs(mi - mf)) <= 1e-12 and np.max(np.abs(gi - gf)) <= 1e-12, (N, level)
        mt, gt, bt = t_inc.level(t_inc.D)
        for n in range(mt.shape[0]):
            t0, t1 = _subtree(N + a, c, t_inc.D, n)
            for j in range(R):
                m_ref = logsumexp(K64[t0:t1] @ ref[j] / math.sqrt(d))
                assert abs(mt[n, j] - m_ref) <= 1e-10 * max(1.0, abs(m_ref)), (N, n, j)
        # routing over a grown tree starts at its new top level
        kept, visited = oracle.route(t_inc, ref, rng.standard_normal(d), 1.0, lib=lib)
        assert visited == sum(-(-(N + a) // c ** l) for l in range(1, t_inc.D + 1))


ALL_PINS = [pin_closed_form_subtree, pin_lower_bound_and_tangent, pin_single_plane_affine,
            pin_exact_leaves_token_topp, pin_dense_at_p1, pin_flat_chunk_topp, pin_routing_invariants,
            pin_ties_lower_id, pin_topp_brute_force, pin_attention_and_sink, pin_bf16_widening,
            pin_append_equivalence, pin_golden_geometry, pin_node_summary_subtree, pin_estimate_many_rows,
            pin_heads_drivers, pin_depth_growth]
