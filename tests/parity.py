"""GPU-vs-oracle comparison protocol, shared by the GPU tests and the smoke check.

Build parity: every stored (m, g, b) of every node agrees with the oracle's
fp64 tree within a relative 1e-5: m relative to max(1, |m|), each g row
relative to max(1, max|g|), and b = m - r.g/sqrt(d) relative to the larger of
its two terms (the subtraction cancels, so fp32 rounding of m shows in b at
the scale of m).

Routing parity (replay): the GPU writes its kept node ids per level and query
head (the trace).  For each head the oracle walks the GPU's own path: at each
level it scores the GPU's frontier in fp64, takes its own top-p cut, and
checks that every node on which the two kept sets differ is ambiguous -- its
oracle probability within 1e-5 of the probability at the cut, or the oracle's
cumulative mass just before or after it within 1e-5 of p.  The next frontier
is the children of the GPU's kept nodes, so one borderline node does not
derail the levels below.  Ambiguous nodes are counted and reported.

Output parity: the oracle's exact attention over the GPU's own token set
(kept leaves plus the sink) matches the GPU output within the dtype's
tolerance; when no level had an ambiguous node the token sets are the
oracle's own, so this is also parity with the oracle's full decode.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

AMBIG = 1e-5
OUT_TOL = {"f32": 1e-5, "bf16": 2e-3}
BUILD_RTOL = 1e-5


def level_count(n_tokens: int, c: int, level: int) -> int:
    return -(-n_tokens // c ** level)


def oracle_trees(K_cpu, ref_cpu, n_tokens: int, c: int, D: int, capacity: int | None = None):
    """One fp64 oracle tree per KV head (K_cpu [H_kv, cap, d] on the host)."""
    return [oracle.build(K_cpu[kh], n_tokens, ref_cpu[kh], c, D, capacity=capacity)
            for kh in range(K_cpu.shape[0])]


def check_build(cache, trees, rtol: float = BUILD_RTOL, levels=None, sample=None, seed=0):
    """Compare the GPU summary store with the oracle trees; returns the worst
    relative errors (m, g, b).  `sample` limits the checked nodes per level."""
    cfg = cache.cfg
    worst = [0.0, 0.0, 0.0]
    rng = np.random.default_rng(seed)
    for level in (levels or range(1, cfg.D + 1)):
        g, b, m = cache.summaries(level)
        n = m.shape[1]
        ids = np.arange(n) if sample is None or n <= sample else np.sort(rng.choice(n, sample, replace=False))
        idt = torch.as_tensor(ids, device=g.device)
        g = g[:, idt].double().cpu().numpy()
        b = b[:, idt].double().cpu().numpy()
        m = m[:, idt].double().cpu().numpy()
        for kh, tree in enumerate(trees):
            mo, go, bo = tree.level(level)
            assert mo.shape[0] == n, (level, mo.shape, n)
            mo, go, bo = mo[ids], go[ids], bo[ids]
            em = np.abs(m[kh] - mo) / np.maximum(1.0, np.abs(mo))
            # b = m - r.g/sqrt(d) cancels: its fp32 error scales with |m| and |r.g|/sqrt(d)
            eb = np.abs(b[kh] - bo) / np.maximum(1.0, np.maximum(np.abs(mo), np.abs(mo - bo)))
            scale_g = np.maximum(1.0, np.abs(go).max(axis=-1, keepdims=True))
            eg = np.abs(g[kh] - go) / scale_g
            worst = [max(worst[0], float(em.max())), max(worst[1], float(eg.max())), max(worst[2], float(eb.max()))]
            assert em.max() <= rtol, ("m", level, kh, float(em.max()))
            assert eg.max() <= rtol, ("g", level, kh, float(eg.max()))
            assert eb.max() <= rtol, ("b", level, kh, float(eb.max()))
    return worst


def replay_head(tree, ref_kh, q_h, p: float, trace_ids, trace_cnt, h: int, n_tokens: int, c: int, D: int):
    """Replay one query head's routing.  Returns (ambiguous count, visited,
    GPU leaves)."""
    amb = 0
    visited = 0
    front = np.arange(level_count(n_tokens, c, D), dtype=np.int64)
    gpu_leaves = None
    for level in range(D, 0, -1):
        cnt = int(trace_cnt[level - 1, h])
        gk = trace_ids[level - 1, h, :cnt].astype(np.int64)
        assert np.all(np.diff(gk) > 0), ("kept ids not ascending", level)
        fset = set(front.tolist())
        assert set(gk.tolist()) <= fset, ("kept node outside the frontier", level)
        est = tree.estimates(level, front, ref_kh, q_h)
        kept_o, prob, cb, rank = oracle.topp(est, front, p)
        ok_set = set(front[kept_o].tolist())
        diff = ok_set ^ set(gk.tolist())
        if diff:
            last = int(np.argmax(np.where(kept_o, rank, -1)))
            p_cut = prob[last]
            pos = {int(n): i for i, n in enumerate(front)}
            for n in diff:
                i = pos[n]
                near = (abs(prob[i] - p_cut) <= AMBIG or abs(cb[i] - p) <= AMBIG or abs(cb[i] + prob[i] - p) <= AMBIG)
                assert near, ("routing differs on a non-ambiguous node", level, n, prob[i], p_cut, cb[i], p)
            amb += len(diff)
        visited += len(front)
        if level == 1:
            gpu_leaves = gk
        else:
            nb = level_count(n_tokens, c, level - 1)
            ch = (gk[:, None] * c + np.arange(c)[None, :]).reshape(-1)
            front = ch[ch < nb]
    return amb, visited, gpu_leaves


def check_decode(res, trees, K_cpu, V_cpu, ref_cpu, q_cpu, p: float, n_tokens: int, c: int, D: int, G: int,
                 kv_dtype: str, heads=None):
    """Full protocol for one decode call; returns the ambiguous-node count."""
    tid = res["trace_ids"].cpu().numpy()
    tcnt = res["trace_counts"].cpu().numpy()
    out = res["out"].double().cpu().numpy()
    n_leaf = res["n_leaf"].cpu().numpy()
    leaf_idx = res["leaf_idx"].cpu().numpy()
    visited = res["visited"].cpu().numpy()
    h_q = out.shape[0]
    amb_total = 0
    for h in (heads if heads is not None else range(h_q)):
        kh = h // G
        amb, vis, leaves = replay_head(trees[kh], ref_cpu[kh], q_cpu[h], p, tid, tcnt, h, n_tokens, c, D)
        amb_total += amb
        assert int(visited[h]) == vis, ("nodes visited", h, int(visited[h]), vis)
        assert int(n_leaf[h]) == len(leaves), ("leaf count", h)
        assert np.array_equal(leaf_idx[h, :len(leaves)].astype(np.int64), leaves), ("leaf ids", h)
        toks = oracle.token_set(leaves, n_tokens, c)
        ref_out = oracle.attend(K_cpu[kh], V_cpu[kh], toks, q_cpu[h])
        err = float(np.max(np.abs(out[h] - ref_out)))
        assert err <= OUT_TOL[kv_dtype], ("output", h, err)
    return amb_total
