"""GPU-vs-oracle comparison protocol, shared by the GPU tests and the smoke check.

Build parity: every stored (m, g, b) of every node agrees with the oracle's
fp64 tree within a relative 1e-5: m relative to max(1, |m|), each g row
relative to max(1, max|g|), and b = m - r.g/sqrt(d) relative to the larger of
its two terms (the subtraction cancels, so fp32 rounding of m shows in b at
the scale of m).

Routing parity (replay): the GPU writes its kept node ids per level and query
head (the trace).  For each head the oracle walks the GPU's own path: at each
level it scores the GPU's frontier in fp64, takes its own top-p cut, and
checks that every node on which the two kept sets differ is ambiguous: its
oracle probability within a relative 1e-5 of the probability at the cut
(|P_i - P_cut| <= 1e-5 max(P_i, P_cut); the band scales with the
probabilities, so it does not swallow a whole level of tiny ones), or the
oracle's cumulative mass just before or after it within 1e-5 of p.  The next
frontier is the children of the GPU's kept nodes, so one borderline node does
not derail the levels below.  Ambiguous nodes are counted, bounded (at most
AMB_FRAC of the kept nodes compared, so none on the small cases) and
appended, one JSON line per check, to the parity log (ZHA_PARITY_LOG, by
default gpurun_out/parity_counts.jsonl at the repository root).

Output parity: the oracle's exact attention over the GPU's own token set
(kept leaves plus the sink) matches the GPU output within the dtype's
tolerance; when no level had an ambiguous node the token sets are the
oracle's own, so this is also parity with the oracle's full decode.
"""
from __future__ import annotations

import json
import os
import time

import numpy as np
import torch

import oracle

AMBIG_REL = 1e-5        # relative band on the probability at the cut
AMBIG_CUM = 1e-5        # band on the cumulative mass around p
AMB_FRAC = 1e-4         # most ambiguous nodes allowed per kept node compared
OUT_TOL = {"f32": 1e-5, "bf16": 2e-3}
BUILD_RTOL = 1e-5


def level_count(n_tokens: int, c: int, level: int) -> int:
    return -(-n_tokens // c ** level)


def oracle_trees(K_cpu, ref_cpu, n_tokens: int, c: int, D: int, capacity: int | None = None):
    """One fp64 oracle tree per KV head (K_cpu [H_kv, cap, d] on the host)."""
    return [oracle.build(K_cpu[kh], n_tokens, ref_cpu[kh], c, D, capacity=capacity)
            for kh in range(K_cpu.shape[0])]


def touched_nodes(t0: int, t1: int, c: int, D: int) -> dict:
    """Node ids of every level whose subtree holds a token of [t0, t1)."""
    return {lv: np.arange(t0 // c ** lv, (t1 - 1) // c ** lv + 1) for lv in range(1, D + 1)}


def check_build(cache, trees, rtol: float = BUILD_RTOL, levels=None, sample=None, seed=0, ids=None,
                heads=None):
    """Compare the GPU summary store with the oracle trees; returns the worst
    relative errors (m, g, b).  `sample` limits the checked nodes per level
    (the last, possibly partial, node is always among them); `ids` (level ->
    node ids) checks exactly those nodes instead; `heads` lists the KV heads
    that `trees` holds, in order (default: all)."""
    cfg = cache.cfg
    worst = [0.0, 0.0, 0.0]
    rng = np.random.default_rng(seed)
    heads = list(range(cfg.h_kv)) if heads is None else list(heads)
    for level in (levels or (sorted(ids) if ids is not None else range(1, cache.depth + 1))):
        g, b, m = cache.summaries(level)
        n = m.shape[1]
        if ids is not None:
            sel = np.asarray(ids[level], dtype=np.int64)
        elif sample is None or n <= sample:
            sel = np.arange(n)
        else:
            sel = np.union1d(rng.choice(n, sample, replace=False), [n - 1])
        ids_l = sel
        idt = torch.as_tensor(ids_l, device=g.device)
        for i, tree in enumerate(trees):
            kh = heads[i]
            gi = g[kh].index_select(0, idt).double().cpu().numpy()
            bi = b[kh].index_select(0, idt).double().cpu().numpy()
            mi = m[kh].index_select(0, idt).double().cpu().numpy()
            mo, go, bo = tree.level(level)
            assert mo.shape[0] == n, (level, mo.shape, n)
            mo, go, bo = mo[ids_l], go[ids_l], bo[ids_l]
            em = np.abs(mi - mo) / np.maximum(1.0, np.abs(mo))
            # b = m - r.g/sqrt(d) cancels: its fp32 error scales with |m| and |r.g|/sqrt(d)
            eb = np.abs(bi - bo) / np.maximum(1.0, np.maximum(np.abs(mo), np.abs(mo - bo)))
            scale_g = np.maximum(1.0, np.abs(go).max(axis=-1, keepdims=True))
            eg = np.abs(gi - go) / scale_g
            worst = [max(worst[0], float(em.max())), max(worst[1], float(eg.max())), max(worst[2], float(eb.max()))]
            assert em.max() <= rtol, ("m", level, kh, float(em.max()))
            assert eg.max() <= rtol, ("g", level, kh, float(eg.max()))
            assert eb.max() <= rtol, ("b", level, kh, float(eb.max()))
    return worst


def router_trees(cache):
    """Oracle trees over the GPU's bf16 router copy (router_dtype ZHA_BF16):
    per KV head, every present level's m (the GPU's fp32 m) and g~ (the
    bf16 copy, widened exactly) as an oracle summary store, so that the
    oracle routes over the same quantised summaries as the GPU."""
    cfg = cache.cfg
    D = cache.depth
    n = cache.n_tokens
    counts = [level_count(n, cfg.c, lv) for lv in range(1, D + 1)]
    off = np.zeros(D, dtype=np.int64)
    off[1:] = np.cumsum(counts)[:-1]
    trees = []
    for kh in range(cfg.h_kv):
        ms, gs, bs = [], [], []
        for lv in range(1, D + 1):
            g16, b16 = cache.router_summaries(lv)
            _, _, m = cache.summaries(lv)
            ms.append(m[kh].double().cpu().numpy())
            gs.append(g16[kh].double().cpu().numpy())
            bs.append(b16[kh].double().cpu().numpy())
        trees.append(oracle.Tree(np.ascontiguousarray(np.concatenate(ms)), np.ascontiguousarray(np.concatenate(gs)),
                                 np.ascontiguousarray(np.concatenate(bs)), off, n, cfg.c, D))
    return trees


def check_router_copy(cache, trees, ref_cpu, rtol: float = BUILD_RTOL):
    """The bf16 router copy against the oracle's exact summaries: every g~
    element is the exact g_j rounded to bf16 (within one bf16 step of it,
    plus the fp32 tolerance), and every plane offset is m_j - r_j.g~_j/sqrt(d)
    recomputed in fp64 from the GPU's own g~ and the oracle's m_j."""
    cfg = cache.cfg
    for lv in range(1, cache.depth + 1):
        g16, b16 = cache.router_summaries(lv)
        for kh, tree in enumerate(trees):
            mo, go, _ = tree.level(lv)
            gq = g16[kh].double().cpu().numpy()
            bq = b16[kh].double().cpu().numpy()
            scale_g = np.maximum(1.0, np.abs(go).max(axis=-1, keepdims=True))
            err = np.abs(gq - go) - 2.0 ** -8 * np.abs(go)
            assert np.max(err / scale_g) <= 2 * rtol, ("router g", lv, kh, float(np.max(err / scale_g)))
            r = np.asarray(ref_cpu[kh], dtype=np.float64)
            b_ref = mo - np.einsum("nrd,rd->nr", gq, r) / np.sqrt(cfg.d)
            eb = np.abs(bq - b_ref) / np.maximum(1.0, np.maximum(np.abs(mo), np.abs(mo - b_ref)))
            assert eb.max() <= rtol, ("router b", lv, kh, float(eb.max()))


def parity_log_path() -> str:
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    return os.environ.get("ZHA_PARITY_LOG") or os.path.join(root, "gpurun_out", "parity_counts.jsonl")


def record(case: str, **fields) -> None:
    """Append one JSON line about a parity check to the parity log."""
    path = parity_log_path()
    try:
        os.makedirs(os.path.dirname(path), exist_ok=True)
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, "time": time.time(), **fields}) + "\n")
    except OSError:
        pass


def amb_bound(kept: int) -> int:
    """Ambiguous nodes allowed when `kept` kept nodes were compared."""
    return int(AMB_FRAC * kept)


def replay_head(tree, ref_kh, q_h, p: float, trace_ids, trace_cnt, h: int, n_tokens: int, c: int, D: int,
                stats=None):
    """Replay one query head's routing.  Returns (ambiguous count, visited,
    GPU leaves); `stats` (a dict) accumulates the kept nodes compared."""
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
                near = (abs(prob[i] - p_cut) <= AMBIG_REL * max(prob[i], p_cut) or abs(cb[i] - p) <= AMBIG_CUM
                        or abs(cb[i] + prob[i] - p) <= AMBIG_CUM)
                assert near, ("routing differs on a non-ambiguous node", level, n, prob[i], p_cut, cb[i], p)
            amb += len(diff)
        if stats is not None:
            stats["kept"] = stats.get("kept", 0) + len(ok_set)
        visited += len(front)
        if level == 1:
            gpu_leaves = gk
        else:
            nb = level_count(n_tokens, c, level - 1)
            ch = (gk[:, None] * c + np.arange(c)[None, :]).reshape(-1)
            front = ch[ch < nb]
    return amb, visited, gpu_leaves


def check_decode(res, trees, K_cpu, V_cpu, ref_cpu, q_cpu, p: float, n_tokens: int, c: int, D: int, G: int,
                 kv_dtype: str, heads=None, case: str | None = None):
    """Full protocol for one decode call; returns the ambiguous-node count,
    after checking it against amb_bound and, when `case` names the check,
    recording it in the parity log."""
    tid = res["trace_ids"].cpu().numpy()
    tcnt = res["trace_counts"].cpu().numpy()
    out = res["out"].double().cpu().numpy()
    n_leaf = res["n_leaf"].cpu().numpy()
    leaf_idx = res["leaf_idx"].cpu().numpy()
    visited = res["visited"].cpu().numpy()
    h_q = out.shape[0]
    amb_total = 0
    stats = {}
    worst = 0.0
    checked = list(heads if heads is not None else range(h_q))
    for h in checked:
        kh = h // G
        amb, vis, leaves = replay_head(trees[kh], ref_cpu[kh], q_cpu[h], p, tid, tcnt, h, n_tokens, c, D, stats)
        amb_total += amb
        assert int(visited[h]) == vis, ("nodes visited", h, int(visited[h]), vis)
        assert int(n_leaf[h]) == len(leaves), ("leaf count", h)
        assert np.array_equal(leaf_idx[h, :len(leaves)].astype(np.int64), leaves), ("leaf ids", h)
        toks = oracle.token_set(leaves, n_tokens, c)
        ref_out = oracle.attend(K_cpu[kh], V_cpu[kh], toks, q_cpu[h])
        err = float(np.max(np.abs(out[h] - ref_out)))
        worst = max(worst, err)
        assert err <= OUT_TOL[kv_dtype], ("output", h, err)
    kept = stats.get("kept", 0)
    if case is not None:
        record(case, heads=len(checked), kept_compared=kept, ambiguous=amb_total, bound=amb_bound(kept),
               max_abs_err=worst, n_tokens=int(n_tokens))
    assert amb_total <= amb_bound(kept), ("ambiguous nodes over the bound", amb_total, kept)
    return amb_total
