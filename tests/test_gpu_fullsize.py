"""CUDA path vs the fp64 oracle at the full sizes of the benchmark workloads,
in the launch configuration the benchmark times (needs a B200).

Each workload runs its own schedule:
  * wide_256k, light_1m: decodes only; the first and the last query of the
    workload are replayed for every query head;
  * deep_256k: 128 steps of (two appends, one decode); four steps are
    replayed, and after the 256 appends every node they touched is checked;
  * extreme_10m: 64 decodes, then 1,024 appends, then one more decode; the
    first and last of the 64 and the decode after the appends are replayed
    for all 16 query heads, and every node the appends touched is checked;
  * light_1m's settings at 3M tokens, 13 queries in one batched decode (the
    leaf level's slices too large to come back on chip), all replayed.
The oracle side runs one KV head at a time (its tree, keys and values), so
the 10M case needs about 10 GB of host memory at once.  Build parity is
checked on sampled nodes of every level (always including the last, partial
node) plus the appended nodes.  Each replay appends its ambiguous-node count
to the parity log (see parity.py).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_build, check_decode, touched_nodes

import tree_indexed_sparse_b200 as zha

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def _gpu_cache(w, inp):
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity)
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    return cache


def _decode(cache, q, p, trace_cap):
    """One traced decode; host copies of its outputs."""
    res = cache.decode(q, p, trace_cap=trace_cap)
    torch.cuda.synchronize()
    assert cache.status() == zha.ZHA_OK
    return {k: v.cpu() for k, v in res.items()}


def _heads(kh, G):
    return range(kh * G, (kh + 1) * G)


@pytest.mark.parametrize("name", ["wide_256k", "light_1m"])
def test_fullsize_parity(name):
    w = W[name]
    inp = workloads.generate(w, "cuda")
    cache = _gpu_cache(w, inp)
    trace_cap = oracle.level_nodes(w.capacity, w.c, 1)
    steps = [0, w.steps - 1]
    res = {s: _decode(cache, inp.Q[s], w.p, trace_cap) for s in steps}
    K_cpu, V_cpu, ref_cpu = inp.K.cpu(), inp.V.cpu(), inp.ref.cpu()
    ht = oracle.build_heads(K_cpu, w.n_tokens, ref_cpu, w.c, w.D)
    trees = [ht.head(kh) for kh in range(w.h_kv)]
    worst = check_build(cache, trees, sample=64)
    print(f"{name}: build worst relative error m={worst[0]:.2e} g={worst[1]:.2e} b={worst[2]:.2e}")
    for s in steps:
        amb = check_decode(res[s], trees, K_cpu, V_cpu, ref_cpu, inp.Q[s].cpu(), w.p, w.n_tokens, w.c, w.D,
                           w.group, w.kv_dtype, case=f"{name} step {s}")
        print(f"{name}: step {s}, {w.h_q} heads, ambiguous nodes {amb}")


def test_fullsize_deep_schedule():
    """deep_256k with its own schedule: two appends before every decode."""
    w = W["deep_256k"]
    assert w.appends_per_step == 2
    inp = workloads.generate(w, "cuda")
    cache = _gpu_cache(w, inp)
    trace_cap = oracle.level_nodes(w.capacity, w.c, 1)
    checked = [0, 1, w.steps // 2, w.steps - 1]
    res = {}
    app = 0
    for s in range(w.steps):
        for _ in range(w.appends_per_step):
            cache.append(inp.K_app[app], inp.V_app[app])
            app += 1
        if s in checked:
            res[s] = _decode(cache, inp.Q[s], w.p, trace_cap)
        else:
            cache.decode(inp.Q[s], w.p)
    torch.cuda.synchronize()
    assert cache.status() == zha.ZHA_OK
    assert cache.n_tokens == w.n_tokens + w.total_appends
    # the appended rows are in the device cache now; the oracle replays the
    # schedule on its own tree, one KV head at a time
    G = w.group
    for kh in range(w.h_kv):
        K_h, V_h, ref_h = inp.K[kh].cpu(), inp.V[kh].cpu(), inp.ref[kh].cpu()
        tree = oracle.build(K_h, w.n_tokens, ref_h, w.c, w.D, capacity=w.capacity)
        n = w.n_tokens
        for s in range(w.steps):
            for _ in range(w.appends_per_step):
                oracle.append_update(tree, K_h, ref_h)
                n += 1
            if s in checked:
                amb = check_decode(res[s], {kh: tree}, {kh: K_h}, {kh: V_h}, {kh: ref_h}, inp.Q[s].cpu(), w.p, n,
                                   w.c, w.D, G, w.kv_dtype, heads=_heads(kh, G),
                                   case=f"deep_256k step {s} kv head {kh}")
                print(f"deep_256k: step {s} (after {n - w.n_tokens} appends), KV head {kh}, ambiguous {amb}")
        check_build(cache, [tree], heads=[kh], ids=touched_nodes(w.n_tokens, n, w.c, w.D))
        check_build(cache, [tree], heads=[kh], sample=64, seed=kh)


def test_fullsize_extreme_10m():
    """extreme_10m with its own schedule: 64 decodes, then 1,024 appends."""
    w = W["extreme_10m"]
    assert w.appends_after == 1024 and w.appends_per_step == 0
    inp = workloads.generate(w, "cuda")
    cache = _gpu_cache(w, inp)
    trace_cap = oracle.level_nodes(w.capacity, w.c, 1)
    checked = [0, w.steps - 1]
    res = {}
    for s in range(w.steps):
        if s in checked:
            res[s] = _decode(cache, inp.Q[s], w.p, trace_cap)
        else:
            cache.decode(inp.Q[s], w.p)
    for i in range(w.appends_after):
        cache.append(inp.K_app[i], inp.V_app[i])
    res["after"] = _decode(cache, inp.Q[0], w.p, trace_cap)
    n_end = w.n_tokens + w.appends_after
    assert cache.n_tokens == n_end
    G = w.group
    for kh in range(w.h_kv):
        K_h, V_h, ref_h = inp.K[kh].cpu(), inp.V[kh].cpu(), inp.ref[kh].cpu()
        tree = oracle.build(K_h, w.n_tokens, ref_h, w.c, w.D, capacity=w.capacity)
        one = ({kh: tree}, {kh: K_h}, {kh: V_h}, {kh: ref_h})
        for s in checked:
            amb = check_decode(res[s], *one, inp.Q[s].cpu(), w.p, w.n_tokens, w.c, w.D, G, w.kv_dtype,
                               heads=_heads(kh, G), case=f"extreme_10m step {s} kv head {kh}")
            print(f"extreme_10m: step {s}, KV head {kh}, ambiguous nodes {amb}")
        for _ in range(w.appends_after):
            oracle.append_update(tree, K_h, ref_h)
        assert tree.n_tokens == n_end
        check_build(cache, [tree], heads=[kh], ids=touched_nodes(w.n_tokens, n_end, w.c, w.D))
        check_build(cache, [tree], heads=[kh], sample=256, seed=kh)
        amb = check_decode(res["after"], *one, inp.Q[0].cpu(), w.p, n_end, w.c, w.D, G, w.kv_dtype,
                           heads=_heads(kh, G), case=f"extreme_10m after appends kv head {kh}")
        print(f"extreme_10m: after {w.appends_after} appends, KV head {kh}, ambiguous nodes {amb}")
        del tree, K_h, V_h


def test_batch_with_spilled_leaf_slices():
    """13 queries of the 1M light workload's settings, at 3M tokens, in one
    zha_decode_batch: 52 virtual KV heads, so teams of two CTAs, whose leaf
    level slices (12K-60K slots each by the oracle's routing of these
    queries, beyond the 7,808 that come back on chip) stay in global memory
    and run the chunked histogram and classification passes.  Every query's routing and
    output are replayed against the oracle for all 16 query heads."""
    from parity import oracle_trees

    n_q = 13
    w = W["light_1m"].scaled(3_000_000, steps=n_q)
    inp = workloads.generate(w, "cuda")
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, max_batch=n_q)
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    cap = oracle.level_nodes(w.capacity, w.c, 1)
    qs = inp.Q[:n_q].contiguous()
    res = cache.decode_batch(qs, w.p, trace_cap=cap)
    torch.cuda.synchronize()
    assert cache.status() == zha.ZHA_OK
    res = {k: v.cpu() for k, v in res.items()}
    K_cpu, V_cpu, ref_cpu = inp.K.cpu(), inp.V.cpu(), inp.ref.cpu()
    del inp, cache
    torch.cuda.empty_cache()
    trees = oracle_trees(K_cpu, ref_cpu, w.n_tokens, w.c, w.D, capacity=w.capacity)
    h_q = w.h_q
    qs = qs.cpu()
    for t in range(n_q):
        res_t = {"out": res["out"][t], "leaf_idx": res["leaf_idx"][t], "n_leaf": res["n_leaf"][t],
                 "visited": res["visited"][t], "trace_ids": res["trace_ids"][:, t * h_q:(t + 1) * h_q],
                 "trace_counts": res["trace_counts"][:, t * h_q:(t + 1) * h_q]}
        check_decode(res_t, trees, K_cpu, V_cpu, ref_cpu, qs[t].double().numpy(), w.p, w.n_tokens, w.c, w.D,
                     w.group, w.kv_dtype, case=f"light settings at 3M, batch of {n_q}, query {t}")
