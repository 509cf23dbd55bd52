"""CUDA path vs the fp64 oracle at the full sizes of the benchmark workloads,
in the launch configuration the benchmark times (needs a B200).

Build parity is checked on sampled nodes of every level.  Decode parity
replays the GPU's routing trace of one decode step per workload against the
oracle (every query head for the 256K and 1M workloads; the four query heads
of KV head 0 for the 10M one, whose oracle estimates are computed node by node
from the raw keys instead of a stored tree) and checks the outputs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_build, check_decode

import tree_indexed_sparse_b200 as zha

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


class LazyTree:
    """Oracle estimates of any node, from its subtree's raw keys."""

    def __init__(self, K, n_tokens, c, D):
        self.K, self.n_tokens, self.c, self.D = K, n_tokens, c, D

    def estimates(self, l, ids, ref, q):
        out = np.empty(len(ids))
        for i, n in enumerate(ids):
            m, g, _ = oracle.node_summary(self.K, self.n_tokens, ref, self.c, l, int(n))
            out[i] = oracle.estimate(m, g, ref, q)
        return out


def _gpu_cache(w, inp):
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity)
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    return cache


@pytest.mark.parametrize("name", ["wide_256k", "deep_256k", "light_1m"])
def test_fullsize_parity(name):
    w = W[name]
    inp = workloads.generate(w, "cuda")
    cache = _gpu_cache(w, inp)
    K_cpu, V_cpu, ref_cpu = inp.K.cpu(), inp.V.cpu(), inp.ref.cpu()
    trees = [oracle.build(K_cpu[kh], w.n_tokens, ref_cpu[kh], w.c, w.D) for kh in range(w.h_kv)]
    worst = check_build(cache, trees, sample=64)
    print(f"{name}: build worst relative error m={worst[0]:.2e} g={worst[1]:.2e} b={worst[2]:.2e}")
    trace_cap = oracle.level_nodes(w.n_tokens, w.c, 1)
    res = cache.decode(inp.Q[0], w.p, trace_cap=trace_cap)
    torch.cuda.synchronize()
    assert cache.status() == zha.ZHA_OK
    amb = check_decode(res, trees, K_cpu, V_cpu, ref_cpu, inp.Q[0].cpu(), w.p, w.n_tokens, w.c, w.D, w.group,
                       w.kv_dtype)
    print(f"{name}: one decode step, {w.h_q} heads, ambiguous nodes {amb}")


def test_fullsize_parity_10m():
    w = W["extreme_10m"]
    inp = workloads.generate(w, "cuda")
    cache = _gpu_cache(w, inp)
    K0 = inp.K[0].cpu()
    V0 = inp.V[0].cpu()
    ref0 = inp.ref[0].cpu()
    # build parity: a few nodes of every level of KV head 0, from the raw keys
    rng = np.random.default_rng(0)
    for level in range(1, w.D + 1):
        g, b, m = cache.summaries(level)
        n = m.shape[1]
        for node in sorted(set(rng.integers(0, n, 3).tolist()) | {n - 1}):
            mo, go, bo = oracle.node_summary(K0, w.n_tokens, ref0, w.c, level, node)
            mg = m[0, node].double().cpu().numpy()
            gg = g[0, node].double().cpu().numpy()
            assert np.max(np.abs(mg - mo) / np.maximum(1.0, np.abs(mo))) <= 1e-5, ("m", level, node)
            assert np.max(np.abs(gg - go) / np.maximum(1.0, np.abs(go).max())) <= 1e-5, ("g", level, node)
    trace_cap = oracle.level_nodes(w.n_tokens, w.c, 1)
    res = cache.decode(inp.Q[0], w.p, trace_cap=trace_cap)
    torch.cuda.synchronize()
    assert cache.status() == zha.ZHA_OK
    tree0 = LazyTree(K0, w.n_tokens, w.c, w.D)
    K_cpu = [K0]
    V_cpu = [V0]
    amb = check_decode(res, [tree0], K_cpu, V_cpu, [ref0], inp.Q[0].cpu(), w.p, w.n_tokens, w.c, w.D, w.group,
                       w.kv_dtype, heads=range(w.group))
    print(f"extreme_10m: one decode step, KV head 0 ({w.group} heads), ambiguous nodes {amb}")
