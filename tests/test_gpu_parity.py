"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Cases are the tiny fp32 workload at its own size (all 64 queries) and the
other workloads' structures at sizes the oracle finishes in seconds (several
top nodes, ragged tails); the full-size workloads are in test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import OUT_TOL, check_build, check_decode, oracle_trees

import tree_indexed_sparse_b200 as zha

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS
CASES = {
    "tiny_f32": W["tiny_f32_16k"],  # the tiny workload itself: 16,384 tokens, all 64 queries
    "wide": W["wide_256k"].scaled(16384 + 100, steps=3),
    "deep": W["deep_256k"].scaled(16384 + 37, steps=3),
    "light": W["light_1m"].scaled(300000 + 5, steps=3),
}


class Case:
    def __init__(self, w):
        self.w = w
        self.inp = workloads.generate(w, "cpu")
        self.K = self.inp.K.clone()          # host copy that also receives appended rows
        self.V = self.inp.V.clone()
        self.dK = self.inp.K.cuda()
        self.dV = self.inp.V.cuda()
        self.dref = self.inp.ref.cuda()
        dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
        self.cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity)
        self.cache.build(self.dK, self.dV, w.n_tokens, self.dref)
        self.trees = oracle_trees(self.K, self.inp.ref, w.n_tokens, w.c, w.D, capacity=w.capacity)
        self.n = w.n_tokens

    def append(self, i):
        w = self.w
        k = self.inp.K_app[i].cuda()
        v = self.inp.V_app[i].cuda()
        self.cache.append(k, v)
        self.K[:, self.n] = self.inp.K_app[i]
        self.V[:, self.n] = self.inp.V_app[i]
        for kh in range(w.h_kv):
            oracle.append_update(self.trees[kh], self.K[kh], self.inp.ref[kh])
        self.n += 1


_cases = {}


def get_case(name):
    if name not in _cases:
        _cases[name] = Case(CASES[name])
    return _cases[name]


@pytest.mark.parametrize("name", list(CASES))
def test_build_parity(name):
    c = get_case(name)
    worst = check_build(c.cache, c.trees)
    print(f"{name}: worst relative error m={worst[0]:.2e} g={worst[1]:.2e} b={worst[2]:.2e}")
    assert c.cache.status() == 0


@pytest.mark.parametrize("name", list(CASES))
def test_decode_parity(name):
    c = get_case(name)
    w = c.w
    trace_cap = oracle.level_nodes(w.capacity, w.c, 1)
    amb = 0
    app = 0
    for s in range(w.steps):
        for _ in range(w.appends_per_step):
            c.append(app)
            app += 1
        q = c.inp.Q[s]
        res = c.cache.decode(q.cuda(), w.p, trace_cap=trace_cap)
        torch.cuda.synchronize()
        assert c.cache.status() == 0
        amb += check_decode(res, c.trees, c.K, c.V, c.inp.ref, q.double().numpy(), w.p, c.n, w.c, w.D, w.group,
                            w.kv_dtype, case=f"{name} step {s}")
    print(f"{name}: {w.steps} steps, ambiguous nodes {amb}")


@pytest.mark.parametrize("name", list(CASES))
def test_dense_parity(name):
    c = get_case(name)
    w = c.w
    q = c.inp.Q[0]
    out = c.cache.dense(q.cuda()).double().cpu().numpy()
    for h in range(w.h_q):
        kh = h // w.group
        ref = oracle.attend(c.K[kh], c.V[kh], np.arange(c.n), q[h].double().numpy())
        assert np.max(np.abs(out[h] - ref)) <= OUT_TOL[w.kv_dtype], h


@pytest.mark.parametrize("name", ["tiny_f32", "wide", "light"])
def test_p1_is_dense(name):
    """p = 1 keeps every leaf: the routed output is dense attention."""
    c = get_case(name)
    q = c.inp.Q[1].cuda()
    res = c.cache.decode(q, 1.0)
    dense = c.cache.dense(q)
    tol = OUT_TOL[c.w.kv_dtype]
    assert torch.max(torch.abs(res["out"] - dense)).item() <= tol
    nl = oracle.level_nodes(c.n, c.w.c, 1)
    assert torch.all(res["n_leaf"] == nl)


def test_decode_deterministic():
    c = get_case("light")
    q = c.inp.Q[2].cuda()
    cap = oracle.level_nodes(c.w.capacity, c.w.c, 1)
    r1 = c.cache.decode(q, c.w.p, trace_cap=cap)
    r2 = c.cache.decode(q, c.w.p, trace_cap=cap)
    for k in ("out", "n_leaf", "visited", "trace_counts"):
        assert torch.equal(r1[k], r2[k]), k
    for h in range(c.w.h_q):
        n = int(r1["n_leaf"][h])
        assert torch.equal(r1["leaf_idx"][h, :n], r2["leaf_idx"][h, :n])
        for level in range(c.w.D):
            m = int(r1["trace_counts"][level, h])
            assert torch.equal(r1["trace_ids"][level, h, :m], r2["trace_ids"][level, h, :m])


def _small_cache(N, c, D, R, h_kv, h_q, d, dtype, seed, cap=None):
    g = torch.Generator().manual_seed(seed)
    cap = cap or N
    tdt = torch.float32 if dtype == zha.ZHA_F32 else torch.bfloat16
    K = torch.zeros(h_kv, cap, d, dtype=tdt)
    V = torch.zeros(h_kv, cap, d, dtype=tdt)
    K[:, :N] = torch.randn(h_kv, N, d, generator=g).to(tdt)
    V[:, :N] = torch.randn(h_kv, N, d, generator=g).to(tdt)
    ref = torch.randn(h_kv, R, d, generator=g)
    if dtype == zha.ZHA_BF16:
        ref = ref.to(torch.bfloat16).float()
    cache = zha.ZhaCache(h_kv, h_q, d, R, c, D, dtype, cap)
    dK, dV, dref = K.cuda(), V.cuda(), ref.cuda()
    cache.build(dK, dV, N, dref)
    return cache, (K, V, ref), (dK, dV, dref)


@pytest.mark.parametrize("N,c,D,R,h_kv,h_q,d,dtype", [
    (1, 4, 3, 16, 1, 1, 64, zha.ZHA_F32),        # a single token
    (3, 4, 2, 16, 1, 4, 64, zha.ZHA_F32),        # one partial leaf
    (16, 4, 2, 1, 2, 8, 128, zha.ZHA_BF16),      # exactly c^D tokens
    (17, 4, 2, 16, 2, 8, 128, zha.ZHA_BF16),     # c^D + 1: a second top node
    (1000, 2, 9, 1, 1, 4, 128, zha.ZHA_BF16),    # deep binary tree
    (5000, 256, 1, 16, 1, 4, 128, zha.ZHA_BF16),  # wide leaves, ragged tail
    (3000, 4, 3, 16, 4, 4, 64, zha.ZHA_F32),     # one query head per KV head: sorted, redundant and team cuts
    (2000, 4, 3, 16, 2, 8, 64, zha.ZHA_BF16),    # d = 64 with groups of 4
])
def test_edge_shapes(N, c, D, R, h_kv, h_q, d, dtype):
    cache, (K, V, ref), _ = _small_cache(N, c, D, R, h_kv, h_q, d, dtype, seed=N + c)
    trees = oracle_trees(K, ref, N, c, D)
    check_build(cache, trees)
    kv = "f32" if dtype == zha.ZHA_F32 else "bf16"
    g = torch.Generator().manual_seed(7)
    for p in (0.5, 0.9, 1.0):
        q = torch.randn(h_q, d, generator=g) * 2
        res = cache.decode(q.cuda(), p, trace_cap=oracle.level_nodes(N, c, 1))
        check_decode(res, trees, K, V, ref, q.double().numpy(), p, N, c, D, h_q // h_kv, kv)
    assert cache.status() == 0


@pytest.mark.parametrize("n_leaves", [400, 2048])
def test_tied_nodes_keep_lowest_ids(n_leaves):
    """Every leaf chunk holds the same keys, so every node has the same
    estimate for every query (exact ties).  The cut must keep the lowest ids:
    ceil(p * n) of them.  400 leaves: a team level small enough for each CTA
    to cut alone (the candidates ranked by id); 2048 leaves: the team's
    histogram with a boundary bucket too crowded to rank (taken in id
    order)."""
    c, D, R, h_kv, h_q, d = 4, 1, 16, 1, 4, 128
    N = n_leaves * c
    g = torch.Generator().manual_seed(n_leaves)
    chunk = torch.randn(h_kv, c, d, generator=g)
    K = chunk.repeat(1, n_leaves, 1).to(torch.bfloat16)
    V = torch.randn(h_kv, N, d, generator=g).to(torch.bfloat16)
    ref = torch.randn(h_kv, R, d, generator=g).to(torch.bfloat16).float()
    cache = zha.ZhaCache(h_kv, h_q, d, R, c, D, zha.ZHA_BF16, N)
    dK, dV, dref = K.cuda(), V.cuda(), ref.cuda()
    cache.build(dK, dV, N, dref)
    trees = oracle_trees(K, ref, N, c, D)
    p = 0.3003  # p * n is not an integer: the boundary sits inside a node, away from rounding
    want = int(np.ceil(p * n_leaves))
    q = torch.randn(h_q, d, generator=g)
    res = cache.decode(q.cuda(), p, trace_cap=n_leaves)
    torch.cuda.synchronize()
    assert cache.status() == 0
    n_leaf = res["n_leaf"].cpu()
    idx = res["leaf_idx"].cpu()
    for h in range(h_q):
        assert int(n_leaf[h]) == want, (h, int(n_leaf[h]), want)
        assert torch.equal(idx[h, :want], torch.arange(want, dtype=torch.int32)), h
    check_decode(res, trees, K, V, ref, q.double().numpy(), p, N, c, D, h_q // h_kv, "bf16")


def test_append_matches_rebuild_bitexact():
    """Appending tokens one by one stores exactly the summaries of a fresh
    build over the longer cache (same device functions, same order)."""
    N, a, c, D, R, h_kv, h_q, d = 4090, 13, 4, 6, 16, 2, 8, 128
    cache, (K, V, ref), (dK, dV, dref) = _small_cache(N, c, D, R, h_kv, h_q, d, zha.ZHA_BF16, 11, cap=N + a)
    g = torch.Generator().manual_seed(5)
    knew = torch.randn(a, h_kv, d, generator=g).to(torch.bfloat16)
    vnew = torch.randn(a, h_kv, d, generator=g).to(torch.bfloat16)
    for i in range(a):
        cache.append(knew[i].cuda(), vnew[i].cuda())
    K[:, N:N + a] = knew.transpose(0, 1)
    V[:, N:N + a] = vnew.transpose(0, 1)
    fresh = zha.ZhaCache(h_kv, h_q, d, R, c, D, zha.ZHA_BF16, N + a)
    fK, fV = K.cuda(), V.cuda()
    fresh.build(fK, fV, N + a, dref)
    torch.cuda.synchronize()
    assert cache.n_tokens == N + a
    assert torch.equal(dK, fK) and torch.equal(dV, fV)
    for level in range(1, D + 1):
        for x, y in zip(cache.summaries(level), fresh.summaries(level)):
            assert torch.equal(x, y), level
    trees = oracle_trees(K, ref, N + a, c, D)
    check_build(cache, trees)


def test_errors_and_capacity():
    N, c, D, R, h_kv, h_q, d = 64, 4, 2, 16, 1, 4, 64
    cfg = zha.zha_config(h_kv, h_q, d, R, c, D, zha.ZHA_F32, 0, N)
    ws = torch.empty(zha.zha_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    ctx = zha.zha_create(cfg, ws, ws.numel())
    q = torch.randn(h_q, d, device="cuda")
    out = torch.empty(h_q, d, device="cuda")
    with pytest.raises(zha.ZhaError) as e:
        zha.zha_decode(ctx, q, 0.9, out)
    assert e.value.code == zha.ZHA_ERR_NOT_BUILT
    zha.zha_destroy(ctx)
    cache, _, _ = _small_cache(N, c, D, R, h_kv, h_q, d, zha.ZHA_F32, 3)
    k = torch.zeros(h_kv, d, device="cuda")
    with pytest.raises(zha.ZhaError) as e:
        cache.append(k, k)
    assert e.value.code == zha.ZHA_ERR_CAPACITY
    with pytest.raises(zha.ZhaError) as e:
        cache.decode(q, 0.0)
    assert e.value.code == zha.ZHA_ERR_BAD_ARG
    # a leaf list shorter than the kept set: clipped, status says capacity
    res = cache.decode(q, 1.0, leaf_cap=2)
    torch.cuda.synchronize()
    assert cache.status() == zha.ZHA_ERR_CAPACITY
    assert torch.all(res["n_leaf"] == 16)
    assert cache.status() == 0


def test_barrier_timeout_reports_status_and_next_decode_is_clean():
    """A team or grid barrier wait that runs out of its clock budget ends the
    decode with ZHA_ERR_TIMEOUT in the device status word (the kernel
    returns; nothing traps), and the next decode at the normal budget is
    valid.  A budget of 0 cycles makes every wait that is not satisfied at
    its first poll give up."""
    c = get_case("light")
    w = c.w
    q = c.inp.Q[0].cuda()
    cap = oracle.level_nodes(c.w.capacity, c.w.c, 1)
    zha.zha_set_wait_budget(c.cache.ctx, 0)
    seen = []
    try:
        for _ in range(3):
            c.cache.decode(q, w.p, trace_cap=cap)
            torch.cuda.synchronize()
            st = c.cache.status()
            seen.append(st)
            assert st in (zha.ZHA_OK, zha.ZHA_ERR_TIMEOUT), st
            if st == zha.ZHA_ERR_TIMEOUT:
                break
    finally:
        zha.zha_set_wait_budget(c.cache.ctx, 2_000_000_000)
    assert zha.ZHA_ERR_TIMEOUT in seen, seen
    res = c.cache.decode(q, w.p, trace_cap=cap)
    torch.cuda.synchronize()
    assert c.cache.status() == zha.ZHA_OK
    check_decode(res, c.trees, c.K, c.V, c.inp.ref, c.inp.Q[0].double().numpy(), w.p, c.n, w.c, w.D, w.group,
                 w.kv_dtype, case="light after a timed-out decode")
    with pytest.raises(zha.ZhaError) as e:
        zha.zha_set_wait_budget(c.cache.ctx, -1)
    assert e.value.code == zha.ZHA_ERR_BAD_ARG


def test_injected_host_faults(monkeypatch):
    """ZHA_FAULT makes the host side report a failure without touching the
    GPU: cuda_launch fails zha_build before its launch, capacity fails
    zha_append; with the variable unset both work again."""
    N, c, D, R, h_kv, h_q, d = 200, 4, 2, 16, 1, 4, 64
    cache, (K, V, ref), (dK, dV, dref) = _small_cache(N, c, D, R, h_kv, h_q, d, zha.ZHA_F32, 9, cap=N + 1)
    monkeypatch.setenv("ZHA_FAULT", "cuda_launch")
    with pytest.raises(zha.ZhaError) as e:
        cache.build(dK, dV, N, dref)
    assert e.value.code == zha.ZHA_ERR_CUDA
    monkeypatch.setenv("ZHA_FAULT", "capacity")
    k = torch.zeros(h_kv, d, device="cuda")
    with pytest.raises(zha.ZhaError) as e:
        cache.append(k, k)
    assert e.value.code == zha.ZHA_ERR_CAPACITY
    monkeypatch.delenv("ZHA_FAULT")
    cache.build(dK, dV, N, dref)
    cache.append(k, k)
    torch.cuda.synchronize()
    assert cache.n_tokens == N + 1 and cache.status() == zha.ZHA_OK
    K[:, N] = 0.0
    V[:, N] = 0.0
    trees = oracle_trees(K, ref, N + 1, c, D)
    check_build(cache, trees)


@pytest.mark.parametrize("N,a,c,D,Dm,R,h_kv,h_q,d,dtype", [
    (16384 - 2, 6, 4, 6, 8, 16, 1, 1, 64, zha.ZHA_F32),    # the tiny workload's tree grows from 6 to 7 levels
    (510, 5, 8, 2, 4, 1, 2, 8, 128, zha.ZHA_BF16),         # chunk 8: grows from 2 to 3 levels
])
def test_depth_growth(N, a, c, D, Dm, R, h_kv, h_q, d, dtype):
    """A tree whose depth grows with the context: the append that leaves c + 1
    top nodes adds a new top level.  Before, across and after the step the
    summaries and the routing match the oracle growing the same way, and the
    grown tree is bit-identical to a fresh build over all the tokens."""
    g = torch.Generator().manual_seed(N + c)
    tdt = torch.float32 if dtype == zha.ZHA_F32 else torch.bfloat16
    cap = N + a
    K = torch.zeros(h_kv, cap, d, dtype=tdt)
    V = torch.zeros(h_kv, cap, d, dtype=tdt)
    K[:, :cap] = torch.randn(h_kv, cap, d, generator=g).to(tdt)
    V[:, :cap] = torch.randn(h_kv, cap, d, generator=g).to(tdt)
    ref = torch.randn(h_kv, R, d, generator=g)
    if dtype == zha.ZHA_BF16:
        ref = ref.to(torch.bfloat16).float()
    kv = "f32" if dtype == zha.ZHA_F32 else "bf16"
    cache = zha.ZhaCache(h_kv, h_q, d, R, c, D, dtype, cap, max_depth=Dm)
    dK, dV, dref = K.cuda(), V.cuda(), ref.cuda()
    dK[:, N:] = 0
    dV[:, N:] = 0
    cache.build(dK, dV, N, dref)
    trees = [oracle.build(K[kh], N, ref[kh], c, D, capacity=cap, max_depth=Dm) for kh in range(h_kv)]
    assert cache.depth == trees[0].D == oracle.depth_for(N, c, D, Dm)
    D_start = cache.depth
    qs = torch.randn(a + 1, h_q, d, generator=g) * 2
    n = N
    for i in range(a + 1):
        if i > 0:
            cache.append(K[:, n].cuda(), V[:, n].cuda())
            for kh in range(h_kv):
                oracle.append_update(trees[kh], K[kh], ref[kh])
            n += 1
        torch.cuda.synchronize()
        assert cache.depth == trees[0].D, (n, cache.depth, trees[0].D)
        check_build(cache, trees)
        res = cache.decode(qs[i].cuda(), 0.9, trace_cap=oracle.level_nodes(cap, c, 1))
        torch.cuda.synchronize()
        assert cache.status() == zha.ZHA_OK
        check_decode(res, trees, K, V, ref, qs[i].double().numpy(), 0.9, n, c, cache.depth, h_q // h_kv, kv,
                     case=f"depth growth N={n} c={c} depth {cache.depth}")
    assert cache.depth == D_start + 1
    fresh = zha.ZhaCache(h_kv, h_q, d, R, c, D, dtype, cap, max_depth=Dm)
    fK, fV = K.cuda(), V.cuda()
    fresh.build(fK, fV, n, dref)
    torch.cuda.synchronize()
    assert fresh.depth == cache.depth
    for level in range(1, cache.depth + 1):
        for x, y in zip(cache.summaries(level), fresh.summaries(level)):
            assert torch.equal(x, y), level


def test_depth_growth_build_starts_deeper():
    """With room to grow, a build starts at the least depth whose top level
    holds at most c nodes (here 4 levels where 2 are the minimum)."""
    N, c, D, Dm, R, h_kv, h_q, d = 5000, 8, 2, 4, 1, 2, 8, 128
    cache, (K, V, ref), _ = _small_cache(N, c, D, R, h_kv, h_q, d, zha.ZHA_BF16, 21)
    assert cache.depth == D  # a fixed-depth cache of the same data
    grow = zha.ZhaCache(h_kv, h_q, d, R, c, D, zha.ZHA_BF16, N, max_depth=Dm)
    dK, dV, dref = K.cuda(), V.cuda(), ref.cuda()
    grow.build(dK, dV, N, dref)
    torch.cuda.synchronize()
    assert grow.depth == oracle.depth_for(N, c, D, Dm) == 4
    trees = [oracle.build(K[kh], N, ref[kh], c, D, max_depth=Dm) for kh in range(h_kv)]
    check_build(grow, trees)
    q = torch.randn(h_q, d, generator=torch.Generator().manual_seed(3)) * 2
    res = grow.decode(q.cuda(), 0.8, trace_cap=oracle.level_nodes(N, c, 1))
    torch.cuda.synchronize()
    assert grow.status() == zha.ZHA_OK
    check_decode(res, trees, K, V, ref, q.double().numpy(), 0.8, N, c, grow.depth, h_q // h_kv, "bf16",
                 case="depth growth build N=5000 c=8 depth 4")


ROUTER_CASES = {
    "wide": W["wide_256k"].scaled(16384 + 100, steps=2),
    "deep": W["deep_256k"].scaled(16384 + 37, steps=2),
    "light": W["light_1m"].scaled(300000 + 5, steps=2),
}


@pytest.mark.parametrize("name", list(ROUTER_CASES))
def test_bf16_router(name):
    """router_dtype ZHA_BF16: the routing reads a bf16 copy of every g row.
    The copy is the oracle's exact g rounded to bf16, its plane offsets are
    recomputed from it, and the GPU's routing matches the oracle routing over
    that same quantised store (the attention is exact as always); appends
    keep the copy current."""
    from parity import check_router_copy, router_trees
    w = ROUTER_CASES[name]
    inp = workloads.generate(w, "cpu")
    K, V = inp.K.clone(), inp.V.clone()
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, zha.ZHA_BF16, w.capacity, router_dtype=zha.ZHA_BF16)
    dK, dV, dref = inp.K.cuda(), inp.V.cuda(), inp.ref.cuda()
    cache.build(dK, dV, w.n_tokens, dref)
    trees = oracle_trees(K, inp.ref, w.n_tokens, w.c, w.D, capacity=w.capacity)
    n = w.n_tokens
    app = 0
    for s in range(w.steps):
        for _ in range(w.appends_per_step):
            cache.append(inp.K_app[app].cuda(), inp.V_app[app].cuda())
            K[:, n] = inp.K_app[app]
            V[:, n] = inp.V_app[app]
            for kh in range(w.h_kv):
                oracle.append_update(trees[kh], K[kh], inp.ref[kh])
            n += 1
            app += 1
        torch.cuda.synchronize()
        check_build(cache, trees)
        check_router_copy(cache, trees, inp.ref)
        q = inp.Q[s]
        res = cache.decode(q.cuda(), w.p, trace_cap=oracle.level_nodes(w.capacity, w.c, 1))
        torch.cuda.synchronize()
        assert cache.status() == zha.ZHA_OK
        check_decode(res, router_trees(cache), K, V, inp.ref, q.double().numpy(), w.p, n, w.c, w.D, w.group,
                     w.kv_dtype, case=f"bf16 router {name} step {s}")


@pytest.mark.parametrize("name,n_q", [("tiny_f32", 4), ("wide", 3), ("deep", 4), ("light", 4)])
def test_batch_decode(name, n_q):
    """zha_decode_batch: n_q queries against the same cache in one launch,
    each (query, KV head) pair routed by its own team of CTAs.  Every query's
    routing and output match the oracle, and its output matches the
    one-query decode of the same query."""
    c = get_case(name)
    w = c.w
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, max_batch=n_q)
    cache.build(c.dK, c.dV, c.n, c.dref)
    qs = torch.stack([c.inp.Q[s % c.inp.Q.shape[0]] for s in range(n_q)])
    cap = oracle.level_nodes(w.capacity, w.c, 1)
    res = cache.decode_batch(qs.cuda(), w.p, trace_cap=cap)
    torch.cuda.synchronize()
    assert cache.status() == zha.ZHA_OK
    h_q = w.h_q
    for t in range(n_q):
        res_t = {"out": res["out"][t], "leaf_idx": res["leaf_idx"][t], "n_leaf": res["n_leaf"][t],
                 "visited": res["visited"][t], "trace_ids": res["trace_ids"][:, t * h_q:(t + 1) * h_q],
                 "trace_counts": res["trace_counts"][:, t * h_q:(t + 1) * h_q]}
        check_decode(res_t, c.trees, c.K, c.V, c.inp.ref, qs[t].double().numpy(), w.p, c.n, w.c, w.D, w.group,
                     w.kv_dtype, case=f"batch {name} query {t} of {n_q}")
        one = cache.decode(qs[t].cuda(), w.p)
        torch.cuda.synchronize()
        assert torch.max(torch.abs(one["out"] - res["out"][t])).item() <= OUT_TOL[w.kv_dtype]
    with pytest.raises(zha.ZhaError) as e:
        cache.decode_batch(torch.zeros(n_q + 1, h_q, w.d, device="cuda"), w.p)
    assert e.value.code == zha.ZHA_ERR_BAD_ARG


@pytest.mark.parametrize("name,world", [("wide", 2), ("light", 4), ("deep", 3)])
def test_kv_head_shards(name, world):
    """A cache split by KV head (tree_indexed_sparse_b200.shard): every
    shard, built from its heads' slices and decoding its query heads, passes
    the oracle protocol on those heads and matches the whole cache's decode
    of them (leaf sets exactly, outputs within the tolerance).  The shards
    run one after another on this GPU: their decodes never exchange data."""
    from tree_indexed_sparse_b200.shard import ShardedZhaCache

    c = get_case(name)
    w = c.w
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    cap = oracle.level_nodes(w.capacity, w.c, 1)
    q = c.inp.Q[0]
    whole = c.cache.decode(q.cuda(), w.p)
    torch.cuda.synchronize()
    covered = []
    for rank in range(world):
        sh = ShardedZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, rank=rank, world=world)
        # the whole cache may have appended rows past n: shards take the same prefix
        sh.build(sh.local_kv(c.dK).contiguous(), sh.local_kv(c.dV).contiguous(), c.n, sh.local_kv(c.dref).contiguous())
        res = sh.decode(q.cuda(), w.p, trace_cap=cap)
        torch.cuda.synchronize()
        assert sh.status() == zha.ZHA_OK
        k0, k1, q0, q1 = sh.kv0, sh.kv1, sh.q0, sh.q1
        covered += list(range(k0, k1))
        check_decode(res, c.trees[k0:k1], c.K[k0:k1], c.V[k0:k1], c.inp.ref[k0:k1], q[q0:q1].double().numpy(), w.p,
                     c.n, w.c, w.D, w.group, w.kv_dtype, case=f"{name} KV-head shard {rank} of {world}")
        assert torch.equal(res["n_leaf"], whole["n_leaf"][q0:q1])
        for h in range(q1 - q0):
            n = int(res["n_leaf"][h])
            assert torch.equal(res["leaf_idx"][h, :n], whole["leaf_idx"][q0 + h, :n])
        assert torch.max(torch.abs(res["out"] - whole["out"][q0:q1])).item() <= OUT_TOL[w.kv_dtype]
        sh.close()
    assert covered == list(range(w.h_kv))
