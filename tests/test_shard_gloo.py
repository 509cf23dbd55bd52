"""KV-head sharding (tree_indexed_sparse_b200.shard) on the host: the head
partition, the slicing of whole-layer tensors, and the assembly of the
layer's output from the ranks' shares with two gloo ranks on the CPU.

The per-rank cache here is a stand-in with the library cache's interface
that attends over every stored token of each of its heads (plain softmax
attention, fp64): sharding only decides which heads a rank computes, so
the assembled output must equal the same stand-in run over all heads."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from tree_indexed_sparse_b200.shard import ShardedZhaCache, head_range  # noqa: E402


class DenseStandIn:
    """The cache interface over host tensors: exact attention of every head."""

    def __init__(self, h_kv, h_q, d, R, c, D, kv_dtype, capacity_tokens):
        self.h_kv, self.h_q, self.d, self.G = h_kv, h_q, d, h_q // h_kv
        self.K = torch.zeros(h_kv, capacity_tokens, d, dtype=torch.float64)
        self.V = torch.zeros_like(self.K)
        self.n = 0

    def build(self, K, V, n_tokens, ref):
        assert K.shape[0] == self.h_kv and ref.shape[0] == self.h_kv
        self.K[:, :n_tokens] = K[:, :n_tokens].double()
        self.V[:, :n_tokens] = V[:, :n_tokens].double()
        self.n = n_tokens

    def append(self, k, v):
        assert k.shape == (self.h_kv, self.d)
        self.K[:, self.n] = k.double()
        self.V[:, self.n] = v.double()
        self.n += 1

    def decode(self, q, p):
        assert q.shape == (self.h_q, self.d)
        out = torch.empty(self.h_q, self.d, dtype=torch.float32)
        for h in range(self.h_q):
            kh = h // self.G
            s = self.K[kh, :self.n] @ q[h].double() / self.d ** 0.5
            out[h] = (torch.softmax(s, 0) @ self.V[kh, :self.n]).float()
        return {"out": out, "n_leaf": torch.full((self.h_q,), self.n, dtype=torch.int32)}

    def status(self):
        return 0

    @property
    def n_tokens(self):
        return self.n


def _inputs(h_kv, h_q, d, n, cap, seed=7):
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(h_kv, cap, d, generator=g)
    V = torch.randn(h_kv, cap, d, generator=g)
    ref = torch.randn(h_kv, 1, d, generator=g)
    q = torch.randn(h_q, d, generator=g)
    kn = torch.randn(h_kv, d, generator=g)
    vn = torch.randn(h_kv, d, generator=g)
    return K, V, ref, q, kn, vn


@pytest.mark.parametrize("h_kv", [1, 2, 3, 4, 7, 8, 64])
def test_head_range_partitions_every_head_once(h_kv):
    for world in range(1, h_kv + 1):
        spans = [head_range(h_kv, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == h_kv
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 == b0
        sizes = [b - a for a, b in spans]
        assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_head_range_rejects_more_ranks_than_heads():
    with pytest.raises(ValueError):
        head_range(4, 5, 0)
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def test_shards_in_one_process_cover_the_layer():
    """Without a process group: explicit rank and world; the shards' outputs
    put side by side are the whole layer's."""
    h_kv, h_q, d, n, cap = 3, 12, 16, 40, 48
    K, V, ref, q, kn, vn = _inputs(h_kv, h_q, d, n, cap)
    whole = DenseStandIn(h_kv, h_q, d, 1, 4, 2, 0, cap)
    whole.build(K, V, n, ref)
    whole.append(kn, vn)
    want = whole.decode(q, 1.0)["out"]
    parts = []
    for rank in range(2):
        sh = ShardedZhaCache(h_kv, h_q, d, 1, 4, 2, 0, cap, rank=rank, world=2, cache_factory=DenseStandIn)
        sh.build(sh.local_kv(K), sh.local_kv(V), n, sh.local_kv(ref))
        sh.append(sh.local_kv(kn), sh.local_kv(vn))
        res = sh.decode(q, 1.0)
        assert res["out"].shape == (sh.q1 - sh.q0, d)
        parts.append(res["out"])
        with pytest.raises(ValueError):  # 3 heads over 2 ranks: unequal shares
            sh.gather_out(res["out"])
    assert torch.equal(torch.cat(parts), want)


def test_slicing_checks_head_counts():
    sh = ShardedZhaCache(4, 16, 8, 1, 4, 2, 0, 16, rank=1, world=2, cache_factory=DenseStandIn)
    assert (sh.kv0, sh.kv1, sh.q0, sh.q1) == (2, 4, 8, 16)
    with pytest.raises(ValueError):
        sh.local_kv(torch.zeros(3, 16, 8))
    with pytest.raises(ValueError):
        sh.local_q(torch.zeros(15, 8))
    with pytest.raises(ValueError):
        ShardedZhaCache(4, 10, 8, 1, 4, 2, 0, 16, rank=0, world=1, cache_factory=DenseStandIn)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q_out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from tree_indexed_sparse_b200.shard import ShardedZhaCache as S

    h_kv, h_q, d, n, cap = 4, 16, 32, 50, 64
    K, V, ref, q, kn, vn = _inputs(h_kv, h_q, d, n, cap)
    sh = S(h_kv, h_q, d, 1, 4, 2, 0, cap, cache_factory=DenseStandIn)  # rank and world from the group
    sh.build(sh.local_kv(K), sh.local_kv(V), n, sh.local_kv(ref))
    sh.append(sh.local_kv(kn), sh.local_kv(vn))
    local = sh.decode(q, 1.0)["out"]
    full = sh.decode(q, 1.0, gather=True)["out"]
    q_out.put((rank, sh.kv0, sh.kv1, local, full))
    dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_layer_output():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=120) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    h_kv, h_q, d, n, cap = 4, 16, 32, 50, 64
    K, V, ref, qv, kn, vn = _inputs(h_kv, h_q, d, n, cap)
    whole = DenseStandIn(h_kv, h_q, d, 1, 4, 2, 0, cap)
    whole.build(K, V, n, ref)
    whole.append(kn, vn)
    want = whole.decode(qv, 1.0)["out"]
    assert [(g[1], g[2]) for g in got] == [(0, 2), (2, 4)]
    for rank, kv0, kv1, local, full in got:
        assert torch.equal(local, want[kv0 * 4:kv1 * 4])
        assert torch.equal(full, want)
