"""A ZHA cache split by KV head over the ranks of a process group.

The KV heads of a layer are independent under ZHA: each has its own tree,
its query heads route and attend over it alone, and nothing passes between
heads until the outputs meet the output projection.  A cache too large for
one GPU ("Zyphra 分层注意力（ZHA）…", section "局限与权衡：未被压缩的 KV 缓存和模型速度":
the full KV cache stays resident) therefore splits across GPUs by KV head
with no exchange on the decode path: rank r holds KV heads
[h_kv r / N, h_kv (r + 1) / N) -- their K, V, reference queries and tree --
and decodes the query heads of its own group.  Each rank's outputs are its
slice of the layer's [h_q, d] output, the layout a row-parallel output
projection consumes; ``decode(..., gather=True)`` assembles the whole output
on every rank with one NCCL all-gather for callers that need it.

Everything a rank computes runs in the library's kernels through
``ZhaCache``; this module only picks the rank's heads, slices tensors and
calls torch.distributed.
"""
from __future__ import annotations


def head_range(h_kv: int, world: int, rank: int) -> tuple[int, int]:
    """KV heads [first, last) of `rank` among `world` ranks: contiguous,
    sizes differing by at most one, every rank at least one head."""
    if not 1 <= world <= h_kv:
        raise ValueError(f"{world} ranks for {h_kv} KV heads: every rank needs at least one head")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    return h_kv * rank // world, h_kv * (rank + 1) // world


class ShardedZhaCache:
    """This rank's share of a cache split by KV head.

    ``rank``/``world`` default to the process group's (one rank, no group,
    when torch.distributed is not initialised).  ``cache_factory`` builds the
    rank's cache (``ZhaCache`` of this package: the CUDA path) from
    (h_kv, h_q, d, R, c, D, kv_dtype, capacity_tokens, **kwargs).

    Tensors passed to ``build`` and ``append`` are the rank's slices
    (``local_kv`` cuts them from whole-layer tensors); ``decode`` takes the
    layer's whole query [h_q, d] and uses the rank's rows.
    """

    def __init__(self, h_kv: int, h_q: int, d: int, R: int, c: int, D: int, kv_dtype: int,
                 capacity_tokens: int, *, rank: int | None = None, world: int | None = None, group=None,
                 cache_factory=None, **kwargs):
        import torch.distributed as dist

        if h_q % h_kv:
            raise ValueError(f"{h_q} query heads do not group evenly over {h_kv} KV heads")
        if world is None or rank is None:
            on = dist.is_available() and dist.is_initialized()
            world = dist.get_world_size(group) if on else 1
            rank = dist.get_rank(group) if on else 0
        self.rank, self.world, self.group = rank, world, group
        self.h_kv, self.h_q, self.d = h_kv, h_q, d
        self.G = h_q // h_kv
        self.kv0, self.kv1 = head_range(h_kv, world, rank)
        self.q0, self.q1 = self.kv0 * self.G, self.kv1 * self.G
        if cache_factory is None:
            from . import ZhaCache as cache_factory
        self.local = cache_factory(self.kv1 - self.kv0, self.q1 - self.q0, d, R, c, D, kv_dtype, capacity_tokens,
                                   **kwargs)

    # ---- slicing -------------------------------------------------------------
    def local_kv(self, x):
        """This rank's KV heads of a whole-layer tensor [h_kv, ...]."""
        if x.shape[0] != self.h_kv:
            raise ValueError(f"expected {self.h_kv} KV heads in dimension 0, got {x.shape[0]}")
        return x[self.kv0:self.kv1]

    def local_q(self, q):
        """This rank's query heads of a whole-layer query [h_q, d]."""
        if q.shape[0] != self.h_q:
            raise ValueError(f"expected {self.h_q} query heads in dimension 0, got {q.shape[0]}")
        return q[self.q0:self.q1]

    # ---- the path ------------------------------------------------------------
    def build(self, K, V, n_tokens: int, ref, **kw) -> None:
        """K, V [h_local, capacity, d] and ref [h_local, R, d]: this rank's heads."""
        self.local.build(K, V, n_tokens, ref, **kw)

    def append(self, k, v, **kw) -> None:
        """k, v [h_local, d]: the new token's rows of this rank's heads."""
        self.local.append(k, v, **kw)

    def decode(self, q, p: float, gather: bool = False, **kw):
        """Decode the layer's query q [h_q, d] over this rank's heads.  Returns
        the rank's result (out [h_q_local, d], leaf_idx, n_leaf, visited: its
        query heads q0 .. q1 - 1); with gather=True, "out" is the whole layer's
        [h_q, d] on every rank (ranks must hold equal numbers of heads)."""
        res = self.local.decode(self.local_q(q).contiguous(), p, **kw)
        if gather:
            res["out"] = self.gather_out(res["out"])
        return res

    def gather_out(self, out_local):
        """The whole layer's output [h_q, d] from every rank's [h_q_local, d]."""
        import torch
        import torch.distributed as dist

        if self.world == 1:
            return out_local
        if self.h_kv % self.world:
            raise ValueError(f"gather needs equal shards: {self.h_kv} KV heads over {self.world} ranks")
        full = torch.empty(self.h_q, self.d, dtype=out_local.dtype, device=out_local.device)
        dist.all_gather_into_tensor(full, out_local.contiguous(), group=self.group)
        return full

    def status(self) -> int:
        return self.local.status()

    @property
    def n_tokens(self) -> int:
        return self.local.n_tokens

    def close(self) -> None:
        close = getattr(self.local, "close", None)
        if close is not None:
            close()
