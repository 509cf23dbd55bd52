"""fp64 CPU oracle of the ZHA decode hot path -- TEST INFRASTRUCTURE ONLY.

This package is the checker the CUDA library is compared against.  Only the
test suite, the smoke check and the CPU-baseline leg of the benchmark may
import it; the library under ``tree_indexed_sparse_b200`` never does, and this
package never imports that one.  The arithmetic lives in ``zha_oracle.c``
(plain C, double precision); this module only marshals numpy arrays.

Every function cites the page passage it states; the page titles are listed
at the top of ``zha_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zha_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1


def compile_oracle(src: str = _SRC, out: str = _LIB_PATH, openmp: bool = True) -> str:
    """Compile the C oracle with gcc (strict IEEE double: no fast-math, no FMA
    contraction) into a shared library and return its path."""
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", src, "-o", out, "-lm"]
    if openmp:
        cmd.insert(1, "-fopenmp")
    subprocess.run(cmd, check=True)
    return out


def _stale(lib: str, src: str) -> bool:
    return (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(src)


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int
_D = ctypes.c_double


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    lib.orc_level_nodes.argtypes = [_I64, _I32, _I32]
    lib.orc_level_nodes.restype = _I64
    lib.orc_leaf_summary.argtypes = [_P, _I32, _I64, _I64, _I32, _P, _I32, _P, _P, _P]
    lib.orc_leaf_summary.restype = None
    lib.orc_estimate.argtypes = [_P, _P, _I32, _I32, _P, _P]
    lib.orc_estimate.restype = _D
    lib.orc_parent_summary.argtypes = [_P, _P, _I32, _I32, _P, _I32, _P, _P, _P]
    lib.orc_parent_summary.restype = None
    lib.orc_build.argtypes = [_P, _I32, _I64, _I32, _P, _I32, _I32, _I32, _P, _P, _P, _P]
    lib.orc_build.restype = None
    lib.orc_append_update.argtypes = [_P, _I32, _I64, _I32, _P, _I32, _I32, _I32, _P, _P, _P, _P]
    lib.orc_append_update.restype = None
    lib.orc_topp.argtypes = [_P, _P, _I64, _D, _P, _P, _P, _P]
    lib.orc_topp.restype = _I64
    lib.orc_route.argtypes = [_P, _P, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _D, _P, _P, _P]
    lib.orc_route.restype = _I32
    lib.orc_attend.argtypes = [_P, _P, _I32, _I32, _P, _I64, _P, _P]
    lib.orc_attend.restype = None
    lib.orc_token_set.argtypes = [_P, _I64, _I64, _I32, _P]
    lib.orc_token_set.restype = _I64
    lib.orc_decode_heads.argtypes = [_P, _P, _I32, _I64, _I64, _I32, _I32, _I32, _P, _I64, _P,
                                     _I64, _P, _I32, _I32, _I32, _P, _P, _D, _P, _P, _I64, _P,
                                     _P, _P, _I64]
    lib.orc_decode_heads.restype = None
    lib.orc_build_heads.argtypes = [_P, _I32, _I64, _I64, _I32, _I32, _P, _I32, _I32, _I32, _P,
                                    _I64, _P, _I64, _P, _P]
    lib.orc_build_heads.restype = None
    lib.orc_estimate_many.argtypes = [_P, _P, _I64, _P, _I64, _I32, _I32, _P, _P, _P]
    lib.orc_estimate_many.restype = None
    lib.orc_node_summary.argtypes = [_P, _I32, _I64, _I32, _P, _I32, _I32, _I32, _I64, _P, _P, _P]
    lib.orc_node_summary.restype = None
    lib.orc_depth_for.argtypes = [_I64, _I32, _I32, _I32]
    lib.orc_depth_for.restype = _I32
    lib.orc_build_level.argtypes = [_P, _I32, _I64, _I32, _P, _I32, _I32, _I32, _P, _P, _P, _P]
    lib.orc_build_level.restype = None
    lib.orc_set_threads.argtypes = [_I32]
    lib.orc_set_threads.restype = None
    return lib


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (compiling first if missing or stale) the oracle library.  A
    non-default ``path`` loads that build instead (used by the tests that
    check the pins reject deliberately broken copies of the oracle)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        if _stale(_LIB_PATH, _SRC):
            compile_oracle()
        _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def kv_array(x) -> tuple[np.ndarray, int]:
    """Stored keys/values as a contiguous numpy array plus the dtype code.
    Accepts numpy float32 / uint16 (bf16 bits) arrays or torch float32 /
    bfloat16 tensors (bf16 bits are passed through unchanged)."""
    if hasattr(x, "detach"):
        import torch

        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), BF16
        if x.dtype == torch.float32:
            return x.numpy(), F32
        raise TypeError(f"unsupported key/value dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"unsupported key/value dtype {x.dtype}")


def f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        import torch

        x = x.detach().cpu().to(torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def set_threads(n: int, lib=None) -> None:
    """Threads of the OpenMP drivers (build_heads, decode_heads)."""
    (lib or load()).orc_set_threads(int(n))


def level_nodes(n_tokens: int, c: int, level: int, lib=None) -> int:
    """ceil(N / c^level): node count of a level (1 = leaf chunks)."""
    return int((lib or load()).orc_level_nodes(n_tokens, c, level))


def leaf_summary(K, t0: int, t1: int, ref, lib=None):
    """(m[R], g[R,d], b[R]) of the leaf chunk holding tokens [t0, t1) of one
    head's keys K[N, d] -- the tangent planes of the chunk's log mass."""
    lib = lib or load()
    Ka, dt = kv_array(K)
    ref = f64(ref)
    R, d = ref.shape
    m = np.zeros(R)
    g = np.zeros((R, d))
    b = np.zeros(R)
    lib.orc_leaf_summary(_ptr(Ka), dt, t0, t1, d, _ptr(ref), R, _ptr(m), _ptr(g), _ptr(b))
    return m, g, b


def parent_summary(cm, cg, ref, lib=None):
    """(m[R], g[R,d], b[R]) of a parent from its children's m[nch,R], g[nch,R,d]."""
    lib = lib or load()
    cm = f64(cm)
    cg = f64(cg)
    ref = f64(ref)
    R, d = ref.shape
    m = np.zeros(R)
    g = np.zeros((R, d))
    b = np.zeros(R)
    lib.orc_parent_summary(_ptr(cm), _ptr(cg), cm.shape[0], d, _ptr(ref), R, _ptr(m), _ptr(g), _ptr(b))
    return m, g, b


def estimate(m, g, ref, q, lib=None) -> float:
    """max_j [m_j + (q - r_j).g_j / sqrt(d)] for one node."""
    lib = lib or load()
    m = f64(m)
    g = f64(g)
    ref = f64(ref)
    q = f64(q)
    R, d = ref.shape
    return float(lib.orc_estimate(_ptr(m), _ptr(g), R, d, _ptr(ref), _ptr(q)))


def estimate_many(m_all, g_all, level_row0: int, ids, ref, q, lib=None) -> np.ndarray:
    """Estimates of the listed node ids of one level (a tree's m, g store;
    the level starts at row level_row0)."""
    lib = lib or load()
    ref = f64(ref)
    q = f64(q)
    ids = np.ascontiguousarray(ids, dtype=np.int64)
    R, d = ref.shape
    out = np.zeros(ids.shape[0])
    lib.orc_estimate_many(_ptr(m_all), _ptr(g_all), int(level_row0), _ptr(ids), ids.shape[0], R, d,
                          _ptr(ref), _ptr(q), _ptr(out))
    return out


def node_summary(K, n_tokens: int, ref, c: int, level: int, n: int, lib=None):
    """(m, g, b) of node n of `level`, computed from its subtree's raw keys."""
    lib = lib or load()
    Ka, dt = kv_array(K)
    ref = f64(ref)
    R, d = ref.shape
    m = np.zeros(R)
    g = np.zeros((R, d))
    b = np.zeros(R)
    lib.orc_node_summary(_ptr(Ka), dt, int(n_tokens), d, _ptr(ref), R, c, int(level), int(n), _ptr(m), _ptr(g),
                         _ptr(b))
    return m, g, b


def depth_for(n_tokens: int, c: int, D0: int, max_depth: int = 0, lib=None) -> int:
    """Depth of a tree that grows with the context: the smallest depth in
    [D0, max_depth] whose top level holds at most c nodes (max_depth <= D0:
    the depth stays D0)."""
    return int((lib or load()).orc_depth_for(int(n_tokens), int(c), int(D0), int(max_depth)))


@dataclass
class Tree:
    """Summary store of one head.  Node (level l, id n) is row
    ``level_off[l-1] + n`` of m[rows, R], g[rows, R, d], b[rows, R].  D is
    the current depth; with max_depth > D0 the store has room for
    max_depth levels and D grows as tokens are appended."""

    m: np.ndarray
    g: np.ndarray
    b: np.ndarray
    level_off: np.ndarray
    n_tokens: int
    c: int
    D: int
    D0: int = 0
    max_depth: int = 0

    def estimates(self, l: int, ids, ref, q, lib=None) -> np.ndarray:
        """Estimates for query q of the listed node ids of level l."""
        return estimate_many(self.m, self.g, int(self.level_off[l - 1]), ids, ref, q, lib=lib)

    def level(self, l: int):
        """(m, g, b) views of the nodes currently present at level l."""
        n = level_nodes(self.n_tokens, self.c, l)
        o = int(self.level_off[l - 1])
        return self.m[o:o + n], self.g[o:o + n], self.b[o:o + n]


def _alloc_tree(capacity: int, R: int, d: int, c: int, D: int) -> Tree:
    sizes = [level_nodes(capacity, c, l) for l in range(1, D + 1)]
    off = np.zeros(D, dtype=np.int64)
    off[1:] = np.cumsum(sizes)[:-1]
    rows = int(sum(sizes))
    return Tree(np.zeros((rows, R)), np.zeros((rows, R, d)), np.zeros((rows, R)), off, 0, c, D)


def build(K, n_tokens: int, ref, c: int, D: int, capacity: int | None = None, max_depth: int = 0,
          lib=None) -> Tree:
    """Tree of one head over its first n_tokens keys K[>=n_tokens, d].  D is
    the depth, or with max_depth > D the least depth: the tree then starts
    at depth_for(n_tokens, c, D, max_depth) and has room to grow to
    max_depth levels."""
    lib = lib or load()
    Ka, dt = kv_array(K)
    ref = f64(ref)
    R, d = ref.shape
    Dm = max(D, max_depth)
    t = _alloc_tree(max(capacity or n_tokens, n_tokens), R, d, c, Dm)
    t.D = depth_for(n_tokens, c, D, max_depth, lib=lib)
    t.D0, t.max_depth = D, max_depth
    t.n_tokens = n_tokens
    lib.orc_build(_ptr(Ka), dt, n_tokens, d, _ptr(ref), R, c, t.D, _ptr(t.m), _ptr(t.g), _ptr(t.b),
                  _ptr(t.level_off))
    return t


def append_update(tree: Tree, K, ref, lib=None) -> None:
    """Tree maintenance after the caller stored one new key at row
    tree.n_tokens of K: the count grows by one and the new token's leaf and
    all its ancestors are recomputed.  When the top level then holds more
    than c nodes and the tree may still grow, a new top level is built over
    it (every node of the new level, from its children)."""
    lib = lib or load()
    Ka, dt = kv_array(K)
    ref = f64(ref)
    R, d = ref.shape
    tree.n_tokens += 1
    lib.orc_append_update(_ptr(Ka), dt, tree.n_tokens, d, _ptr(ref), R, tree.c, tree.D,
                          _ptr(tree.m), _ptr(tree.g), _ptr(tree.b), _ptr(tree.level_off))
    D_new = depth_for(tree.n_tokens, tree.c, tree.D0 or tree.D, tree.max_depth, lib=lib)
    while tree.D < D_new:
        tree.D += 1
        lib.orc_build_level(_ptr(Ka), dt, tree.n_tokens, d, _ptr(ref), R, tree.c, tree.D, _ptr(tree.m),
                            _ptr(tree.g), _ptr(tree.b), _ptr(tree.level_off))


def topp(est, ids, p: float, lib=None):
    """Top-p cut of one frontier.  Returns (kept[bool], prob, cum_before, rank)."""
    lib = lib or load()
    est = f64(est)
    ids = np.ascontiguousarray(ids, dtype=np.int64)
    F = est.shape[0]
    kept = np.zeros(F, dtype=np.uint8)
    prob = np.zeros(F)
    cb = np.zeros(F)
    rank = np.zeros(F, dtype=np.int64)
    lib.orc_topp(_ptr(est), _ptr(ids), F, float(p), _ptr(kept), _ptr(prob), _ptr(cb), _ptr(rank))
    return kept.astype(bool), prob, cb, rank


def route(tree: Tree, ref, q, p: float, lib=None):
    """Route one query.  Returns (kept, visited) with kept[l-1] the ascending
    kept ids at level l."""
    lib = lib or load()
    ref = f64(ref)
    q = f64(q)
    R, d = ref.shape
    D = tree.D
    bufs = [np.zeros(level_nodes(tree.n_tokens, tree.c, l) + 1, dtype=np.int64) for l in range(1, D + 1)]
    arr = (ctypes.c_void_p * D)(*[b.ctypes.data for b in bufs])
    cnt = np.zeros(D, dtype=np.int64)
    vis = np.zeros(1, dtype=np.int64)
    lib.orc_route(_ptr(tree.m), _ptr(tree.g), _ptr(tree.level_off), tree.n_tokens, R, d, tree.c, D,
                  _ptr(ref), _ptr(q), float(p), arr, _ptr(cnt), _ptr(vis))
    return [bufs[l][:cnt[l]].copy() for l in range(D)], int(vis[0])


def token_set(leaves, n_tokens: int, c: int, lib=None) -> np.ndarray:
    """Tokens of the kept leaf chunks plus the sink token 0, ascending."""
    lib = lib or load()
    leaves = np.ascontiguousarray(leaves, dtype=np.int64)
    out = np.zeros(leaves.shape[0] * c + 1, dtype=np.int64)
    T = lib.orc_token_set(_ptr(leaves), leaves.shape[0], n_tokens, c, _ptr(out))
    return out[:T].copy()


def attend(K, V, tokens, q, lib=None) -> np.ndarray:
    """Exact softmax attention of q over the listed tokens of one head."""
    lib = lib or load()
    Ka, dt = kv_array(K)
    Va, dv = kv_array(V)
    assert dt == dv
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    q = f64(q)
    d = q.shape[0]
    out = np.zeros(d)
    lib.orc_attend(_ptr(Ka), _ptr(Va), dt, d, _ptr(tokens), tokens.shape[0], _ptr(q), _ptr(out))
    return out


def decode_one(K, V, tree: Tree, ref, q, p: float, lib=None):
    """One query head: route, gather, attend.  Returns (out, leaves, visited)."""
    kept, visited = route(tree, ref, q, p, lib=lib)
    toks = token_set(kept[0], tree.n_tokens, tree.c, lib=lib)
    return attend(K, V, toks, q, lib=lib), kept[0], visited


class HeadsTrees:
    """Trees of all KV heads in one contiguous store (for the OpenMP drivers)."""

    def __init__(self, H_kv: int, capacity: int, R: int, d: int, c: int, D: int):
        sizes = [level_nodes(capacity, c, l) for l in range(1, D + 1)]
        self.level_off = np.zeros(D, dtype=np.int64)
        self.level_off[1:] = np.cumsum(sizes)[:-1]
        self.rows = int(sum(sizes))
        self.m = np.zeros((H_kv, self.rows, R))
        self.g = np.zeros((H_kv, self.rows, R, d))
        self.b = np.zeros((H_kv, self.rows, R))
        self.H_kv, self.R, self.d, self.c, self.D = H_kv, R, d, c, D
        self.n_tokens = 0

    def head(self, kh: int) -> Tree:
        return Tree(self.m[kh], self.g[kh], self.b[kh], self.level_off, self.n_tokens, self.c, self.D)


def build_heads(K, n_tokens: int, ref, c: int, D: int, capacity: int | None = None, lib=None) -> HeadsTrees:
    """Trees of every KV head of K[H_kv, cap, d] (OpenMP over heads)."""
    lib = lib or load()
    Ka, dt = kv_array(K)
    ref = f64(ref)
    H_kv, R, d = ref.shape
    ht = HeadsTrees(H_kv, max(capacity or n_tokens, n_tokens), R, d, c, D)
    ht.n_tokens = n_tokens
    lib.orc_build_heads(_ptr(Ka), dt, Ka.shape[1], n_tokens, d, H_kv, _ptr(ref), R, c, D,
                        _ptr(ht.m), ht.rows * R, _ptr(ht.g), ht.rows * R * d, _ptr(ht.b),
                        _ptr(ht.level_off))
    return ht


def decode_heads(K, V, ht: HeadsTrees, ref, Q, p: float, lib=None):
    """All query heads of one decoded token (OpenMP over heads); query head h
    reads KV head h // (H_q / H_kv).  Returns (out[H_q,d], leaves list, visited[H_q])."""
    lib = lib or load()
    Ka, dt = kv_array(K)
    Va, _ = kv_array(V)
    ref = f64(ref)
    Q = f64(Q)
    H_q, d = Q.shape
    N = ht.n_tokens
    nl1 = level_nodes(N, ht.c, 1)
    kept_stride = sum(level_nodes(N, ht.c, l) for l in range(1, ht.D + 1))
    out = np.zeros((H_q, d))
    leaf = np.zeros((H_q, nl1), dtype=np.int64)
    nleaf = np.zeros(H_q, dtype=np.int64)
    vis = np.zeros(H_q, dtype=np.int64)
    kept = np.zeros(H_q * kept_stride, dtype=np.int64)
    lib.orc_decode_heads(_ptr(Ka), _ptr(Va), dt, Ka.shape[1], N, d, ht.H_kv, H_q, _ptr(ht.m),
                         ht.rows * ht.R, _ptr(ht.g), ht.rows * ht.R * d, _ptr(ht.level_off), ht.R,
                         ht.c, ht.D, _ptr(ref), _ptr(Q), float(p), _ptr(out), _ptr(leaf), nl1,
                         _ptr(nleaf), _ptr(vis), _ptr(kept), kept_stride)
    return out, [leaf[h, :nleaf[h]].copy() for h in range(H_q)], vis
