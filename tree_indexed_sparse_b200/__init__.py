"""Python binding of libzha.so: ZHA tree-indexed sparse decode attention on B200.

The functions below carry the C ABI's names (``include/zha.h``) and only
marshal arguments: every step of the hot path runs in the library's CUDA
kernels.  ``ZhaCache`` is a convenience owner of the device buffers (torch
tensors) around one context.  There is no fallback: if ``libzha.so`` is
missing or cannot load, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# ZHA_LIB selects another build of the same library (e.g. an instrumented one)
LIB_PATH = os.environ.get("ZHA_LIB") or os.path.join(_HERE, "libzha.so")

ZHA_OK = 0
ZHA_ERR_BAD_ARG = -1
ZHA_ERR_CAPACITY = -2
ZHA_ERR_NOT_BUILT = -3
ZHA_ERR_CUDA = -4
ZHA_ERR_TIMEOUT = -5
ZHA_ERR_UNSUPPORTED = -6
ZHA_F32 = 0
ZHA_BF16 = 1

# every symbol include/zha.h declares
EXPORTS = ["zha_workspace_bytes", "zha_create", "zha_destroy", "zha_build", "zha_append", "zha_decode",
           "zha_decode_batch",
           "zha_dense_decode", "zha_dense_decode_static", "zha_device_status", "zha_set_phase_timer",
           "zha_set_wait_budget", "zha_depth", "zha_n_tokens", "zha_summary_layout", "zha_router_layout",
           "zha_strerror"]


class ZhaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {zha_strerror(code)} ({code})")


class zha_config(ctypes.Structure):
    _fields_ = [("h_kv", ctypes.c_int32), ("h_q", ctypes.c_int32), ("d", ctypes.c_int32),
                ("R", ctypes.c_int32), ("c", ctypes.c_int32), ("D", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32), ("max_depth", ctypes.c_int32),
                ("capacity_tokens", ctypes.c_int64), ("router_dtype", ctypes.c_int32),
                ("max_batch", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python tree_indexed_sparse_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    CFG = ctypes.POINTER(zha_config)
    lib.zha_workspace_bytes.argtypes = [CFG]
    lib.zha_workspace_bytes.restype = I64
    lib.zha_create.argtypes = [CFG, P, I64, ctypes.POINTER(P)]
    lib.zha_create.restype = ctypes.c_int
    lib.zha_destroy.argtypes = [P]
    lib.zha_destroy.restype = None
    lib.zha_build.argtypes = [P, P, P, I64, P, I32, I32, P]
    lib.zha_build.restype = ctypes.c_int
    lib.zha_append.argtypes = [P, P, P, P]
    lib.zha_append.restype = ctypes.c_int
    lib.zha_decode.argtypes = [P, P, F, P, P, I32, P, P, P, P, I32, P]
    lib.zha_decode.restype = ctypes.c_int
    lib.zha_decode_batch.argtypes = [P, P, I32, F, P, P, I32, P, P, P, P, I32, P]
    lib.zha_decode_batch.restype = ctypes.c_int
    lib.zha_dense_decode.argtypes = [P, P, P, P]
    lib.zha_dense_decode.restype = ctypes.c_int
    lib.zha_dense_decode_static.argtypes = [CFG, P, P, I64, P, P, P, P]
    lib.zha_dense_decode_static.restype = ctypes.c_int
    lib.zha_device_status.argtypes = [P, ctypes.POINTER(I32), P]
    lib.zha_device_status.restype = ctypes.c_int
    lib.zha_set_phase_timer.argtypes = [P, P]
    lib.zha_set_phase_timer.restype = ctypes.c_int
    lib.zha_set_wait_budget.argtypes = [P, I64]
    lib.zha_set_wait_budget.restype = ctypes.c_int
    lib.zha_depth.argtypes = [P]
    lib.zha_depth.restype = I32
    lib.zha_n_tokens.argtypes = [P]
    lib.zha_n_tokens.restype = I64
    lib.zha_summary_layout.argtypes = [P, I32, ctypes.POINTER(I64), ctypes.POINTER(I64),
                                       ctypes.POINTER(I64), ctypes.POINTER(I64)]
    lib.zha_summary_layout.restype = ctypes.c_int
    lib.zha_router_layout.argtypes = [P, I32, ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I64)]
    lib.zha_router_layout.restype = ctypes.c_int
    lib.zha_strerror.argtypes = [ctypes.c_int]
    lib.zha_strerror.restype = ctypes.c_char_p
    return lib


lib = _load()


def _check(code: int, where: str) -> None:
    if code != ZHA_OK:
        raise ZhaError(code, where)


def _vp(x) -> ctypes.c_void_p:
    """Device pointer of a tensor, or a raw integer address, or None."""
    if x is None:
        return ctypes.c_void_p(0)
    if hasattr(x, "data_ptr"):
        return ctypes.c_void_p(x.data_ptr())
    return ctypes.c_void_p(int(x))


# ---- the C ABI, name for name ------------------------------------------------

def zha_strerror(code: int) -> str:
    return lib.zha_strerror(code).decode()


def zha_workspace_bytes(cfg: zha_config) -> int:
    return int(lib.zha_workspace_bytes(ctypes.byref(cfg)))


def zha_create(cfg: zha_config, d_workspace, ws_bytes: int) -> ctypes.c_void_p:
    ctx = ctypes.c_void_p()
    _check(lib.zha_create(ctypes.byref(cfg), _vp(d_workspace), int(ws_bytes), ctypes.byref(ctx)), "zha_create")
    return ctx


def zha_destroy(ctx) -> None:
    lib.zha_destroy(ctx)


def zha_build(ctx, d_K, d_V, n_tokens: int, d_ref_q, c: int, D: int, stream=None) -> None:
    _check(lib.zha_build(ctx, _vp(d_K), _vp(d_V), int(n_tokens), _vp(d_ref_q), int(c), int(D), _vp(stream)),
           "zha_build")


def zha_append(ctx, d_k, d_v, stream=None) -> None:
    _check(lib.zha_append(ctx, _vp(d_k), _vp(d_v), _vp(stream)), "zha_append")


def zha_decode(ctx, d_q, p: float, d_out, d_leaf_idx=None, leaf_cap: int = 0, d_n_leaf=None,
               d_nodes_visited=None, d_trace_ids=None, d_trace_counts=None, trace_cap: int = 0,
               stream=None) -> None:
    _check(lib.zha_decode(ctx, _vp(d_q), float(p), _vp(d_out), _vp(d_leaf_idx), int(leaf_cap), _vp(d_n_leaf),
                          _vp(d_nodes_visited), _vp(d_trace_ids), _vp(d_trace_counts), int(trace_cap),
                          _vp(stream)), "zha_decode")


def zha_decode_batch(ctx, d_q, n_q: int, p: float, d_out, d_leaf_idx=None, leaf_cap: int = 0, d_n_leaf=None,
                     d_nodes_visited=None, d_trace_ids=None, d_trace_counts=None, trace_cap: int = 0,
                     stream=None) -> None:
    _check(lib.zha_decode_batch(ctx, _vp(d_q), int(n_q), float(p), _vp(d_out), _vp(d_leaf_idx), int(leaf_cap),
                                _vp(d_n_leaf), _vp(d_nodes_visited), _vp(d_trace_ids), _vp(d_trace_counts),
                                int(trace_cap), _vp(stream)), "zha_decode_batch")


def zha_dense_decode(ctx, d_q, d_out, stream=None) -> None:
    _check(lib.zha_dense_decode(ctx, _vp(d_q), _vp(d_out), _vp(stream)), "zha_dense_decode")


def zha_dense_decode_static(cfg: zha_config, d_K, d_V, n_tokens: int, d_q, d_out, d_status, stream=None) -> None:
    _check(lib.zha_dense_decode_static(ctypes.byref(cfg), _vp(d_K), _vp(d_V), int(n_tokens), _vp(d_q), _vp(d_out),
                                       _vp(d_status), _vp(stream)), "zha_dense_decode_static")


def zha_device_status(ctx, stream=None) -> int:
    st = ctypes.c_int32(0)
    _check(lib.zha_device_status(ctx, ctypes.byref(st), _vp(stream)), "zha_device_status")
    return int(st.value)


def zha_set_phase_timer(ctx, d_ns) -> None:
    """d_ns: device int64 tensor of D + 3 entries for the decode phase stamps
    (global timer, ns), or None to clear.  Keep it alive while set."""
    _check(lib.zha_set_phase_timer(ctx, _vp(d_ns)), "zha_set_phase_timer")


def zha_set_wait_budget(ctx, cycles: int) -> None:
    """Testing hook: clock cycles each inter-CTA wait of zha_decode may take."""
    _check(lib.zha_set_wait_budget(ctx, int(cycles)), "zha_set_wait_budget")


def zha_depth(ctx) -> int:
    return int(lib.zha_depth(ctx))


def zha_n_tokens(ctx) -> int:
    return int(lib.zha_n_tokens(ctx))


def zha_summary_layout(ctx, level: int):
    g, b, m, n = (ctypes.c_int64() for _ in range(4))
    _check(lib.zha_summary_layout(ctx, int(level), ctypes.byref(g), ctypes.byref(b), ctypes.byref(m),
                                  ctypes.byref(n)), "zha_summary_layout")
    return int(g.value), int(b.value), int(m.value), int(n.value)


def zha_router_layout(ctx, level: int):
    g, b, n = (ctypes.c_int64() for _ in range(3))
    _check(lib.zha_router_layout(ctx, int(level), ctypes.byref(g), ctypes.byref(b), ctypes.byref(n)),
           "zha_router_layout")
    return int(g.value), int(b.value), int(n.value)


# ---- convenience owner of one context's device buffers ----------------------

class ZhaCache:
    """One KV cache and its tree on the current CUDA device.

    Owns the workspace (a torch uint8 tensor); keeps references to the K, V and
    reference-query tensors handed to ``build`` so they outlive the context.
    """

    def __init__(self, h_kv: int, h_q: int, d: int, R: int, c: int, D: int, kv_dtype: int,
                 capacity_tokens: int, device="cuda", max_depth: int = 0, router_dtype: int = ZHA_F32,
                 max_batch: int = 1):
        import torch

        self.cfg = zha_config(h_kv, h_q, d, R, c, D, kv_dtype, max_depth, capacity_tokens, router_dtype, max_batch)
        nbytes = zha_workspace_bytes(self.cfg)
        if nbytes < 0:
            raise ZhaError(nbytes, "zha_workspace_bytes")
        self.device = torch.device(device)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.ctx = zha_create(self.cfg, self.workspace, nbytes)
        self._keep = ()

    def close(self) -> None:
        # at interpreter shutdown the module globals may already be gone
        if getattr(self, "ctx", None) and lib is not None and zha_destroy is not None:
            zha_destroy(self.ctx)
        self.ctx = None

    def __del__(self):
        self.close()

    @staticmethod
    def _stream(stream):
        import torch

        s = stream if stream is not None else torch.cuda.current_stream()
        return s.cuda_stream

    def build(self, K, V, n_tokens: int, ref, stream=None) -> None:
        self._keep = (K, V, ref)
        zha_build(self.ctx, K, V, n_tokens, ref, self.cfg.c, self.cfg.D, self._stream(stream))

    def append(self, k, v, stream=None) -> None:
        zha_append(self.ctx, k, v, self._stream(stream))

    @property
    def n_tokens(self) -> int:
        return zha_n_tokens(self.ctx)

    @property
    def depth(self) -> int:
        """Current depth (routing levels) of the tree."""
        return zha_depth(self.ctx)

    def decode(self, q, p: float, leaf_cap: int | None = None, trace_cap: int = 0, stream=None, out=None):
        """Returns a dict of device tensors: out, leaf_idx, n_leaf, visited
        (+ trace_ids, trace_counts when trace_cap > 0)."""
        import torch

        h_q, D = self.cfg.h_q, self.depth
        dev = self.device
        if leaf_cap is None:
            leaf_cap = -(-self.n_tokens // self.cfg.c)
        res = {
            "out": out if out is not None else torch.empty(h_q, self.cfg.d, dtype=torch.float32, device=dev),
            "leaf_idx": torch.empty(h_q, max(leaf_cap, 1), dtype=torch.int32, device=dev),
            "n_leaf": torch.empty(h_q, dtype=torch.int32, device=dev),
            "visited": torch.empty(h_q, dtype=torch.int64, device=dev),
        }
        tid = tcnt = None
        if trace_cap > 0:
            tid = res["trace_ids"] = torch.full((D, h_q, trace_cap), -1, dtype=torch.int32, device=dev)
            tcnt = res["trace_counts"] = torch.zeros(D, h_q, dtype=torch.int32, device=dev)
        zha_decode(self.ctx, q, p, res["out"], res["leaf_idx"], leaf_cap, res["n_leaf"], res["visited"],
                   tid, tcnt, trace_cap, self._stream(stream))
        return res

    def decode_batch(self, qs, p: float, leaf_cap: int | None = None, trace_cap: int = 0, stream=None, out=None):
        """Decode n_q queries qs [n_q, h_q, d] in one launch.  Returns a dict of
        device tensors: out [n_q, h_q, d], leaf_idx [n_q, h_q, leaf_cap],
        n_leaf and visited [n_q, h_q] (+ trace_ids [D, n_q * h_q, trace_cap]
        and trace_counts [D, n_q * h_q] when trace_cap > 0)."""
        import torch

        n_q, h_q, D = qs.shape[0], self.cfg.h_q, self.depth
        dev = self.device
        if leaf_cap is None:
            leaf_cap = -(-self.n_tokens // self.cfg.c)
        res = {
            "out": out if out is not None else torch.empty(n_q, h_q, self.cfg.d, dtype=torch.float32, device=dev),
            "leaf_idx": torch.empty(n_q, h_q, max(leaf_cap, 1), dtype=torch.int32, device=dev),
            "n_leaf": torch.empty(n_q, h_q, dtype=torch.int32, device=dev),
            "visited": torch.empty(n_q, h_q, dtype=torch.int64, device=dev),
        }
        tid = tcnt = None
        if trace_cap > 0:
            tid = res["trace_ids"] = torch.full((D, n_q * h_q, trace_cap), -1, dtype=torch.int32, device=dev)
            tcnt = res["trace_counts"] = torch.zeros(D, n_q * h_q, dtype=torch.int32, device=dev)
        zha_decode_batch(self.ctx, qs, n_q, p, res["out"], res["leaf_idx"], leaf_cap, res["n_leaf"], res["visited"],
                         tid, tcnt, trace_cap, self._stream(stream))
        return res

    def dense(self, q, out=None, stream=None):
        import torch

        o = out if out is not None else torch.empty(self.cfg.h_q, self.cfg.d, dtype=torch.float32,
                                                    device=self.device)
        zha_dense_decode(self.ctx, q, o, self._stream(stream))
        return o

    def status(self, stream=None) -> int:
        return zha_device_status(self.ctx, self._stream(stream))

    def summaries(self, level: int):
        """(g [h_kv, nodes, R, d], b [h_kv, nodes, R], m [h_kv, nodes, R]) fp32
        views of level `level` for the nodes present now."""
        import torch

        go, bo, mo, cap = zha_summary_layout(self.ctx, level)
        c = self.cfg
        n = -(-self.n_tokens // c.c ** level) if self.n_tokens else 0
        ws = self.workspace

        def view(off, shape):
            count = 1
            for s in shape:
                count *= s
            return ws[off:off + 4 * count].view(torch.float32).view(*shape)

        g = view(go, (c.h_kv, cap, c.R, c.d))[:, :n]
        b = view(bo, (c.h_kv, cap, c.R))[:, :n]
        m = view(mo, (c.h_kv, cap, c.R))[:, :n]
        return g, b, m

    def router_summaries(self, level: int):
        """(g~ [h_kv, nodes, R, d] bf16, b~ [h_kv, nodes, R] fp32): the bf16
        router copy of level `level` (router_dtype ZHA_BF16)."""
        import torch

        go, bo, cap = zha_router_layout(self.ctx, level)
        c = self.cfg
        n = -(-self.n_tokens // c.c ** level) if self.n_tokens else 0
        ws = self.workspace
        g = ws[go:go + 2 * c.h_kv * cap * c.R * c.d].view(torch.bfloat16).view(c.h_kv, cap, c.R, c.d)[:, :n]
        b = ws[bo:bo + 4 * c.h_kv * cap * c.R].view(torch.float32).view(c.h_kv, cap, c.R)[:, :n]
        return g, b
