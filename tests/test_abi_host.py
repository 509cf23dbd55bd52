"""The C ABI library on the host: loads without a GPU, exports every symbol
include/zha.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import workloads
import tree_indexed_sparse_b200 as zha

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "zha.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(zha_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert names == sorted(zha.EXPORTS)
    for n in names:
        assert hasattr(zha.lib, n), n
        assert ctypes.cast(getattr(zha.lib, n), ctypes.c_void_p).value


def _cfg(w):
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    return zha.zha_config(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, 0, w.capacity)


@pytest.mark.parametrize("name", workloads.ORDER)
def test_workspace_sizes(name):
    w = workloads.WORKLOADS[name]
    nbytes = zha.zha_workspace_bytes(_cfg(w))
    assert nbytes > 0
    # at least the fp32 summary store of every level
    store = 0
    for level in range(1, w.D + 1):
        nodes = -(-w.capacity // w.c ** level)
        store += w.h_kv * nodes * w.R * (w.d + 2) * 4
    assert store <= nbytes <= store * 2 + (1 << 28)


@pytest.mark.parametrize("field,value,code", [
    ("h_kv", 0, zha.ZHA_ERR_BAD_ARG), ("h_q", 6, zha.ZHA_ERR_BAD_ARG), ("c", 1, zha.ZHA_ERR_BAD_ARG),
    ("D", 0, zha.ZHA_ERR_BAD_ARG), ("D", 17, zha.ZHA_ERR_BAD_ARG), ("kv_dtype", 7, zha.ZHA_ERR_BAD_ARG),
    ("capacity_tokens", 0, zha.ZHA_ERR_BAD_ARG), ("d", 96, zha.ZHA_ERR_UNSUPPORTED),
    ("R", 3, zha.ZHA_ERR_UNSUPPORTED), ("max_depth", 1, zha.ZHA_ERR_BAD_ARG),
    ("max_depth", 17, zha.ZHA_ERR_BAD_ARG), ("max_depth", -1, zha.ZHA_ERR_BAD_ARG),
])
def test_bad_config(field, value, code):
    cfg = _cfg(workloads.WORKLOADS["wide_256k"])
    setattr(cfg, field, value)
    assert zha.zha_workspace_bytes(cfg) == code
    with pytest.raises(zha.ZhaError) as e:
        zha.zha_create(cfg, 1 << 20, 1 << 40)
    assert e.value.code == code


def test_create_rejects_workspace_before_cuda():
    cfg = _cfg(workloads.WORKLOADS["tiny_f32_16k"])
    need = zha.zha_workspace_bytes(cfg)
    for ptr, size in [(0, need), (256 * 1000, need - 1), (256 * 1000 + 8, need)]:
        with pytest.raises(zha.ZhaError) as e:
            zha.zha_create(cfg, ptr, size)
        assert e.value.code == zha.ZHA_ERR_BAD_ARG


def test_null_context_calls():
    assert zha.zha_n_tokens(None) == 0
    for fn, args in [(zha.lib.zha_build, (None, None, None, 1, None, 4, 2, None)),
                     (zha.lib.zha_append, (None, None, None, None)),
                     (zha.lib.zha_dense_decode, (None, None, None, None))]:
        assert fn(*args) == zha.ZHA_ERR_BAD_ARG
    assert zha.zha_strerror(zha.ZHA_ERR_CAPACITY) == "capacity exceeded"
    assert zha.zha_strerror(12345) == "unknown status"


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "tree_indexed_sparse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "zha_oracle" not in text and "liboracle" not in text, f
