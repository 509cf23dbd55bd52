"""zha_dense_decode_static (dense decode with the library's fixed scratch, no
context, no workspace) against zha_dense_decode on the same cache (needs a
B200).  Kept in a file collected last so that it also runs after every other
GPU test in the same process; it passes alone in a fresh process too.
"""
import pytest
import torch

import workloads
from parity import OUT_TOL

import tree_indexed_sparse_b200 as zha

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS
CASES = {
    "bf16_g4_d128": W["wide_256k"].scaled(16384 + 100, steps=2),
    "f32_tiny": W["tiny_f32_16k"].scaled(16384 - 3, steps=2),
}


def _case(w):
    inp = workloads.generate(w, "cpu")
    dK, dV, dref = inp.K.cuda(), inp.V.cuda(), inp.ref.cuda()
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity)
    cache.build(dK, dV, w.n_tokens, dref)
    return inp, dK, dV, cache, dt


@pytest.mark.parametrize("name", list(CASES))
def test_static_dense_matches_context_dense(name):
    w = CASES[name]
    inp, dK, dV, cache, dt = _case(w)
    tol = OUT_TOL[w.kv_dtype]
    cfg = zha.zha_config(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, 0, w.capacity)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):  # two calls in a row on the same scratch
        q = inp.Q[call % inp.Q.shape[0]].cuda().contiguous()
        ref_out = cache.dense(q)
        out = torch.full((w.h_q, w.d), float("nan"), dtype=torch.float32, device="cuda")
        zha.zha_dense_decode_static(cfg, dK, dV, w.n_tokens, q, out, status, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == zha.ZHA_OK
        assert cache.status() == zha.ZHA_OK
        err = (out - ref_out).abs().max().item()
        print(f"{name} call {call}: max |static - context| = {err:.3e}")
        assert torch.isfinite(out).all()
        assert err <= tol


def test_static_dense_rejects_oversized_and_bad_args():
    # partials of h_q = 128 heads at d = 128 on every SM exceed the fixed scratch
    cfg = zha.zha_config(32, 128, 128, 1, 16, 1, zha.ZHA_BF16, 0, 1024)
    K = torch.zeros(32, 1024, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(128, 128, dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(zha.ZhaError) as e:
        zha.zha_dense_decode_static(cfg, K, K, 1024, q, out, status)
    assert e.value.code == zha.ZHA_ERR_CAPACITY
    small = zha.zha_config(2, 8, 128, 1, 16, 1, zha.ZHA_BF16, 0, 1024)
    with pytest.raises(zha.ZhaError) as e:  # n_tokens beyond the capacity
        zha.zha_dense_decode_static(small, K, K, 1025, q, out, status)
    assert e.value.code == zha.ZHA_ERR_BAD_ARG
    with pytest.raises(zha.ZhaError) as e:  # no status word
        zha.zha_dense_decode_static(small, K, K, 16, q, out, None)
    assert e.value.code == zha.ZHA_ERR_BAD_ARG
    torch.cuda.synchronize()
