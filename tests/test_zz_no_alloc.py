"""zha_dense_decode_static (dense decode with the library's fixed scratch, no
context, no workspace) against zha_dense_decode on the same cache and against
the fp64 oracle's dense attention (needs a B200).  Kept in a file collected
last so that it also runs after every other GPU test in the same process; it
passes alone in a fresh process too.

The entry point serves callers that may not allocate device memory while
they serve.  After its first call on a device (which loads the module and
with it the fixed scratch), further calls must leave the device's free
memory unchanged.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import OUT_TOL

import tree_indexed_sparse_b200 as zha

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS
CASES = {
    "bf16_g4_d128": W["wide_256k"].scaled(16384 + 100, steps=2),
    "f32_tiny": W["tiny_f32_16k"].scaled(16384 - 3, steps=2),
}
SCRATCH = 8 * 1024 * 1024  # ZHA_STATIC_SCRATCH_BYTES of include/zha.h


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
    qs = [inp.Q[call % inp.Q.shape[0]].cuda().contiguous() for call in range(2)]
    outs = [torch.full((w.h_q, w.d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
    ref_outs = [cache.dense(q) for q in qs]
    torch.cuda.synchronize()
    for call in range(2):  # two calls in a row on the same scratch
        zha.zha_dense_decode_static(cfg, dK, dV, w.n_tokens, qs[call], outs[call], status, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == zha.ZHA_OK
        assert cache.status() == zha.ZHA_OK
        err = (outs[call] - ref_outs[call]).abs().max().item()
        print(f"{name} call {call}: max |static - context| = {err:.3e}")
        assert torch.isfinite(outs[call]).all()
        assert err <= tol
        # and directly against the oracle's exact dense attention
        out = outs[call].double().cpu().numpy()
        q = qs[call].double().cpu().numpy()
        for h in range(w.h_q):
            kh = h // w.group
            ref = oracle.attend(inp.K[kh], inp.V[kh], np.arange(w.n_tokens), q[h])
            assert np.max(np.abs(out[h] - ref)) <= tol, (name, call, h)


def test_static_dense_allocates_nothing_after_its_first_call():
    w = CASES["bf16_g4_d128"]
    inp, dK, dV, cache, dt = _case(w)
    cfg = zha.zha_config(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, 0, w.capacity)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = inp.Q[0].cuda().contiguous()
    out = torch.empty(w.h_q, w.d, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    zha.zha_dense_decode_static(cfg, dK, dV, w.n_tokens, q, out, status, stream)  # set-up call
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        zha.zha_dense_decode_static(cfg, dK, dV, w.n_tokens, q, out, status, stream)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert int(status.item()) == zha.ZHA_OK


def _fits(n_sm, h_kv, h_q, d):
    """The header's bound: partials of one CTA per SM (at most 256 CTAs), each
    h_q (d + 4) fp32, rounded up to 256 bytes, plus h_kv 4-byte tickets."""
    n_cta = min(256, n_sm)
    part = -(-(n_cta * h_q * (d + 4) * 4) // 256) * 256
    return part + h_kv * 4 <= SCRATCH


@pytest.mark.parametrize("d", [64, 128])
def test_static_dense_capacity_boundary(d):
    """The largest configuration that fits the fixed scratch is accepted and
    the next one up is rejected with ZHA_ERR_CAPACITY, on this GPU's SM count
    (groups of 4 query heads per KV head)."""
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    h_kv = 1
    while h_kv < 64 and _fits(n_sm, h_kv + 1, 4 * (h_kv + 1), d):
        h_kv += 1
    assert _fits(n_sm, h_kv, 4 * h_kv, d)
    n = 64
    tdt = torch.bfloat16
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for hk, ok in ((h_kv, True), (h_kv + 1, _fits(n_sm, h_kv + 1, 4 * (h_kv + 1), d))):
        if hk > 64:
            continue
        cfg = zha.zha_config(hk, 4 * hk, d, 1, 16, 1, zha.ZHA_BF16, 0, n)
        K = torch.randn(hk, n, d, device="cuda").to(tdt)
        q = torch.randn(4 * hk, d, device="cuda")
        out = torch.empty_like(q)
        if ok:
            zha.zha_dense_decode_static(cfg, K, K, n, q, out, status)
            torch.cuda.synchronize()
            assert int(status.item()) == zha.ZHA_OK
        else:
            with pytest.raises(zha.ZhaError) as e:
                zha.zha_dense_decode_static(cfg, K, K, n, q, out, status)
            assert e.value.code == zha.ZHA_ERR_CAPACITY


def test_static_dense_rejects_bad_args():
    K = torch.zeros(2, 1024, 128, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(8, 128, dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    small = zha.zha_config(2, 8, 128, 1, 16, 1, zha.ZHA_BF16, 0, 1024)
    with pytest.raises(zha.ZhaError) as e:  # n_tokens beyond the capacity
        zha.zha_dense_decode_static(small, K, K, 1025, q, out, status)
    assert e.value.code == zha.ZHA_ERR_BAD_ARG
    with pytest.raises(zha.ZhaError) as e:  # no status word
        zha.zha_dense_decode_static(small, K, K, 16, q, out, None)
    assert e.value.code == zha.ZHA_ERR_BAD_ARG
    torch.cuda.synchronize()
