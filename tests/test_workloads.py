"""The seeded generators: determinism, shapes and the needle recipe (CPU)."""
import math

import torch

import workloads


def test_deterministic_and_shapes():
    w = workloads.WORKLOADS["deep_256k"].scaled(9000, steps=3)
    a = workloads.generate(w)
    b = workloads.generate(w)
    for x, y in zip((a.K, a.V, a.ref, a.Q, a.needle_pos, a.K_app, a.V_app),
                    (b.K, b.V, b.ref, b.Q, b.needle_pos, b.K_app, b.V_app)):
        assert torch.equal(x, y)
    assert a.K.shape == (4, 9000 + 6, 128) and a.K.dtype == torch.bfloat16
    assert a.Q.shape == (3, 16, 128) and a.K_app.shape == (6, 4, 128)
    assert torch.all(a.K[:, 9000:] == 0)
    # reference queries are bf16-representable for a bf16 cache
    assert torch.equal(a.ref, a.ref.to(torch.bfloat16).float())


def test_needles():
    w = workloads.WORKLOADS["wide_256k"].scaled(20000, steps=4)
    inp = workloads.generate(w)
    G = w.group
    for kh in range(w.h_kv):
        pos = inp.needle_pos[kh].reshape(-1)
        assert pos.unique().numel() == pos.numel()
        assert pos.min() >= 1 and pos.max() < w.n_tokens
        tail = (pos >= w.n_tokens - workloads.TAIL).sum().item()
        assert tail == pos.numel() // 4
        for s in range(w.steps):
            for g in range(G):
                q = inp.Q[s, kh * G + g]
                k = inp.K[kh, inp.needle_pos[kh, s, g]].float()
                base = 3 * math.sqrt(w.d) * q / q.norm()
                noise = k - base
                # noise variance 0.1 (bf16 rounding of a norm-34 vector adds little)
                assert abs(noise.var().item() - 0.1) < 0.05


def test_mixture_segments():
    w = workloads.WORKLOADS["light_1m"].scaled(4096, steps=1)
    inp = workloads.generate(w)
    K = inp.K[0, :4096].float()
    needles = set(inp.needle_pos[0].reshape(-1).tolist())
    keep = torch.tensor([i not in needles for i in range(4096)])
    seg = torch.arange(4096) // workloads.SEGMENT
    # within a 512-token segment the keys scatter by sigma 0.5 around one mean
    for s in range(8):
        ks = K[(seg == s) & keep]
        assert abs(ks.std(dim=0).mean().item() - 0.5) < 0.05
