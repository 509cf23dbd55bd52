"""Seeded synthetic inputs for the ZHA decode workloads.

This module is shared by the CUDA-path tests, the oracle tests and the
benchmark.  It holds no arithmetic of the method itself: it only draws the
keys, values, reference queries, decode queries, planted needles and appended
rows, from ``torch`` generators seeded per workload.

Recipe (one generator, seeded with the workload's seed; draws in this order):

1. reference queries ``ref[H_kv, R, d] ~ N(0, I)``; for bf16 caches they are
   rounded to bf16-representable values (kept as fp32), so a bf16 key times a
   reference query is exact in fp32;
2. decode queries ``Q[steps, H_q, d] ~ N(0, I)`` (fp32);
3. keys, one KV head at a time: either ``N(0, I)``, or a 64-component
   Gaussian mixture -- means ``mu[64, d] ~ N(0, I)`` drawn per KV head, one
   component ``z ~ U{0..63}`` per segment of 512 contiguous tokens, key
   ``mu[z] + 0.5 * N(0, I)``;
4. values ``V ~ N(0, I)``, one KV head at a time;
5. needles: every (step, query head) owns ``needles`` positions in its KV
   head, all distinct within the KV head; a quarter of them (when the
   workload asks for a tail) lie in the last 4,096 tokens (the last N/2 for
   N < 8,192), the rest are uniform over the tokens before that window from
   token 1 on (over ``[1, N)`` without a tail).  The key
   at a needle of query ``q`` is ``3 * q / |q| * sqrt(d) + eps`` with
   ``eps ~ N(0, 0.1 I)`` (variance 0.1);
6. the cache is cast to its storage dtype (bf16 or fp32);
7. appended rows (``k, v`` per KV head), drawn like the keys/values above;
   mixture keys continue the segment/component sequence past ``N``.

The pages' own workloads are a trained model's KV caches on long-context
benchmarks, which are not available here; these synthetic caches stand in for
them with the shapes of the five workloads below.  A generator on ``cuda``
draws different numbers than one on ``cpu`` for the same seed; every test and
benchmark generates on one device and moves copies to the other.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

SEGMENT = 512          # tokens sharing one mixture component
COMPONENTS = 64        # mixture components
TAIL = 4096            # "last 4K tokens" window for a quarter of the needles
NEEDLE_SCALE = 3.0
NEEDLE_NOISE_VAR = 0.1
MIX_SIGMA = 0.5


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    h_kv: int
    h_q: int
    d: int
    n_tokens: int
    c: int
    D: int
    R: int
    p: float
    steps: int
    kv_dtype: str             # "f32" or "bf16"
    keys: str                 # "normal" or "mixture"
    needles: int              # needles per (step, query head)
    needle_tail: bool         # a quarter of the needles in the last 4,096 tokens
    appends_per_step: int = 0  # appends before each decode step
    appends_after: int = 0     # appends after the decode steps

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def total_appends(self) -> int:
        return self.steps * self.appends_per_step + self.appends_after

    @property
    def capacity(self) -> int:
        return self.n_tokens + self.total_appends

    @property
    def torch_dtype(self):
        return torch.float32 if self.kv_dtype == "f32" else torch.bfloat16

    def scaled(self, n_tokens: int, steps: int | None = None, **kw) -> "Workload":
        """Same structure at another context length (for quick parity cases)."""
        return replace(self, n_tokens=n_tokens, steps=steps if steps is not None else self.steps,
                       name=f"{self.name}@{n_tokens}", **kw)


WORKLOADS = {
    # tiny fp32 case the oracle finishes in seconds: 4 top nodes of 4,096 tokens
    "tiny_f32_16k": Workload("tiny_f32_16k", 0, 1, 1, 64, 16384, 4, 6, 16, 0.95, 64, "f32",
                             "normal", 8, False),
    # wide tree: 1,024 leaf chunks of 256 tokens, one routing level
    "wide_256k": Workload("wide_256k", 1, 4, 16, 128, 262144, 256, 1, 16, 0.95, 128, "bf16",
                          "normal", 16, True),
    # deep tree: chunk 4, depth 6, two appends before every decode step
    "deep_256k": Workload("deep_256k", 2, 4, 16, 128, 262144, 4, 6, 16, 0.95, 128, "bf16",
                          "normal", 16, True, appends_per_step=2),
    # lightweight router: one reference query, chunk 8, depth 6, p = 0.75
    "light_1m": Workload("light_1m", 3, 4, 16, 128, 1048576, 8, 6, 1, 0.75, 128, "bf16",
                         "mixture", 16, True),
    # extreme length: 10M tokens, chunk 8, depth 7, 1,024 appends after decoding
    "extreme_10m": Workload("extreme_10m", 4, 4, 16, 128, 10485760, 8, 7, 1, 0.75, 64, "bf16",
                            "mixture", 16, True, appends_after=1024),
}

# the five workloads in the order the benchmark configuration lists them
ORDER = ["tiny_f32_16k", "wide_256k", "deep_256k", "light_1m", "extreme_10m"]


@dataclass
class Inputs:
    w: Workload
    K: torch.Tensor        # [H_kv, capacity, d] storage dtype; rows >= n_tokens are zero
    V: torch.Tensor
    ref: torch.Tensor      # [H_kv, R, d] fp32
    Q: torch.Tensor        # [steps, H_q, d] fp32
    needle_pos: torch.Tensor  # [H_kv, steps, G, needles] int64
    K_app: torch.Tensor    # [total_appends, H_kv, d] storage dtype
    V_app: torch.Tensor


def _keys(w: Workload, gen, device, n: int, seg0: int, means, comps_needed):
    """n keys of one KV head starting at segment index seg0."""
    if w.keys == "normal":
        return torch.randn(n, w.d, generator=gen, device=device)
    nseg = comps_needed
    z = torch.randint(0, COMPONENTS, (nseg,), generator=gen, device=device)
    seg = (torch.arange(n, device=device) + seg0 * SEGMENT) // SEGMENT - seg0
    return means[z[seg]] + MIX_SIGMA * torch.randn(n, w.d, generator=gen, device=device)


def generate(w: Workload, device: str = "cpu") -> Inputs:
    """Draw every input of workload ``w`` on ``device`` (see the module recipe)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    H, N, d, G = w.h_kv, w.n_tokens, w.d, w.group
    ref = torch.randn(H, w.R, d, generator=gen, device=device)
    if w.kv_dtype == "bf16":
        ref = ref.to(torch.bfloat16).to(torch.float32)
    Q = torch.randn(w.steps, w.h_q, d, generator=gen, device=device)

    K = torch.zeros(H, w.capacity, d, dtype=w.torch_dtype, device=device)
    V = torch.zeros(H, w.capacity, d, dtype=w.torch_dtype, device=device)
    means = []
    for kh in range(H):
        mu = torch.randn(COMPONENTS, d, generator=gen, device=device) if w.keys == "mixture" else None
        means.append(mu)
        nseg = math.ceil(N / SEGMENT)
        K[kh, :N] = _keys(w, gen, device, N, 0, mu, nseg).to(w.torch_dtype)
    for kh in range(H):
        V[kh, :N] = torch.randn(N, d, generator=gen, device=device).to(w.torch_dtype)

    # needles: [H_kv, steps, G, needles]
    per_kv = w.steps * G * w.needles
    pos = torch.empty(H, per_kv, dtype=torch.int64, device=device)
    for kh in range(H):
        if w.needle_tail:
            n_tail = w.steps * G * (w.needles // 4)
            n_body = per_kv - n_tail
            win = min(TAIL, N // 2)
            tail = (N - win) + torch.randperm(win, generator=gen, device=device)[:n_tail]
            body = 1 + torch.randperm(N - win - 1, generator=gen, device=device)[:n_body]
            # per query: needles//4 tail positions then the body positions
            tail = tail.view(w.steps * G, w.needles // 4)
            body = body.view(w.steps * G, w.needles - w.needles // 4)
            pos[kh] = torch.cat([tail, body], dim=1).reshape(-1)
        else:
            pos[kh] = 1 + torch.randperm(N - 1, generator=gen, device=device)[:per_kv]
    needle_pos = pos.view(H, w.steps, G, w.needles)
    for kh in range(H):
        qh = Q[:, kh * G:(kh + 1) * G, :]                            # [steps, G, d]
        unit = qh / qh.norm(dim=-1, keepdim=True)
        base = NEEDLE_SCALE * math.sqrt(d) * unit                      # [steps, G, d]
        noise = math.sqrt(NEEDLE_NOISE_VAR) * torch.randn(w.steps, G, w.needles, d,
                                                          generator=gen, device=device)
        keys = base[:, :, None, :] + noise
        K[kh, needle_pos[kh].reshape(-1)] = keys.reshape(-1, d).to(w.torch_dtype)

    n_app = w.total_appends
    K_app = torch.zeros(n_app, H, d, dtype=w.torch_dtype, device=device)
    V_app = torch.zeros(n_app, H, d, dtype=w.torch_dtype, device=device)
    if n_app:
        for kh in range(H):
            if w.keys == "mixture":
                seg0 = N // SEGMENT
                # the segment holding token N continues its own component draw
                nseg = math.ceil((N + n_app) / SEGMENT) - seg0
                z = torch.randint(0, COMPONENTS, (nseg,), generator=gen, device=device)
                seg = (torch.arange(N, N + n_app, device=device) // SEGMENT) - seg0
                k = means[kh][z[seg]] + MIX_SIGMA * torch.randn(n_app, d, generator=gen, device=device)
            else:
                k = torch.randn(n_app, d, generator=gen, device=device)
            K_app[:, kh] = k.to(w.torch_dtype)
        for kh in range(H):
            V_app[:, kh] = torch.randn(n_app, d, generator=gen, device=device).to(w.torch_dtype)
    return Inputs(w, K, V, ref, Q, needle_pos, K_app, V_app)
