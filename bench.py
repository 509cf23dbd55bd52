#!/usr/bin/env python
"""Decode-step benchmark of the ZHA hot path on B200 (one JSON line on rank 0).

Metric: microseconds per decoded token per layer (batch 1, every query head),
plus HBM GB/s on the bytes the step must touch, next to a dense flash-decode
kernel over the same cache.

One step = what one decoded token costs one layer: zha_append of the token's
k, v (tree maintenance: the leaf and every ancestor are recomputed) followed by
zha_decode of its query (routing over every level, then exact attention over
the kept leaves plus the sink).  The full tree build is timed separately and
reported as build tokens/s.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launch stream; a 256 MiB buffer is written between steps (L2 flush)
outside the events.  The routing of every step is replayed first in an
untimed, traced pass (the decode is deterministic) to count the algorithmic
bytes; the cache is then rebuilt and the timed pass runs without tracing.
Inside a timed step nothing separates the append from the decode: the decode
is launched as a programmatic dependent of the append, and an event between
them would serialise that overlap.  The per-kernel split (append, decode,
and the decode's in-kernel phase stamps) therefore comes from a second pass
over the same K steps from a rebuilt cache, with a third event between the
two launches; the roofline entry uses that pass's decode durations.

--impl reference times the fp64 CPU oracle on the same workload instead.
Multi-GPU: --gpus N runs N replicas (each rank the whole workload on its
GPU); --kv-shards N times the workload split by KV head over N GPUs, each
shard alone on this GPU (shards exchange nothing while decoding).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "µs per decoded token per layer and HBM GB/s (ZHA vs dense) at 256K–10M ctx, 1 B200"
UNIT = "us/token"
DEFAULT_WORKLOAD = "extreme_10m"
APPEND_BURST = 256  # appends timed on their own for a workload whose schedule has none
FLUSH_BYTES = 256 << 20
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the measured copy peak is the roofline's denominator)
# a bounded GPU-side delay queued before each timed step, so the host has
# enqueued the whole step before the GPU reaches its first event
HOLD_CYCLES = 400_000


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def kernel_source_hash() -> str:
    """Hash of the CUDA sources: ncu counters stay valid only for the kernels
    they were taken on."""
    import glob
    import hashlib

    csrc = os.path.join(ROOT, "tree_indexed_sparse_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    """(bytes, note): per-launch DRAM bytes (read + write) of k_decode from the
    committed ncu record, or None with the reason when there is none for this
    workload or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "k_decode_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None, "no ncu record"
    if rec.get("source_hash") != kernel_source_hash():
        return None, "the kernel sources changed since the ncu capture"
    entry = rec.get("workloads", {}).get(workload)
    if not entry:
        return None, rec.get("not_captured", {}).get(workload, "this workload was not captured")
    return entry["dram_bytes"], (f"ncu capture of decode launch {entry['launch']} "
                                 f"(algorithmic {entry['algorithmic_bytes']:.0f} B, "
                                 f"dram/algorithmic {entry['dram_bytes'] / entry['algorithmic_bytes']:.3f})")


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value of x over all ranks (the job's time is its slowest
    rank's); x itself with one rank."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank: int, world: int, ms_max: float) -> float:
    """Replicas: every rank decodes its own token stream; whole-job microseconds
    per decoded token = slowest rank's time over all ranks' tokens."""
    return ms_max * 1000.0 / (units_per_rank * world)


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, local):
        self.proc = None
        # raw samples: ZHA_CLOCKS_DIR when set (to keep them), else a temp dir
        import tempfile

        out_dir = os.environ.get("ZHA_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"zha_clocks_rank{local}.csv")
        vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
        self.index = vis[local].strip() if local < len(vis) else str(local)

    def _lines(self):
        try:
            with open(self.path) as f:
                return sum(1 for line in f if line.count(",") >= 8)
        except OSError:
            return 0

    def start(self):
        """Launch the sampler and wait (up to 5 s) for its first sample, so that
        samples cover the timed region that follows."""
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while self._lines() < 1 and time.time() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.first = self._lines()
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # one more sample after the timed region, then stop
        t0 = time.time()
        n0 = self._lines()
        while self._lines() <= n0 and time.time() - t0 < 2.0 and self.proc.poll() is None:
            time.sleep(0.005)
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def step_bytes(w, trace_ids, trace_cnt, n_tokens, router_bf16=False):
    """Algorithmic bytes of one decode from its per-level kept sets.

    Routing reads each node of the union frontier of a KV head once (g and b:
    R*(d+1)*4 bytes, or R*(2d+4) with the bf16 router copy), whatever the
    number of its query heads that need it;
    attention reads the K and V rows of the union of the heads' token sets
    once; plus the queries and outputs."""
    c, D, d, R, G = w.c, w.D, w.d, w.R, w.group
    e = 4 if w.kv_dtype == "f32" else 2
    node = R * (2 * d + 4) if router_bf16 else R * (d + 1) * 4
    route = 0
    attn = 0
    slots_total = 0
    slots_level = [0] * (D + 1)
    for kh in range(w.h_kv):
        heads = range(kh * G, (kh + 1) * G)
        for level in range(D, 0, -1):
            if level == D:
                nodes = -(-n_tokens // c ** D)
            else:
                kept = set()
                for h in heads:
                    kept.update(trace_ids[level, h, :trace_cnt[level, h]].tolist())
                nb = -(-n_tokens // c ** level)
                nodes = sum(min(c, nb - k * c) for k in kept)
            route += nodes * node
            slots_total += nodes
            slots_level[level] += nodes
        leaves = set()
        sink = False
        for h in heads:
            lv = trace_ids[0, h, :trace_cnt[0, h]]
            leaves.update(lv.tolist())
            if len(lv) == 0 or lv[0] != 0:
                sink = True
        toks = sum(min(c, n_tokens - lf * c) for lf in leaves) + (1 if sink and 0 not in leaves else 0)
        attn += toks * 2 * d * e
    qo = w.h_q * d * 8
    return route, attn + qo, slots_total, slots_level


def append_bytes(w, n_after):
    """Bytes one zha_append must move: the new k, v rows, the leaf's keys,
    each ancestor's children (read) and the D recomputed nodes (written)."""
    c, D, d, R = w.c, w.D, w.d, w.R
    e = 4 if w.kv_dtype == "f32" else 2
    node_w = R * (d + 2) * 4
    node_r = R * (d + 1) * 4
    pos = n_after - 1
    leaf = pos // c
    b = 2 * d * e + (n_after - leaf * c) * d * e + D * node_w
    n = leaf
    for level in range(2, D + 1):
        n //= c
        nbelow = -(-n_after // c ** (level - 1))
        b += min(c, nbelow - n * c) * node_r
    return b * w.h_kv


def bench_workload(base, W, K):
    """The workload with room for the benchmark's appends: W + K steps of the
    workload's own appends per step, then its appends after the decodes (or,
    for a workload without appends, APPEND_BURST appends timed on their own)."""
    burst = base.appends_after or APPEND_BURST
    total = (W + K) * base.appends_per_step + burst
    return dataclasses.replace(base, appends_per_step=0, appends_after=total), base.appends_per_step, burst


def run_zha(args, rank, world, local):
    import tree_indexed_sparse_b200 as zha

    base = workloads.WORKLOADS[args.workload]
    W, K = args.warmup, args.steps
    w, per_step, burst = bench_workload(base, W, K)
    dev = torch.device("cuda", torch.cuda.current_device())
    t0 = time.time()
    inp = workloads.generate(w, "cuda")
    torch.cuda.synchronize()
    gen_s = time.time() - t0
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    router_bf16 = args.router == "bf16"
    nb = args.batch
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, device=dev,
                         router_dtype=zha.ZHA_BF16 if router_bf16 else zha.ZHA_F32, max_batch=nb)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    n1cap = -(-w.capacity // w.c)

    # build (timed, after one warm-up build)
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    torch.cuda.synchronize()
    flush.zero_()
    eb0, eb1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    eb0.record(stream)
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    eb1.record(stream)
    torch.cuda.synchronize()
    build_ms = eb0.elapsed_time(eb1)

    out = torch.empty(nb, w.h_q, w.d, dtype=torch.float32, device=dev)
    leaf_idx = torch.empty(nb, w.h_q, n1cap, dtype=torch.int32, device=dev)
    n_leaf = torch.empty(nb, w.h_q, dtype=torch.int32, device=dev)
    visited = torch.empty(nb, w.h_q, dtype=torch.int64, device=dev)
    # the queries of step i: [nb, h_q, d], consecutive queries of the workload
    qsteps = torch.stack([torch.stack([inp.Q[(i * nb + t) % w.steps] for t in range(nb)])
                          for i in range(max(w.steps, 1))])
    qs = qsteps if nb > 1 else inp.Q

    def decode(q, trace=None):
        if trace is None:
            zha.zha_decode_batch(cache.ctx, q, nb, w.p, out, leaf_idx, n1cap, n_leaf, visited, None, None, 0,
                                 stream.cuda_stream)
        else:
            zha.zha_decode_batch(cache.ctx, q, nb, w.p, out, leaf_idx, n1cap, n_leaf, visited, trace[0], trace[1],
                                 n1cap, stream.cuda_stream)

    def appends(i):
        """The appends of step i (the workload's own count per step)."""
        for j in range(per_step):
            r = i * per_step + j
            cache.append(inp.K_app[r], inp.V_app[r])

    # pass A: traced, untimed -- algorithmic bytes of every step, warm-up
    # steps included (one k_decode launch per step, in step order)
    tr_ids = torch.empty(w.D, nb * w.h_q, n1cap, dtype=torch.int32, device=dev)
    tr_cnt = torch.empty(w.D, nb * w.h_q, dtype=torch.int32, device=dev)
    per_step_all = []
    leaves_per_head, vis_per_head = [], []
    for i in range(W + K):
        appends(i)
        decode(qs[i % w.steps], (tr_ids, tr_cnt))
        ids = tr_ids.cpu().numpy()
        cnt = tr_cnt.cpu().numpy()
        n_now = w.n_tokens + (i + 1) * per_step
        rb, ab, slots, slots_level = 0, 0, 0, [0] * (w.D + 1)
        for t in range(nb):  # every query's own routing and token set
            sl = slice(t * w.h_q, (t + 1) * w.h_q)
            r_, a_, s_, l_ = step_bytes(w, ids[:, sl], cnt[:, sl], n_now, router_bf16)
            rb, ab, slots = rb + r_, ab + a_, slots + s_
            slots_level = [x + y for x, y in zip(slots_level, l_)]
        app_b = sum(append_bytes(w, n_now - per_step + j + 1) for j in range(per_step))
        per_step_all.append((rb, ab, app_b, slots, n_now, slots_level))
        if i >= W:
            leaves_per_head.append(n_leaf.float().mean().item())
            vis_per_head.append(visited.float().mean().item())
    timed_b = per_step_all[W:]
    ref_out = out.clone()
    assert cache.status() == 0, "device status not OK after the traced pass"
    if os.environ.get("ZHA_STEP_BYTES"):
        # per-launch algorithmic bytes of every k_decode of this pass, for
        # checking an ncu DRAM capture of launch i against its own step
        with open(os.environ["ZHA_STEP_BYTES"], "w") as f:
            json.dump({"workload": w.name, "warmup": W, "steps": K, "appends_per_step": per_step,
                       "decode_bytes": [r + a for r, a, *_ in per_step_all]}, f)

    # pass B: timed
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    stamps = torch.zeros(w.D + 3, dtype=torch.int64, device=dev)
    zha.zha_set_phase_timer(cache.ctx, stamps)
    ea, eb, ec = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    t_step, t_app, t_route, t_attn, t_merge, t_lvl, t_dec_c = [], [], [], [], [], [], []
    clocks = Clocks(local)
    for i in range(W):
        flush.zero_()
        appends(i)
        decode(qs[i % w.steps])
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    wall0 = time.time()
    for i in range(W, W + K):
        flush.zero_()
        torch.cuda._sleep(HOLD_CYCLES)
        ea.record(stream)
        appends(i)
        decode(qs[i % w.steps])
        ec.record(stream)
        torch.cuda.synchronize()
        t_step.append(ea.elapsed_time(ec))
    torch.cuda.synchronize()
    wall = time.time() - wall0
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    same = torch.equal(out, ref_out)
    total_ms = sum(t_step)
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_step = total_ms / K
    us_token = job_value(K * nb, world, total_ms)

    # appends after the decode steps (the workload's own count, or a burst of
    # APPEND_BURST for a workload without appends), back to back, one event
    # pair around all of them
    n_before = cache.n_tokens
    flush.zero_()
    torch.cuda._sleep(HOLD_CYCLES)
    ea.record(stream)
    for j in range(burst):
        r = (W + K) * per_step + j
        cache.append(inp.K_app[r], inp.V_app[r])
    eb.record(stream)
    torch.cuda.synchronize()
    burst_ms = ea.elapsed_time(eb)
    burst_b = sum(append_bytes(w, n_before + j + 1) for j in range(burst))
    assert cache.status() == 0

    # pass C: the same steps from a rebuilt cache, split per kernel by events
    # (appends, then the decode), with the decode's in-kernel stamps
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    for i in range(W + K):
        flush.zero_()
        torch.cuda._sleep(HOLD_CYCLES)
        ea.record(stream)
        appends(i)
        eb.record(stream)
        decode(qs[i % w.steps])
        ec.record(stream)
        torch.cuda.synchronize()
        if i < W:
            continue
        ns = stamps.tolist()
        if per_step:
            t_app.append(ea.elapsed_time(eb))
        dec = eb.elapsed_time(ec)
        t_dec_c.append(dec)
        # in-kernel stamps split the decode kernel; launch latency goes to routing
        t_route.append(dec - (ns[w.D + 2] - ns[w.D]) * 1e-6)
        t_attn.append((ns[w.D + 1] - ns[w.D]) * 1e-6)
        t_merge.append((ns[w.D + 2] - ns[w.D + 1]) * 1e-6)
        # levels D .. 1 as seen by the first CTA of KV head 0 (kernel start to
        # the end of level D, ..., end of level 2 to the end of the routing)
        t_lvl.append([(ns[j + 1] - ns[j]) * 1e-3 for j in range(w.D)])
    torch.cuda.synchronize()

    route_b = [s[0] for s in timed_b]
    attn_b = [s[1] for s in timed_b]
    app_b = [s[2] for s in timed_b]
    step_b = [r + a + p for r, a, p in zip(route_b, attn_b, app_b)]
    peak, peak_kind = peaks()
    gbs = sum(step_b) / (sum(t_step) * 1e-3) / 1e9
    phases = {
        "route": {"us": 1e3 * statistics.mean(t_route), "bytes": statistics.mean(route_b),
                  "gbs": sum(route_b) / (sum(t_route) * 1e-3) / 1e9},
        "attention": {"us": 1e3 * statistics.mean(t_attn), "bytes": statistics.mean(attn_b),
                      "gbs": sum(attn_b) / (sum(t_attn) * 1e-3) / 1e9},
        "merge": {"us": 1e3 * statistics.mean(t_merge)},
        "route_levels_us": {f"level_{w.D - i}": statistics.mean(x[i] for x in t_lvl) for i in range(w.D)},
    }
    if per_step:
        phases["appends_in_step"] = {"count": per_step, "us": 1e3 * statistics.mean(t_app),
                                     "bytes": statistics.mean(app_b),
                                     "gbs": sum(app_b) / (sum(t_app) * 1e-3) / 1e9}
    # the decode is one kernel (routing levels + attention + merge): its
    # algorithmic bytes over its event-timed duration (pass C)
    t_dec = t_dec_c
    dec_b = [r + a for r, a in zip(route_b, attn_b)]
    achieved = sum(dec_b) / (sum(t_dec) * 1e-3) / 1e9
    traffic, traffic_note = measured_traffic(w.name)
    roofline = {"bound": "hbm", "kernel": "k_decode", "launches_per_step": 1,
                "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                "peak_kind": f"{peak_kind} copy bandwidth (burst)", "traffic": traffic,
                "traffic_note": traffic_note,
                "algorithmic_bytes_per_launch": statistics.mean(dec_b), "us_per_launch": 1e3 * statistics.mean(t_dec)}

    # dense flash-decode over the same cache (every row present now)
    n_dense = cache.n_tokens
    e = 4 if w.kv_dtype == "f32" else 2
    dense_bytes = n_dense * w.h_kv * 2 * w.d * e + w.h_q * w.d * 8
    t_dense = []
    dout = torch.empty_like(out)
    for i in range(W + K):
        flush.zero_()
        torch.cuda._sleep(HOLD_CYCLES)
        ea.record(stream)
        zha.zha_dense_decode(cache.ctx, qs[i % w.steps], dout, stream.cuda_stream)
        eb.record(stream)
        torch.cuda.synchronize()
        if i >= W:
            t_dense.append(ea.elapsed_time(eb))
    dense_us = 1e3 * statistics.mean(t_dense)
    dense = {"us_per_token": dense_us, "hbm_gbs": dense_bytes / (dense_us * 1e-6) / 1e9,
             "frac": dense_bytes / (dense_us * 1e-6) / 1e9 / peak, "bytes": dense_bytes, "n_tokens": n_dense}

    # e2e: host buffers through the API, copies inside the timed region.  A
    # step's inputs (q, then the k and v of each of its appends) sit packed
    # in one pinned host row, so they cross in a single copy, as a serving
    # loop would send them; the device views of that row are the API's inputs.
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    qc, kc, vc = qs.cpu(), inp.K_app.cpu(), inp.V_app.cpu()
    qb = nb * w.h_q * w.d * 4
    kb = w.h_kv * w.d * kc.element_size()
    rows = []
    for i in range(W + K):
        parts = [qc[i % w.steps].contiguous().view(torch.uint8).flatten()]
        for j in range(per_step):
            r = i * per_step + j
            parts += [kc[r].contiguous().view(torch.uint8).flatten(), vc[r].contiguous().view(torch.uint8).flatten()]
        rows.append(torch.cat(parts))
    hin = torch.stack(rows).pin_memory()
    hout = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    din = torch.empty(qb + 2 * kb * per_step, dtype=torch.uint8, device=dev)
    dq = din[:qb].view(torch.float32).view(*qs.shape[1:])
    dkv = [(din[qb + 2 * kb * j:qb + 2 * kb * j + kb].view(inp.K.dtype).view(w.h_kv, w.d),
            din[qb + 2 * kb * j + kb:qb + 2 * kb * (j + 1)].view(inp.K.dtype).view(w.h_kv, w.d))
           for j in range(per_step)]
    t_e2e = []
    for i in range(W + K):
        flush.zero_()
        torch.cuda._sleep(HOLD_CYCLES)
        ea.record(stream)
        din.copy_(hin[i], non_blocking=True)
        for dk, dv in dkv:
            cache.append(dk, dv)
        decode(dq)
        hout.copy_(out, non_blocking=True)
        eb.record(stream)
        torch.cuda.synchronize()
        if i >= W:
            t_e2e.append(ea.elapsed_time(eb))
    h2d = din.numel()
    d2h = hout.numel() * 4
    e2e_us = 1e3 * sum(t_e2e) / K / world
    e2e_us = max_over_ranks(e2e_us, world, dev)

    step_desc = (f"{per_step} zha_append calls then one zha_decode" if per_step else "one zha_decode") + \
        (f" of one token, all query heads, batch 1, one layer" if nb == 1 else
         f"_batch of {nb} query tokens against the same cache, all query heads, one layer; value per query token")
    res = {
        "metric": METRIC, "value": us_token, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_step, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "n_tokens": w.n_tokens, "h_kv": w.h_kv, "h_q": w.h_q, "d": w.d,
                   "c": w.c, "D": w.D, "R": w.R, "p": w.p, "kv_dtype": w.kv_dtype, "keys": w.keys,
                   "step": step_desc,
                   "appends_after_steps": burst if base.appends_after else 0,
                   "router": "bf16 copy of g (reduced-precision router)" if router_bf16 else "fp32",
                   "queries_per_decode": nb,
                   "l2": "256 MiB written between steps, outside the per-step events",
                   "parallelism": f"replicas x{world}"},
        "hbm_gbs": gbs, "hbm_frac": gbs / peak,
        "step_us": {"mean": 1e3 * statistics.mean(t_step), "median": 1e3 * statistics.median(t_step),
                    "p10": 1e3 * float(np.percentile(t_step, 10)), "p90": 1e3 * float(np.percentile(t_step, 90))},
        "phases": phases,
        "roofline": roofline,
        "dense": dense, "speedup_vs_dense": dense_us / (1e3 * statistics.mean(t_step)),
        "build": {"ms": build_ms, "tokens_per_s": w.n_tokens / (build_ms * 1e-3)},
        "append": {"count": burst, "in_workload_schedule": bool(base.appends_after),
                   "us_per_append": 1e3 * burst_ms / burst, "tokens_per_s": burst / (burst_ms * 1e-3),
                   "bytes_per_append": burst_b / burst, "gbs": burst_b / (burst_ms * 1e-3) / 1e9},
        "routing": {"kept_leaves_per_head": statistics.mean(leaves_per_head),
                    "nodes_visited_per_head": statistics.mean(vis_per_head),
                    "keys_touched_frac": statistics.mean(leaves_per_head) * w.c / w.n_tokens,
                    "union_slots_per_step": statistics.mean(s[3] for s in timed_b),
                    "union_slots_per_level": {f"level_{lv}": statistics.mean(s[5][lv] for s in timed_b)
                                              for lv in range(w.D, 0, -1)},
                    "timed_pass_reproduces_traced": bool(same)},
        "e2e": {"value": e2e_us / nb, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk,
        "gpu_launches": K * (per_step + 1),
        "dense_note": "dense is timed for one query token per call",
        "gen_s": gen_s, "wall_timed_s": wall,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        del cache, flush
        torch.cuda.empty_cache()
        res["cpu_baseline"] = cpu_baseline(base, inp, args.cpu_seconds, W, K)
    return res


def cpu_baseline(base, inp, budget_s, W, K, steps_cap=None):
    """The fp64 oracle as it stands, on the host cores, on a bounded sample of
    the workload: the full build of every KV head's tree (OpenMP over KV
    heads), then steps of the workload's schedule (its appends, then the
    decode of every query head, OpenMP over query heads) until the time
    budget is spent; then a few steps on one thread.  Needs the host memory
    of the cache plus its fp64 trees."""
    import oracle

    nproc = os.cpu_count() or 1
    cores = min(16, nproc)
    w, per_step, _ = bench_workload(base, W, K)
    oracle.set_threads(cores)
    K_h = inp.K.cpu()
    V_h = inp.V.cpu()
    ref = inp.ref.cpu()
    Q = inp.Q.cpu()
    Ka = inp.K_app.cpu()
    Va = inp.V_app.cpu()
    # the workload's own rows (the device cache may hold appended rows)
    K_h[:, w.n_tokens:] = 0
    V_h[:, w.n_tokens:] = 0
    t0 = time.time()
    ht = oracle.build_heads(K_h, w.n_tokens, ref, w.c, w.D, capacity=w.capacity)
    build_s = time.time() - t0
    trees = [ht.head(kh) for kh in range(w.h_kv)]
    n = [w.n_tokens]

    def step(i):
        for j in range(per_step):
            r = i * per_step + j
            K_h[:, n[0]] = Ka[r]
            V_h[:, n[0]] = Va[r]
            for kh in range(w.h_kv):
                oracle.append_update(trees[kh], K_h[kh], ref[kh])
            n[0] += 1
            ht.n_tokens = n[0]
        oracle.decode_heads(K_h, V_h, ht, ref, Q[i % w.steps], w.p)

    done = 0
    t1 = time.time()
    while True:
        step(done)
        done += 1
        el = time.time() - t1
        if el > budget_s or done >= (steps_cap or (W + K)):
            break
    us = el / done * 1e6
    # one thread, a third of the budget
    oracle.set_threads(1)
    done1 = 0
    t2 = time.time()
    while True:
        step(done + done1)
        done1 += 1
        el1 = time.time() - t2
        if el1 > budget_s / 3 or done + done1 >= W + K:
            break
    oracle.set_threads(cores)
    sched = f"{per_step} appends + " if per_step else ""
    return {"value": us, "unit": UNIT, "cores": cores, "nproc": nproc, "kind": "oracle",
            "sample": f"{w.name}: full fp64 build of all {w.h_kv} KV-head trees ({build_s:.1f} s, "
                      f"{w.n_tokens / build_s:.0f} tokens/s, OpenMP over KV heads), then {done} steps of "
                      f"{sched}the decode of all {w.h_q} query heads (OpenMP over heads, {cores} threads)",
            "build_tokens_per_s": w.n_tokens / build_s,
            "single_thread": {"value": el1 / done1 * 1e6, "unit": UNIT, "steps": done1}}


def run_reference(args, rank, world):
    """The fp64 oracle as the reference arm, on rank 0 only."""
    if rank != 0:
        return None
    base = workloads.WORKLOADS[args.workload]
    W, K = args.warmup, args.steps
    w, _, _ = bench_workload(base, W, K)
    inp = workloads.generate(w, "cuda" if torch.cuda.is_available() else "cpu")
    cb = cpu_baseline(base, inp, args.cpu_seconds * 4, W, K, steps_cap=W + K)
    return {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": cb["value"] / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "n_tokens": w.n_tokens, "h_kv": w.h_kv, "h_q": w.h_q, "d": w.d,
                       "c": w.c, "D": w.D, "R": w.R, "p": w.p, "kv_dtype": w.kv_dtype},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_growth(args, local):
    """A tree whose depth grows with the context, measured where it grows:
    the light workload's settings (chunk 8, depth 6, R = 1, p = 0.75,
    mixture keys) at 2,097,152 - 4 tokens (8 top nodes of 262,144 tokens)
    with room for a 7th level.  Device times (L2 flushed before each call):
    decodes at depth 6, the appends up to and past 2,097,152 tokens (the
    5th adds the new top level), decodes at depth 7."""
    import tree_indexed_sparse_b200 as zha

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    base = workloads.WORKLOADS["light_1m"]
    steps, n_app = 16, 8
    N = base.c ** (base.D + 1) - 4
    w = dataclasses.replace(base.scaled(N, steps=steps), appends_per_step=0, appends_after=n_app)
    inp = workloads.generate(w, dev)
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, device=dev, max_depth=w.D + 1)
    cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
    out = torch.empty(w.h_q, w.d, dtype=torch.float32, device=dev)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        flush.zero_()
        torch.cuda._sleep(HOLD_CYCLES)
        ea.record(stream)
        fn()
        eb.record(stream)
        torch.cuda.synchronize()
        return ea.elapsed_time(eb) * 1e3

    depth0 = cache.depth
    before = [timed(lambda: cache.decode(inp.Q[i % steps], w.p, out=out)) for i in range(3 + steps)][3:]
    apps = []
    for i in range(n_app):
        d0 = cache.depth
        us = timed(lambda: cache.append(inp.K_app[i], inp.V_app[i]))
        apps.append({"n_tokens": cache.n_tokens, "depth": cache.depth, "adds_level": cache.depth > d0, "us": us})
    after = [timed(lambda: cache.decode(inp.Q[i % steps], w.p, out=out)) for i in range(3 + steps)][3:]
    assert cache.status() == 0
    grow = [x["us"] for x in apps if x["adds_level"]]
    plain = [x["us"] for x in apps if not x["adds_level"]]
    return {"metric": "growing depth: decode before and after the tree adds a level, and the append that adds it",
            "unit": "us", "n_gpus": 1, "steps": steps, "data": "synthetic",
            "config": {"workload": f"light_1m settings at {N} tokens, depth {w.D} growing to {w.D + 1}",
                       "l2": "256 MiB written before every call"},
            "depth_before": depth0, "depth_after": cache.depth,
            "decode_us_before": statistics.median(before), "decode_us_after": statistics.median(after),
            "append_us_adding_level": grow[0] if grow else None,
            "append_us_other": statistics.median(plain) if plain else None, "appends": apps}


CROSSOVER_N = [16384, 32768, 49152, 65536, 98304, 131072, 196608, 262144, 524288, 1048576]


def run_crossover(args, local):
    """The light workload's settings (chunk 8, R = 1, p = 0.75, mixture keys)
    at growing context lengths: device time of one routed decode and of one
    dense decode per length (L2 flushed between calls), and the length at
    which the two curves cross (linear interpolation)."""
    import tree_indexed_sparse_b200 as zha

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    base = workloads.WORKLOADS["light_1m"]
    steps = 32
    rows = []
    for n in CROSSOVER_N:
        D = 1  # deepest tree with at least 4 top nodes, as at 1M (c^D * 4 <= n)
        while D < base.D and base.c ** (D + 1) * 4 <= n:
            D += 1
        w = dataclasses.replace(base.scaled(n, steps=steps), D=D, appends_per_step=0, appends_after=0)
        inp = workloads.generate(w, dev)
        dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
        cache = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, device=dev)
        cache.build(inp.K, inp.V, w.n_tokens, inp.ref)
        out = torch.empty(w.h_q, w.d, dtype=torch.float32, device=dev)
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tz, td = [], []
        for i in range(3 + steps):
            q = inp.Q[i % steps]
            for fn, acc in ((lambda: cache.decode(q, w.p, out=out), tz), (lambda: cache.dense(q, out=out), td)):
                flush.zero_()
                torch.cuda._sleep(HOLD_CYCLES)
                ea.record(stream)
                fn()
                eb.record(stream)
                torch.cuda.synchronize()
                if i >= 3:
                    acc.append(ea.elapsed_time(eb) * 1e3)
        assert cache.status() == 0
        rows.append({"n_tokens": n, "D": D, "zha_us": statistics.median(tz), "dense_us": statistics.median(td)})
        del cache, inp
        torch.cuda.empty_cache()
    cross = None
    for a, b in zip(rows, rows[1:]):
        da, db = a["zha_us"] - a["dense_us"], b["zha_us"] - b["dense_us"]
        if da >= 0 > db:
            cross = a["n_tokens"] + (b["n_tokens"] - a["n_tokens"]) * da / (da - db)
            break
    if cross is None and rows and rows[0]["zha_us"] < rows[0]["dense_us"]:
        cross = f"< {rows[0]['n_tokens']}"
    return {"metric": "crossover context length, routed vs dense decode (light workload settings)",
            "unit": "tokens", "value": cross, "higher_is_better": False, "n_gpus": 1, "steps": steps,
            "data": "synthetic", "rows": rows,
            "config": {"workload": "light_1m settings at each n_tokens (depth: at least 4 top nodes)",
                       "l2": "256 MiB written before every call"}}


def run_kv_shards(args, local):
    """KV-head sharding of the workload over N GPUs, measured on one GPU: each
    shard (its KV heads' cache, built from the same inputs) decodes every
    step alone, L2 flushed before each call; shards share no data on the
    decode path, so an N-GPU job's time per token is the slowest shard's.
    The whole cache is timed beside them on the same steps."""
    import tree_indexed_sparse_b200 as zha
    from tree_indexed_sparse_b200.shard import ShardedZhaCache

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    w = workloads.WORKLOADS[args.workload]
    N = args.kv_shards
    W, K = args.warmup, args.steps
    inp = workloads.generate(w, dev)
    dt = zha.ZHA_BF16 if w.kv_dtype == "bf16" else zha.ZHA_F32
    whole = zha.ZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, device=dev)
    whole.build(inp.K, inp.V, w.n_tokens, inp.ref)
    shards = []
    for r in range(N):
        sh = ShardedZhaCache(w.h_kv, w.h_q, w.d, w.R, w.c, w.D, dt, w.capacity, rank=r, world=N, device=dev)
        sh.build(sh.local_kv(inp.K).contiguous(), sh.local_kv(inp.V).contiguous(), w.n_tokens,
                 sh.local_kv(inp.ref).contiguous())
        shards.append(sh)
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        flush.zero_()
        torch.cuda._sleep(HOLD_CYCLES)
        ea.record(stream)
        fn()
        eb.record(stream)
        torch.cuda.synchronize()
        return ea.elapsed_time(eb) * 1e3

    t_whole, t_shard = [], [[] for _ in range(N)]
    clocks = Clocks(local)
    for i in range(W + K):
        q = inp.Q[i % w.steps]
        if i == W:
            clocks.start()
        tw = timed(lambda: whole.decode(q, w.p))
        ts = [timed(lambda: sh.decode(q, w.p)) for sh in shards]
        if i >= W:
            t_whole.append(tw)
            for r in range(N):
                t_shard[r].append(ts[r])
    clk = clocks.stop()
    assert whole.status() == 0 and all(sh.status() == 0 for sh in shards)
    per_step = [max(t_shard[r][i] for r in range(N)) for i in range(K)]
    job_us = statistics.mean(per_step)
    return {"metric": "us per decoded token per layer, KV heads split over N GPUs (each shard timed alone on one GPU)",
            "unit": "us/token", "value": job_us, "higher_is_better": False, "n_gpus_emulated": N, "steps": K,
            "warmup": W, "scaling": "strong", "data": "synthetic",
            "whole_cache_us": statistics.mean(t_whole), "speedup": statistics.mean(t_whole) / job_us,
            "shards": [{"kv_heads": [sh.kv0, sh.kv1], "us": statistics.mean(t_shard[r])} for r, sh in enumerate(shards)],
            "clocks": clk,
            "config": {"workload": w.name, "parallelism": f"kv-heads x{N} (emulated: shards run one after another)",
                       "l2": "256 MiB written before every call"}}


def record_traffic(csv_path: str, steps_path: str, launch: int) -> None:
    """Write profiles/k_decode_traffic.json from one ncu capture: the DRAM
    bytes (read + write) of k_decode launch `launch` (0-based, the first
    traced pass of this script runs the decodes in step order) from the ncu
    CSV, next to that launch's algorithmic bytes from the ZHA_STEP_BYTES file
    of the same command, under the hash of the kernel sources they were
    taken on."""
    import csv

    rows = list(csv.reader(open(csv_path)))
    hdr = next(i for i, r in enumerate(rows) if "Metric Name" in r)
    cols = rows[hdr]
    name_i, metric_i, value_i = cols.index("Kernel Name"), cols.index("Metric Name"), cols.index("Metric Value")
    unit_i = cols.index("Metric Unit")
    scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "ns": 1e-3, "usecond": 1.0, "us": 1.0,
             "msecond": 1e3, "ms": 1e3}
    vals = {}  # bytes, or microseconds for the duration
    for r in rows[hdr + 1:]:
        if len(r) > value_i and "k_decode" in r[name_i]:
            vals[r[metric_i]] = float(r[value_i].replace(",", "")) * scale.get(r[unit_i], 1.0)
    dram = vals["dram__bytes_read.sum"] + vals["dram__bytes_write.sum"]
    steps = json.load(open(steps_path))
    algo = steps["decode_bytes"][launch]
    path = os.path.join(ROOT, "profiles", "k_decode_traffic.json")
    try:
        rec = json.load(open(path))
    except (OSError, ValueError):
        rec = {}
    if rec.get("source_hash") != kernel_source_hash():
        rec = {"source_hash": kernel_source_hash(), "workloads": {}, "not_captured": rec.get("not_captured", {})}
    rec["not_captured"]["extreme_10m"] = ("not captured: its cache holds about 24 GB on the device, above the size "
                                          "at which a counter capture may run on this pool")
    rec["workloads"][steps["workload"]] = {"launch": launch, "dram_bytes": dram, "algorithmic_bytes": algo,
                                           "ncu_duration_us": vals.get("gpu__time_duration.sum")}
    with open(path, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec["workloads"][steps["workload"]]))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["zha", "reference"], default="zha")
    ap.add_argument("--workload", choices=workloads.ORDER, default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--crossover", action="store_true",
                    help="sweep the light workload's settings over context lengths, routed vs dense")
    ap.add_argument("--batch", type=int, default=1,
                    help="query tokens per decode call (zha_decode_batch); value is per query token")
    ap.add_argument("--router", choices=["f32", "bf16"], default="f32",
                    help="summaries the routing reads: fp32 (default) or the bf16 router copy")
    ap.add_argument("--growth", action="store_true",
                    help="time the step where a tree with room to grow adds a level (light settings, 2M tokens)")
    ap.add_argument("--kv-shards", type=int, default=0, metavar="N",
                    help="time the workload split by KV head over N GPUs, each shard alone on this GPU")
    ap.add_argument("--record-traffic", nargs=3, metavar=("NCU_CSV", "STEP_BYTES_JSON", "LAUNCH"),
                    help="write profiles/k_decode_traffic.json from an ncu capture of k_decode (no GPU needed)")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args.record_traffic[0], args.record_traffic[1], int(args.record_traffic[2]))
        return
    args.warmup = max(args.warmup, 3)
    rank, world, local = dist_setup(args.gpus)
    if args.crossover or args.growth or args.kv_shards:
        if rank == 0:
            run = run_crossover if args.crossover else run_growth if args.growth else run_kv_shards
            print(json.dumps(run(args, local)), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_zha(args, rank, world, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
