"""Benchmark: coefficient-domain decode attention over the int8 block-DCT
archive (archive GB/s and fraction of the HBM roofline) plus prefill
compression tokens/s, on synthetic AR(1) K/V.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fc|reference]
                    [--workload long]

One step is one decode step of the workload over one batch: append one token
per (batch, kv head) to K and V (every R-th step archives a block through the
compress + quantise path) and run decode attention over archive + raw tail.
Inputs stay resident in HBM; ``copies`` independent archives (together more
than twice the L2) are visited round-robin so no step reads the previous
one's archive from L2. The K steps are captured once into a CUDA graph with
their per-step arguments and replayed; replays rewrite identical bytes, so
every replay is exactly K steps of work.

For N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the workload (weak scaling: (batch, kv head) work shards with no exchange);
times are the max over ranks.
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
Q_POOL = 64


# ----------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    """One process per GPU; the process group only carries the barrier and
    the max-over-ranks timing (the replicas exchange no data)."""
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(
                seconds=120), device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(
                seconds=120))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank_step: float, world: int,
                  max_step_s: float) -> float:
    """Weak scaling: every rank streams its own replica of the workload, so
    the job moves world x the per-rank bytes per step in the slowest rank's
    step time."""
    return world * bytes_per_rank_step / max_step_s / 1e9


def measured_hbm_gbs():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" +
                 self.FIELDS, "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.15)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        if not getattr(self, "out", ""):
            return None
        rows = [r for r in csv.reader(io.StringIO(self.out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# the files the tensor-core decode-attention kernel is compiled from
DECODE_SOURCES = ("include/fc.h",
                  "compressed_decode_attention_blockwise_b200/csrc/fc_internal.cuh",
                  "compressed_decode_attention_blockwise_b200/csrc/fc_encode.cuh",
                  "compressed_decode_attention_blockwise_b200/csrc/fc_decode.cuh",
                  "compressed_decode_attention_blockwise_b200/csrc/fc_tc_ptx.cuh",
                  "compressed_decode_attention_blockwise_b200/csrc/fc_decode_tc.cu")


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(rel.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(name: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, or None when absent or taken on different kernel sources."""
    p = os.path.join(ROOT, "profiles", name)
    try:
        txt = open(p).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    hsh = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", txt)
    if not m or not hsh or hsh.group(1) != kernel_source_hash():
        return None
    return float(m.group(1))


# ------------------------------------------------------------ the fc arm

def attention_bytes(cache, Hq: int, q_elem: int, out_elem: int) -> int:
    """Algorithmic bytes of one decode-attention launch: live archive (codes
    and scales, K and V) + live raw tail (K and V) + q + out."""
    b = cache.k.storage_bytes() + cache.v.storage_bytes()
    return b + cache.B * Hq * cache.D * (q_elem + out_elem)


ROOF_LAUNCHES = 600
# fc_decode_attention flag modes of the roofline legs: (overlap, q_final)
MODES = {"isolated": (False, False), "overlap": (True, False),
         "overlap_q_final": (True, True)}


def attention_modes(caches, q_pool, out_bufs, n_launch, W, world,
                    modes=MODES):
    """Mean per-launch time of fc_decode_attention in each flag mode: one
    CUDA graph of ``n_launch`` launches over the archive copies round-robin
    (each launch reads a different copy than the previous one), timed with
    CUDA events on the launching stream after W warm-up replays.
    isolated: no flags, each launch starts after the previous one completed;
    overlap: FC_DECODE_OVERLAP, the next launch streams its archive while the
    previous drains (valid in any decode loop); overlap_q_final: also
    FC_DECODE_Q_FINAL (q final before the previous launch started)."""
    copies = len(caches)
    ev0, ev1 = torch.cuda.Event(True), torch.cuda.Event(True)
    res = {}
    for name, (ov, qf) in modes.items():
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n_launch):
                c = i % copies
                caches[c].attention(q_pool[i % len(q_pool)], out=out_bufs[c],
                                    overlap=ov, q_final=qf)
        for _ in range(max(W, 3)):
            g.replay()
        torch.cuda.synchronize()
        barrier(world)
        ev0.record()
        g.replay()
        ev1.record()
        torch.cuda.synchronize()
        res[name] = max_over_ranks(ev0.elapsed_time(ev1) / 1e3 / n_launch,
                                   world)
        del g
    return res


def bench_workload(name, peak, W, world, dev, l2, budget_s=0.25):
    """Decode-attention throughput of one more workload at its full size
    (archive copies round-robin above twice the L2), in the three flag
    modes; the number of launches per graph keeps each replay near
    ``budget_s``."""
    from compressed_decode_attention_blockwise_b200 import CodecKVCache
    w = synth.WORKLOADS[name]
    tok_dt = synth.torch_dtype(w.in_dtype)
    esz = torch.tensor([], dtype=tok_dt).element_size()
    data = synth.generate(w.replace(steps=0), q_steps=Q_POOL)
    kd, vd = data["k"].to(dev), data["v"].to(dev)
    del data["k"], data["v"]
    arc_bytes = None
    caches = []
    while True:
        c = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                         token_dtype=tok_dt, device=dev)
        c.prefill(kd[:, :, :w.T], vd[:, :, :w.T])
        caches.append(c)
        arc_bytes = c.storage_bytes()
        if len(caches) * arc_bytes > 2 * l2:
            break
    del kd, vd
    q_pool = data["q"].to(dev)
    outs = [torch.empty((w.B, w.Hq, 1, w.D), dtype=torch.float32,
                        device=dev) for _ in caches]
    for i, c in enumerate(caches):
        c.attention(q_pool[0], out=outs[i])
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    caches[0].attention(q_pool[0], out=outs[0])
    torch.cuda.synchronize()
    one = max(time.perf_counter() - t0, 1e-6)
    n = int(max(20, min(ROOF_LAUNCHES, budget_s / one)))
    modes = attention_modes(caches, q_pool, outs, n, W, world)
    nbytes = attention_bytes(caches[0], w.Hq, esz, 4)
    entry = {"bytes_per_launch": int(nbytes), "launches": n,
             "archive_copies": len(caches),
             "kernel": "tensor-core" if caches[0].tensor_core_path(w.Hq)
             else "cuda-core"}
    for m, t in modes.items():
        entry[m] = {"us_per_launch": round(t * 1e6, 3),
                    "GB_per_s": round(nbytes / t / 1e9, 2),
                    "frac": round(nbytes / t / 1e9 / peak, 4)}
    del caches, outs
    torch.cuda.empty_cache()
    return entry


def bench_layers(w, kd, vd, q_pool, dev, W, world, n_layers=8,
                 n_steps=16):
    """Decode steps of n_layers independent layer caches of the workload:
    one fc_decode_step_layers launch per step against n_layers separate
    fc_decode_step launches, each plain and with the overlap flags. CUDA
    graphs of n_steps steps; microseconds per layer-step."""
    from compressed_decode_attention_blockwise_b200 import (
        CodecKVCache, decode_step_layers)
    tok_dt = synth.torch_dtype(w.in_dtype)
    esz = torch.tensor([], dtype=tok_dt).element_size()
    need = (w.T + n_steps) // w.R + 1

    def make():
        cs = []
        for _ in range(n_layers):
            c = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                             token_dtype=tok_dt, device=dev, capacity=need)
            c.prefill(kd[:, :, :w.T], vd[:, :, :w.T])
            cs.append(c)
        return cs

    outs = [torch.empty((w.B, w.Hq, 1, w.D), dtype=torch.float32,
                        device=dev) for _ in range(n_layers)]
    ev0, ev1 = torch.cuda.Event(True), torch.cuda.Event(True)
    res = {"layers": n_layers, "steps": n_steps}
    modes = {"one_launch": (False, False), "separate": (False, False),
             "one_launch_overlap_q_final": (True, True),
             "separate_overlap_q_final": (True, True)}
    for name, flags in modes.items():
        caches = make()
        for c in caches:
            c.workspace(w.Hq, c.num_splits(w.Hq))
        torch.cuda.synchronize()
        step_bytes = []
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for s in range(n_steps):
                t = w.T + s
                q = q_pool[s % len(q_pool)]
                kn, vn = kd[:, :, t:t + 1], vd[:, :, t:t + 1]
                if name.startswith("one_launch"):
                    decode_step_layers(caches, [q] * n_layers,
                                       [kn] * n_layers, [vn] * n_layers,
                                       outs=outs, overlap=flags[0],
                                       q_final=flags[1])
                else:
                    for l, c in enumerate(caches):
                        c.step(q, kn, vn, out=outs[l], overlap=flags[0],
                               q_final=flags[1])
                step_bytes.append(sum(attention_bytes(c, w.Hq, esz, 4)
                                      for c in caches))
        for _ in range(max(W, 3)):
            g.replay()
        torch.cuda.synchronize()
        barrier(world)
        ev0.record()
        g.replay()
        ev1.record()
        torch.cuda.synchronize()
        t_rep = max_over_ranks(ev0.elapsed_time(ev1) / 1e3, world)
        per = t_rep / (n_steps * n_layers)
        res[name] = {"us_per_layer": round(per * 1e6, 3),
                     "GB_per_s": round(sum(step_bytes) / t_rep / 1e9, 2)}
        del g, caches
        torch.cuda.empty_cache()
    return res


def run_fc(args, world, rank, local):
    from compressed_decode_attention_blockwise_b200 import CodecKVCache, _lib

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    K, W = args.steps, args.warmup
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    tok_dt = synth.torch_dtype(w.in_dtype)
    esz = torch.tensor([], dtype=tok_dt).element_size()
    per_block = 0
    for coeff in (w.k_coeff, w.v_coeff):
        per_block += w.S * w.D * {"i8": 1, "bf16": 2, "f32": 4}[coeff] + \
            (w.S * 4 if coeff == "i8" else 0)
    arc_bytes = w.B * w.Hk * w.n_blocks * per_block
    copies = args.copies or max(1, math.ceil(2 * l2 / max(arc_bytes, 1)))
    if arc_bytes < 2 * l2:
        copies = max(copies, 2)
    per_copy = -(-K // copies)
    extra = 2 * per_copy + 1          # graph steps, then the e2e steps
    data = synth.generate(w.replace(steps=extra), q_steps=Q_POOL)
    k_all, v_all = data["k"], data["v"]
    q_pool = data["q"].to(dev)
    need_blocks = (w.T + extra) // w.R + 1

    caches = []
    kd, vd = k_all.to(dev), v_all.to(dev)
    for _ in range(copies):
        c = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                         token_dtype=tok_dt, device=dev, capacity=need_blocks)
        c.prefill(kd[:, :, :w.T], vd[:, :, :w.T])
        caches.append(c)
    torch.cuda.synchronize()
    caps = [c.k.capacity for c in caches]

    # ---------------- prefill compression (rows a2, a3): tokens/s
    scratch = CodecKVCache(w.B, w.Hk, w.D, w.R, w.S, w.k_coeff, w.v_coeff,
                           token_dtype=tok_dt, device=dev,
                           capacity=w.n_blocks)
    kp, vp = kd[:, :, :w.T], vd[:, :, :w.T]

    def compress_once():
        for st, x in ((scratch.k, kp), (scratch.v, vp)):
            st.arc.n_blocks = 0
            st.tail_desc.len = 0
            _lib.fc_compress_blocks(x, st.arc, st.tail_desc)

    n_comp = max(3, min(K, 30))
    for _ in range(max(W, 3)):
        compress_once()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(True), torch.cuda.Event(True)
    barrier(world)
    ev0.record()
    for _ in range(n_comp):
        compress_once()
    ev1.record()
    torch.cuda.synchronize()
    comp_s = max_over_ranks(ev0.elapsed_time(ev1) / 1e3 / n_comp, world)
    comp_bytes = 2 * w.B * w.Hk * w.T * w.D * esz + arc_bytes
    del scratch

    # ---------------- reconstructed view: every archived block of K and V
    # decoded to the token dtype plus the raw tails (fc_read_view)
    views = [torch.empty((w.B, w.Hk, w.T, w.D), dtype=tok_dt, device=dev)
             for _ in range(2)]

    def view_once():
        for st, o in zip((caches[0].k, caches[0].v), views):
            _lib.fc_read_view(st.arc, st.tail_desc, 0, o)

    n_view = max(3, min(K, 30))
    for _ in range(max(W, 3)):
        view_once()
    torch.cuda.synchronize()
    barrier(world)
    ev0.record()
    for _ in range(n_view):
        view_once()
    ev1.record()
    torch.cuda.synchronize()
    view_s = max_over_ranks(ev0.elapsed_time(ev1) / 1e3 / n_view, world)
    view_bytes = arc_bytes + 2 * w.B * w.Hk * w.D * esz * (w.T + w.n_tail)
    del views

    Hq = w.Hq
    out_bufs = [torch.empty((w.B, Hq, 1, w.D), dtype=torch.float32,
                            device=dev) for _ in range(copies)]
    for i, c in enumerate(caches):      # allocate workspaces before capture
        c.attention(q_pool[0], out=out_bufs[i])
    torch.cuda.synchronize()

    # ---------------- attention-only graphs: per-launch duration (roofline)
    # ROOF_LAUNCHES launches whatever --steps is, so that the first launch of
    # a replay (which cannot overlap the previous replay) weighs little
    att_bytes = [attention_bytes(c, Hq, esz, 4) for c in caches]
    modes = attention_modes(caches, q_pool, out_bufs, ROOF_LAUNCHES, W, world)
    att_launch_s = modes["overlap_q_final"]
    iso_launch_s = modes["isolated"]
    att_bytes_mean = sum(att_bytes[i % copies]
                         for i in range(ROOF_LAUNCHES)) / ROOF_LAUNCHES

    # ---------------- decode steps (append + attention), CUDA graph
    step_bytes = []
    g_step = torch.cuda.CUDAGraph()
    pos = [w.T] * copies
    with torch.cuda.graph(g_step):
        for i in range(K):
            c = i % copies
            t = pos[c]
            caches[c].step(q_pool[i % Q_POOL], kd[:, :, t:t + 1],
                           vd[:, :, t:t + 1], out=out_bufs[c],
                           overlap=True, q_final=True)
            pos[c] += 1
            step_bytes.append(attention_bytes(caches[c], Hq, esz, 4))
    assert [c.k.capacity for c in caches] == caps, "archive grew in capture"
    for _ in range(max(W, 3)):
        g_step.replay()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev0.record()
        g_step.replay()
        ev1.record()
        torch.cuda.synchronize()
    step_s = max_over_ranks(ev0.elapsed_time(ev1) / 1e3 / K, world)
    bytes_per_step = sum(step_bytes) / K

    # ---------------- e2e through the C ABI with host buffers
    # each step's inputs (new K and V token, query) as one contiguous pinned
    # host block, copied to the device inside the call
    n_e2e = min(K, per_copy * copies)
    nk = w.B * w.Hk * w.D
    nq = w.B * Hq * w.D
    host_in = torch.empty((n_e2e, 2 * nk + nq), dtype=tok_dt,
                          pin_memory=True)
    pos_e = list(pos)
    for i in range(n_e2e):
        c = i % copies
        t = pos_e[c]
        host_in[i, :nk] = k_all[:, :, t].reshape(-1)
        host_in[i, nk:2 * nk] = v_all[:, :, t].reshape(-1)
        host_in[i, 2 * nk:] = data["q"][i % Q_POOL].reshape(-1)
        pos_e[c] += 1
    host_out = torch.empty((copies, w.B, Hq, 1, w.D), dtype=torch.float32,
                           pin_memory=True)
    # one fc_decode_step_host call per step (host block in, host output
    # out, the copies and the fused step inside the call), its arguments
    # marshalled before the timed region
    staging = [torch.empty(_lib.fc_decode_step_staging_bytes(
        w.B, w.Hk, Hq, w.D, tok_dt, torch.float32), dtype=torch.uint8,
        device=dev) for _ in range(copies)]
    calls = []
    for i in range(n_e2e):
        c = i % copies
        calls.append(_lib.HostStep(
            caches[c], Hq, host_in[i], host_out[c], staging[c],
            caches[c].workspace(Hq, caches[c].num_splits(Hq)),
            overlap=True, q_final=True))
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    ev0.record()
    for call in calls:
        call()
    ev1.record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    e2e_s = max_over_ranks(max(ev0.elapsed_time(ev1) / 1e3, wall) / n_e2e,
                           world)
    # bytes streamed per step: the archives and tails as the loop left them
    # differ from the per-step values by at most one token per step, so the
    # mean is taken from the state before and after the loop
    e2e_bytes = 0.5 * (sum(step_bytes[-copies:]) / copies +
                       sum(attention_bytes(cc, Hq, esz, 4)
                           for cc in caches) / copies)
    h2d = (2 * w.B * w.Hk * w.D * esz) + w.B * Hq * w.D * esz
    d2h = w.B * Hq * w.D * 4
    assert torch.isfinite(host_out).all()

    peak, peak_kind = measured_hbm_gbs()
    achieved = att_bytes_mean / att_launch_s / 1e9
    value = whole_job_gbs(bytes_per_step, world, step_s)
    res = {
        "metric": "decode-attn archive GB/s (coefficient-domain split-K "
                  "decode step: append + attention)",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(step_s * 1e3, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic AR(1) K/V (seeded), int8 block-DCT archive",
        "config": {
            "workload": w.name, "B": w.B, "Hq": w.Hq, "Hk": w.Hk, "D": w.D,
            "T": w.T, "R": w.R, "S": w.S, "k_coeff": w.k_coeff,
            "v_coeff": w.v_coeff, "q_tail_dtype": w.in_dtype, "rho": w.rho,
            "outlier_frac": w.outlier_frac, "seed": w.seed,
            "archive_copies": copies,
            "l2": "inputs larger than L2: %d archive copies (%.0f MB) visited "
                  "round-robin" % (copies, copies * arc_bytes / 1e6),
            "timing": "one CUDA-graph replay of K captured steps, CUDA events",
            "launch": "decode step = fc_decode_step (append + attention in one launch) with FC_DECODE_OVERLAP | FC_DECODE_Q_FINAL (programmatic dependent launch after the previous step; q is written before the graph runs); roofline: fc_decode_attention alone, same flags",
            "parallelism": "replicas" if world > 1 else "single",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "decode attention (split-K + fused combine)",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_kind": peak_kind,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "traffic": profiled_traffic("decode_attention_%s.md" % w.name),
            "bytes_per_launch": int(att_bytes_mean),
            "us_per_launch": round(att_launch_s * 1e6, 3),
            "launches": ROOF_LAUNCHES,
            "timing": "mean over %d back-to-back launches (one CUDA-graph "
                      "replay, independent of --steps) with FC_DECODE_OVERLAP"
                      " | FC_DECODE_Q_FINAL (each launch's start overlaps the "
                      "previous one's drain; independent archives)"
                      % ROOF_LAUNCHES,
            "modes": {m: {"us_per_launch": round(t * 1e6, 3),
                          "achieved": round(att_bytes_mean / t / 1e9, 2),
                          "frac": round(att_bytes_mean / t / 1e9 / peak, 4)}
                      for m, t in modes.items()},
            "modes_note": "isolated: no flags, each launch starts after the "
                          "previous one completed; overlap: FC_DECODE_OVERLAP "
                          "only (the dependency a layer-by-layer decode "
                          "has); overlap_q_final: the headline mode",
        },
        "compress": {
            "tokens_per_s": round(w.B * w.T / comp_s, 1),
            "GB_per_s": round(comp_bytes / comp_s / 1e9, 2),
            "us_per_prefill": round(comp_s * 1e6, 2),
            "frac_of_peak": round(comp_bytes / comp_s / 1e9 / peak, 4),
        },
        "read_view": {
            "kernel": "fc_read_view: every archived block of K and V decoded "
                      "to the token dtype, plus the raw tails",
            "us": round(view_s * 1e6, 2),
            "GB_per_s": round(view_bytes / view_s / 1e9, 2),
            "frac_of_peak": round(view_bytes / view_s / 1e9 / peak, 4),
            "bytes": int(view_bytes),
            "l2": "each pass writes %.0f MB (> L2), evicting the archive "
                  "before the next pass" % (2 * w.B * w.Hk * w.T * w.D * esz
                                            / 1e6),
        },
        "us_per_layer": round(step_s * 1e6, 3),
        "e2e": {"value": round(whole_job_gbs(e2e_bytes, world, e2e_s), 2),
                "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "us_per_step": round(e2e_s * 1e6, 2), "steps": n_e2e,
                "api": "fc_decode_step_host (C ABI; pinned host block in, "
                       "host output out; copies and fused step inside the "
                       "call, arguments marshalled once)"},
        "gpu_launches": K,
        "clocks": clk.summary(),
    }
    if args.layers > 0:
        lay = bench_layers(w, kd, vd, q_pool, dev, W, world,
                           n_layers=args.layers)
        lay["peak"] = peak
        for m in ("one_launch", "separate", "one_launch_overlap_q_final",
                  "separate_overlap_q_final"):
            lay[m]["frac"] = round(lay[m]["GB_per_s"] / peak, 4)
        lay["note"] = ("decode steps (append + attention) of %d independent "
                       "layer caches of this workload: one "
                       "fc_decode_step_layers launch per step against one "
                       "fc_decode_step launch per layer, each plain and with "
                       "FC_DECODE_OVERLAP | FC_DECODE_Q_FINAL" % args.layers)
        res["layers"] = lay
    if args.workloads and args.workloads != "none":
        wl = {}
        for name in args.workloads.split(","):
            if name and name != w.name:
                wl[name] = bench_workload(name, peak, W, world, dev, l2)
        res["workloads"] = wl
    return res


# ------------------------------------------------------- oracle baseline

def oracle_sample_step(arc, q, heads, R):
    """One bounded oracle step: decompress-then-softmax over the sampled kv
    heads of the archive. Returns the bytes of archive streamed."""
    import oracle
    nbytes = 0
    for b, h in heads:
        ck, cv, tk, tv, qg, bpb = arc[(b, h)]
        oracle.decode_attention_reference(qg, ck, cv, tk, tv, R)
        nbytes += bpb
    return nbytes


def prepare_oracle_sample(w, blocks=None, heads=((0, 0),)):
    """Oracle-side archive of a bounded sample of the workload: the first
    ``blocks`` blocks of the listed (b, kv head) pairs, encoded by the oracle
    itself, plus the matching queries."""
    import oracle
    nb = w.n_blocks if blocks is None else min(blocks, w.n_blocks)
    sub = w.replace(B=max(b for b, _ in heads) + 1)
    data = synth.generate(sub.replace(T=nb * w.R + w.n_tail), q_steps=0)
    G = w.G
    arc = {}
    for b, h in heads:
        x = data["k"][b:b + 1, h:h + 1].to(torch.float64).numpy()
        y = data["v"][b:b + 1, h:h + 1].to(torch.float64).numpy()
        ek = oracle.encode_stream(x, w.R, w.S, w.k_coeff)
        ev = oracle.encode_stream(y, w.R, w.S, w.v_coeff)
        qg = data["q"][b:b + 1, h * G:(h + 1) * G].to(torch.float64).numpy()
        per_block = sum(w.S * w.D * {"i8": 1, "bf16": 2, "f32": 4}[c] +
                        (w.S * 4 if c == "i8" else 0)
                        for c in (w.k_coeff, w.v_coeff))
        bpb = nb * per_block
        arc[(b, h)] = (ek["C_hat"], ev["C_hat"], ek["tail"], ev["tail"], qg,
                       bpb)
    return arc


def host_cores():
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def blas_limit(n=1):
    """Context that pins the BLAS / OpenMP pools to n threads (the oracle's
    einsums then run on one core), or a no-op without threadpoolctl."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=n)
    except Exception:
        import contextlib
        return contextlib.nullcontext()


def cpu_cores_used():
    """(threads the oracle runs on, host cores available, BLAS pools)."""
    try:
        from threadpoolctl import threadpool_info
        blas = [p.get("num_threads", 1) for p in threadpool_info()]
    except Exception:
        blas = []
    return 1, host_cores(), blas


def run_cpu_baseline(w, budget_s=10.0):
    """The fp64 oracle (as it stands) timed on this host on a bounded sample
    of the workload: one kv head at a time until ``budget_s`` elapses."""
    heads = [(0, h) for h in range(w.Hk)]
    arc = prepare_oracle_sample(w, blocks=min(w.n_blocks, 2048),
                                heads=heads[:1])
    with blas_limit(1):
        cores, avail, blas = cpu_cores_used()
        t0 = time.perf_counter()
        nbytes = 0
        reps = 0
        while True:
            nbytes += oracle_sample_step(arc, None, list(arc), w.R)
            reps += 1
            if time.perf_counter() - t0 >= budget_s or reps >= 50:
                break
        dt = time.perf_counter() - t0
    nb = min(w.n_blocks, 2048)
    return {"value": round(nbytes / dt / 1e9, 6), "unit": "GB/s",
            "cores": cores, "host_cores": avail, "blas_threads": blas,
            "kind": "oracle",
            "sample": "%d x decode attention of 1 kv head (%d q heads) over "
                      "the first %d blocks + %d tail tokens of the %s "
                      "workload, decompress-then-softmax in float64 "
                      "(%.1f s) on one thread (BLAS pools pinned to 1 of %d "
                      "host cores)" % (reps, w.G, nb, w.n_tail, w.name, dt,
                                       avail)}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = synth.WORKLOADS[args.workload]
    blocks = 256
    arc = prepare_oracle_sample(w, blocks=blocks, heads=((0, 0),))
    with blas_limit(1):
        cores, avail, _ = cpu_cores_used()
        for _ in range(args.warmup):
            oracle_sample_step(arc, None, list(arc), w.R)
        t0 = time.perf_counter()
        nbytes = 0
        for _ in range(args.steps):
            nbytes += oracle_sample_step(arc, None, list(arc), w.R)
        dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = ("each step: decode attention of 1 kv head (%d q heads) over "
              "%d blocks + %d tail tokens of the %s workload, fp64 oracle "
              "decompress-then-softmax" % (w.G, blocks, w.n_tail, w.name))
    return {
        "impl": "reference",
        "metric": "decode-attn archive GB/s (coefficient-domain split-K "
                  "decode step: append + attention)",
        "value": round(value, 6), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic AR(1) K/V (seeded)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hk": w.Hk,
                   "D": w.D, "T": w.T, "R": w.R, "S": w.S},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s",
                         "cores": cores, "host_cores": avail,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "GB/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["fc", "reference"], default="fc")
    ap.add_argument("--workload", default="long",
                    choices=sorted(synth.WORKLOADS))
    ap.add_argument("--copies", type=int, default=0,
                    help="archive copies visited round-robin (0 = enough to "
                         "exceed twice the L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=8,
                    help="layer caches of the multi-layer leg (0 = skip)")
    ap.add_argument("--workloads", default="tiny,gqa,large,stream",
                    help="comma-separated further workloads whose decode "
                         "attention is timed at full size ('none' = none)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    init_dist(world, local)
    try:
        res = run_fc(args, world, rank, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = run_cpu_baseline(
                    synth.WORKLOADS[args.workload])
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
