#!/usr/bin/env python
"""Benchmark of one Wave Forcing layer-round on B200 through libwf.

A step is one pass of the whole hot path over one layer of one wavefront
round: wf_publish_kv (3D rotary + paged scatter of every live slot),
wf_round_attention (M_WF-masked attention of every live slot, with the
readiness check) and wf_advance_round (page recycling + table rewrite). The
pool is first driven through pipeline fill so every timed step is a steady
round. Inputs live in HBM before timing starts; the working set (pool, q, k,
v, q_rot, out) is larger than the 126 MB L2, so no flush is needed between
steps.

value = unmasked attention FLOPs of the timed steps / device time of those
steps (TFLOP/s), summed over ranks (each rank runs an independent replica).

The default run also measures, in the same process, the 14B-shaped layer, the
5-step layer and the 30-layer x 200-round streaming rollout (key
"other_workloads"), times the float64 oracle on the host cores
("cpu_baseline") and the same step from pinned host buffers ("e2e").

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With --gpus N > 1 and no torchrun environment, the script relaunches itself as
N ranks (one process per GPU) under torch.distributed.run.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "WF round attention TFLOP/s (unmasked)"
UNIT = "TFLOP/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="wan13b_bf16")
    ap.add_argument("--fused", action="store_true",
                    help="step = wf_project_publish (QKV projection + RoPE + publication from "
                         "activations and dummy weights) + attention + advance")
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16",
                    help="pool storage: bf16, or E4M3 codes with block scales and FP8 "
                         "tensor-core attention")
    ap.add_argument("--mask", choices=["wf", "rf"], default="wf",
                    help="wf: M_WF chunk-causal mask; rf: bidirectional live window")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=None,
                    help="oracle time per reference step (default: ~150 s over the run)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra measurements of the 14B-shaped layer, the 5-step layer "
                         "and the 30-layer streaming rollout")
    ap.add_argument("--extra-steps", type=int, default=20)
    ap.add_argument("--stream-rounds", type=int, default=200)
    return ap.parse_args()


# ----------------------------------------------------------------------------- utils

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity when not
    distributed). Uses a tensor on ``device`` (the rank's GPU under NCCL, the
    CPU under gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    if device is None:
        device = torch.device("cpu") if dist.get_backend() == "gloo" else torch.device(
            "cuda", torch.cuda.current_device())
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_rate(units_per_rank, ms_max, n_ranks):
    """Units per second of the whole job: every rank processes units_per_rank
    in its timed region, and the job takes as long as its slowest rank."""
    return n_ranks * units_per_rank / (ms_max * 1e-3)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def pick_peak(peaks, timed_s, clocks, key="bf16_tflops"):
    """The measured peak that matches the conditions the kernel ran under: the
    sustained figure (a seconds-long loop under the 1 kW cap) only when the
    timed region lasted seconds AND the sampled clocks saw sw_power_cap; the
    burst figure otherwise. Returns (peak, basis)."""
    capped = bool(clocks) and "sw_power_cap" in (clocks.get("reasons") or [])
    sustained = peaks.get(key + "_sustained")
    if timed_s >= 2.0 and capped and sustained:
        return sustained, "sustained"
    return peaks[key], "burst"


def source_sha(path):
    """Hash of a kernel source's code: line comments and blank lines are left
    out, so that a comment edit does not void the recorded counters."""
    with open(path, encoding="utf-8") as f:
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in f]
    code = "\n".join(ln for ln in lines if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def read_traffic(kernel_file, variant=None):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or None
    when the kernel source has changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    key = os.path.basename(kernel_file) + (f":{variant}" if variant else "")
    e = d.get(key)
    if not e or e.get("source_sha") != source_sha(kernel_file):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.remove(self.path)
        if not rows:
            return None
        mhz = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def unmasked_flops(layout, cfg):
    """4 * C * (keys visible to the slot) * d * heads summed over live slots:
    QK^T and PV multiply-adds over unmasked (query, key) pairs only. Under the
    WF mask a slot reads the context prefix up to its own entry; under RF the
    whole context."""
    total = 0
    for idx, (kind, chunk, slot, tag, pages) in enumerate(layout):
        if slot is None:
            continue
        nvis = len(layout) if cfg.mask == "rf" else idx + 1
        total += 4 * cfg.chunk_tokens * nvis * cfg.chunk_tokens * cfg.head_dim * cfg.num_heads
    return total


def publish_bytes(layout, cfg, kv="bf16"):
    """Algorithmic HBM bytes of one publish: read q, k, v and write q_rot, K, V
    pages (rows of live slots; the zeroed page tail counted as written). FP8
    pools read bf16 and write 1-byte codes plus one fp32 scale per block."""
    live = sum(1 for r in layout if r[2] is not None)
    elt_in = 2 if cfg.dtype == "bf16" else 4
    elt_out = 1 if kv == "fp8" else elt_in
    hd = cfg.num_heads * cfg.head_dim
    tail = cfg.pages_per_chunk * cfg.page_tokens - cfg.chunk_tokens
    scales = 3 * cfg.pages_per_chunk * cfg.num_heads * 4 if kv == "fp8" else 0
    return live * (3 * cfg.chunk_tokens * hd * (elt_in + elt_out) + 2 * tail * hd * elt_out + scales)


# ------------------------------------------------------------------------- our arm

def run_stream(args, ws, rank, local):
    """Streaming rollout: a step is one whole round (publish + attention for
    every layer, then one advance), timed from round 0 so the pipeline-fill
    rounds are included; steady-state rounds are reported separately. Inputs
    are a few pre-generated seeded N(0,1) sets cycled over (round, layer)."""
    import torch
    import wf_inputs
    from chunk_causal_wavefront_b200 import KVPool, make_config

    cfg = wf_inputs.CONFIGS[args.config]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    L = cfg.num_layers
    rounds = args.steps
    npages = (cfg.num_stages + 1 + cfg.anchor_chunks + cfg.history_chunks) * cfg.pages_per_chunk
    pcfg = make_config(num_stages=cfg.num_stages, chunk_tokens=cfg.chunk_tokens,
                       num_heads=cfg.num_heads, head_dim=cfg.head_dim,
                       anchor_chunks=cfg.anchor_chunks, history_chunks=cfg.history_chunks,
                       page_tokens=cfg.page_tokens, num_layers=L, dtype=cfg.dtype, rope=cfg.rope,
                       frames_per_chunk=cfg.frames_per_chunk, grid_h=cfg.grid_h, grid_w=cfg.grid_w,
                       rope_split=cfg.rope_split, rope_base=cfg.rope_base,
                       max_rounds=max(rounds, args.warmup) + 2)
    order = wf_inputs.draw_page_order(npages, cfg.seed + 1)
    shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed * 1000 + rank)
    sets = [[torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
             for _ in range(3)] for _ in range(3)]
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    out = torch.empty(shape, dtype=torch.bfloat16, device=dev)

    def one_round(pool, k):
        for layer in range(L):
            x = sets[(k * L + layer) % len(sets)]
            pool.publish(layer, x[0], x[1], x[2], q_rot)
            pool.attention(layer, q_rot, out)
        pool.advance()

    pool = KVPool(pcfg, device=dev, page_order=order)
    for k in range(args.warmup):
        one_round(pool, k)
    if pool.check_status() != 0:
        raise RuntimeError("device status after warm-up")
    mem = pool.mem
    pool.close()
    pool = KVPool(pcfg, device=dev, page_order=order, mem=mem)   # fresh rollout from round 0

    import torch.distributed as dist
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(rounds + 1)]
    flops = []
    clocks = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    evs[0].record(stream)
    for k in range(rounds):
        flops.append(L * unmasked_flops(pool.layout(), cfg))
        one_round(pool, k)
        evs[k + 1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if pool.check_status() != 0:
        raise RuntimeError("device status after timed rounds")
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(rounds)]
    steady = cfg.steady_round()
    ms = sum(per)
    steady_ms = sum(per[steady:]) if rounds > steady else float("nan")
    ms, steady_ms = max_over_ranks([ms, steady_ms], dev)
    pool.close()
    return {"ms": ms, "steady_ms": steady_ms, "flops_total": sum(flops),
            "flops_steady": sum(flops[steady:]), "rounds": rounds, "steady_rounds": max(0, rounds - steady),
            "layers": L, "clocks": clk}



def run_ours(args, ws, rank, local):
    import torch
    import wf_inputs
    from chunk_causal_wavefront_b200 import KVPool, make_config

    cfg = wf_inputs.CONFIGS[args.config].replace(mask=args.mask)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    steady = cfg.steady_round()
    total_rounds = steady + args.warmup + args.steps + (0 if args.no_e2e else args.e2e_steps + 2) + 4
    npages = (cfg.num_stages + 1 + cfg.anchor_chunks + cfg.history_chunks) * cfg.pages_per_chunk
    pool = KVPool(make_config(num_stages=cfg.num_stages, chunk_tokens=cfg.chunk_tokens,
                              num_heads=cfg.num_heads, head_dim=cfg.head_dim,
                              anchor_chunks=cfg.anchor_chunks, history_chunks=cfg.history_chunks,
                              page_tokens=cfg.page_tokens, num_layers=1,
                              dtype="fp8" if args.kv == "fp8" else cfg.dtype,
                              rope=cfg.rope, frames_per_chunk=cfg.frames_per_chunk,
                              grid_h=cfg.grid_h, grid_w=cfg.grid_w, rope_split=cfg.rope_split,
                              rope_base=cfg.rope_base, max_rounds=total_rounds, mask=cfg.mask),
                  device=dev, page_order=wf_inputs.draw_page_order(npages, cfg.seed + 1))
    shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed * 1000 + rank)
    inputs = []
    for _ in range(2):   # two rounds of q, k, v, cycled
        inputs.append([torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(tdt)
                       for _ in range(3)])
    if cfg.k_outlier_frac > 0:
        for x in inputs:
            m = torch.rand(shape[:3], generator=gen, device=dev) < cfg.k_outlier_frac
            x[1] = torch.where(m[..., None], x[1].float() * cfg.k_outlier_scale, x[1].float()).to(tdt)
    q_rot = torch.empty(shape, dtype=torch.uint8 if args.kv == "fp8" else tdt, device=dev)
    out = torch.empty(shape, dtype=tdt, device=dev)
    hidden = cfg.num_heads * cfg.head_dim
    if args.fused:
        # activations [S+1][C][hidden] and dummy weights [3*hidden][hidden], N(0, 1/hidden)
        acts = [torch.randn((cfg.num_slots, cfg.chunk_tokens, hidden), generator=gen, device=dev,
                            dtype=torch.float32).to(tdt) for _ in range(2)]
        w_qkv = (torch.randn((3 * hidden, hidden), generator=gen, device=dev, dtype=torch.float32)
                 / math.sqrt(hidden)).to(tdt)

    def publish_step(i):
        if args.fused:
            pool.project_publish(0, acts[i & 1], w_qkv, q_rot)
        else:
            x = inputs[i & 1]
            pool.publish(0, x[0], x[1], x[2], q_rot)

    def step(i):
        publish_step(i)
        pool.attention(0, q_rot, out)
        pool.advance()

    # pipeline fill (untimed, not counted as warm-up)
    for i in range(steady):
        step(i)
    for i in range(args.warmup):
        step(i)
    st = pool.check_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    layout = pool.layout()
    flops = unmasked_flops(layout, cfg)
    pbytes = publish_bytes(layout, cfg, args.kv)

    import torch.distributed as dist
    ev = lambda: torch.cuda.Event(enable_timing=True)
    e_pub = [(ev(), ev()) for _ in range(args.steps)]
    e_att = [(ev(), ev()) for _ in range(args.steps)]
    t0, t1 = ev(), ev()
    clocks = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record(stream)
    for i in range(args.steps):
        e_pub[i][0].record(stream)
        publish_step(i)
        e_pub[i][1].record(stream)
        e_att[i][0].record(stream)
        pool.attention(0, q_rot, out)
        e_att[i][1].record(stream)
        pool.advance()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if ws > 1:
        dist.barrier()
    st = pool.check_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timed steps")
    ms = t0.elapsed_time(t1)
    att_ms = statistics.mean(a.elapsed_time(b) for a, b in e_att)
    pub_ms = statistics.mean(a.elapsed_time(b) for a, b in e_pub)
    ms, = max_over_ranks([ms], dev)

    live = sum(1 for r in layout if r[2] is not None)
    proj_flops = 2 * live * cfg.chunk_tokens * (3 * hidden) * hidden if args.fused else 0
    res = {"ms": ms, "att_ms": att_ms, "pub_ms": pub_ms, "flops": flops, "pbytes": pbytes,
           "clocks": clk, "layout_positions": len(layout), "proj_flops": proj_flops}

    # End to end: the step's q, k, v come from pinned host buffers and out goes
    # back to pinned host memory, all inside the timed region. The copies are
    # pipelined the way a caller would: H2D of step i+1 on one copy stream and
    # D2H of step i-1 on another overlap the kernels of step i (double-buffered
    # device inputs and outputs, ordered by events).
    if not args.no_e2e and not args.fused:
        host_in = [[t.cpu().pin_memory() for t in x] for x in inputs]
        host_out = torch.empty(shape, dtype=tdt).pin_memory()
        dev_in = [[torch.empty(shape, dtype=tdt, device=dev) for _ in range(3)] for _ in range(2)]
        dev_out = [torch.empty(shape, dtype=tdt, device=dev) for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host_in[0])
        d2h = host_out.numel() * host_out.element_size()
        s_h2d = torch.cuda.Stream(dev)
        s_d2h = torch.cuda.Stream(dev)
        n = args.e2e_steps
        ev_in = [ev() for _ in range(n)]        # inputs of step i are on the device
        ev_pub = [ev() for _ in range(n)]       # publish of step i has read its inputs
        ev_att = [ev() for _ in range(n)]       # attention of step i has written out
        ev_out = [ev() for _ in range(n)]       # out of step i is back on the host

        def upload(i):
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(ev_pub[i - 2])          # buffer set reused
                for d, h in zip(dev_in[i & 1], host_in[i & 1]):
                    d.copy_(h, non_blocking=True)
                ev_in[i].record(s_h2d)

        a, b = ev(), ev()
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        a.record(stream)
        s_h2d.wait_event(a)
        s_d2h.wait_event(a)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            stream.wait_event(ev_in[i])
            x = dev_in[i & 1]
            pool.publish(0, x[0], x[1], x[2], q_rot)
            ev_pub[i].record(stream)
            if i >= 2:
                stream.wait_event(ev_out[i - 2])             # out buffer reused
            pool.attention(0, q_rot, dev_out[i & 1])
            ev_att[i].record(stream)
            pool.advance()
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_att[i])
                host_out.copy_(dev_out[i & 1], non_blocking=True)
                ev_out[i].record(s_d2h)
        stream.wait_event(ev_out[n - 1])
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b)
        e_ms, = max_over_ranks([e_ms], dev)
        res["e2e"] = {"ms": e_ms, "steps": args.e2e_steps, "h2d": h2d, "d2h": d2h}
        st = pool.check_status()
        if st != 0:
            raise RuntimeError(f"device status {st} after e2e steps")
    pool.close()
    return res


# ------------------------------------------------------------------- oracle timing

ORACLE_SAMPLE_ROWS = 64


def oracle_sample_rate(cfg, seconds, seed=0, nrows=ORACLE_SAMPLE_ROWS):
    """Time the float64 oracle on a fixed, bounded sample of one steady round:
    the first `nrows` query rows of every live slot, one head, against each
    slot's full visible context, rotary included, repeated until `seconds`
    have passed (at least once). The CPU baseline and the reference arm both
    time this same sample. Returns (TFLOP/s, description)."""
    import numpy as np
    from oracle import wf_oracle as O
    S, A, H = cfg.num_stages, cfg.anchor_chunks, cfg.history_chunks
    lay = O.round_layout(S, A, H, cfg.steady_round())
    rng = np.random.default_rng(seed)
    C, d = cfg.chunk_tokens, cfg.head_dim

    def rope(x, chunk):
        if not cfg.rope:
            return x
        return O.rope_3d(x, chunk, cfg.frames_per_chunk, cfg.grid_h, cfg.grid_w,
                         cfg.rope_split, cfg.rope_base)

    keys = {p.chunk: rng.standard_normal((C, 1, d)) for p in lay}
    vals = {p.chunk: rng.standard_normal((C, 1, d)) for p in lay}
    q = rng.standard_normal((C, 1, d))

    def once(rows):
        kk = {c: rope(x, c) for c, x in keys.items()}
        qr = {p.slot: rope(q, p.chunk) for p in lay if p.slot is not None}
        O.attention_slot_prefix(qr, kk, vals, lay, rows=rows)
        return _unmasked_rows_flops(lay, len(rows), C, d)

    rows = np.arange(min(nrows, C))
    fl, reps = 0, 0
    t0 = time.perf_counter()
    while True:
        fl += once(rows)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    desc = (f"{reps} x ({len(rows)} query rows x 1 head of every live slot of a steady round, "
            f"each against its full visible context, rotary included), {dt:.1f} s")
    return fl / dt / 1e12, desc


def _unmasked_rows_flops(lay, nrows, C, d):
    tot = 0
    for idx, p in enumerate(lay):
        if p.slot is not None:
            tot += 4 * nrows * (idx + 1) * C * d
    return tot


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:
        return None


def run_reference(args, ws, rank):
    import wf_inputs
    cfg = wf_inputs.CONFIGS[args.config]
    if rank != 0:
        return
    per_step = (args.ref_step_seconds if args.ref_step_seconds is not None
                else max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        oracle_sample_rate(cfg, per_step / 4)
    rates = []
    t0 = time.perf_counter()
    descs = None
    for _ in range(args.steps):
        r, descs = oracle_sample_rate(cfg, per_step)
        rates.append(r)
    wall = time.perf_counter() - t0
    v = statistics.mean(rates)
    cores = len(os.sched_getaffinity(0))
    line = {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(cfg, args.gpus),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": blas_threads() or cores,
                             "kind": "oracle", "sample": descs},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(cfg, n, fused=False, kv="bf16"):
    return {"workload": f"{cfg.name}{'' if cfg.mask == 'wf' else ' (RF mask)'}"
                        f"{' (fused QKV projection)' if fused else ''}"
                        f"{' (E4M3 pool: FP8 K/V pages + scales, FP8 attention)' if kv == 'fp8' else ''}"
                        f": one layer-round, S={cfg.num_stages}+store, "
                        f"C={cfg.chunk_tokens}, heads={cfg.num_heads}x{cfg.head_dim}, "
                        f"anchor={cfg.anchor_chunks}, history={cfg.history_chunks}, "
                        f"page={cfg.page_tokens}, steady state",
            "step": ("wf_project_publish" if fused else "wf_publish_kv")
                    + " + wf_round_attention + wf_advance_round",
            "l2": "working set > 126 MB L2 (pool 233 MB + q/k/v/q_rot/out 360 MB); no flush",
            "parallelism": f"replicas x{n}" if n > 1 else "single GPU"}


def spawn_ranks(n, argv):
    """Run this script as n ranks of one node under torch.distributed.run (one
    process per GPU, rendezvous on 127.0.0.1) and return its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def attention_block(att_ms, flops, timed_s, clocks, peaks, ratio):
    """Achieved TFLOP/s of the attention kernel, with the fraction of the
    measured bf16 peak that matches the run's conditions (x ratio for FP8)."""
    tflops = flops / (att_ms * 1e-3) / 1e12
    peak, basis = pick_peak(peaks, timed_s, clocks)
    return {"ms_per_launch": att_ms, "tflops": tflops, "flops_per_launch": flops,
            "pct_peak_burst": 100 * tflops / (ratio * peaks["bf16_tflops"]),
            "pct_peak_sustained": 100 * tflops / (ratio * peaks.get("bf16_tflops_sustained",
                                                                     peaks["bf16_tflops"])),
            "peak": ratio * peak, "peak_basis": basis, "frac": tflops / (ratio * peak)}


def run_deliver(local, peaks, launches=50):
    """wf_deliver_kv of one live slot's K/V (one layer of the 1.3B-shaped
    workload) into a second pool on the same device: a same-device copy, so it
    measures the kernels, not the NVLink path the call is for on several GPUs."""
    import torch
    import wf_inputs
    from chunk_causal_wavefront_b200 import KVPool, make_config
    cfg = wf_inputs.CONFIGS["wan13b_bf16"]
    dev = torch.device("cuda", local)
    npages = (cfg.num_stages + 1 + cfg.anchor_chunks + cfg.history_chunks) * cfg.pages_per_chunk
    steady = cfg.steady_round()
    pc = make_config(num_stages=cfg.num_stages, chunk_tokens=cfg.chunk_tokens, num_heads=cfg.num_heads,
                     head_dim=cfg.head_dim, anchor_chunks=cfg.anchor_chunks,
                     history_chunks=cfg.history_chunks, page_tokens=cfg.page_tokens, num_layers=1,
                     dtype=cfg.dtype, rope=cfg.rope, frames_per_chunk=cfg.frames_per_chunk,
                     grid_h=cfg.grid_h, grid_w=cfg.grid_w, rope_split=cfg.rope_split,
                     rope_base=cfg.rope_base, max_rounds=steady + 2)
    order = wf_inputs.draw_page_order(npages, cfg.seed + 1)
    sender = KVPool(pc, device=dev, page_order=order)
    receiver = KVPool(pc, device=dev, page_order=order)
    shape = (cfg.num_slots, cfg.chunk_tokens, cfg.num_heads, cfg.head_dim)
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed * 1000 + 7)
    x = [torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16) for _ in range(3)]
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    for _ in range(steady):
        sender.advance()
        receiver.advance()
    sender.publish(0, x[0], x[1], x[2], q_rot)
    slot = 0
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        sender.deliver(0, slot, receiver)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(launches)]
    torch.cuda.synchronize()
    for a, b in ev:
        a.record(stream)
        sender.deliver(0, slot, receiver)
        b.record(stream)
    torch.cuda.synchronize()
    if sender.check_status() != 0 or receiver.check_status() != 0:
        raise RuntimeError("device status after the delivery timing")
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    tiles = cfg.pages_per_chunk * 2 * cfg.num_heads
    moved = 2 * tiles * cfg.page_tokens * cfg.head_dim * 2        # read + write, bf16
    sender.close()
    receiver.close()
    gbs = moved / (ms * 1e-3) / 1e9
    return {"kernels": "deliver_copy_kernel + deliver_tags_kernel",
            "what": f"one live slot's K/V of one layer ({cfg.pages_per_chunk} pages x K,V x "
                    f"{cfg.num_heads} heads x {cfg.page_tokens}x{cfg.head_dim} bf16) into a second "
                    "pool on the same device (same-device copy, not the NVLink path)",
            "ms_per_launch": ms, "bytes_per_launch": moved, "same_device_copy_gbs": gbs,
            "pct_hbm": 100 * gbs / peaks["hbm_gbs"], "launches": launches}


def run_extras(args, ws, rank, local, peaks):
    """The other workloads, measured in the same run: the 14B-shaped layer and
    the 5-step layer (steady layer-rounds, publish + attention + advance), the
    Wave Parallelism delivery of one slot (same-device copy), and the 30-layer
    streaming rollout (whole rounds from round 0, fill included)."""
    import argparse as _ap
    extra = {}
    for name in ("wan14b_bf16", "wan13b_5step_bf16"):
        a = _ap.Namespace(**vars(args))
        a.config, a.steps, a.warmup, a.no_e2e = name, args.extra_steps, 3, True
        a.fused, a.kv, a.mask = False, "bf16", "wf"
        r = run_ours(a, ws, rank, local)
        if rank == 0:
            timed_s = r["ms"] * 1e-3
            extra[name] = {
                "layer_rounds_per_s": ws * a.steps / timed_s,
                "tflops": whole_job_rate(r["flops"] * a.steps, r["ms"], ws) / 1e12,
                "ms_per_step": r["ms"] / a.steps, "steps": a.steps,
                "attention": attention_block(r["att_ms"], r["flops"], timed_s, r["clocks"], peaks, 1.0),
                "publish_gbs": r["pbytes"] / (r["pub_ms"] * 1e-3) / 1e9,
                "clocks": r["clocks"]}
    d = run_deliver(local, peaks)
    if rank == 0:
        extra["deliver"] = d
    a = _ap.Namespace(**vars(args))
    a.config, a.steps, a.warmup = "stream_13b_bf16", args.stream_rounds, 3
    r = run_stream(a, ws, rank, local)
    if rank == 0:
        extra["stream_13b_bf16"] = {
            "layers": r["layers"], "rounds": r["rounds"],
            "rounds_per_s": ws * r["rounds"] / (r["ms"] * 1e-3),
            "steady_rounds_per_s": ws * r["steady_rounds"] / (r["steady_ms"] * 1e-3),
            "tflops": ws * r["flops_total"] / (r["ms"] * 1e-3) / 1e12,
            "steady_tflops": ws * r["flops_steady"] / (r["steady_ms"] * 1e-3) / 1e12,
            "clocks": r["clocks"]}
    return extra


def main():
    args = parse()
    if args.fused and args.kv == "fp8":
        raise SystemExit("--fused publishes into bf16 pools only")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: relaunch as args.gpus ranks
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            backend = "nccl"
        else:
            backend = "gloo"   # the reference arm runs on host cores only
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if args.impl == "reference":
        run_reference(args, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return
    import wf_inputs
    cfg = wf_inputs.CONFIGS[args.config]
    peaks, src = read_peaks()
    if cfg.num_layers > 1:
        res = run_stream(args, ws, rank, local)
        if rank == 0:
            value = whole_job_rate(res["flops_total"], res["ms"], ws) / 1e12
            line = {
                "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": res["rounds"],
                "warmup": args.warmup, "ms_per_step": res["ms"] / res["rounds"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
                "data": "synthetic",
                "config": {"workload": f"{cfg.name}: {res['layers']} layers x {res['rounds']} rounds "
                                       f"from round 0 (fill included), S={cfg.num_stages}+store, "
                                       f"C={cfg.chunk_tokens}, heads={cfg.num_heads}x{cfg.head_dim}, "
                                       f"history={cfg.history_chunks}, page recycling",
                           "step": "one round: per layer wf_publish_kv + wf_round_attention; "
                                   "then wf_advance_round",
                           "l2": "working set 7 GB pool + inputs > L2; no flush",
                           "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
                "rounds_per_s": ws * res["rounds"] / (res["ms"] * 1e-3),
                "steady_rounds_per_s": ws * res["steady_rounds"] / (res["steady_ms"] * 1e-3),
                "steady_tflops": ws * res["flops_steady"] / (res["steady_ms"] * 1e-3) / 1e12,
                "clocks": res["clocks"],
                "gpu_launches": res["rounds"] * (2 * res["layers"] + 1),
            }
            print(json.dumps(line), flush=True)
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return
    res = run_ours(args, ws, rank, local)
    extra = None
    if not args.no_extra and args.config == "wan13b_bf16" and not args.fused and args.kv == "bf16" \
            and args.mask == "wf":
        extra = run_extras(args, ws, rank, local, peaks)
    if rank == 0:
        ms_step = res["ms"] / args.steps
        timed_s = res["ms"] * 1e-3
        value = whole_job_rate(res["flops"] * args.steps, res["ms"], ws) / 1e12
        # An E4M3 contraction's peak: the measured bf16 peak times the nominal
        # dense ratio fp8 / bf16 (4.5 / 2.25 PFLOP/s).
        f8 = args.kv == "fp8"
        ratio = 2.0 if f8 else 1.0
        att = attention_block(res["att_ms"], res["flops"], timed_s, res["clocks"], peaks, ratio)
        pub_gbs = res["pbytes"] / (res["pub_ms"] * 1e-3) / 1e9
        kfile = os.path.join(ROOT, "chunk_causal_wavefront_b200", "csrc", "attn_tc.cu")
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if f8 else cfg.dtype,
            "data": "synthetic",
            "config": workload_config(cfg, ws, args.fused, args.kv),
            "layer_rounds_per_s": ws * args.steps / timed_s,
            "attention": att,
            "publish": ({"kernel": ("publish_fp8_kernel" if f8 else
                                    "publish_tma_kernel" if cfg.head_dim == 128 and cfg.page_tokens == 128
                                    else "publish_kernel"),
                         "ms_per_launch": res["pub_ms"], "gbs": pub_gbs,
                         "pct_hbm": 100 * pub_gbs / peaks["hbm_gbs"],
                         "bytes_per_launch": res["pbytes"]} if not args.fused else
                        {"kernel": "project_kernel (QKV GEMM + RoPE + paged publication)",
                         "ms_per_launch": res["pub_ms"],
                         "gemm_tflops": res["proj_flops"] / (res["pub_ms"] * 1e-3) / 1e12,
                         "pct_bf16_peak_burst": 100 * res["proj_flops"] / (res["pub_ms"] * 1e-3)
                         / 1e12 / peaks["bf16_tflops"],
                         "flops_per_launch": res["proj_flops"]}),
            "roofline": {"bound": "tensor", "achieved": att["tflops"], "peak": att["peak"],
                         "unit": "TFLOP/s", "frac": att["frac"],
                         "traffic": read_traffic(kfile, "e4m3" if f8 else "bf16"),
                         "kernel": "attn_tc_kernel<e4m3>" if f8 else "attn_tc_kernel<bf16>",
                         "peak_source": f"{src} bf16_tflops"
                                        + ("_sustained" if att["peak_basis"] == "sustained" else "")
                                        + (" x 2 (nominal fp8/bf16 dense ratio)" if f8 else ""),
                         "peak_basis": att["peak_basis"] + (
                             " (timed region of seconds with sw_power_cap sampled)"
                             if att["peak_basis"] == "sustained" else
                             " (timed region under 2 s or no power cap sampled)"),
                         "frac_burst": att["pct_peak_burst"] / 100,
                         "frac_sustained": att["pct_peak_sustained"] / 100},
            "clocks": res["clocks"],
            "gpu_launches": 3 * args.steps,
        }
        if "e2e" in res:
            e = res["e2e"]
            line["e2e"] = {"value": ws * res["flops"] * e["steps"] / (e["ms"] * 1e-3) / 1e12,
                           "unit": UNIT, "h2d_bytes_per_step": e["h2d"],
                           "d2h_bytes_per_step": e["d2h"], "steps": e["steps"]}
        if extra:
            line["other_workloads"] = extra
        if ws == 1 and not args.no_cpu_baseline:
            v, desc = oracle_sample_rate(cfg, args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": UNIT,
                                    "cores": blas_threads() or len(os.sched_getaffinity(0)),
                                    "kind": "oracle", "sample": desc}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
