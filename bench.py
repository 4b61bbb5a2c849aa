#!/usr/bin/env python
"""Throughput bench of the looped weight-shared decoder on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole forward path over one batch of synthetic
input: for a prefill workload, loop_prefill of B sequences x S tokens (56
layer executions, mHC, attention, linear attention, output head); for the
decode workload, one loop_decode_step of 64 sequences.  Prints one JSON line
(rank 0).  With N > 1 (torchrun) every rank runs an independent replica on its
own GPU (the path shards by sequence; there is no data-path collective) and
the timing is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import seeded  # noqa: E402
from seeded import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "loop9b_prefill_b4_s8192"

# DRAM read + write per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum),
# taken under the capture rules; set to None when the kernel changes:
# - tcgen05 GEMM: mean over five consecutive full-size launches of the 9B
#   prefill (SwiGLU, mHC write at K 12,288 and 4,096, q/k/v/gate; one-pass
#   metrics, see profiles/launches_loop9b_prefill_b4_s8192.md)
# - decode attention: 1.085 GB per launch on the probe_decode_b64_ctx4096
#   workload (64 x 4096 keys), scaled by keys to 32,787
GEMM_TRAFFIC_PER_LAUNCH = 3.94e9
DECODE_ATTN_TRAFFIC_PER_LAUNCH = 1.085e9 * 32787 / 4097
LONG_WORKLOAD = "loop9b_prefill_b1_s262144"
EXTEND_K = 8  # tokens per sequence of the timed loop_extend steps
DATA = "synthetic: seeded SplitMix64 token ids, random-init N(0, 0.02) bf16 weights of the 9B shape"


def args_():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-tokens", type=int, default=12)
    p.add_argument("--no-decode", action="store_true", help="skip the decode measurement of the default run")
    p.add_argument("--decode-steps", type=int, default=None,
                   help="timed decode steps (default: the decode workload's 128)")
    p.add_argument("--no-long", action="store_true", help="skip the 262,144-token prefill of the default run")
    p.add_argument("--long-steps", type=int, default=2)
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def workload_info(name):
    w = W.WORKLOADS[name]
    m = dict(w["model"])
    decode = "decode_steps" in w
    return w, m, decode


def metric_for(name, decode):
    if decode:
        return "looped-decoder decode tokens/s at 9B shape", "tokens/s"
    if W.WORKLOADS[name]["model"]["io_mode"] == 1:
        return "looped 4-layer group prefill tokens/s at 9B width", "tokens/s"
    return "looped-decoder prefill tokens/s at 9B shape", "tokens/s"


# ---------------------------------------------------------------------------- algorithmic work

def layer_weight_bytes(m, full: bool) -> int:
    H, F = m["hidden"], m["ffn"]
    if full:
        nq, nkv = m["n_q"] * m["head_dim"], m["n_kv"] * m["head_dim"]
        w_in, w_o = (nq + 2 * nkv) * H, H * nq
    else:
        d = m["n_lin"] * m["lin_dim"]
        w_in, w_o = (3 * d + m["n_lin"]) * H, H * d
    return 2 * (w_in + w_o + 2 * F * H + H * F)


def prefill_step_flops(m, B: int, S: int) -> dict:
    """Tensor FLOPs one prefill step must do: every layer execution's
    projections (2 x parameters per token), causal attention (QK^T and PV over
    the keys at or before each query), the chunked linear-attention products
    at the pages' chunk length (scores, intra- and inter-chunk outputs, state
    update), and the LM head on the last position of each sequence."""
    execs = list(range(m["n_prelude"])) + [m["n_prelude"] + j for j in range(m["n_block"])] * m["n_loops"] + \
        [m["n_prelude"] + m["n_block"] + j for j in range(m["n_coda"])]
    full = [p % m["group"] == m["full_slot"] for p in execs]
    T = B * S
    proj = sum(2 * T * layer_weight_bytes(m, f) // 2 for f in full)
    d = m["head_dim"]
    attn = sum(full) * B * m["n_q"] * 4 * d * (S * (S + 1) // 2)
    C, dl = m["lin_chunk"], m["lin_dim"]
    gla = (len(full) - sum(full)) * T * m["n_lin"] * (4 * C * dl + 4 * dl * dl)
    head = 2 * B * m["hidden"] * m["vocab"] if m["io_mode"] == 0 else 0
    return {"projections": proj, "attention": attn, "linear_attention": gla, "lm_head": head,
            "total": proj + attn + gla + head}


def decode_step_bytes(m, B: int, ctx: int) -> dict:
    """HBM bytes one decode step must move: every layer execution reads its
    weights (the shared block twice), the head reads E, full attention reads
    the KV cache of its slot, linear attention reads and writes its state."""
    n_phys = m["n_prelude"] + m["n_block"] + m["n_coda"]
    execs = list(range(m["n_prelude"])) + [m["n_prelude"] + j for j in range(m["n_block"])] * m["n_loops"] + \
        [m["n_prelude"] + m["n_block"] + j for j in range(m["n_coda"])]
    full = [p % m["group"] == m["full_slot"] for p in execs]
    weights = sum(layer_weight_bytes(m, f) for f in full) + 2 * m["vocab"] * m["hidden"]
    kv_row = m["n_kv"] * m["head_dim"] * 2 * 2
    kv = sum(full) * B * (ctx + 1) * kv_row
    state = (len(full) - sum(full)) * B * m["n_lin"] * m["lin_dim"] ** 2 * 4 * 2
    return {"weights": weights, "kv": kv, "state": state, "total": weights + kv + state + sum(full) * B * kv_row}


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- our arm

def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time (every rank gets it); x itself on one rank."""
    if world <= 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


def run_ours(a, rank, world, local_rank):
    import torch
    import looped_weight_shared_b200 as L

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w, m, decode = workload_info(a.workload)
    B, S, seed = w["batch"], w["seq"], w["seed"]
    if decode:
        m.update(max_batch=B, max_ctx=S + a.warmup + 2 * a.steps + 2)
    else:
        m.update(max_batch=B, max_ctx=S)
    cfg = L.make_config(**m)
    t0 = time.time()
    g = L.loop_model_create(cfg, seed=seed)
    create_s = time.time() - t0
    stream = torch.cuda.current_stream(dev)
    V, H = m["vocab"], m["hidden"]

    if decode:
        tok = torch.from_numpy(seeded.tokens(seed, B, S, V)).to(dev)
        L.loop_prefill(g, tokens=tok, out=torch.empty((B, V), device=dev))
        nxt = seeded.tokens(seed, B, a.warmup + 2 * a.steps + 2, V, stream=seeded.S_DECODE_TOKENS)
        step_tok = [torch.from_numpy(nxt[:, i].copy()).to(dev) for i in range(nxt.shape[1])]
        out = torch.empty((B, V), device=dev)
        it = iter(step_tok)

        def step():
            L.loop_decode_step(g, next(it), out)
        units = B
    elif m["io_mode"] == 1:
        hid = torch.from_numpy(seeded.hidden(seed, B, S, H)).to(dev)
        out = torch.empty((B, S, H), device=dev)

        def step():
            L.loop_prefill(g, hidden=hid, out=out)
        units = B * S
    else:
        tok = torch.from_numpy(seeded.tokens(seed, B, S, V)).to(dev)
        out = torch.empty((B, V), device=dev)

        def step():
            L.loop_prefill(g, tokens=tok, out=out)
        units = B * S

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    L.loop_timing_read(g, 0, reset=True)
    L.loop_set_timing(g, True)
    launches0 = L.loop_launch_count(g)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        for _ in range(a.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    L.loop_set_timing(g, False)
    launches = L.loop_launch_count(g) - launches0
    ms = max_over_ranks(ev0.elapsed_time(ev1) / a.steps, world, dev)
    if world > 1:
        torch.distributed.barrier()
    value = job_throughput(units, world, ms)
    classes = {}
    for ci, cname in enumerate(L.KERNEL_CLASSES):
        tms, n, work = L.loop_timing_read(g, ci)
        classes[cname] = {"ms_per_step": tms / a.steps, "launches": n, "work": work}
    status = L.loop_device_status()

    # e2e: the same step through the C ABI with host buffers (pinned), the
    # step's inputs copied in and its result read back inside the timed region
    if decode:
        host_in = torch.from_numpy(nxt[:, -a.steps:].T.copy()).pin_memory()
        e2e_out = torch.empty((B, V), pin_memory=True)
        d_tok = torch.empty((B,), dtype=torch.int32, device=dev)
        h2d = B * 4
        d2h = B * V * 4
    elif m["io_mode"] == 1:
        host_in = torch.from_numpy(seeded.hidden(seed, B, S, H)).pin_memory()
        e2e_out = torch.empty((B, S, H), pin_memory=True)
        d_hid = torch.empty((B, S, H), device=dev)
        h2d = B * S * H * 4
        d2h = B * S * H * 4
    else:
        host_in = torch.from_numpy(seeded.tokens(seed, B, S, V)).pin_memory()
        e2e_out = torch.empty((B, V), pin_memory=True)
        d_tok = torch.empty((B, S), dtype=torch.int32, device=dev)
        h2d = B * S * 4
        d2h = B * V * 4

    def e2e_step(i):
        if decode:
            d_tok.copy_(host_in[i % host_in.shape[0]], non_blocking=True)
            L.loop_decode_step(g, d_tok, out)
        elif m["io_mode"] == 1:
            d_hid.copy_(host_in, non_blocking=True)
            L.loop_prefill(g, hidden=d_hid, out=out)
        else:
            d_tok.copy_(host_in, non_blocking=True)
            L.loop_prefill(g, tokens=d_tok, out=out)
        e2e_out.copy_(out, non_blocking=True)

    e2e_steps = a.steps
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ev0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps, world, dev)
    L.loop_model_destroy(g)
    return dict(ms=ms, value=value, classes=classes, clocks=clk.summary(), launches=launches, status=status,
                e2e_ms=e2e_ms, e2e_value=job_throughput(units, world, e2e_ms), h2d=h2d, d2h=d2h,
                create_s=create_s, units=units)


def run_decode(a, world, local_rank):
    """Decode throughput: 64 sequences after a 32,768-token prefill."""
    import numpy as np
    import torch
    import looped_weight_shared_b200 as L

    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS["loop9b_decode_b64_ctx32768"]
    m = dict(w["model"])
    B, S, seed = w["batch"], w["seq"], w["seed"]
    steps = max(a.decode_steps if a.decode_steps is not None else w["decode_steps"], 1)
    warm = max(a.warmup, 3)
    ek, ewarm, esteps = EXTEND_K, 2, 4  # multi-token append (verify) steps after the decode steps
    m.update(max_batch=B, max_ctx=S + warm + 2 * steps + ek * (ewarm + esteps) + 2)
    g = L.loop_model_create(L.make_config(**m), seed=seed)
    V = m["vocab"]
    out = torch.empty((B, V), device=dev)
    L.loop_prefill(g, tokens=torch.from_numpy(seeded.tokens(seed, B, S, V)).to(dev), out=out)
    nxt = seeded.tokens(seed, B, warm + 2 * steps, V, stream=seeded.S_DECODE_TOKENS)
    toks = [torch.from_numpy(nxt[:, i].copy()).to(dev) for i in range(nxt.shape[1])]
    for i in range(warm):
        L.loop_decode_step(g, toks[i], out)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ctx0 = L.loop_seq_len(g, 0)
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the timed steps: no per-launch events
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        for i in range(steps):
            L.loop_decode_step(g, toks[warm + i], out)
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, world, dev)
    # the same steps again with per-launch events, for the per-class split
    L.loop_timing_read(g, 0, reset=True)
    L.loop_set_timing(g, True)
    ev0.record(stream)
    for i in range(steps):
        L.loop_decode_step(g, toks[warm + steps + i], out)
    ev1.record(stream)
    torch.cuda.synchronize()
    L.loop_set_timing(g, False)
    ms_timed = ev0.elapsed_time(ev1) / steps
    classes = {}
    for ci, cname in enumerate(L.KERNEL_CLASSES):
        tms, n, work = L.loop_timing_read(g, ci)
        classes[cname] = {"ms_per_step": tms / steps, "launches": n}
    # loop_extend: k new tokens per sequence in one pass (the verification step
    # of multi-token prediction), timed without per-launch events
    ext = seeded.tokens(seed + 1000, B, ek * (ewarm + esteps), V, stream=seeded.S_DECODE_TOKENS)
    ext_t = [torch.from_numpy(np.ascontiguousarray(ext[:, i * ek:(i + 1) * ek])).to(dev) for i in range(ewarm + esteps)]
    for i in range(ewarm):
        L.loop_extend(g, ext_t[i], out)
    torch.cuda.synchronize()
    ectx0 = L.loop_seq_len(g, 0)
    ev0.record(stream)
    for i in range(esteps):
        L.loop_extend(g, ext_t[ewarm + i], out)
    ev1.record(stream)
    torch.cuda.synchronize()
    ext_ms = max_over_ranks(ev0.elapsed_time(ev1) / esteps, world, dev)
    L.loop_model_destroy(g)
    mid_ctx = ctx0 + steps // 2
    by = decode_step_bytes(m, B, mid_ctx)
    return {"ms": ms, "value": job_throughput(B, world, ms), "bytes": by, "classes": classes, "clocks": clk.summary(),
            "ctx": mid_ctx, "ms_with_launch_events": ms_timed,
            "extend": {"k": ek, "batch": B, "context": ectx0, "steps": esteps, "warmup": ewarm, "ms_per_step": ext_ms,
                       "value": job_throughput(B * ek, world, ext_ms), "unit": "tokens/s"}}


def run_long_prefill(a, world, local_rank):
    """The long-context workload: one 262,144-token prefill of the 9B-shaped
    model, 1 warm-up step and a.long_steps timed steps, per-class split from
    CUDA events around every launch (inside the timed region, as for the
    headline prefill)."""
    import torch
    import looped_weight_shared_b200 as L

    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS[LONG_WORKLOAD]
    m = dict(w["model"])
    B, S, seed = w["batch"], w["seq"], w["seed"]
    m.update(max_batch=B, max_ctx=S)
    g = L.loop_model_create(L.make_config(**m), seed=seed)
    V = m["vocab"]
    tok = torch.from_numpy(seeded.tokens(seed, B, S, V)).to(dev)
    out = torch.empty((B, V), device=dev)
    L.loop_prefill(g, tokens=tok, out=out)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    stream = torch.cuda.current_stream(dev)
    steps = max(a.long_steps, 1)
    L.loop_timing_read(g, 0, reset=True)
    L.loop_set_timing(g, True)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        for _ in range(steps):
            L.loop_prefill(g, tokens=tok, out=out)
        ev1.record(stream)
        torch.cuda.synchronize()
    L.loop_set_timing(g, False)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / steps, world, dev)
    classes = {}
    for ci, cname in enumerate(L.KERNEL_CLASSES):
        tms, n, work = L.loop_timing_read(g, ci)
        classes[cname] = {"ms_per_step": tms / steps, "launches": n, "work": work}
    status = L.loop_device_status()
    L.loop_model_destroy(g)
    return {"ms": ms, "value": job_throughput(B * S, world, ms), "classes": classes, "clocks": clk.summary(),
            "status": status, "steps": steps, "model": m, "batch": B, "seq": S}


# ---------------------------------------------------------------------------- oracle (CPU)

def oracle_sample(a, steps=1):
    """Time the oracle on a bounded sample of the workload on this host's cores."""
    import numpy as np
    import oracle

    w, m, decode = workload_info(a.workload)
    seed = w["seed"]
    s_tok = a.cpu_sample_tokens
    mm = dict(m, max_batch=1, max_ctx=s_tok + steps + 1)
    t0 = time.time()
    o = oracle.Model(oracle.make_config(**mm), seed=seed)
    setup = time.time() - t0
    times = []
    if decode:
        tok = seeded.tokens(seed, 1, s_tok, m["vocab"])
        o.prefill(tok)
        for i in range(steps):
            t = time.time()
            o.decode_step(np.array([int(tok[0, i % s_tok])], dtype=np.int32))
            times.append(time.time() - t)
        units = 1
        sample = (f"decode steps of 1 sequence after a {s_tok}-token prefill at the 9B shape (the workload decodes "
                  f"64 sequences after 32,768 tokens; the oracle's per-token cost there is higher)")
    elif m["io_mode"] == 1:
        h = seeded.hidden(seed, 1, s_tok, m["hidden"])
        for _ in range(steps):
            t = time.time()
            o.prefill(hidden=h)
            times.append(time.time() - t)
        units = s_tok
        sample = f"prefill of 1 x {s_tok} tokens of the workload's model (the workload is {w['batch']} x {w['seq']})"
    else:
        tok = seeded.tokens(seed, 1, s_tok, m["vocab"])
        for _ in range(steps):
            t = time.time()
            o.prefill(tok)
            times.append(time.time() - t)
        units = s_tok
        sample = (f"prefill of 1 x {s_tok} tokens of the workload's model (the workload is {w['batch']} x {w['seq']}); "
                  f"a sample, not an extrapolation: at {s_tok} tokens attention is a negligible share of the oracle's "
                  f"work, at {w['seq']} it is not")
    o.close()
    return dict(value=units / statistics.mean(times), times=times, sample=sample, setup_s=setup,
                cores=int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)))


# ---------------------------------------------------------------------------- main

def main():
    a = args_()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w, m, decode = workload_info(a.workload)
    metric, unit = metric_for(a.workload, decode)
    config = {"workload": a.workload, "batch": w["batch"], "seq_len": w["seq"],
              "l2": "inputs larger than L2: 15.6 GB of weights and >1 GB of activations stream through every step",
              "parallelism": f"replicas x{world}"}
    if decode:
        config["decode_context"] = w["seq"]

    if a.impl == "reference":
        if rank != 0:
            return
        r = oracle_sample(a, steps=a.steps)
        line = {"impl": "reference", "metric": metric, "value": r["value"], "unit": unit, "n_gpus": a.gpus,
                "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * statistics.mean(r["times"]),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": DATA, "config": config,
                "cpu_baseline": {"value": r["value"], "unit": unit, "cores": r["cores"], "kind": "oracle",
                                 "sample": r["sample"]},
                "e2e": {"value": r["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    r = run_ours(a, rank, world, local_rank)
    pk, pk_kind = peaks()
    g = r["classes"]["gemm"]
    ach = g["work"] / (g["ms_per_step"] * a.steps) / 1e9 if g["ms_per_step"] > 0 else 0.0
    peak = pk["bf16_tflops_sustained"]
    roof = {"bound": "tensor", "kernel": "tcgen05 projection GEMM (all launches in the timed steps)",
            "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak if peak else None,
            "peak_kind": f"{pk_kind} sustained bf16", "traffic": GEMM_TRAFFIC_PER_LAUNCH,
            "traffic_note": "DRAM bytes per GEMM launch (ncu, small-capture rule); achieved is over all GEMM "
                            "launches of the steps"}
    step_roof = None
    if not decode:
        fl = prefill_step_flops(m, w["batch"], w["seq"])
        step_tf = fl["total"] / (r["ms"] / 1e3) / 1e12
        step_roof = {"bound": "tensor", "achieved": step_tf, "peak": peak, "unit": "TFLOP/s",
                     "frac": step_tf / peak if peak else None, "peak_kind": f"{pk_kind} sustained bf16",
                     "flops_per_step": fl}
    line = {"metric": metric, "value": r["value"], "unit": unit, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": r["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": DATA, "config": config, "clocks": r["clocks"],
            "roofline": roof,
            "step_roofline": step_roof,
            "e2e": {"value": r["e2e_value"], "unit": unit, "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"]},
            "gpu_launches": r["launches"],
            "kernel_ms_per_step": {k: round(v["ms_per_step"], 3) for k, v in r["classes"].items()},
            "device_status": r["status"]}
    if a.workload == DEFAULT_WORKLOAD and not a.no_decode:
        d = run_decode(a, world, local_rank)
        kv_ms = d["classes"]["attention"]["ms_per_step"]
        kv_gbs = d["bytes"]["kv"] / (kv_ms / 1e3) / 1e9 if kv_ms > 0 else 0.0
        step_gbs = d["bytes"]["total"] / (d["ms"] / 1e3) / 1e9
        line["decode"] = {
            "metric": "looped-decoder decode tokens/s at 9B shape", "value": d["value"], "unit": "tokens/s",
            "ms_per_step": d["ms"], "workload": "loop9b_decode_b64_ctx32768", "batch": 64, "context": d["ctx"],
            "bytes_per_step": d["bytes"],
            "step_roofline": {"bound": "hbm", "achieved": step_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                              "frac": step_gbs / pk["hbm_gbs"], "peak_kind": f"{pk_kind} copy bandwidth"},
            "roofline": {"bound": "hbm", "kernel": "decode attention (KV-cache read)", "achieved": kv_gbs,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": kv_gbs / pk["hbm_gbs"],
                         "traffic": DECODE_ATTN_TRAFFIC_PER_LAUNCH,
                         "traffic_note": "per launch, scaled by context from a 4096-key capture"},
            "kernel_ms_per_step": {k: round(v["ms_per_step"], 3) for k, v in d["classes"].items()},
            "kernel_split_note": "per-class times come from a second run of the same steps with CUDA events around "
                                 "every launch (ms_per_step_with_launch_events); the headline ms_per_step has none",
            "ms_per_step_with_launch_events": d["ms_with_launch_events"],
            "extend": d["extend"],
            "clocks": d["clocks"]}
    if a.workload == DEFAULT_WORKLOAD and not a.no_long:
        lp = run_long_prefill(a, world, local_rank)
        fl = prefill_step_flops(lp["model"], lp["batch"], lp["seq"])
        step_tf = fl["total"] / (lp["ms"] / 1e3) / 1e12
        at = lp["classes"]["attention"]
        at_tf = at["work"] / (at["ms_per_step"] * lp["steps"]) / 1e9 if at["ms_per_step"] > 0 else 0.0
        line["long_prefill"] = {
            "metric": "looped-decoder prefill tokens/s at 9B shape, 262,144-token context", "value": lp["value"],
            "unit": "tokens/s", "ms_per_step": lp["ms"], "steps": lp["steps"], "warmup": 1,
            "workload": LONG_WORKLOAD, "batch": lp["batch"], "seq_len": lp["seq"],
            "step_roofline": {"bound": "tensor", "achieved": step_tf, "peak": peak, "unit": "TFLOP/s",
                              "frac": step_tf / peak if peak else None, "peak_kind": f"{pk_kind} sustained bf16",
                              "flops_per_step": fl},
            "roofline": {"bound": "tensor", "kernel": "tcgen05 causal flash attention (all launches of the steps)",
                         "achieved": at_tf, "peak": peak, "unit": "TFLOP/s", "frac": at_tf / peak if peak else None,
                         "peak_kind": f"{pk_kind} sustained bf16", "traffic": None},
            "kernel_ms_per_step": {k: round(v["ms_per_step"], 3) for k, v in lp["classes"].items()},
            "device_status": lp["status"], "clocks": lp["clocks"]}
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        c = oracle_sample(a, steps=1)
        line["cpu_baseline"] = {"value": c["value"], "unit": unit, "cores": c["cores"], "kind": "oracle",
                                "sample": c["sample"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
