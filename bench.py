#!/usr/bin/env python
"""Benchmark of the SSD mixer core (prefill + decode) through the C ABI.

Workload (one "step"): the small hybrid-shaped mixer, bf16 activations with fp32 state:
batch 2 x 2048 tokens, 32 heads x headdim 64, 8 groups, d_state 128, conv 4, chunk 128.
A step prefills the whole batch (conv + SiLU, softplus, chunked SSD scan, D skip,
gated group RMSNorm) and then decodes one more token per sequence from the prefill's
final states, so every stage of the path runs once per step. ``value`` is tokens
processed per second (prefill + decode tokens) over all ranks.

The same JSON line carries the decode workload (batch 256, 128 heads x 64, 8 groups,
d_state 128, fp32 state, 1000 steps) in ``decode_workload``, the backward pass of the
step's prefill (gradient on y) in ``backward``, the dominant kernel's roofline, an
end-to-end number with host buffers, the clocks seen during the timed region and the fp64
CPU oracle timed on the host cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own replica of the batch
(the mixer core has no exchange step), the time is the max over ranks, and ``value``
is the total over ranks ("weak" scaling).
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Mamba-2 SSD mixer prefill tokens/s & decode steps/s; % of HBM roofline"
WORKLOAD = "small_bf16"
L2_BYTES = 126 * 2**20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target length of the CPU sample")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ algorithmic bytes

def path_bytes(w, batch, seqlen, init_states: bool) -> int:
    """Bytes the prefill must move: read x, z, B, C, dt once, write y once, the final
    states (and read the initial states when given). Parameters are ignored."""
    es = 2 if w.act == "bf16" else 4
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    tok = batch * seqlen
    io_ = tok * (3 * HP + 2 * GN + H) * es
    st = batch * H * w.headdim * w.dstate * 4 + batch * w.xbc_channels * 3 * es
    return io_ + st * (2 if init_states else 1)


def decode_bytes(w, batch) -> int:
    """One decode step: the fp32 state and the conv state read and written, the token's
    inputs read and y written."""
    es = 2 if w.act == "bf16" else 4
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    state = 2 * batch * H * w.headdim * w.dstate * 4
    conv = 2 * batch * w.xbc_channels * 3 * es
    return state + conv + batch * (3 * HP + 2 * GN + H) * es


def backward_bytes(w, batch, seqlen) -> int:
    """Bytes the backward pass must move with gradients on y only and no initial states:
    read x, z, B, C, dt and dy once, write dx, dz, dB, dC and ddt once. Parameters and their
    gradients are ignored."""
    es = 2 if w.act == "bf16" else 4
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    return batch * seqlen * (2 * (2 * HP + 2 * GN + H) + HP) * es


def kernel_bytes(name, w, batch, seqlen) -> int | None:
    """Minimum bytes of one launch of each kernel: its inputs read once, its outputs
    written once (for the fused prefill kernel these are the path's bytes)."""
    es = 2 if w.act == "bf16" else 4
    HP, GN, H, Cc = w.d_inner, w.ngroups * w.dstate, w.nheads, w.xbc_channels
    P, N, Q = w.headdim, w.dstate, w.chunk
    tok = batch * seqlen
    nc = -(-seqlen // Q)
    states = batch * nc * H * P * N * 4
    if name == "conv_silu":
        return tok * Cc * es * 2
    if name == "simt_chunk_state":
        return tok * (HP + GN + H) * es + tok * H * 8 + states
    if name == "simt_state_pass":
        return 2 * states + batch * H * P * N * 4 + tok * H * 4 // Q
    if name == "simt_chunk_scan":
        return tok * Cc * es + tok * H * 8 + states + tok * HP * 4
    if name == "gated_norm":
        return tok * HP * (4 + 2 * es)
    if name == "decode_step":
        return decode_bytes(w, batch)
    if name == "tc_prefill":           # the whole prefill in one kernel
        return path_bytes(w, batch, seqlen, False)
    if name == "tc_norm_finish":       # gated values read and written, partial sums read
        return tok * HP * es * 2 + tok * H * 4 * 4
    return None


# ------------------------------------------------------------------ measured DRAM traffic

KERNEL_SOURCES = {"tc_prefill": ["hybrid_mamba_ssm_causal_b200/csrc/ssd_prefill_ws.cu",
                                 "hybrid_mamba_ssm_causal_b200/csrc/ssd_tc_util.cuh"],
                  "decode_step": ["hybrid_mamba_ssm_causal_b200/csrc/ssd_decode.cu"]}
TRAFFIC_SUMMARIES = {"tc_prefill": "profiles/ssd_prefill_ws_small_bf16.md",
                     "decode_step": "profiles/decode_step_decode_bf16.md"}


def code_only(text: str) -> str:
    """C++/CUDA source without its comments and with whitespace collapsed: the part that
    decides what the compiled kernel does."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":                                   # string or char literal, kept whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def sources_sha256(name: str) -> str:
    """Hash of the code (comments and layout ignored) of the files a kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[name]:
        with open(os.path.join(ROOT, rel)) as f:
            h.update(code_only(f.read()).encode())
    return h.hexdigest()


def measured_traffic(name: str):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch from the committed ncu summary
    of this kernel, or None when there is none or the kernel's sources changed since."""
    if name not in TRAFFIC_SUMMARIES:
        return None
    try:
        with open(os.path.join(ROOT, TRAFFIC_SUMMARIES[name])) as f:
            kv = dict(line.split(":", 1) for line in f.read().splitlines()
                      if line.startswith(("traffic_bytes_per_launch:", "kernel_sources_sha256:")))
    except OSError:
        return None
    if kv.get("kernel_sources_sha256", "").strip() != sources_sha256(name):
        return None
    try:
        return float(kv["traffic_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks

class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, enabled: bool):
        self.proc = None
        self.index = index
        if enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in csv.reader(io.StringIO(out)):
            if len(row) < 8:
                continue
            try:
                sm.append(float(row[0]))
                mx = float(row[1])
            except ValueError:
                continue
            for nm, v in zip(names, row[4:8]):
                if v.strip().lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle

def cpu_oracle_step(w, inp, dec):
    import oracle
    od = oracle.Dims(w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate, w.dconv, w.eps)
    o = oracle.prefill_dict(od, inp)
    oracle.decode_step(od, dec["x"], dec["z"], dec["B"], dec["C"], dec["dt"], inp["A"], inp["D"],
                       inp["conv_w"], inp["conv_b"], inp["dt_bias"], inp["norm_w"], o["final_ssm"],
                       o["final_conv"])


def cpu_baseline(w, inp, dec, seconds: float):
    import oracle
    tok = w.batch * (w.seqlen + 1)
    reps, t0 = 0, time.perf_counter()
    while True:
        cpu_oracle_step(w, inp, dec)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": tok * reps / el, "unit": "tokens/s", "cores": oracle.default_threads(), "kind": "oracle",
            "sample": f"{reps} full steps of the workload (prefill {w.batch}x{w.seqlen} + 1 decode token), "
                      f"fp64, {el:.1f} s"}


def decode_token_inputs(w, seed=11):
    rng = np.random.default_rng(seed)
    from hybrid_mamba_ssm_causal_b200.workloads import round_bf16
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    f = lambda *s: round_bf16(rng.standard_normal(s).astype(np.float32)) if w.act == "bf16" else rng.standard_normal(s).astype(np.float32)
    return {"x": f(w.batch, HP), "z": f(w.batch, HP), "B": f(w.batch, GN), "C": f(w.batch, GN), "dt": f(w.batch, H)}


# ------------------------------------------------------------------ reference arm

def run_reference(a, rank, world):
    """The oracle (fp64, host cores) on the same workload, metric and unit; rank 0 only."""
    if rank != 0:
        return
    from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
    import oracle
    w = WORKLOADS[WORKLOAD]
    inp = make_prefill_inputs(w)
    dec = decode_token_inputs(w)
    for _ in range(a.warmup):
        cpu_oracle_step(w, inp, dec)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        cpu_oracle_step(w, inp, dec)
    el = time.perf_counter() - t0
    tok = w.batch * (w.seqlen + 1)
    v = tok * a.steps / el
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": el / a.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w), "global_batch": w.batch, "seq_len": w.seqlen,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.default_threads(), "kind": "oracle",
                             "sample": f"each step = the full workload step (prefill {w.batch}x{w.seqlen} + 1 decode token)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_desc(w):
    return (f"{w.name}: prefill b{w.batch} L{w.seqlen} H{w.nheads}xP{w.headdim} G{w.ngroups} N{w.dstate} "
            f"conv{w.dconv} Q{w.chunk} {w.act}, then 1 decode step")


# ------------------------------------------------------------------ ranks

def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, units_per_rank_step: int, ms_per_step: float) -> float:
    """Whole-job throughput: the units every rank processed per step over the step time (weak
    scaling: each rank runs its own replica of the workload)."""
    return world * units_per_rank_step / (ms_per_step * 1e-3)


# ------------------------------------------------------------------ our arm

def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        run_reference(a, rank, world)
        return

    import torch
    import torch.distributed as dist
    from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
    from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_decode_inputs, make_prefill_inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    lib = sm.load_library()
    hbm, tf_burst, tf_sus, peak_src = peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(x: float) -> float:
        return max_over_ranks(x, world, dev)

    w = WORKLOADS[WORKLOAD]
    inp = make_prefill_inputs(w)
    dec = decode_token_inputs(w)
    adt = torch.bfloat16 if w.act == "bf16" else torch.float32
    seq_keys = ("x", "z", "B", "C", "dt")

    def dev_t(v, act):
        return torch.from_numpy(np.ascontiguousarray(v)).to(adt if act else torch.float32).to(dev)

    params = {k: dev_t(inp[k], False) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
    d = sm.Dims(w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk, w.dconv, w.eps, w.act)
    dd = sm.Dims(w.batch, 1, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk, w.dconv, w.eps, w.act)
    step_bytes = path_bytes(w, w.batch, w.seqlen, False) + decode_bytes(w, w.batch)
    nsets = max(2, -(-2 * L2_BYTES // step_bytes))       # rotating input sets: > 2x L2 in total
    base = {k: dev_t(inp[k], True) for k in seq_keys}
    dbase = {k: dev_t(dec[k], True) for k in seq_keys}
    sets = []
    for _ in range(nsets):
        sets.append({
            "in": {k: v.clone() for k, v in base.items()},
            "dec": {k: v.clone() for k, v in dbase.items()},
            "y": torch.empty(w.batch, w.seqlen, w.d_inner, dtype=adt, device=dev),
            "ydec": torch.empty(w.batch, w.d_inner, dtype=adt, device=dev),
            "fs": torch.empty(w.batch, w.nheads, w.headdim, w.dstate, device=dev),
            "fc": torch.empty(w.batch, w.xbc_channels, 3, dtype=adt, device=dev),
        })
    ws = sm.alloc_workspace(d, dev)
    P = params

    def step(s):
        t = sets[s % nsets]
        i = t["in"]
        sm.ssd_mixer_prefill(d, i["x"], i["z"], i["B"], i["C"], i["dt"], P["A"], P["D"], P["conv_w"], P["conv_b"],
                             P["dt_bias"], P["norm_w"], None, None, t["y"], t["fs"], t["fc"], ws)
        q = t["dec"]
        sm.ssd_mixer_decode_step(dd, q["x"], q["z"], q["B"], q["C"], q["dt"], P["A"], P["D"], P["conv_w"],
                                 P["conv_b"], P["dt_bias"], P["norm_w"], t["fs"], t["fc"], None, t["ydec"])

    stream = torch.cuda.current_stream()
    for s in range(a.warmup):
        step(s)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = Clocks(local, not a.no_clocks)
    time.sleep(0.3 if not a.no_clocks else 0)
    lib.ssd_mixer_profile_enable(1)
    lib.ssd_mixer_profile_read(*prof_buffers())          # drop anything recorded earlier
    n0 = lib.ssd_mixer_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(a.steps):
        step(a.warmup + s)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = lib.ssd_mixer_launch_count() - n0
    per_kernel = read_profile(lib)
    lib.ssd_mixer_profile_enable(0)
    barrier()
    ms_local = e0.elapsed_time(e1) / a.steps
    ms = rank_max(ms_local)
    tok_step = w.batch * (w.seqlen + 1)
    value = job_value(world, tok_step, ms)

    # dominant kernel and its roofline
    dom = max(per_kernel.items(), key=lambda kv: kv[1][0]) if per_kernel else None
    roofline = None
    if dom:
        name, (tot_ms, n) = dom
        kb = kernel_bytes(name, w, w.batch, w.seqlen)
        avg_ms = tot_ms / n
        ach = kb / (avg_ms * 1e-3) / 1e9 if kb else None
        roofline = {"kernel": name, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                    "frac": (ach / hbm) if ach else None, "traffic": measured_traffic(name), "peak_source": peak_src,
                    "avg_launch_us": avg_ms * 1e3, "algorithmic_bytes_per_launch": kb,
                    "share_of_step": tot_ms / (ms_local * a.steps)}

    # end to end through the C ABI with host buffers (pinned), copies inside the timed region
    e2e = None
    if not a.no_e2e:
        host_in = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(adt).pin_memory() for k in seq_keys}
        host_dec = {k: torch.from_numpy(np.ascontiguousarray(dec[k])).to(adt).pin_memory() for k in seq_keys}
        host_y = torch.empty(w.batch, w.seqlen, w.d_inner, dtype=adt).pin_memory()
        host_yd = torch.empty(w.batch, w.d_inner, dtype=adt).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host_in.values()) + \
            sum(v.numel() * v.element_size() for v in host_dec.values())
        d2h = host_y.numel() * host_y.element_size() + host_yd.numel() * host_yd.element_size()

        def e2e_step(s):
            t = sets[s % nsets]
            for k in seq_keys:
                t["in"][k].copy_(host_in[k], non_blocking=True)
                t["dec"][k].copy_(host_dec[k], non_blocking=True)
            step(s)
            host_y.copy_(t["y"], non_blocking=True)
            host_yd.copy_(t["ydec"], non_blocking=True)

        for s in range(a.warmup):
            e2e_step(s)
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for s in range(a.steps):
            e2e_step(s)
        f1.record(stream)
        torch.cuda.synchronize()
        ems = rank_max(f0.elapsed_time(f1) / a.steps)
        e2e = {"value": job_value(world, tok_step, ems), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems}

    # decode workload: 256 sequences, 1000 single-token steps, state in place
    decode = None
    if not a.no_decode:
        wd = WORKLOADS["decode_bf16"]
        pool = 64                                           # distinct per-step inputs (> L2 in total)
        di = make_decode_inputs(wd, steps=pool)
        ssm = torch.from_numpy(di["init_ssm"]).to(dev)
        conv = torch.from_numpy(di["init_conv"]).to(adt).to(dev)
        dparams = {k: dev_t(di[k], False) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
        dseq = {k: dev_t(di[k], True) for k in seq_keys}
        ydec = torch.empty(wd.batch, wd.d_inner, dtype=adt, device=dev)
        ddims = sm.Dims(wd.batch, 1, wd.nheads, wd.headdim, wd.ngroups, wd.dstate, 1, wd.dconv, wd.eps, wd.act)
        Q = dparams

        def dstep(s):
            j = s % pool
            sm.ssd_mixer_decode_step(ddims, dseq["x"][j], dseq["z"][j], dseq["B"][j], dseq["C"][j], dseq["dt"][j],
                                     Q["A"], Q["D"], Q["conv_w"], Q["conv_b"], Q["dt_bias"], Q["norm_w"],
                                     ssm, conv, None, ydec)

        for s in range(max(3, a.warmup)):
            dstep(s)
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for s in range(a.decode_steps):
            dstep(s)
        g1.record(stream)
        torch.cuda.synchronize()
        dms = rank_max(g0.elapsed_time(g1) / a.decode_steps)
        db = decode_bytes(wd, wd.batch)
        ach = db / (dms * 1e-3) / 1e9
        decode = {"workload": f"decode_bf16: b{wd.batch} H{wd.nheads}xP{wd.headdim} G{wd.ngroups} N{wd.dstate} "
                              f"fp32 state, {a.decode_steps} steps",
                  "value": job_value(world, 1, dms), "unit": "steps/s", "tokens_per_s": job_value(world, wd.batch, dms),
                  "us_per_step": dms * 1e3,
                  "roofline": {"kernel": "decode_step", "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                               "frac": ach / hbm, "traffic": measured_traffic("decode_step"),
                               "algorithmic_bytes_per_launch": db, "peak_source": peak_src}}

    # backward pass of the same prefill (gradient on y only): one call per step
    bwd = None
    if not a.no_backward:
        from hybrid_mamba_ssm_causal_b200.workloads import round_bf16
        HP, GN, H, Cc = w.d_inner, w.ngroups * w.dstate, w.nheads, w.xbc_channels
        rng = np.random.default_rng(13)
        dout = dev_t(round_bf16(rng.standard_normal((w.batch, w.seqlen, HP))).astype(np.float32), True)
        bws = torch.empty(sm.ssd_mixer_backward_workspace_size(d), dtype=torch.uint8, device=dev)
        ga = {k: torch.empty(w.batch, w.seqlen, n, dtype=adt, device=dev)
              for k, n in (("x", HP), ("z", HP), ("B", GN), ("C", GN), ("dt", H))}
        gp = {k: torch.empty(*shape, dtype=torch.float32, device=dev)
              for k, shape in (("A", (H,)), ("D", (H,)), ("conv_w", (Cc, 4)), ("conv_b", (Cc,)),
                               ("dt_bias", (H,)), ("norm_w", (HP,)))}

        def bstep(s):
            i = sets[s % nsets]["in"]
            sm.ssd_mixer_backward(d, i["x"], i["z"], i["B"], i["C"], i["dt"], P["A"], P["D"], P["conv_w"],
                                  P["conv_b"], P["dt_bias"], P["norm_w"], None, None, dout, None, None,
                                  ga["x"], ga["z"], ga["B"], ga["C"], ga["dt"], gp["A"], gp["D"], gp["conv_w"],
                                  gp["conv_b"], gp["dt_bias"], gp["norm_w"], None, None, bws)

        for s in range(max(3, a.warmup)):
            bstep(s)
        torch.cuda.synchronize()
        barrier()
        lib.ssd_mixer_profile_enable(1)
        lib.ssd_mixer_profile_read(*prof_buffers())
        n0 = lib.ssd_mixer_launch_count()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for s in range(a.steps):
            bstep(s)
        b1.record(stream)
        torch.cuda.synchronize()
        blaunch = lib.ssd_mixer_launch_count() - n0
        bk = read_profile(lib)
        lib.ssd_mixer_profile_enable(0)
        bms = rank_max(b0.elapsed_time(b1) / a.steps)
        bb = backward_bytes(w, w.batch, w.seqlen)
        ach = bb / (bms * 1e-3) / 1e9
        bwd = {"workload": f"{w.name} backward: b{w.batch} L{w.seqlen}, gradient on y only, {a.steps} calls",
               "ms_per_call": bms, "tokens_per_s": job_value(world, w.batch * w.seqlen, bms),
               "launches_per_call": blaunch / a.steps,
               "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                            "algorithmic_bytes_per_call": bb, "peak_source": peak_src},
               "kernels": {k: {"ms_per_call": v[0] / a.steps, "launches": v[1]} for k, v in bk.items()}}

    ck = clocks.stop()   # sampled over the prefill, end-to-end, decode and backward timed regions
    cpu = None
    if rank == 0 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, inp, dec, a.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": workload_desc(w), "global_batch": w.batch * world, "seq_len": w.seqlen,
                       "parallelism": f"replicas x{world}",
                       "l2": f"{nsets} rotating input/output sets ({nsets * step_bytes / 2**20:.0f} MiB > L2)"},
            "path_hbm": {"algorithmic_bytes_per_step": step_bytes,
                         "achieved_gbs": step_bytes / (ms * 1e-3) / 1e9,
                         "frac": step_bytes / (ms * 1e-3) / 1e9 / hbm, "peak": hbm},
            "roofline": roofline, "kernels": {k: {"ms_total": v[0], "launches": v[1]} for k, v in per_kernel.items()},
            "gpu_launches": launches, "e2e": e2e, "decode_workload": decode, "backward": bwd, "clocks": ck,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


_PROF = None


def prof_buffers(n=64):
    import ctypes
    global _PROF
    if _PROF is None:
        _PROF = ((ctypes.c_char_p * n)(), (ctypes.c_double * n)(), (ctypes.c_int * n)(), n)
    return _PROF


def read_profile(lib) -> dict:
    names, ms, cnt, n = prof_buffers()
    k = lib.ssd_mixer_profile_read(names, ms, cnt, n)
    return {names[i].decode(): (ms[i], cnt[i]) for i in range(k)}


if __name__ == "__main__":
    main()
