#!/usr/bin/env python
"""Benchmark of the SSD mixer core (prefill + decode) through the C ABI.

Headline workload (one "step"): the large long-context mixer, bf16 activations with fp32
state: one sequence of 32768 tokens run as two chained 16384-token prefill calls (the
second starts from the first call's final SSM and conv states), 256 heads x headdim 64,
8 groups, d_state 128, conv 4, chunk 256; then one decode token from the second call's
final states. Every stage of the path runs each step: conv + SiLU, softplus, the chunked
SSD scan, the D skip, the gated group RMSNorm and the single-token state update. ``value``
is tokens processed per second (prefill + decode tokens) over all ranks.

The same JSON line carries the other workloads of the plan as sub-records under
``workloads`` (each with its own roofline): the tiny fp32 prefill, the small and mid bf16
prefills, and the decode workload (batch 256, 128 heads x 64, 1000 steps); the backward
pass of the small prefill under ``backward``; the dominant kernel's roofline; an
end-to-end number with host buffers; the clocks seen during the timed regions and the fp64
CPU oracle timed on the host cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Timing: CUDA events on the launching stream, W warm-up steps, a barrier and a synchronize
on both sides, the max over ranks. The headline is timed with the library's per-kernel
profiler off; per-kernel times come from a second pass over the same steps with it on.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own replica of the workload
(the mixer core has no exchange step), the time is the max over ranks, and ``value`` is
the total over ranks ("weak" scaling).
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Mamba-2 SSD mixer prefill tokens/s & decode steps/s; % of HBM roofline"
HEADLINE = "long_bf16"
SUB_PREFILL = ("tiny_f32", "small_bf16", "mid_bf16")
L2_BYTES = 126 * 2**20
TRAFFIC_FILE = "profiles/dram_traffic_per_call.json"
# model width of the layer sub-record: Nemotron-3 Nano, whose Mamba mixer has the mid workload's
# 64 heads x 64 (Modalities PR #459, commit notes: dimension 2688)
LAYER_D_MODEL = 2688


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="skip the tiny/small/mid prefill sub-records")
    ap.add_argument("--no-layer", action="store_true", help="skip the whole-layer (projections + core) sub-record")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target length of the CPU sample")
    ap.add_argument("--profile-case", choices=["long_4k", "layer_mid"], default=None,
                    help="run one small case for a profiler (3 warm-up calls, then 1) and exit: a long_bf16-shaped "
                         "prefill of 4096 tokens, or the mid_bf16 layer")
    return ap.parse_args(argv)


def profile_case(name: str) -> None:
    """Three warm-up calls and one more of a case sized for an ncu capture (a few hundred MB on
    the device, still larger than L2), then exit; prints one line, no benchmark figures."""
    import torch
    from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
    from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_params, round_bf16
    dev = torch.device("cuda", 0)
    rng = np.random.default_rng(7)
    if name == "long_4k":
        w = WORKLOADS["long_bf16"].with_(seqlen=4096, calls=1)
    else:
        w = WORKLOADS["mid_bf16"]
    d = sm.Dims(w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk, w.dconv, w.eps, w.act)
    prm = {k: torch.from_numpy(v).float().to(dev) for k, v in make_params(w, rng).items()}
    bf = lambda *shape: torch.from_numpy(round_bf16(rng.standard_normal(shape, dtype=np.float32))).to(torch.bfloat16).to(dev)
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    if name == "long_4k":
        x, z, B, C, dt = bf(w.batch, w.seqlen, HP), bf(w.batch, w.seqlen, HP), bf(w.batch, w.seqlen, GN), \
            bf(w.batch, w.seqlen, GN), bf(w.batch, w.seqlen, H)
        ws = sm.alloc_workspace(d, dev)
        run = lambda: sm.prefill(d, x, z, B, C, dt, prm["A"], prm["D"], prm["conv_w"], prm["conv_b"],
                                 prm["dt_bias"], prm["norm_w"], workspace=ws)
    else:
        width = 2 * HP + 2 * GN + H
        hid = bf(w.batch, w.seqlen, LAYER_D_MODEL)
        Win = (bf(width, LAYER_D_MODEL).float() / np.sqrt(LAYER_D_MODEL)).to(torch.bfloat16)
        Wout = (bf(LAYER_D_MODEL, HP).float() / np.sqrt(HP)).to(torch.bfloat16)
        ws = torch.empty(sm.ssd_mixer_layer_workspace_size(d, LAYER_D_MODEL), dtype=torch.uint8, device=dev)
        run = lambda: sm.layer_prefill(d, hid, Win, Wout, prm["A"], prm["D"], prm["conv_w"], prm["conv_b"],
                                       prm["dt_bias"], prm["norm_w"], workspace=ws)
    for _ in range(4):
        run()
    torch.cuda.synchronize()
    print(f"profile case {name} done", flush=True)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ algorithmic bytes

def path_bytes(w, batch, seqlen, init_states: bool) -> int:
    """Bytes one prefill call must move: read x, z, B, C, dt once, write y once, write the
    final states (and read the initial states when given). Parameters are ignored."""
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


def headline_step_bytes(w) -> int:
    """One headline step: both chained prefill calls (the second reads the first's final
    states) and the decode token."""
    return (path_bytes(w, w.batch, w.seqlen, False) + path_bytes(w, w.batch, w.seqlen, True) +
            decode_bytes(w, w.batch))


def kernel_bytes(name, w, batch, seqlen, init_states=False) -> int | None:
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
        return path_bytes(w, batch, seqlen, init_states)
    if name == "tc_norm_finish":       # gated values read and written, partial sums read
        return tok * HP * es * 2 + tok * H * 4 * 4
    if name == "tc_bc_conv":           # raw B, C read, SiLU(conv) of them written
        return tok * 2 * GN * es * 2
    return None


# ------------------------------------------------------------------ measured DRAM traffic

KERNEL_SOURCES = {"tc_prefill": ["hybrid_mamba_ssm_causal_b200/csrc/ssd_prefill_ws.cu",
                                 "hybrid_mamba_ssm_causal_b200/csrc/ssd_tc_util.cuh"],
                  "decode_step": ["hybrid_mamba_ssm_causal_b200/csrc/ssd_decode.cu"]}


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


def measured_traffic(name: str, workload: str, path: str | None = None):
    """dram__bytes_read.sum + dram__bytes_write.sum per call of kernel ``name`` on ``workload``
    (summed over the call's launches), from the committed ncu figures (a small JSON file beside
    the summaries), or None when there is no entry or the kernel's sources changed since the
    capture."""
    try:
        with open(path or os.path.join(ROOT, TRAFFIC_FILE)) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return None
    for e in data.get("entries", []):
        if e.get("kernel") == name and e.get("workload") == workload:
            if name not in KERNEL_SOURCES or e.get("kernel_sources_sha256") != sources_sha256(name):
                return None
            try:
                return float(e["traffic_bytes_per_call"])
            except (KeyError, TypeError, ValueError):
                return None
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

def decode_token_inputs(w, seed=11):
    rng = np.random.default_rng(seed)
    from hybrid_mamba_ssm_causal_b200.workloads import round_bf16
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    f = lambda *s: round_bf16(rng.standard_normal(s).astype(np.float32)) if w.act == "bf16" else rng.standard_normal(s).astype(np.float32)
    return {"x": f(w.batch, HP), "z": f(w.batch, HP), "B": f(w.batch, GN), "C": f(w.batch, GN), "dt": f(w.batch, H)}


def oracle_sample(w, inp, dec, tokens: int) -> None:
    """The oracle on the first ``tokens`` tokens of every row of the workload, followed by one
    decode token from the resulting states (a bounded sample of one headline step)."""
    import oracle
    od = oracle.Dims(w.batch, tokens, w.nheads, w.headdim, w.ngroups, w.dstate, w.dconv, w.eps)
    part = {k: (v[:, :tokens] if k in ("x", "z", "B", "C", "dt") else v) for k, v in inp.items()}
    o = oracle.prefill_dict(od, part)
    oracle.decode_step(od, dec["x"], dec["z"], dec["B"], dec["C"], dec["dt"], inp["A"], inp["D"],
                       inp["conv_w"], inp["conv_b"], inp["dt_bias"], inp["norm_w"], o["final_ssm"],
                       o["final_conv"])


def calibrate_sample(w, inp, dec, seconds: float) -> int:
    """Token count of an oracle sample that takes about ``seconds`` on the host cores."""
    t0 = time.perf_counter()
    oracle_sample(w, inp, dec, 64)
    per_tok = max(time.perf_counter() - t0, 1e-4) / 64
    tok = int(seconds / per_tok) // 64 * 64
    return int(min(max(tok, 64), w.seqlen))


def cpu_baseline(w, inp, dec, seconds: float):
    import oracle
    tok = calibrate_sample(w, inp, dec, seconds)
    t0 = time.perf_counter()
    oracle_sample(w, inp, dec, tok)
    el = time.perf_counter() - t0
    units = w.batch * (tok + 1)
    return {"value": units / el, "unit": "tokens/s", "cores": min(oracle.default_threads(), w.batch * w.ngroups),
            "kind": "oracle",
            "sample": f"fp64 oracle on the first {tok} tokens of each of the {w.batch} row(s) of {w.name} "
                      f"(all {w.nheads} heads) plus 1 decode token, {el:.1f} s; its threads run independent "
                      f"(row, group) units, {w.batch * w.ngroups} here"}


# ------------------------------------------------------------------ reference arm

def workload_desc(w):
    return (f"{w.name}: one sequence of {w.total_seqlen} tokens as {w.calls} chained prefill calls of {w.seqlen} "
            f"(b{w.batch} H{w.nheads}xP{w.headdim} G{w.ngroups} N{w.dstate} conv{w.dconv} Q{w.chunk} {w.act}, "
            f"final states passed between the calls), then 1 decode token")


def headline_config(w, world):
    return {"workload": workload_desc(w), "global_batch": w.batch * world, "seq_len": w.total_seqlen,
            "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2 ({headline_step_bytes(w) / 2**30:.2f} GiB moved per step)"}


def run_reference(a, rank, world):
    """The oracle (fp64, host cores) on the headline workload, metric and unit; rank 0 only.
    Each step is a bounded sample of the headline step (the first tokens of the sequence)."""
    if rank != 0:
        return
    from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
    import oracle
    w = WORKLOADS[HEADLINE]
    inp = make_prefill_inputs(w.with_(calls=1, seqlen=2048))     # the sample's tokens only
    dec = decode_token_inputs(w)
    per_step = max(1.0, 150.0 / max(1, a.steps + a.warmup))     # seconds per step: the run ends in minutes
    tok = calibrate_sample(w.with_(seqlen=2048), inp, dec, per_step)
    for _ in range(a.warmup):
        oracle_sample(w, inp, dec, tok)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        oracle_sample(w, inp, dec, tok)
    el = time.perf_counter() - t0
    units = w.batch * (tok + 1)
    v = units * a.steps / el
    cores = min(oracle.default_threads(), w.batch * w.ngroups)
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": el / a.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": headline_config(w, 1),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step = the fp64 oracle on the first {tok} tokens of the {w.name} "
                                       f"sequence (all {w.nheads} heads) plus 1 decode token"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


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


# ------------------------------------------------------------------ profiler

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


def profiled(lib, fn, n):
    """Run fn(i) for i < n with the library's per-kernel CUDA events on; returns
    {kernel: (total ms, launches)}. Used only outside the headline's timed region."""
    import torch
    torch.cuda.synchronize()
    lib.ssd_mixer_profile_enable(1)
    read_profile(lib)                                    # drop anything recorded earlier
    for i in range(n):
        fn(i)
    torch.cuda.synchronize()
    out = read_profile(lib)
    lib.ssd_mixer_profile_enable(0)
    return out


def roofline_of(per_kernel: dict, bytes_of, hbm: float, peak_src: str, traffic=None, calls=None):
    """Roofline of the kernel with the largest device time: algorithmic bytes per call over its
    device time per call (the sum of the call's launches: the main prefill kernel runs a call
    as several launches when its rows are split into pieces), against the measured copy
    bandwidth. ``calls``: the calls in the profiled region (default: one per launch)."""
    if not per_kernel:
        return None
    name, (tot_ms, n) = max(per_kernel.items(), key=lambda kv: kv[1][0])
    kb = bytes_of(name)
    nc = calls or n
    call_ms = tot_ms / nc
    ach = kb / (call_ms * 1e-3) / 1e9 if kb else None
    return {"kernel": name, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
            "frac": (ach / hbm) if ach else None, "traffic": traffic(name) if traffic else None,
            "peak_source": peak_src, "us_per_call": call_ms * 1e3, "launches_per_call": n / nc,
            "avg_launch_us": tot_ms / n * 1e3, "algorithmic_bytes_per_call": kb,
            "share_of_kernel_time": tot_ms / sum(v[0] for v in per_kernel.values())}


# ------------------------------------------------------------------ our arm

def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        run_reference(a, rank, world)
        return
    if a.profile_case:
        profile_case(a.profile_case)
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
    seq_keys = ("x", "z", "B", "C", "dt")

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(x: float) -> float:
        return max_over_ranks(x, world, dev)

    def dims(w, seqlen=None, batch=None):
        return sm.Dims(w.batch if batch is None else batch, w.seqlen if seqlen is None else seqlen, w.nheads,
                       w.headdim, w.ngroups, w.dstate, w.chunk, w.dconv, w.eps, w.act)

    def to_dev(v, act, adt):
        return torch.from_numpy(np.ascontiguousarray(v)).to(adt if act else torch.float32).to(dev)

    stream = torch.cuda.current_stream()

    def timed(fn, steps, warmup):
        """Average ms per call of fn(i) over `steps` calls after `warmup`, CUDA events on the
        launching stream, barrier + synchronize on both sides, max over ranks; and the number
        of this library's kernels launched in the timed region."""
        for i in range(warmup):
            fn(i)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        n0 = lib.ssd_mixer_launch_count()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            fn(warmup + i)
        e1.record(stream)
        torch.cuda.synchronize()
        launches = lib.ssd_mixer_launch_count() - n0
        barrier()
        return rank_max(e0.elapsed_time(e1) / steps), launches

    clocks = Clocks(local, not a.no_clocks)

    # ---------------- headline: long_bf16, two chained 16384-token calls + one decode token
    w = WORKLOADS[HEADLINE]
    adt = torch.bfloat16
    inp = make_prefill_inputs(w)
    dec = decode_token_inputs(w)
    P_ = {k: to_dev(inp[k], False, adt) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
    X = {k: to_dev(inp[k], True, adt) for k in seq_keys}          # [1, 32768, width]
    DQ = {k: to_dev(dec[k], True, adt) for k in seq_keys}
    L1, T = w.seqlen, w.total_seqlen
    d1, dd = dims(w), dims(w, seqlen=1)
    y = torch.empty(w.batch, T, w.d_inner, dtype=adt, device=dev)
    ydec = torch.empty(w.batch, w.d_inner, dtype=adt, device=dev)
    fs = torch.empty(w.batch, w.nheads, w.headdim, w.dstate, device=dev)
    fc = torch.empty(w.batch, w.xbc_channels, 3, dtype=adt, device=dev)
    ws = sm.alloc_workspace(d1, dev)
    half = lambda t, k: t[:, k * L1:(k + 1) * L1]

    def call(k, s=None):
        i = {n: half(X[n], k) for n in seq_keys}
        init = (None, None) if k == 0 else (fs, fc)
        sm.ssd_mixer_prefill(d1, i["x"], i["z"], i["B"], i["C"], i["dt"], P_["A"], P_["D"], P_["conv_w"],
                             P_["conv_b"], P_["dt_bias"], P_["norm_w"], init[0], init[1], half(y, k), fs, fc, ws, s)

    def decode(s=None):
        sm.ssd_mixer_decode_step(dd, DQ["x"], DQ["z"], DQ["B"], DQ["C"], DQ["dt"], P_["A"], P_["D"], P_["conv_w"],
                                 P_["conv_b"], P_["dt_bias"], P_["norm_w"], fs, fc, None, ydec, s)

    def step(_i):
        call(0)
        call(1)
        decode()

    time.sleep(0.3 if not a.no_clocks else 0)
    ms, launches = timed(step, a.steps, a.warmup)
    tok_step = w.batch * (T + 1)
    value = job_value(world, tok_step, ms)
    step_bytes = headline_step_bytes(w)
    per_kernel = profiled(lib, step, a.steps)
    call_bytes = (path_bytes(w, w.batch, L1, False) + path_bytes(w, w.batch, L1, True)) // 2

    def head_bytes(name):
        if name == "tc_prefill":
            return call_bytes
        return kernel_bytes(name, w, w.batch, L1)

    roofline = roofline_of(per_kernel, head_bytes, hbm, peak_src, lambda n: measured_traffic(n, HEADLINE),
                           calls=2 * a.steps)
    if roofline:
        roofline["units_per_call"] = f"{w.batch * L1} tokens x {w.nheads} heads (one 16384-token call)"

    # ---------------- end to end: pinned host inputs, copies inside the timed region
    e2e = None
    if not a.no_e2e:
        host = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(adt).pin_memory() for k in seq_keys}
        hdec = {k: torch.from_numpy(np.ascontiguousarray(dec[k])).to(adt).pin_memory() for k in seq_keys}
        hy = torch.empty(w.batch, T, w.d_inner, dtype=adt).pin_memory()
        hyd = torch.empty(w.batch, w.d_inner, dtype=adt).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values()) + \
            sum(v.numel() * v.element_size() for v in hdec.values())
        d2h = hy.numel() * hy.element_size() + hyd.numel() * hyd.element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        call_done, y_copied = [ev(), ev()], [ev(), ev()]
        for e_ in call_done + y_copied:
            e_.record(stream)
        dec_done, ydec_copied = ev(), ev()
        dec_done.record(stream)
        ydec_copied.record(stream)

        def e2e_step(_i):
            # inputs of each call go in on their own stream as soon as the previous step's call
            # has finished reading that half; y leaves on a third stream as soon as it is written
            ins = []
            for k in (0, 1):
                s_in.wait_event(call_done[k])
                with torch.cuda.stream(s_in):
                    for n in seq_keys:
                        half(X[n], k).copy_(half(host[n], k), non_blocking=True)
                    if k == 1:
                        s_in.wait_event(dec_done)
                        for n in seq_keys:
                            DQ[n].copy_(hdec[n], non_blocking=True)
                e_in = ev()
                e_in.record(s_in)
                ins.append(e_in)
            for k in (0, 1):
                stream.wait_event(ins[k])
                stream.wait_event(y_copied[k])
                call(k)
                call_done[k].record(stream)
            stream.wait_event(ydec_copied)
            decode()
            dec_done.record(stream)
            with torch.cuda.stream(s_out):
                for k in (0, 1):
                    s_out.wait_event(call_done[k])
                    half(hy, k).copy_(half(y, k), non_blocking=True)
                    y_copied[k].record(s_out)
                s_out.wait_event(dec_done)
                hyd.copy_(ydec, non_blocking=True)
                ydec_copied.record(s_out)

        def e2e_timed(fn, steps, warmup):
            for i in range(warmup):
                fn(i)
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            s_in.wait_event(f0)
            s_out.wait_event(f0)
            for i in range(steps):
                fn(warmup + i)
            stream.wait_event(y_copied[1])
            stream.wait_event(ydec_copied)
            f1.record(stream)
            torch.cuda.synchronize()
            barrier()
            return rank_max(f0.elapsed_time(f1) / steps)

        ems = e2e_timed(e2e_step, a.steps, max(3, min(a.warmup, 5)))

        def h2d_step(_i):   # the step's host-to-device copies alone, on the same copy stream
            with torch.cuda.stream(s_in):
                for k in (0, 1):
                    for n in seq_keys:
                        half(X[n], k).copy_(half(host[n], k), non_blocking=True)
                for n in seq_keys:
                    DQ[n].copy_(hdec[n], non_blocking=True)

        def copies_timed(fn, steps):
            fn(0)
            torch.cuda.synchronize()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(s_in)
            for i in range(steps):
                fn(i)
            f1.record(s_in)
            torch.cuda.synchronize()
            return rank_max(f0.elapsed_time(f1) / steps)

        h2d_ms = copies_timed(h2d_step, max(3, min(a.steps, 10)))
        e2e = {"value": job_value(world, tok_step, ems), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems, "h2d_only_ms_per_step": h2d_ms,
               "how": "pinned host buffers; each call's inputs copied in on a copy stream, y copied out on "
                      "another, overlapped with the other call's compute; h2d_only_ms_per_step times the "
                      "host-to-device copies of a step alone"}
        del host, hy
    del X, y

    # ---------------- the other prefill workloads (sub-records)
    subs = {}
    if not a.no_sub:
        for name in SUB_PREFILL:
            wsub = WORKLOADS[name]
            sadt = torch.bfloat16 if wsub.act == "bf16" else torch.float32
            sinp = make_prefill_inputs(wsub)
            init = sinp["init_ssm"] is not None
            cb = path_bytes(wsub, wsub.batch, wsub.seqlen, init)
            nsets = max(1, min(2048, -(-2 * L2_BYTES // cb)))       # rotating sets: > 2x L2 in total
            sp = {k: to_dev(sinp[k], False, sadt) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
            base = {k: to_dev(sinp[k], True, sadt) for k in seq_keys}
            i_ssm = to_dev(sinp["init_ssm"], False, sadt) if init else None
            i_conv = to_dev(sinp["init_conv"], True, sadt) if sinp["init_conv"] is not None else None
            sets = []
            for _ in range(nsets):
                sets.append({"in": {k: v.clone() for k, v in base.items()} if nsets > 1 else base,
                             "y": torch.empty(wsub.batch, wsub.seqlen, wsub.d_inner, dtype=sadt, device=dev),
                             "fs": torch.empty(wsub.batch, wsub.nheads, wsub.headdim, wsub.dstate, device=dev),
                             "fc": torch.empty(wsub.batch, wsub.xbc_channels, 3, dtype=sadt, device=dev)})
            dsub = dims(wsub)
            wsp = sm.alloc_workspace(dsub, dev)

            def scall(i, t=None, d_=dsub, sets_=sets, p_=sp, ws_=wsp, ii=i_ssm, ic=i_conv):
                t = sets_[i % len(sets_)]
                q = t["in"]
                sm.ssd_mixer_prefill(d_, q["x"], q["z"], q["B"], q["C"], q["dt"], p_["A"], p_["D"], p_["conv_w"],
                                     p_["conv_b"], p_["dt_bias"], p_["norm_w"], ii, ic, t["y"], t["fs"], t["fc"],
                                     ws_)

            sms, sl = timed(scall, max(a.steps, 20), max(3, a.warmup))
            pk = profiled(lib, scall, max(a.steps, 20))
            rf = roofline_of(pk, lambda n, ww=wsub: kernel_bytes(n, ww, ww.batch, ww.seqlen, init), hbm, peak_src,
                             lambda n, nm=name: measured_traffic(n, nm), calls=max(a.steps, 20))
            subs[name] = {
                "workload": f"{name}: prefill b{wsub.batch} L{wsub.seqlen} H{wsub.nheads}xP{wsub.headdim} "
                            f"G{wsub.ngroups} N{wsub.dstate} Q{wsub.chunk} {wsub.act}"
                            + (", initial states given" if init else ""),
                "value": job_value(world, wsub.batch * wsub.seqlen, sms), "unit": "tokens/s",
                "us_per_call": sms * 1e3, "launches_per_call": sl / max(a.steps, 20),
                "path_hbm": {"algorithmic_bytes_per_call": cb, "achieved_gbs": cb / (sms * 1e-3) / 1e9,
                             "frac": cb / (sms * 1e-3) / 1e9 / hbm, "peak": hbm},
                "roofline": rf,
                "kernels": {k: {"us_per_call": v[0] * 1e3 / max(a.steps, 20), "launches": v[1]} for k, v in pk.items()},
                "l2": f"{nsets} rotating input/output set(s), {nsets * cb / 2**20:.0f} MiB",
            }
            if name == "tiny_f32":
                subs[name]["note"] = "fp32 CUDA-core path; latency-bound at this size (no roofline claim)"
            del sets, base, wsp

    # ---------------- the whole mixer layer (in_proj -> core -> out_proj) on the mid workload
    layer = None
    if not a.no_layer:
        from hybrid_mamba_ssm_causal_b200.workloads import make_params, round_bf16
        wl = WORKLOADS["mid_bf16"]
        d_model = LAYER_D_MODEL
        HP, GN, H = wl.d_inner, wl.ngroups * wl.dstate, wl.nheads
        width = 2 * HP + 2 * GN + H
        rows = wl.batch * wl.seqlen
        rng = np.random.default_rng(5)
        lp = make_params(wl, rng)
        hid = torch.from_numpy(round_bf16(rng.standard_normal((wl.batch, wl.seqlen, d_model), dtype=np.float32))).to(adt).to(dev)
        Win = torch.from_numpy(round_bf16((rng.standard_normal((width, d_model), dtype=np.float32) /
                                           np.float32(np.sqrt(d_model))))).to(adt).to(dev)
        Wout = torch.from_numpy(round_bf16((rng.standard_normal((d_model, HP), dtype=np.float32) /
                                            np.float32(np.sqrt(HP))))).to(adt).to(dev)
        LP = {k: to_dev(lp[k], False, adt) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
        dlay = dims(wl)
        lws = torch.empty(sm.ssd_mixer_layer_workspace_size(dlay, d_model), dtype=torch.uint8, device=dev)
        lout = (torch.empty(wl.batch, wl.seqlen, d_model, dtype=adt, device=dev),
                torch.empty(wl.batch, H, wl.headdim, wl.dstate, device=dev),
                torch.empty(wl.batch, wl.xbc_channels, 3, dtype=adt, device=dev))

        def lstep(_i):
            sm.layer_prefill(dlay, hid, Win, Wout, LP["A"], LP["D"], LP["conv_w"], LP["conv_b"], LP["dt_bias"],
                             LP["norm_w"], None, None, workspace=lws, out=lout)

        lms, llaunch = timed(lstep, max(3, a.steps // 2), max(3, a.warmup))
        lk = profiled(lib, lstep, max(3, a.steps // 2))

        def lstep_fused(_i):
            sm.layer_prefill(dlay, hid, Win, Wout, LP["A"], LP["D"], LP["conv_w"], LP["conv_b"], LP["dt_bias"],
                             LP["norm_w"], None, None, workspace=lws, out=lout, norm_in_out_proj=True)

        lms_fused, _ = timed(lstep_fused, max(3, a.steps // 2), max(3, a.warmup))
        nrep = max(3, a.steps // 2)
        fl_in, fl_out = 2.0 * rows * d_model * width, 2.0 * rows * HP * d_model
        gem = {}
        gemm_ms = sum(v[0] for k, v in lk.items() if k.startswith("tc_gemm"))
        if gemm_ms > 0:
            # two GEMM launches per call: in_proj, then out_proj (with the norm prologue when the
            # group is wider than a cluster)
            gem = {"kernel": "tc_gemm (in_proj + out_proj)", "bound": "tensor", "unit": "TFLOP/s",
                   "achieved": (fl_in + fl_out) * nrep / (gemm_ms * 1e-3) / 1e12,
                   "peak": tf_burst, "peak_source": peak_src}
            gem["frac"] = gem["achieved"] / tf_burst
        layer = {"workload": f"mid_bf16 layer: b{wl.batch} L{wl.seqlen}, d_model {d_model}, in_proj {d_model}->{width}, "
                             f"core H{H}xP{wl.headdim} G{wl.ngroups} N{wl.dstate}, out_proj {HP}->{d_model}",
                 "value": job_value(world, rows, lms), "unit": "tokens/s", "ms_per_call": lms,
                 "ms_per_call_norm_in_out_proj": lms_fused,
                 "launches_per_call": llaunch / nrep, "gemm_flops_per_call": fl_in + fl_out,
                 "roofline": gem or None,
                 "kernels": {k: {"ms_per_call": v[0] / nrep, "launches": v[1]} for k, v in lk.items()}}
        del hid, Win, Wout, lws, lout

    # ---------------- decode workload: 256 sequences, 1000 single-token steps, state in place
    decode_rec = None
    if not a.no_decode:
        wd = WORKLOADS["decode_bf16"]
        pool = 64                                           # distinct per-step inputs (> L2 in total)
        di = make_decode_inputs(wd, steps=pool)
        ssm = torch.from_numpy(di["init_ssm"]).to(dev)
        conv = torch.from_numpy(di["init_conv"]).to(adt).to(dev)
        dparams = {k: to_dev(di[k], False, adt) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
        dseq = {k: to_dev(di[k], True, adt) for k in seq_keys}
        ydd = torch.empty(wd.batch, wd.d_inner, dtype=adt, device=dev)
        ddims = sm.Dims(wd.batch, 1, wd.nheads, wd.headdim, wd.ngroups, wd.dstate, 1, wd.dconv, wd.eps, wd.act)
        Q = dparams

        def dstep(s):
            j = s % pool
            sm.ssd_mixer_decode_step(ddims, dseq["x"][j], dseq["z"][j], dseq["B"][j], dseq["C"][j], dseq["dt"][j],
                                     Q["A"], Q["D"], Q["conv_w"], Q["conv_b"], Q["dt_bias"], Q["norm_w"],
                                     ssm, conv, None, ydd)

        dms, _ = timed(dstep, a.decode_steps, max(3, a.warmup))
        db = decode_bytes(wd, wd.batch)
        ach = db / (dms * 1e-3) / 1e9
        decode_rec = {"workload": f"decode_bf16: b{wd.batch} H{wd.nheads}xP{wd.headdim} G{wd.ngroups} N{wd.dstate} "
                                  f"fp32 state, {a.decode_steps} steps",
                      "value": job_value(world, 1, dms), "unit": "steps/s",
                      "tokens_per_s": job_value(world, wd.batch, dms), "us_per_step": dms * 1e3,
                      "roofline": {"kernel": "decode_step", "bound": "hbm", "achieved": ach, "peak": hbm,
                                   "unit": "GB/s", "frac": ach / hbm,
                                   "traffic": measured_traffic("decode_step", "decode_bf16"),
                                   "algorithmic_bytes_per_launch": db, "peak_source": peak_src}}
        subs["decode_bf16"] = decode_rec

    # ---------------- backward pass of the small prefill (gradient on y only): one call per step
    bwd = None
    if not a.no_backward:
        from hybrid_mamba_ssm_causal_b200.workloads import round_bf16
        wb = WORKLOADS["small_bf16"]
        binp = make_prefill_inputs(wb)
        HP, GN, H, Cc = wb.d_inner, wb.ngroups * wb.dstate, wb.nheads, wb.xbc_channels
        rng = np.random.default_rng(13)
        dout = to_dev(round_bf16(rng.standard_normal((wb.batch, wb.seqlen, HP))).astype(np.float32), True, adt)
        bp = {k: to_dev(binp[k], False, adt) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
        bi = {k: to_dev(binp[k], True, adt) for k in seq_keys}
        db_ = dims(wb)
        bws = torch.empty(sm.ssd_mixer_backward_workspace_size(db_), dtype=torch.uint8, device=dev)
        ga = {k: torch.empty(wb.batch, wb.seqlen, n, dtype=adt, device=dev)
              for k, n in (("x", HP), ("z", HP), ("B", GN), ("C", GN), ("dt", H))}
        gp = {k: torch.empty(*shape, dtype=torch.float32, device=dev)
              for k, shape in (("A", (H,)), ("D", (H,)), ("conv_w", (Cc, 4)), ("conv_b", (Cc,)),
                               ("dt_bias", (H,)), ("norm_w", (HP,)))}

        def bstep(_s):
            sm.ssd_mixer_backward(db_, bi["x"], bi["z"], bi["B"], bi["C"], bi["dt"], bp["A"], bp["D"], bp["conv_w"],
                                  bp["conv_b"], bp["dt_bias"], bp["norm_w"], None, None, dout, None, None,
                                  ga["x"], ga["z"], ga["B"], ga["C"], ga["dt"], gp["A"], gp["D"], gp["conv_w"],
                                  gp["conv_b"], gp["dt_bias"], gp["norm_w"], None, None, bws)

        bms, blaunch = timed(bstep, a.steps, max(3, a.warmup))
        bk = profiled(lib, bstep, a.steps)
        bb = backward_bytes(wb, wb.batch, wb.seqlen)
        ach = bb / (bms * 1e-3) / 1e9
        bwd = {"workload": f"small_bf16 backward: b{wb.batch} L{wb.seqlen}, gradient on y only, {a.steps} calls",
               "ms_per_call": bms, "tokens_per_s": job_value(world, wb.batch * wb.seqlen, bms),
               "launches_per_call": blaunch / a.steps,
               "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                            "algorithmic_bytes_per_call": bb, "peak_source": peak_src},
               "kernels": {k: {"ms_per_call": v[0] / a.steps, "launches": v[1]} for k, v in bk.items()}}

    ck = clocks.stop()   # sampled over every timed region above
    cpu = None
    if rank == 0 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, inp, dec, a.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": headline_config(w, world),
            "path_hbm": {"algorithmic_bytes_per_step": step_bytes,
                         "achieved_gbs": step_bytes / (ms * 1e-3) / 1e9,
                         "frac": step_bytes / (ms * 1e-3) / 1e9 / hbm, "peak": hbm, "peak_source": peak_src},
            "roofline": roofline, "kernels": {k: {"ms_per_step": v[0] / a.steps, "launches": v[1]}
                                              for k, v in per_kernel.items()},
            "gpu_launches": launches, "e2e": e2e, "workloads": subs, "layer": layer, "decode_workload": decode_rec,
            "backward": bwd, "clocks": ck, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
