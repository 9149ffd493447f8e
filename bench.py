#!/usr/bin/env python
"""Benchmark of the gated delta-rule hot path on B200; prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline: prefill tokens/s of the gated delta rule at H=32, d=128 (the
Qwen3-Next-like workload: B=2, T=8192, 16 q/k heads repeated to 32 v heads,
bf16 q/k/v, fp32 gates/betas/state).  A step is one dr_chunk_fwd call over the
whole batch; L2 is flushed (256 MiB write) before every timed step and each step
is timed with CUDA events on the launching stream.  Also reported in the same
line: the decode step (B=256, H=32, d=128, in-place fp32 state, state GB/s) and
the varlen long-context prefill (8 sequences of 512..16384 tokens + one of
65536), each against its roofline.

Multi-GPU (torchrun): the path needs no exchange, so every rank runs an
independent replica of the workload (weak scaling); timings are the max over
ranks; value = tokens of all ranks / that time.

--impl reference times the fp64 CPU oracle (the only reference this method has)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s (gated delta rule, H=32 d=128)"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true", help="skip decode/varlen lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ------------------------------------------------------------------ process group


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        if self.world > 1:
            import datetime

            torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            if torch.distributed.get_backend() == "nccl":
                torch.distributed.barrier(device_ids=[self.local])
            else:
                torch.distributed.barrier()

    def max(self, x: float, device=None) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            torch.distributed.destroy_process_group()


# ------------------------------------------------------------------ accounting


def prefill_bytes(B, T, Hqk, Hv, dk, dv, in_bytes, out_bytes, n_states, with_state_in):
    """Algorithmic HBM bytes of one prefill call: every input read once, every output written once."""
    tok = B * T
    b = tok * Hqk * dk * in_bytes * 2          # q, k (once per q/k head)
    b += tok * Hv * dv * in_bytes              # v
    b += tok * Hv * dv * out_bytes             # o
    b += tok * Hv * 4 * 2                      # g, beta
    b += n_states * Hv * dk * dv * 4 * (2 if with_state_in else 1)  # state in / out
    return b


def prefill_flops(tokens_heads, dk, dv, C=64):
    """Dense-tile tensor FLOPs per token and v-head: 2C(3dk + 2dv) + 6 dk dv."""
    return tokens_heads * (2 * C * (3 * dk + 2 * dv) + 6 * dk * dv)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# Sources each profiled kernel is compiled from (the first names the kernel in profiles/).
KERNEL_SOURCES = {
    "chunk_pair.cuh": ("chunk_pair.cuh", "chunk_tc.cuh", "tc_ptx.cuh"),
    "decode.cuh": ("decode.cuh",),
    "chunk_simt.cuh": ("chunk_simt.cuh",),
}


def kernel_source_sha(name: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(name, (name,)):
        with open(os.path.join(ROOT, "gated_delta_rule_59_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it covers the current source.

    Summaries under profiles/ carry lines of the form
        bench-traffic: <kernel source file> <workload> <bytes per launch> <source sha256[:16]>
    """
    sha = kernel_source_sha(kernel_file)
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith((".md", ".txt")):
            continue
        for line in open(os.path.join(pdir, fn)):
            m = re.match(r"\s*bench-traffic:\s*(\S+)\s+(\S+)\s+(\d+)\s+(\w+)", line)
            if m and m.group(1) == kernel_file and m.group(2) == workload and m.group(4) == sha:
                return int(m.group(3))
    return None


# ------------------------------------------------------------------ clocks


def smi_index(local: int) -> str:
    """nvidia-smi id of the GPU this process uses (CUDA_VISIBLE_DEVICES entry or ordinal)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the GPU is timed."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ our arm


def time_steps(fn, steps, stream, flush=None):
    """Per-step CUDA-event durations (ms) on `stream`, L2 flushed before each step."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        evs[i][0].record(stream)
        fn(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def run_ours(args, dist: Dist):
    import gated_delta_rule_59_b200 as dr
    from gated_delta_rule_59_b200 import inputs

    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    dist.init("nccl")
    stream = torch.cuda.current_stream(dev)
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    clocks = ClockSampler(smi_index(dist.local))

    # ---------------- headline: gated prefill, B=2 T=8192 Hqk=16 Hv=32 d=128
    host = inputs.config(2)
    B, T, Hqk, dk = host.q.shape
    Hv, dv = host.v.shape[2], host.v.shape[3]
    p = host.to(dev)
    o = torch.empty((B, T, Hv, dv), dtype=torch.float32, device=dev)
    st = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=dev)
    kernel = dr.prefill_kernel(p.q.dtype, dk, dv)

    def step(_):
        dr.chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, None, o=o, state_out=st)

    clocks.start()
    for i in range(args.warmup):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    assert dr.device_status(dev) == 0
    dist.barrier()
    torch.cuda.synchronize()
    durs = time_steps(step, args.steps, stream, flush)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(sum(durs) / len(durs), dev)
    tokens = B * T
    value = dist.world * tokens / (ms / 1e3)
    algo_bytes = prefill_bytes(B, T, Hqk, Hv, dk, dv, 2, 4, B, True)
    flops = prefill_flops(tokens * Hv, dk, dv)
    achieved = algo_bytes / (ms / 1e3) / 1e9
    kfile = "chunk_pair.cuh" if kernel == "tc_bf16" else "chunk_simt.cuh"
    roofline = {
        "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
        "frac": round(achieved / hbm_peak, 4),
        "traffic": profiled_traffic(kfile, "gated_prefill_B2_T8192_Hqk16_Hv32_d128"),
        "peak_kind": peak_kind, "kernel": kernel, "algorithmic_bytes_per_launch": algo_bytes,
        "tensor": {"flops_per_launch_dense_tile": flops,
                   "achieved_tflops": round(flops / (ms / 1e3) / 1e12, 2),
                   "peak_tflops": tc_peak, "frac": round(flops / (ms / 1e3) / 1e12 / tc_peak, 4)},
    }

    # ---------------- e2e: pinned host inputs -> H2D -> dr_chunk_fwd -> D2H
    pin = lambda t: t.pin_memory()
    hq, hk, hv, hg, hb, hs = (pin(t) for t in (host.q, host.k, host.v, host.g, host.beta, host.state_in))
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hst = torch.empty(st.shape, dtype=st.dtype).pin_memory()
    dq, dk_, dv_, dg, db, ds = (torch.empty_like(t, device=dev) for t in (hq, hk, hv, hg, hb, hs))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hg, hb, hs))
    d2h = ho.numel() * ho.element_size() + hst.numel() * hst.element_size()

    def e2e_step(_):
        for d_, h_ in ((dq, hq), (dk_, hk), (dv_, hv), (dg, hg), (db, hb), (ds, hs)):
            d_.copy_(h_, non_blocking=True)
        dr.chunk_fwd(dq, dk_, dv_, dg, db, ds, None, o=o, state_out=st)
        ho.copy_(o, non_blocking=True)
        hst.copy_(st, non_blocking=True)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    dist.barrier()
    e_durs = time_steps(e2e_step, max(3, min(args.steps, 10)), stream, None)
    dist.barrier()
    e_ms = dist.max(sum(e_durs) / len(e_durs), dev)
    e2e = {"value": round(dist.world * tokens / (e_ms / 1e3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4)}
    del dq, dk_, dv_, dg, db, ds

    secondary = {}
    if not args.no_secondary:
        # the headline workload with the kernel's q/k L2 normalisation (DR_QK_L2NORM)
        def l2_step(_):
            dr.chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, None, o=o, state_out=st,
                         qk_l2norm=True)

        for i in range(2):
            flush.zero_()
            l2_step(i)
        torch.cuda.synchronize()
        assert dr.device_status(dev) == 0
        dist.barrier()
        l_durs = time_steps(l2_step, max(3, min(args.steps, 10)), stream, flush)
        dist.barrier()
        l_ms = dist.max(sum(l_durs) / len(l_durs), dev)
        secondary["prefill_qk_l2norm"] = {
            "metric": "prefill tokens/s with in-kernel q/k L2 normalisation (same workload)",
            "value": round(dist.world * tokens / (l_ms / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(l_ms, 4),
            "roofline": {"bound": "hbm", "frac": round(algo_bytes / (l_ms / 1e3) / 1e9 / hbm_peak, 4),
                         "peak": hbm_peak, "unit": "GB/s", "peak_kind": peak_kind},
        }
        # the headline workload also returning the state after every 64-token chunk
        n_cs = dr.chunk_state_rows(None, B, T)
        cs = torch.empty((n_cs, Hv, dk, dv), dtype=torch.float32, device=dev)

        def cs_step(_):
            dr.chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, None, o=o, state_out=st,
                         chunk_states=cs)

        for i in range(2):
            flush.zero_()
            cs_step(i)
        torch.cuda.synchronize()
        assert dr.device_status(dev) == 0
        dist.barrier()
        c_durs = time_steps(cs_step, max(3, min(args.steps, 10)), stream, flush)
        dist.barrier()
        c_ms = dist.max(sum(c_durs) / len(c_durs), dev)
        cs_bytes = algo_bytes + n_cs * Hv * dk * dv * 4
        secondary["prefill_chunk_states"] = {
            "metric": "prefill tokens/s also writing the state after every 64-token chunk "
                      "(same workload)",
            "value": round(dist.world * tokens / (c_ms / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(c_ms, 4), "chunk_state_bytes": n_cs * Hv * dk * dv * 4,
            "roofline": {"bound": "hbm", "algorithmic_bytes_per_launch": cs_bytes,
                         "achieved": round(cs_bytes / (c_ms / 1e3) / 1e9, 1),
                         "frac": round(cs_bytes / (c_ms / 1e3) / 1e9 / hbm_peak, 4),
                         "peak": hbm_peak, "unit": "GB/s", "peak_kind": peak_kind,
                         "traffic": profiled_traffic(
                             kfile, "gated_prefill_chunk_states_B2_T8192_Hqk16_Hv32_d128")},
        }
        del cs
        secondary["prefill_channel_gates"] = guarded(bench_channel_gates, dev, dist, stream,
                                                     flush, hbm_peak, peak_kind, args)
        layer_lines = guarded(bench_layer_steps, dev, dist, stream, flush, hbm_peak, peak_kind)
        if isinstance(layer_lines, dict):  # the error record
            layer_lines = (layer_lines, layer_lines)
        secondary["prologue_conv_silu"], secondary["epilogue_norm_gate"] = layer_lines
        secondary["decode"] = guarded(bench_decode, dev, dist, stream, hbm_peak, peak_kind)
        secondary["varlen"] = guarded(bench_varlen, dev, dist, stream, flush, hbm_peak,
                                      peak_kind)
    clk = clocks.stop()

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if kernel == "tc_bf16" else "f32",
        "data": "synthetic (seeded; shapes and distributions of the gated prefill workload)",
        "config": {"workload": host.name, "global_batch": B * dist.world, "seq_len": T,
                   "heads_qk": Hqk, "heads_v": Hv, "d_k": dk, "d_v": dv, "chunk": 64,
                   "out_dtype": "f32", "parallelism": f"replicas x{dist.world}",
                   "l2": "flushed before every timed step (256 MiB write)"},
        "roofline": roofline, "e2e": e2e, "gpu_launches": args.steps, "clocks": clk,
    }
    line.update(secondary)
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(host, n_tok=host.q.shape[1])
    del p, o, st, flush
    dist.close()
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def guarded(fn, *args):
    """A secondary line that raises on the host is reported as an error record instead of
    costing the headline line.  Every rank runs the same code, so all raise at the same point."""
    try:
        return fn(*args)
    except (ValueError, RuntimeError, AssertionError) as e:
        return {"error": f"{type(e).__name__}: {e}"}


def bench_channel_gates(dev, dist, stream, flush, hbm_peak, peak_kind, args):
    """The headline shape with per-key-channel gates (g [B, T, Hv, dk]): the CUDA-core kernel."""
    import gated_delta_rule_59_b200 as dr
    from gated_delta_rule_59_b200 import inputs

    B, T, Hqk, Hv, d = 2, 8192, 16, 32, 128
    p = inputs.prefill(B, T, Hqk, Hv, d, d, torch.bfloat16, gated=True, state_std=0.02,
                       seed=inputs.SEED_BASE + 2, channel_gates=True).to(dev)
    o = torch.empty((B, T, Hv, d), dtype=torch.float32, device=dev)
    st = torch.empty((B, Hv, d, d), dtype=torch.float32, device=dev)

    def step(_):
        dr.chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, None, o=o, state_out=st)

    for i in range(2):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    assert dr.device_status(dev) == 0
    dist.barrier()
    durs = time_steps(step, 3, stream, flush)
    dist.barrier()
    ms = dist.max(sum(durs) / len(durs), dev)
    algo = prefill_bytes(B, T, Hqk, Hv, d, d, 2, 4, B, True) + B * T * Hv * (d - 1) * 4
    return {
        "metric": "prefill tokens/s with per-key-channel gates (same shape; CUDA-core kernel)",
        "value": round(dist.world * B * T / (ms / 1e3), 1), "unit": "tokens/s",
        "ms_per_step": round(ms, 4), "kernel": dr.prefill_kernel(torch.bfloat16, d, d, True),
        "roofline": {"bound": "alu", "hbm_frac": round(algo / (ms / 1e3) / 1e9 / hbm_peak, 4),
                     "algorithmic_bytes_per_launch": algo, "peak_kind": peak_kind},
        "gpu_launches": 3,
    }


def bench_layer_steps(dev, dist, stream, flush, hbm_peak, peak_kind):
    """The steps either side of the rule on the headline shapes (bf16 activations):
    conv + SiLU of q, k, v (K = 4, conv state out), and RMSNorm + SiLU gate of o (fp32) with
    z (bf16) into bf16.  Both are HBM bound: bytes = every element read and written once."""
    import gated_delta_rule_59_b200 as dr

    B, T, Hqk, Hv, d, K = 2, 8192, 16, 32, 128, 4
    gen = torch.Generator().manual_seed(77)
    xs = [torch.randn((B, T, H, d), generator=gen).to(torch.bfloat16).to(dev)
          for H in (Hqk, Hqk, Hv)]
    ws = [(0.5 * torch.randn((H, d, K), generator=gen)).to(dev) for H in (Hqk, Hqk, Hv)]
    o = torch.randn((B, T, Hv, d), generator=gen).to(dev)
    z = torch.randn((B, T, Hv, d), generator=gen).to(torch.bfloat16).to(dev)
    wt = torch.ones(d, device=dev)
    y = torch.empty((B, T, Hv, d), dtype=torch.bfloat16, device=dev)

    def conv_step(_):
        for x, w in zip(xs, ws):
            dr.short_conv_silu(x, w)

    def norm_step(_):
        dr.norm_gate(o, wt, z=z, y=y)

    out = []
    for fn, nbytes, launches, metric in (
            (conv_step, sum(4 * x.numel() + B * x[0, 0].numel() * (K - 1) * 4 for x in xs), 6,
             "conv + SiLU of q, k, v (K=4) on the headline shape, bf16 in and out"),
            (norm_step, o.numel() * 4 + z.numel() * 2 + y.numel() * 2, 1,
             "RMSNorm + SiLU gate of o (fp32) with z (bf16) into bf16, headline shape")):
        for i in range(3):
            flush.zero_()
            fn(i)
        torch.cuda.synchronize()
        assert dr.device_status(dev) == 0
        dist.barrier()
        durs = time_steps(fn, 10, stream, flush)
        dist.barrier()
        ms = dist.max(sum(durs) / len(durs), dev)
        gbs = nbytes / (ms / 1e3) / 1e9
        out.append({"metric": metric, "value": round(gbs, 1), "unit": "GB/s",
                    "ms_per_step": round(ms, 4), "gpu_launches": 10 * launches,
                    "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak,
                                 "frac": round(gbs / hbm_peak, 4), "unit": "GB/s",
                                 "algorithmic_bytes_per_step": nbytes,
                                 "peak_kind": peak_kind}})
    return out[0], out[1]


def bench_decode(dev, dist, stream, hbm_peak, peak_kind):
    import gated_delta_rule_59_b200 as dr
    from gated_delta_rule_59_b200 import inputs

    n_steps = 64
    state0, steps = inputs.decode_config(n_steps=n_steps)
    state = state0.to(dev)
    dsteps = [s.to(dev) for s in steps]
    B, Hv, dk, dv = state.shape
    Hqk = dsteps[0].q.shape[1]
    o = torch.empty((B, Hv, dv), dtype=torch.float32, device=dev)

    def step(i):
        s = dsteps[i % n_steps]
        dr.recurrent_step(s.q, s.k, s.v, s.g, s.beta, state, o=o)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    dist.barrier()
    durs = time_steps(step, n_steps, stream, None)  # 512 MiB state >> L2: no flush needed
    dist.barrier()
    med = dist.max(statistics.median(durs), dev)
    state_bytes = 2 * B * Hv * dk * dv * 4
    io_bytes = B * (2 * Hqk * dk + Hv * dv) * 2 + B * Hv * dv * 4 + 2 * B * Hv * 4
    gbs = (state_bytes + io_bytes) / (med / 1e3) / 1e9
    res = {
        "metric": "decode-step state HBM GB/s (gated, B=256 H=32 d=128, fp32 state in place)",
        "value": round(dist.world * gbs, 1), "unit": "GB/s",
        "ms_per_step_median": round(med, 4), "steps": n_steps,
        "tokens_per_s": round(dist.world * B / (med / 1e3), 1),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(gbs / hbm_peak, 4), "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": state_bytes + io_bytes,
                     "traffic": profiled_traffic("decode.cuh", "decode_B256_H32_d128")},
        "gpu_launches": n_steps,
    }
    del state, dsteps, o
    return res


def bench_varlen(dev, dist, stream, flush, hbm_peak, peak_kind):
    import gated_delta_rule_59_b200 as dr
    from gated_delta_rule_59_b200 import inputs

    host = inputs.config(4)
    p = host.to(dev)
    _, T, Hqk, dk = p.q.shape
    Hv, dv = p.v.shape[2], p.v.shape[3]
    N = p.cu_seqlens.numel() - 1
    o = torch.empty((1, T, Hv, dv), dtype=torch.float32, device=dev)
    st = torch.empty((N, Hv, dk, dv), dtype=torch.float32, device=dev)

    def step(_):
        dr.chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, p.cu_seqlens, o=o, state_out=st)

    step(0)
    torch.cuda.synchronize()
    assert dr.device_status(dev) == 0
    dist.barrier()
    durs = time_steps(step, 3, stream, flush)
    dist.barrier()
    ms = dist.max(sum(durs) / len(durs), dev)
    algo = prefill_bytes(1, T, Hqk, Hv, dk, dv, 2, 4, N, True)
    gbs = algo / (ms / 1e3) / 1e9
    res = {
        "metric": "varlen prefill tokens/s (8 x U[512,16384] + 65536 tokens, H=16 d=128)",
        "value": round(dist.world * T / (ms / 1e3), 1), "unit": "tokens/s",
        "ms_per_step": round(ms, 4), "tokens": T, "sequences": N,
        "longest": int((p.cu_seqlens[1:] - p.cu_seqlens[:-1]).max().item()),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(gbs / hbm_peak, 4), "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": algo},
    }
    del p, o, st
    return res


# ------------------------------------------------------------------ oracle legs


def _usable_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_sample(host, n_tok):
    """The first n_tok tokens of every sequence, all heads (a bounded sample of the workload)."""
    import oracle

    q, k, v = host.q[:, :n_tok], host.k[:, :n_tok], host.v[:, :n_tok]
    g = None if host.g is None else host.g[:, :n_tok]
    beta = host.beta[:, :n_tok]
    threads = _usable_cores()
    t0 = time.perf_counter()
    oracle.run(q, k, v, g, beta, host.state_in, threads=threads)
    dt = time.perf_counter() - t0
    return dt, threads, q.shape[0] * q.shape[1]


def cpu_baseline(host, n_tok):
    dt, threads, tokens = oracle_sample(host, n_tok)
    return {"value": round(tokens / dt, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 C oracle (form 2), first {n_tok} tokens of each of the "
                      f"{host.q.shape[0]} sequences, all {host.v.shape[2]} v-heads "
                      f"({tokens} tokens, {dt:.2f} s wall)"}


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return
    from gated_delta_rule_59_b200 import inputs

    host = inputs.config(2)
    n_tok = 512
    for _ in range(args.warmup):
        oracle_sample(host, n_tok)
    times = []
    threads = tokens = 0
    for _ in range(args.steps):
        dt, threads, tokens = oracle_sample(host, n_tok)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = tokens / (ms / 1e3)
    B, T = host.q.shape[:2]
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": host.name, "global_batch": B, "seq_len": T,
                   "parallelism": "cpu threads"},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"first {n_tok} tokens of each sequence, all heads, per step"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
    else:
        if args.warmup < 3:
            raise SystemExit("--warmup must be >= 3")
        run_ours(args, dist)


if __name__ == "__main__":
    main()
