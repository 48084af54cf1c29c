#!/usr/bin/env python
"""KDA benchmark: long-context chunkwise prefill on B200 (plus the recurrent decode workload).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]

Step = one kda_chunk_fwd over the long-context batch (B=1, H=32, T=131072, d_k=d_v=128, bf16 q/k/v,
fp32 gates, h0 ~ N(0, 0.02)): chunk prep + state passing + output + final state.  Inputs (6.4 GB
per step) are larger than L2, so no flush is needed between steps.  Timing: W untimed warm-up steps,
then K steps between a barrier + synchronize on both sides, CUDA events on the launching stream,
max over ranks.  N > 1 runs independent replicas (weak scaling, no data-path collective).

--impl reference times the fp64 CPU oracle (test infrastructure) on a bounded sample of the same
workload on the host cores; rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (H=32,d=128,T=128K) & % roofline; decode HBM GB/s"
UNIT = "tokens/s"

# Algorithmic traffic (bytes) and work, per token-head of the prefill (bf16 q,k,v,o; fp32 gates):
#   q, k, v 3 x 256 B, log_alpha 512 B, beta 4 B, o 256 B.
PREFILL_BYTES_PER_TOKEN_HEAD = 768 + 512 + 4 + 256
PREFILL_FLOP_PER_TOKEN_HEAD = 180224          # five C x d and three d x d products per token at C=64, d=128
STATE_BYTES = 128 * 128 * 4                    # one fp32 state (h0 read or h_T write)
DECODE_BYTES_PER_STATE = 2 * STATE_BYTES + 3 * 256 + 512 + 4 + 256  # S read+write, q/k/v, gates, beta, o
MULTI_TQ = (4, 16)  # tokens per kda_decode_multi call in the decode benchmark


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["kda", "reference"], default="kda")
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--decode-steps", type=int, default=1024)
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-backward", action="store_true")
    p.add_argument("--no-cp", action="store_true")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the training-shape and packed-varlen prefill legs")
    p.add_argument("--backward-steps", type=int, default=3)
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle sample (0 skips the CPU baseline)")
    p.add_argument("--profile-range", action="store_true",
                   help="after the warm-up, run one long-context step between cudaProfilerStart and "
                        "cudaProfilerStop and exit (for a profiler's range replay of the whole concurrent call)")
    p.add_argument("--seq-len", type=int, default=131072,
                   help="override T of the long-context workload (small cases for profiler captures)")
    return p.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm_gbs=float(pk["hbm_gbs"]), bf16_tflops=float(pk["bf16_tflops"]),
                    bf16_tflops_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="kda_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                cols = [c.strip() for c in line.split(",")]
                if len(cols) < len(self.FIELDS):
                    continue
                try:
                    sm.append(float(cols[1]))
                    mx.append(float(cols[2]))
                except ValueError:
                    continue
                for name, val in zip(names, cols[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle timing
def oracle_sample(target_s: float, seed: int = 0):
    """Time the fp64 oracle on the first T_s tokens (all 32 heads) of the long-context workload,
    T_s sized so the timed call takes about target_s seconds.  Returns a cpu_baseline dict."""
    import torch

    import oracle
    from kimi_delta_attention_29_b200 import inputs as gen

    shp = gen.LONG

    def run(T_s):
        x = gen.make_prefill(1, T_s, shp.H, shp.dk, shp.dv, shp.dtype, shp.gate_shift, shp.h0_std, seed, "cpu")
        f = lambda t: t.float().numpy()
        args = (f(x["q"]), f(x["k"]), f(x["v"]), f(x["log_alpha"]), f(x["beta"]), f(x["h0"]))
        t0 = time.perf_counter()
        oracle.recurrent(*args)
        return time.perf_counter() - t0

    probe_T = 256
    t_probe = run(probe_T)
    T_s = int(max(64, min(shp.T, probe_T * target_s / max(t_probe, 1e-3))) // 64 * 64)
    dt = run(T_s)
    cores = oracle.num_threads()
    return {"value": T_s / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"fp64 recurrent oracle on tokens 0..{T_s - 1} of B=1,H=32,T=131072,d=128 "
                      f"(all 32 heads, h0 included); {dt:.1f} s on {cores} threads",
            "seconds": dt, "tokens": T_s}


def config_dict(T: int = 131072):
    return {"workload": f"long_B1_H32_T{T}_d128", "model": "KDA operator (chunkwise prefill)", "B": 1,
            "T": T, "H": 32, "dk": 128, "dv": 128, "chunk": 64, "global_batch": 1, "seq_len": T,
            "gates": "log_alpha=-softplus(N(0,1)+2), beta=sigmoid(N(0,1)), h0~N(0,0.02)",
            "l2": f"no flush: inputs ({T * 32 * 1284 / 1e9:.2f} GB per step) are larger than the 126 MB L2",
            "parallelism": "replicas (independent problems per GPU)"}


def reference_arm(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample(max(1.0, args.cpu_seconds / 4))
    samples = [oracle_sample(max(1.0, args.cpu_seconds / 2)) for _ in range(args.steps)]
    tok = sum(s["tokens"] for s in samples)
    sec = sum(s["seconds"] for s in samples)
    value = tok / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * 131072 / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": samples[0]["cores"], "kind": "oracle",
                             "sample": f"{args.steps} steps, each the fp64 oracle on the first "
                                       f"{samples[0]['tokens']} tokens x 32 heads of the workload"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def launches_of(traces) -> int:
    """Kernel launches behind the library's trace entries: the tensor-core prefill's entry brackets
    two concurrent kernels (the state kernel and the intra-chunk kernel), every other entry one."""
    return sum(2 if name.startswith("kda_tc_prefill") else 1 for name, _ in traces)


def kernel_stats(traces):
    out = {}
    for name, ms in traces:
        d = out.setdefault(name, {"launches": 0, "total_ms": 0.0})
        d["launches"] += 1
        d["total_ms"] += ms
    total = sum(d["total_ms"] for d in out.values()) or 1.0
    for d in out.values():
        d["avg_ms"] = d["total_ms"] / d["launches"]
        d["share"] = d["total_ms"] / total
    return out


def reduce_max(x: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (a timing collective, not part of the data path)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, steps: int, world: int, elapsed_ms_max: float) -> float:
    """Units per second for the whole job: every rank processes its own units (weak scaling) and the
    job takes as long as its slowest rank."""
    return world * units_per_step_per_rank * steps / (elapsed_ms_max / 1e3)


def sources_sha256(paths) -> str | None:
    """sha256 over the concatenated bytes of the repo-relative source files (None if one is missing)."""
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        full = os.path.join(ROOT, p)
        if not os.path.exists(full):
            return None
        with open(full, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(kernel: str, units: int):
    """DRAM bytes per launch of `kernel` for `units` work units, scaled from the committed ncu capture
    in profiles/ncu_traffic.json, or None when any source the kernel is compiled from (its .cu file
    and the headers it includes) changed since that capture."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or "sources" not in rec:
        return None
    if sources_sha256(rec["sources"]) != rec["sources_sha256"]:
        return None
    return rec["dram_bytes"] / rec["units"] * units


def prefill_rooflines(kst, token_heads, chunk_heads, states, ms_per_step, peaks):
    """Roofline objects of one prefill step on the operator's algorithmic basis: 1,540 B and
    180,224 FLOP per token-head plus h0 read and h_T written (64 KiB each per (sequence, head)).
    `roofline` divides those bytes by the dominant kernel's average launch duration (an upper bound
    on what that kernel alone achieves); `operator_roofline` divides them by the whole step."""
    dominant = max(kst, key=lambda n: kst[n]["total_ms"])
    op_bytes = token_heads * PREFILL_BYTES_PER_TOKEN_HEAD + 2 * states * STATE_BYTES
    op_flop = token_heads * PREFILL_FLOP_PER_TOKEN_HEAD
    dom_s = kst[dominant]["avg_ms"] / 1e3
    achieved = op_bytes / dom_s / 1e9
    traffic = {n: ncu_traffic(n, chunk_heads) for n in kst}
    traffic_step = None if any(v is None for v in traffic.values()) else sum(traffic.values())
    roofline = {"kernel": dominant, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic[dominant], "peak_source": peaks["source"],
                "algorithmic_bytes_per_launch": op_bytes, "avg_ms": kst[dominant]["avg_ms"],
                "tensor_frac_burst": op_flop / dom_s / 1e12 / peaks["bf16_tflops"],
                "basis": "operator bytes (1,540 B per token-head + h0 + h_T) / the dominant kernel's average "
                         "launch time; traffic = that kernel's DRAM read+write bytes per launch from "
                         "profiles/ncu_traffic.json (null if its sources changed since the capture)"}
    step_s = ms_per_step / 1e3
    operator_roofline = {"bytes_per_step": op_bytes, "achieved_gbs": op_bytes / step_s / 1e9,
                         "hbm_frac": op_bytes / step_s / 1e9 / peaks["hbm_gbs"], "flop_per_step": op_flop,
                         "achieved_tflops": op_flop / step_s / 1e12,
                         "tensor_frac_burst": op_flop / step_s / 1e12 / peaks["bf16_tflops"],
                         "tensor_frac_sustained": op_flop / step_s / 1e12 / peaks["bf16_tflops_sustained"],
                         "dram_bytes_per_step": traffic_step,
                         "dram_over_algorithmic": None if traffic_step is None else traffic_step / op_bytes,
                         "note": "whole call (all kernels) against the operator's algorithmic bytes / FLOPs"}
    return roofline, operator_roofline


def workload_bench(shape, args, dev, stream, peaks, barrier, max_over_ranks, world, cpu_seconds):
    """kda_chunk_fwd on another of the page-shaped workloads (training shape, packed varlen batch):
    tokens/s, the same roofline objects and an oracle sample on the host cores."""
    import torch
    import kimi_delta_attention_29_b200 as kda
    from kimi_delta_attention_29_b200 import inputs as gen
    x = gen.make_prefill_for(shape, seed=0, device=dev)
    B, T, H = x["q"].shape[0], x["q"].shape[1], x["q"].shape[2]
    cu = x["cu_seqlens"]
    N = B if cu is None else cu.numel() - 1
    ws = kda.Workspace(dev)

    def step():
        kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], cu, workspace=ws,
                          stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    assert kda.kda_get_status(ws) == 0, "device status after warm-up"
    barrier()
    steps = max(args.steps, 10)
    kda.kda_trace_begin(16 * steps + 16)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    traces = kda.kda_trace_end()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    kst = kernel_stats(traces)
    tokens = B * T
    if cu is None:
        chunk_heads = B * ((T + 63) // 64) * H
    else:
        lens = (cu[1:] - cu[:-1]).cpu()
        chunk_heads = int(((lens + 63) // 64).sum()) * H
    roof, op_roof = prefill_rooflines(kst, tokens * H, chunk_heads, N * H, ms, peaks)
    out = {"workload": shape.name, "tokens": tokens, "sequences": N, "ms_per_step": ms, "steps": steps,
           "tokens_per_s": whole_job_rate(tokens, 1, world, ms), "roofline": roof, "operator_roofline": op_roof,
           "kernels": kst, "l2": "inputs larger than the 126 MB L2: no flush"}
    if cpu_seconds > 0:
        out["cpu_baseline"] = oracle_sample_shape(x, cpu_seconds)
    return out


def oracle_sample_shape(x, target_s):
    """The fp64 oracle on the first tokens of every sequence of a workload (all heads), sized to take
    about target_s seconds; tokens/s over the tokens it covered."""
    import torch
    import oracle
    q, k, v, la, beta = (x[n].cpu() for n in ("q", "k", "v", "log_alpha", "beta"))
    cu = x["cu_seqlens"]
    B, T, H = q.shape[:3]
    starts = [0] * B if cu is None else [int(c) for c in cu[:-1].cpu()]
    lens = [T] * B if cu is None else [int(b - a) for a, b in zip(cu[:-1].cpu(), cu[1:].cpu())]
    f = lambda t: t.float().numpy()

    def run(n_tok):
        rows_q, rows_k, rows_v, rows_la, rows_b, cus = [], [], [], [], [], [0]
        for i, (a, L) in enumerate(zip(starts, lens)):
            m = min(L, n_tok)
            b = i if cu is None else 0
            rows_q.append(q[b, a:a + m]); rows_k.append(k[b, a:a + m]); rows_v.append(v[b, a:a + m])
            rows_la.append(la[b, a:a + m]); rows_b.append(beta[b, a:a + m]); cus.append(cus[-1] + m)
        cat = lambda rs: torch.cat(rs, 0)[None]
        t0 = time.perf_counter()
        oracle.recurrent(f(cat(rows_q)).astype("float64"), f(cat(rows_k)).astype("float64"),
                         f(cat(rows_v)).astype("float64"), f(cat(rows_la)).astype("float64"),
                         f(cat(rows_b)).astype("float64"), None, cu_seqlens=__import__("numpy").array(cus))
        return time.perf_counter() - t0, cus[-1]

    dt, tok = run(64)
    n_tok = int(max(64, min(max(lens), 64 * target_s / max(dt, 1e-3))))
    dt, tok = run(n_tok)
    cores = oracle.num_threads()
    return {"value": tok / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"fp64 recurrent oracle on the first {n_tok} tokens of each of the {len(lens)} sequences "
                      f"(all {H} heads; {tok} tokens); {dt:.1f} s on {cores} threads"}


def gpu_arm(args):
    import torch
    import torch.distributed as dist

    import kimi_delta_attention_29_b200 as kda
    from kimi_delta_attention_29_b200 import inputs as gen

    rank, local_rank, world = dist_env()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    peaks = load_peaks()
    import dataclasses
    shp = dataclasses.replace(gen.LONG, T=args.seq_len)
    x = gen.make_prefill_for(shp, seed=rank, device=dev)
    B, T, H, D = shp.B, shp.T, shp.H, shp.dk
    o = torch.empty(B, T, H, D, dtype=shp.dtype, device=dev)
    hT = torch.empty(B, H, D, D, dtype=torch.float32, device=dev)
    ws = kda.Workspace(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, o=o, h_T=hT,
                          workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert kda.kda_get_status(ws) == 0, "device status after warm-up"
    if args.profile_range:  # one step inside a profiler range (both kernels of the call, concurrent)
        torch.cuda.cudart().cudaProfilerStart()
        step()
        torch.cuda.synchronize(dev)
        torch.cuda.cudart().cudaProfilerStop()
        assert kda.kda_get_status(ws) == 0, "device status after the profiled step"
        print(json.dumps({"profile_range": shp.name, "T": T, "H": H, "tokens": B * T}))
        if world > 1:
            dist.destroy_process_group()
        return

    clocks = ClockSampler(dev.index)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    kda.kda_trace_begin(16 * args.steps + 16)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    traces = kda.kda_trace_end()
    barrier()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(ev0.elapsed_time(ev1))
    ms_per_step = elapsed_ms / args.steps
    tokens_per_step = B * T
    value = whole_job_rate(tokens_per_step, args.steps, world, elapsed_ms)

    # per-kernel timing (live, CUDA events around each library kernel in the timed region)
    kst = kernel_stats(traces)
    token_heads = B * T * H
    chunk_heads = B * ((T + 63) // 64) * H
    roofline, operator_roofline = prefill_rooflines(kst, token_heads, chunk_heads, B * H, ms_per_step, peaks)

    # end to end through the public API with host buffers: pinned H2D of the step's inputs, the call,
    # D2H of the results (o and h_T), all inside the timed region
    host = {kk: x[kk].cpu().pin_memory() for kk in ("q", "k", "v", "log_alpha", "beta", "h0")}
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hT_h = torch.empty(hT.shape, dtype=hT.dtype, pin_memory=True)
    dx = {kk: torch.empty_like(x[kk]) for kk in host}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + hT_h.numel() * hT_h.element_size()

    def e2e_step():
        for kk in host:
            dx[kk].copy_(host[kk], non_blocking=True)
        kda.kda_chunk_fwd(dx["q"], dx["k"], dx["v"], dx["log_alpha"], dx["beta"], dx["h0"], None, o=o, h_T=hT,
                          workspace=ws, stream=stream)
        o_h.copy_(o, non_blocking=True)
        hT_h.copy_(hT, non_blocking=True)

    e2e = None
    if args.e2e_steps > 0:
        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / args.e2e_steps
        e2e = {"value": world * tokens_per_step / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": args.e2e_steps}
    del host, dx, o_h, hT_h

    # the same prefill with the layer prologue fused in (q/k L2 normalisation, gate activation from the
    # gate projection g; here g = the workload's log_alpha values, A_log = 0, dt_bias = 0)
    A_log = torch.zeros(H, device=dev)
    flags = kda.KDA_PROLOGUE_L2NORM_QK | kda.KDA_PROLOGUE_GATE

    def step_pro():
        kda.kda_chunk_fwd_ex(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, flags=flags,
                             A_log=A_log, o=o, h_T=hT, workspace=ws, stream=stream)

    for _ in range(2):
        step_pro()
    torch.cuda.synchronize(dev)
    barrier()
    pe0, pe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pe0.record(stream)
    for _ in range(args.steps):
        step_pro()
    pe1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    pro_ms = max_over_ranks(pe0.elapsed_time(pe1)) / args.steps
    prologue = {"ms_per_step": pro_ms, "tokens_per_s": whole_job_rate(tokens_per_step, 1, world, pro_ms),
                "flags": "l2norm_qk|gate", "vs_plain": ms_per_step / pro_ms}

    # the layer's output epilogue on this step's output: RMSNorm x weight x sigmoid(g) per (token, head)
    # row, HBM-bound (reads o and g, writes out: 3 x 2 bytes per element, 3.2 GB at this size)
    g_out = torch.randn(o.shape, generator=torch.Generator(device=dev).manual_seed(77), device=dev).to(o.dtype)
    w_out = torch.ones(o.shape[-1], device=dev)
    out_e = torch.empty_like(o)
    for _ in range(2):
        kda.kda_output_gate_norm(o, g_out, w_out, eps=1e-6, out=out_e, stream=stream)
    torch.cuda.synchronize(dev)
    barrier()
    ee0, ee1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    for _ in range(args.steps):
        kda.kda_output_gate_norm(o, g_out, w_out, eps=1e-6, out=out_e, stream=stream)
    ee1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    epi_ms = max_over_ranks(ee0.elapsed_time(ee1)) / args.steps
    epi_bytes = 3 * o.numel() * o.element_size() + w_out.numel() * 4
    epilogue = {"kernel": "kda_output_gate_norm_kernel", "ms_per_call": epi_ms,
                "tokens_per_s": whole_job_rate(tokens_per_step, 1, world, epi_ms),
                "bytes_per_call": epi_bytes, "hbm_gbs": epi_bytes / (epi_ms * 1e6),
                "frac": epi_bytes / (epi_ms * 1e6) / peaks["hbm_gbs"],
                "traffic": ncu_traffic("kda_output_gate_norm_kernel", o.numel() // o.shape[-1])}
    del g_out, out_e

    cp_line = None
    if not args.no_cp and world == 1 and args.seq_len == 131072:
        cp_line = cp_bench(x, dev, stream, ms_per_step)

    backward = None
    if not args.no_backward:
        backward = backward_bench(args, dev, stream, barrier, max_over_ranks, world)

    decode = None
    if not args.no_decode:
        decode = decode_bench(args, dev, stream, peaks, barrier, max_over_ranks)

    workloads = None
    if not args.no_workloads:
        workloads = [workload_bench(shp, args, dev, stream, peaks, barrier, max_over_ranks, world,
                                    args.cpu_seconds / 2 if rank == 0 and world == 1 else 0)
                     for shp in (gen.TRAIN, gen.VARLEN)]

    cpu_baseline = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu_baseline = oracle_sample(args.cpu_seconds)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(T),
            "roofline": roofline, "operator_roofline": operator_roofline, "cpu_baseline": cpu_baseline,
            "e2e": e2e, "gpu_launches": launches_of(traces), "clocks": clk, "prologue": prologue, "epilogue": epilogue, "backward": backward, "context_parallel": cp_line, "decode": decode,
            "workloads": workloads,
            "kernels": kst, "peaks": peaks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def backward_bench(args, dev, stream, barrier, max_over_ranks, world):
    """kda_chunk_bwd on the training shape (B=4, H=16, T=4096, d=128, bf16), next to kda_chunk_fwd on the
    same inputs; kernel split from the library's trace."""
    import torch
    import kimi_delta_attention_29_b200 as kda
    from kimi_delta_attention_29_b200 import inputs as gen
    shp = gen.TRAIN
    x = gen.make_prefill_for(shp, seed=0, device=dev)
    g = torch.Generator(device=dev).manual_seed(11)
    do = torch.randn(x["v"].shape, generator=g, device=dev).to(x["v"].dtype)
    N = shp.B
    ws = torch.empty(kda.kda_chunk_bwd_workspace_size(shp.B, shp.T, shp.H, shp.dk, shp.dv, N, 64, shp.dtype),
                     dtype=torch.uint8, device=dev)
    fws = kda.Workspace()

    def bwd():
        return kda.kda_chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, do=do,
                                 want_dh0=False, workspace=ws, stream=stream)

    def fwd():
        return kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, workspace=fws,
                                 stream=stream)

    def timed(fn, n):
        fn()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1)) / n

    fwd_ms = timed(fwd, max(args.backward_steps, 3))
    bwd_ms = timed(bwd, args.backward_steps)
    kda.kda_trace_begin(64)
    bwd()
    per = {}
    for name, ms in kda.kda_trace_end():
        per[name] = per.get(name, 0.0) + ms
    tokens = shp.B * shp.T
    return {"workload": shp.name, "ms_per_call": bwd_ms, "tokens_per_s": whole_job_rate(tokens, 1, world, bwd_ms),
            "forward_ms_same_shape": fwd_ms, "bwd_over_fwd": bwd_ms / fwd_ms,
            "kernels_ms": per, "arith": "fp32 on CUDA cores"}


def cp_bench(x, dev, stream, single_ms):
    """Context parallelism on the long-context sequence: the work ONE rank does for R segments (its map
    [M | b] in one pass, the composition of R maps, one pass from its incoming state), timed on this GPU
    for the last segment, with the time of each of the three steps.  The all-gather between GPUs is not
    part of it."""
    import torch
    import kimi_delta_attention_29_b200 as kda
    from kimi_delta_attention_29_b200 import cp
    T = x["q"].shape[1]
    rows = []
    for R in (2, 4, 8):
        a, e = T - T // R, T
        part = [x[n][:, a:e].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")]
        Mb_all = torch.zeros(R, x["q"].shape[2], 128, 256, device=dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        split = [0.0, 0.0, 0.0]

        def rank_work(timed):
            if timed:
                ev[0].record(stream)
            _, Mb = cp.segment_map(*part, stream=stream, want_o=False)  # a rank > 0 keeps no map-pass outputs
            Mb_all[R - 1].copy_(Mb)
            if timed:
                ev[1].record(stream)
            S_in, _ = kda.kda_state_compose(Mb_all, None, stream=stream)
            if timed:
                ev[2].record(stream)
            o = cp.segment_from(*part, S_in[R - 1], stream=stream)
            if timed:
                ev[3].record(stream)
                torch.cuda.synchronize(dev)
                for i in range(3):
                    split[i] += ev[i].elapsed_time(ev[i + 1])
            return o

        rank_work(False)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            rank_work(False)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / 3
        for _ in range(3):
            rank_work(True)
        rows.append({"R": R, "segment_tokens": e - a, "rank_ms": ms, "single_gpu_ms": single_ms,
                     "rank_over_single": ms / single_ms, "map_pass_ms": split[0] / 3, "compose_ms": split[1] / 3,
                     "rerun_ms": split[2] / 3})
    return {"workload": "long_B1_H32_T131072_d128 split into R segments", "per_rank": rows,
            "exchange": "all-gather of [M | b] (32 x 128 x 256 fp32 = 4 MiB per rank) not measured: one GPU"}


def decode_bench(args, dev, stream, peaks, barrier, max_over_ranks):
    """256 x 32 fp32 states (128 x 128), `decode_steps` single-token steps, state updated in place."""
    import torch

    import kimi_delta_attention_29_b200 as kda
    from kimi_delta_attention_29_b200 import inputs as gen

    shp = gen.DECODE
    S = gen.make_decode_state(shp.N, shp.H, shp.dk, shp.dv, std=shp.s0_std, seed=0, device=dev)
    pool = [gen.make_decode_token(shp.N, shp.H, shp.dk, shp.dv, dtype=shp.dtype, seed=1000 + s, device=dev)
            for s in range(8)]
    o = torch.empty(shp.N, shp.H, shp.dv, dtype=shp.dtype, device=dev)

    def step(s):
        t = pool[s % len(pool)]
        kda.kda_decode_step(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], S, o=o, stream=stream)

    for s in range(16):
        step(s)
    torch.cuda.synchronize(dev)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for s in range(args.decode_steps):
        step(s)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1)) / args.decode_steps
    nbytes = shp.N * shp.H * DECODE_BYTES_PER_STATE
    gbs = nbytes / (ms / 1e3) / 1e9
    traffic = ncu_traffic("kda_decode_kernel", shp.N * shp.H)
    out = {"workload": shp.name, "steps": args.decode_steps, "ms_per_step": ms,
           "tokens_per_s": shp.N / (ms / 1e3), "hbm_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
           "frac": gbs / peaks["hbm_gbs"], "bytes_per_step": nbytes, "traffic": traffic,
           "note": "inputs cycle through 8 pre-drawn token sets; the 512 MiB state streams from HBM each step"}
    out["multi_token"] = [decode_multi_bench(args, dev, stream, peaks, barrier, max_over_ranks, S, tq)
                          for tq in MULTI_TQ]
    return out


def decode_multi_bench(args, dev, stream, peaks, barrier, max_over_ranks, pool, tq):
    """The same 256 x 32 states as a slot pool, `tq` tokens per call (kda_decode_multi), slots a fixed
    permutation, committed in place; decode_steps tokens in all."""
    import torch

    import kimi_delta_attention_29_b200 as kda
    from kimi_delta_attention_29_b200 import inputs as gen

    shp = gen.DECODE
    perm = torch.randperm(shp.N, generator=torch.Generator().manual_seed(3)).to(torch.int32).to(dev)
    toks = [gen.make_decode_tokens(shp.N, tq, shp.H, shp.dk, shp.dv, dtype=shp.dtype, seed=3000 + s, device=dev)
            for s in range(4)]
    o = torch.empty(shp.N, tq, shp.H, shp.dv, dtype=shp.dtype, device=dev)
    calls = max(1, args.decode_steps // tq)

    def call(s):
        t = toks[s % len(toks)]
        kda.kda_decode_multi(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], pool, slot_in=perm, slot_out=perm,
                             o=o, stream=stream)

    for s in range(8):
        call(s)
    torch.cuda.synchronize(dev)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for s in range(calls):
        call(s)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1)) / calls
    states = shp.N * shp.H
    nbytes = states * (2 * shp.dk * shp.dv * 4 + tq * (DECODE_BYTES_PER_STATE - 2 * shp.dk * shp.dv * 4))
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"tq": tq, "calls": calls, "ms_per_call": ms, "tokens_per_s": shp.N * tq / (ms / 1e3),
            "hbm_gbs": gbs, "frac": gbs / peaks["hbm_gbs"], "bytes_per_call": nbytes}


def main():
    args = parse_args()
    if args.impl == "reference":
        return reference_arm(args)
    return gpu_arm(args)


if __name__ == "__main__":
    sys.exit(main())
