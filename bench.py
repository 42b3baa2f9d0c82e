#!/usr/bin/env python
"""Benchmark of the KDA operator on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long]
                    [--impl reference]

A step is one pass of the hot path over one batch of synthetic input: one
``kda_chunk_fwd`` call over the long-prefill workload (B=1, H=32, T=131072,
dk=dv=128, bf16 q/k/v, fp32 gate/beta/state).  ``value`` is prefill tokens/s
with the inputs resident in HBM; ``e2e`` is the same metric through the public
API with host (pinned) buffers, host<->device copies inside the timed region.
The batched decode step (256 requests x 32 heads) is timed in the same run and
reported under ``decode`` (HBM GB/s).  With N > 1 (torchrun) the ranks split
the heads (rank r takes a contiguous range, as tensor parallelism over heads
would hand it; no data-path collective): the whole job stays the workload's
tokens over all heads (strong scaling) and the time is the maximum over
ranks.  With few heads per rank the automatic choice runs the segmented
(sequence-parallel) prefill.

``--impl reference`` times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload and prints the same metric with impl=reference.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "KDA prefill tokens/s + % bf16 tensor peak; decode-step HBM GB/s"
UNIT = "tokens/s"
FLOP_PER_TOKEN_HEAD = 6 * 128 * 128 + 10 * 64 * 128     # 180,224 dense-tile count
FLOP_PER_TOKEN_HEAD_TRI = 6 * 128 * 128 + 5 * 64 * 128  # 139,264 triangular count
BYTES_PER_TOKEN_HEAD_BF16 = 3 * 256 + 512 + 4 + 256     # q,k,v + g + beta + out = 1540
STATE_BYTES = 128 * 128 * 4
NOMINAL_HBM_GBS = 8000.0


def bwd_flop_per_chunk_head(C: int = 64, d: int = 128) -> int:
    """FLOPs of one chunk and head of the backward pass, each product of its
    three launches counted once: the forward recompute (A, P, U, P U:
    8C^2 d; V - Kt S0, Qt S0, the state update: 6 C d^2; the triangular
    solve C^3 / 3), the reverse chain (A, P, Pt dO, Tt dU: 8 C^2 d; Kh Z,
    Qt^T dO, Kt^T dR: 6 C d^2; C^3 / 3) and the per-chunk gradients (A, U,
    dT, dP and the four products with Kh, Kt, Qt: 16 C^2 d; R, dO S0^T,
    dR S0^T, U Z^T, S0 + Kh^T U: 10 C d^2; dM M^T and M^T X: 4 C^3; C^3 / 3)."""
    solve = C ** 3 // 3
    fwd = 8 * C * C * d + 6 * C * d * d + solve
    chain = 8 * C * C * d + 6 * C * d * d + solve
    chunk = 16 * C * C * d + 10 * C * d * d + 4 * C ** 3 + solve
    return fwd + chain + chunk


# FP32 FMA peak of one B200 at its maximum SM clock: SMs x 128 FP32 lanes x 2
NOMINAL_SM_MHZ = 1965.0
FP32_LANES_PER_SM = 128


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class Clocks:
    """Samples SM clock and throttle reasons with nvidia-smi during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            p = torch.cuda.get_device_properties(device)
            self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            self.bus = None

    def start(self):
        if not self.bus:
            return
        import tempfile
        self.path = tempfile.mktemp(suffix=".csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi takes a while to start: wait (up to 3 s) for its first
        # sample so that it samples the whole timed region that follows
        t0 = time.time()
        while time.time() - t0 < 3.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 8:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        smax = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("chunk_tc.cu", "chunk_split.cu", "chunk_common.cuh", "sm100_ptx.cuh", "kda_internal.h"):
        p = os.path.join(ROOT, "gated_delta_rule_103_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the prefill kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = kernel_source_sha()
    for line in open(p):
        f = line.split()
        if len(f) >= 3 and not line.startswith("#") and f[0] == workload and f[1] == sha:
            return float(f[2])
    return None


def time_prefill(x, steps, warmup, stream, pg, l2norm_qk=False, out_gate=None, out_weight=None,
                 raw_gate=False):
    import gated_delta_rule_103_b200 as kda
    out = torch.empty_like(x["v"])
    fs = torch.empty(x["N"], x["H"], 128, 128, device=x["q"].device, dtype=torch.float32)
    # the caller-owned workspace, allocated once outside the timed region
    need = kda.chunk_fwd_workspace_bytes(x["B"], x["T"], x["H"], x["N"], x["q"].dtype)
    ws = torch.empty(need, dtype=torch.uint8, device=x["q"].device) if need else None

    def step():
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                      initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                      scale=x["scale"], out=out, final_state=fs, stream=stream,
                      l2norm_qk=l2norm_qk, out_gate=out_gate, out_weight=out_weight,
                      workspace=ws, raw_gate=raw_gate)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if pg is not None:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if pg is not None:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    return total_ms, launch_ms


def time_prefill_e2e(x_host, steps, stream):
    """Host buffers -> device -> kernel -> host, all inside the timed region."""
    import gated_delta_rule_103_b200 as kda
    dev = torch.device("cuda", torch.cuda.current_device())
    names = [n for n in ("q", "k", "v", "log_alpha", "beta", "initial_state", "cu_seqlens")
             if x_host.get(n) is not None]
    dbuf = {n: torch.empty_like(x_host[n], device=dev) for n in names}
    out_h = torch.empty(x_host["v"].shape, dtype=x_host["v"].dtype, pin_memory=True)
    fs_h = torch.empty(x_host["N"], x_host["H"], 128, 128, dtype=torch.float32, pin_memory=True)
    out_d = torch.empty_like(dbuf["v"])
    fs_d = torch.empty(fs_h.shape, dtype=torch.float32, device=dev)
    h2d = sum(x_host[n].numel() * x_host[n].element_size() for n in names)
    d2h = out_h.numel() * out_h.element_size() + fs_h.numel() * 4

    def step():
        with torch.cuda.stream(stream):
            for n in names:
                dbuf[n].copy_(x_host[n], non_blocking=True)
            kda.chunk_fwd(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["log_alpha"], dbuf["beta"],
                          initial_state=dbuf.get("initial_state"),
                          cu_seqlens=dbuf.get("cu_seqlens"),
                          scale=x_host["scale"], out=out_d, final_state=fs_d, stream=stream)
            out_h.copy_(out_d, non_blocking=True)
            fs_h.copy_(fs_d, non_blocking=True)

    step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps, h2d, d2h


def time_backward(x, steps, warmup, stream, pg):
    """kda_chunk_bwd on the workload, adjoints drawn once; mean ms per call
    (three launches each: the forward recompute of the chunk states, the
    reverse state-adjoint chain, the per-chunk gradients)."""
    import gated_delta_rule_103_b200 as kda
    from gated_delta_rule_103_b200 import inputs
    d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), x["N"], x["H"], seed=7,
                                          device=x["q"].device)
    dev = x["q"].device
    ws = torch.empty(kda.chunk_bwd_workspace_bytes(x["B"], x["T"], x["H"], x["N"],
                                                   x["cu_seqlens"] is not None, x["q"].dtype),
                     dtype=torch.uint8, device=dev)
    B, T, H, N = x["B"], x["T"], x["H"], x["N"]
    f32 = dict(dtype=torch.float32, device=dev)
    grads = (torch.empty(B, T, H, 128, **f32), torch.empty(B, T, H, 128, **f32),
             torch.empty(B, T, H, 128, **f32), torch.empty(B, T, H, 128, **f32),
             torch.empty(B, T, H, **f32), torch.empty(N, H, 128, 128, **f32))

    def step():
        kda.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_out,
                      initial_state=x["initial_state"], d_final_state=dfs,
                      cu_seqlens=x["cu_seqlens"], scale=x["scale"], stream=stream,
                      workspace=ws, grads=grads)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    torch.cuda.synchronize()
    if pg is not None:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
    torch.cuda.synchronize()
    if pg is not None:
        torch.distributed.barrier()
    return t0.elapsed_time(t1) / steps


def time_decode(N, H, steps, warmup, stream, seed=1005):
    """`steps` consecutive decode steps on one state (updated in place), each
    with its own inputs drawn beforehand on the device; mean ms per step."""
    import gated_delta_rule_103_b200 as kda
    from gated_delta_rule_103_b200 import inputs
    dev = torch.device("cuda", torch.cuda.current_device())
    state = inputs.decode_state(N, H, seed=seed, std=0.1, device=dev)
    xs = [inputs.decode_inputs(N, H, seed=seed, step=s + 1, device=dev) for s in range(steps)]
    out = torch.empty(N, H, 128, dtype=torch.bfloat16, device=dev)

    def step(x):
        kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state,
                           scale=x["scale"], out=out, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(warmup):
            step(xs[i % steps])
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(xs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    units = N * H
    nbytes = units * (2 * STATE_BYTES + 3 * 256 + 512 + 4 + 256)
    return ms, nbytes


def cpu_baseline(workload: dict, budget_s: float = 15.0) -> dict:
    """The fp64 oracle, as it stands, on a bounded sample of the workload:
    all its heads' first `t` tokens of the one sequence, t grown until the
    sample takes a few seconds, then repeated to about `budget_s`; then the
    same oracle on one host core on a 256-token sample."""
    import oracle
    from gated_delta_rule_103_b200.configs import make_prefill
    cores = oracle.max_threads()
    H = workload["H"]
    t = 256
    spent, token_heads = 0.0, 0
    while spent < budget_s:
        x = make_prefill("long", T=t)
        a = time.perf_counter()
        oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], scale=x["scale"])
        dt = time.perf_counter() - a
        spent += dt
        token_heads += t * H
        if dt < budget_s / 4:
            t *= 2
    tokens_per_s = token_heads / H / spent
    # one core: the first 256 tokens of all heads
    x = make_prefill("long", T=256)
    a = time.perf_counter()
    oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], scale=x["scale"],
                       nthreads=1)
    one = 256 / (time.perf_counter() - a)
    return {"value": tokens_per_s, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"long-prefill recipe, H={H}, first {t} tokens of the sequence "
                      f"(doubling from 256), {token_heads} token-heads in {spent:.1f} s",
            "single_core": {"value": one, "unit": UNIT, "cores": 1,
                            "sample": f"first 256 tokens x {H} heads of the long-prefill recipe"}}


def kernel_only(args, dev, stream):
    """Launches only the workload's kernel (warmup + steps times) and prints
    the mean CUDA-event time per launch: the case the ncu captures use."""
    import gated_delta_rule_103_b200 as kda
    from gated_delta_rule_103_b200.configs import WORKLOADS, make_prefill
    if args.workload == "decode":
        ms, nbytes = time_decode(256, 32, args.steps, args.warmup, stream)
        print(json.dumps({"kernel": "decode", "ms": ms, "GB_per_s": nbytes / ms / 1e6}))
        return
    if args.workload == "backward":
        x = make_prefill("short", device=dev, **({"T": args.T} if args.T else {}))
        ms = time_backward(x, args.steps, args.warmup, stream, None)
        print(json.dumps({"kernel": "chunk_bwd", "workload": "short", "T": x["T"], "ms": ms}))
        return
    over = {}
    if args.T:
        over["T"] = args.T
    if args.H:
        over["H"] = args.H
    x = make_prefill(args.workload, device=dev, **over)
    total_ms, launch_ms = time_prefill(x, args.steps, args.warmup, stream, None)
    print(json.dumps({"kernel": "chunk_fwd", "workload": args.workload, "T": x["T"], "H": x["H"],
                      "prefill_kernel": kda.binding.prefill_kernel_choice(x["B"], x["T"], x["H"],
                                                                          x["N"]),
                      "ms": total_ms / args.steps}))


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from gated_delta_rule_103_b200.configs import WORKLOADS
    w = WORKLOADS["long"]
    import oracle
    from gated_delta_rule_103_b200.configs import make_prefill
    cores = oracle.max_threads()
    t = 512
    x = make_prefill("long", T=t)
    times = []
    for i in range(args.warmup + args.steps):
        a = time.perf_counter()
        oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], scale=x["scale"])
        if i >= args.warmup:
            times.append(time.perf_counter() - a)
    ms = 1000.0 * sum(times) / len(times)
    value = t / (ms / 1000.0)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "long prefill B=1 H=32 T=131072 dk=dv=128 (sampled)",
                       "sample_tokens": t},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"first {t} tokens x {w['H']} heads of the long-prefill "
                                       "recipe per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="long", choices=["long", "short", "varlen", "decode", "backward"])
    ap.add_argument("--T", type=int, default=None,
                    help="override the workload's sequence length (profiling cases)")
    ap.add_argument("--H", type=int, default=None,
                    help="override the workload's head count (profiling cases)")
    ap.add_argument("--kernel-only", action="store_true",
                    help="only launch the workload's kernel warmup + steps times and print its "
                         "CUDA-event time (the short case ncu captures run)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = torch.distributed.group.WORLD
    import gated_delta_rule_103_b200 as kda
    from gated_delta_rule_103_b200.configs import WORKLOADS, make_prefill
    from gated_delta_rule_103_b200.sharding import head_range, max_over_ranks
    kda.load_library()
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream()
    if args.kernel_only:
        return kernel_only(args, dev, stream)
    if args.workload in ("decode", "backward"):
        raise SystemExit(f"the {args.workload} step is timed inside every run; "
                         "use --kernel-only to time it alone")
    w = WORKLOADS[args.workload]
    H_all = args.H or w["H"]
    # N ranks split the heads (tensor-parallel style, no data-path
    # collective): the whole job is the workload's tokens over all heads
    h0, h1 = head_range(H_all, ws, rank)
    over = {"H": h1 - h0, "seed": w["seed"] + 7919 * h0}
    if args.T:
        over["T"] = args.T
    x = make_prefill(args.workload, device=dev, **over)
    clocks = Clocks(local)

    clocks.start()
    total_ms, launch_ms = time_prefill(x, args.steps, args.warmup, stream, pg)
    clk = clocks.stop()
    ms_step = max_over_ranks(total_ms / args.steps, device=dev)
    tokens = x["B"] * x["T"]
    value = tokens / (ms_step / 1000.0)

    pk = peaks()
    th = tokens * x["H"]
    alg_bytes = th * BYTES_PER_TOKEN_HEAD_BF16 + x["N"] * x["H"] * STATE_BYTES * (
        (1 if x["initial_state"] is not None else 0) + 1)
    launch_avg = sum(launch_ms) / len(launch_ms)
    achieved_gbs = alg_bytes / (launch_avg / 1000.0) / 1e9
    tflops = th * FLOP_PER_TOKEN_HEAD / (launch_avg / 1000.0) / 1e12
    traffic = recorded_traffic(args.workload) if ws == 1 and not args.T and not args.H else None
    kernel = kda.binding.prefill_kernel_choice(x["B"], x["T"], x["H"], x["N"])

    # end to end through the public API with host buffers
    x_host = {n: (v.cpu().pin_memory() if isinstance(v, torch.Tensor) else v)
              for n, v in x.items()}
    e2e_ms, h2d, d2h = time_prefill_e2e(x_host, args.e2e_steps, stream)
    e2e_ms = max_over_ranks(e2e_ms, device=dev)
    del x_host

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload} prefill: B={x['B']} H={H_all} T={x['T']} "
                               f"dk=dv=128 chunk=64, bf16 q/k/v, fp32 log_alpha/beta/state",
                   "tokens_per_step": tokens, "heads_per_gpu": x["H"],
                   "l2": "inputs > L2 (no flush needed)", "prefill_kernel": kernel,
                   "prefill_segments": kda.binding.prefill_segments(x["B"], x["T"], x["H"], x["N"]),
                   "parallelism": f"heads split over {ws} GPU(s) ({x['H']} per GPU), "
                                  "no data-path collective"},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": pk["hbm"], "unit": "GB/s",
                     "frac": achieved_gbs / pk["hbm"], "traffic": traffic,
                     "peak_source": pk["source"],
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "tensor": {"achieved_tflops": tflops, "peak_burst": pk["bf16"],
                                "frac_burst": tflops / pk["bf16"],
                                "frac_sustained": tflops / pk["bf16_sustained"],
                                "flop_per_token_head": FLOP_PER_TOKEN_HEAD,
                                "frac_burst_triangular_count":
                                    tflops * FLOP_PER_TOKEN_HEAD_TRI / FLOP_PER_TOKEN_HEAD / pk["bf16"]}},
        "e2e": {"value": tokens / (e2e_ms / 1000.0), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * (1 if kernel != "segmented" else 3),
        "clocks": clk,
    }
    if ws == 1:
        line.update(context_entries(args, x, dev, stream, pg, pk, tokens))
        if rank == 0 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
    if pg is not None:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def context_entries(args, x, dev, stream, pg, pk, tokens) -> dict:
    """The other entries of a one-GPU run, each timed by the same rules: the
    headline step with the fused L2Norm and with the output epilogue, the
    other prefill workloads, the few-chain long-context case, the backward
    pass and the batched decode step."""
    import gated_delta_rule_103_b200 as kda
    from gated_delta_rule_103_b200 import inputs as _inputs
    from gated_delta_rule_103_b200.configs import make_prefill
    out = {}
    # the same step with the fused L2Norm of q and k (KDA_FLAG_L2NORM_QK)
    l2_ms, _ = time_prefill(x, args.steps, args.warmup, stream, pg, l2norm_qk=True)
    out["l2norm_qk"] = {"ms_per_step": l2_ms / args.steps,
                        "value": tokens / (l2_ms / args.steps / 1000.0), "unit": UNIT,
                        "note": "same step, q and k L2-normalised inside the kernel"}
    # with the gate given as pre-activations (KDA_FLAG_RAW_GATE; the same
    # decays: z = logit(alpha) of the workload's gate)
    xr = dict(x, log_alpha=(x["log_alpha"] - torch.log(-torch.expm1(x["log_alpha"]))).contiguous())
    rg_ms, _ = time_prefill(xr, args.steps, args.warmup, stream, pg, raw_gate=True)
    del xr
    out["raw_gate"] = {"ms_per_step": rg_ms / args.steps,
                       "value": tokens / (rg_ms / args.steps / 1000.0), "unit": UNIT,
                       "note": "same step, log alpha = log sigmoid(z) from pre-activations z "
                               "inside the kernel"}
    # and with the output RMSNorm + sigmoid gate (KDA_FLAG_OUT_NORM_GATE)
    gate, weight = _inputs.out_gate_inputs(tuple(x["v"].shape), x["v"].dtype, seed=7, device=dev)
    ng_ms, _ = time_prefill(x, args.steps, args.warmup, stream, pg, out_gate=gate, out_weight=weight)
    del gate, weight
    out["out_norm_gate"] = {"ms_per_step": ng_ms / args.steps,
                            "value": tokens / (ng_ms / args.steps / 1000.0), "unit": UNIT,
                            "note": "same step plus the output RMSNorm and sigmoid gate"}

    # the other prefill configurations, for context (same timing rules)
    others = {}
    for name in ("short", "varlen"):
        xo = make_prefill(name, device=dev)
        o_ms, _ = time_prefill(xo, args.steps, args.warmup, stream, pg)
        o_ms /= args.steps
        o_tok = xo["B"] * xo["T"]
        others[name] = {"ms_per_step": o_ms, "value": o_tok / (o_ms / 1000.0), "unit": UNIT,
                        "tokens_per_step": o_tok,
                        "prefill_kernel": kda.binding.prefill_kernel_choice(
                            xo["B"], xo["T"], xo["H"], xo["N"])}
        del xo
    out["other_prefill"] = others

    # few (sequence, head) chains at a long context: 8 heads (a 4-way head
    # split of the 32) over 512k tokens, segmented by the automatic choice,
    # against the unsegmented cluster kernel
    xf = make_prefill("long", device=dev, H=8, T=524288, seed=1006)
    f_ms, f_launch = time_prefill(xf, args.steps, args.warmup, stream, pg)
    f_ms /= args.steps
    kda.binding.set_prefill_kernel("cluster")
    try:
        c_ms, _ = time_prefill(xf, args.steps, args.warmup, stream, pg)
    finally:
        kda.binding.set_prefill_kernel("auto")
    c_ms /= args.steps
    f_th = xf["T"] * xf["H"]
    f_bytes = f_th * BYTES_PER_TOKEN_HEAD_BF16 + xf["H"] * STATE_BYTES
    out["few_chains_long_context"] = {
        "workload": "B=1 H=8 T=524288 dk=dv=128, long-prefill recipe",
        "ms_per_step": f_ms, "value": xf["T"] / (f_ms / 1000.0), "unit": UNIT,
        "prefill_kernel": kda.binding.prefill_kernel_choice(1, xf["T"], 8, 1),
        "prefill_segments": kda.binding.prefill_segments(1, xf["T"], 8, 1),
        "cluster_kernel_ms_per_step": c_ms,
        "speedup_vs_cluster": c_ms / f_ms,
        "hbm_frac": f_bytes / (f_ms / 1000.0) / 1e9 / pk["hbm"]}
    del xf

    # the backward pass on the short-prefill configuration
    xb = make_prefill("short", device=dev)
    bwd_ms = time_backward(xb, 3, 3, stream, pg)
    bwd_tok = xb["B"] * xb["T"]
    bwd_flop = bwd_tok * xb["H"] * bwd_flop_per_chunk_head() / 64.0
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    fp32_peak = sms * FP32_LANES_PER_SM * 2 * NOMINAL_SM_MHZ * 1e6 / 1e12
    bwd_tflops = bwd_flop / (bwd_ms / 1000.0) / 1e12
    del xb
    out["backward"] = {
        "workload": "short prefill B=4 H=32 T=4096, adjoints of out and final state",
        "ms_per_step": bwd_ms, "value": bwd_tok / (bwd_ms / 1000.0), "unit": UNIT,
        "steps": 3, "note": "kda_chunk_bwd, fp32 FFMA: chunk-state recompute, reverse "
                            "state-adjoint chain, per-chunk gradients",
        "roofline": {"bound": "alu", "achieved": bwd_tflops, "peak": fp32_peak,
                     "unit": "TFLOP/s", "frac": bwd_tflops / fp32_peak,
                     "peak_source": f"{sms} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 "
                                    f"x {NOMINAL_SM_MHZ:.0f} MHz",
                     "flop_per_chunk_head": bwd_flop_per_chunk_head()}}

    dec_ms, dec_bytes = time_decode(256, 32, args.decode_steps, 3, stream)
    dec_gbs = dec_bytes / (dec_ms / 1000.0) / 1e9
    out["decode"] = {"workload": "256 requests x 32 heads, one token each, dk=dv=128, "
                                 f"{args.decode_steps} consecutive steps on one state",
                     "ms_per_step": dec_ms, "GB_per_s": dec_gbs, "frac_hbm": dec_gbs / pk["hbm"],
                     "frac_8TBps": dec_gbs / NOMINAL_HBM_GBS, "steps": args.decode_steps}
    return out


if __name__ == "__main__":
    main()
