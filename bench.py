#!/usr/bin/env python
"""Benchmark of ReHyAt's temporally chunked hybrid attention forward on B200.

Default workload (one GPU): Wan2.1-1.3B 480p attention shape, B=1, H=12,
d=128, F=21 latent frames x 30x52 = 1560 tokens (32,760 tokens), T_c=3,
T_o=1, bf16, Gaussian Q/K/V with RMS-normalised Q/K (seeded, synthetic).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config wan13b|wan14b|recurrent] [--sweep]

A step = one pass of the whole path over one batch: the states stage
(phi(K), per-segment phi(K)^T V, chunk scan) and the fused chunk attention.
Under torchrun each rank runs its own batch (weak scaling, no collective on
the data path); the step time is the max over ranks.  Rank 0 prints one JSON
line.  --impl reference times the fp64 CPU oracle on bounded row samples.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "hybrid-attention tokens/s on 1 B200 and % of roofline, Wan2.1-1.3B 480p shape"
UNIT = "tokens/s"

CONFIGS = {
    "wan13b": dict(workload="Wan2.1-1.3B 480p attention shape", B=1, H=12, d=128, F=21, S_tok=1560,
                   T_c=3, T_o=1, seed=1),
    "wan14b": dict(workload="Wan2.1-14B 720p-like attention shape", B=1, H=40, d=128, F=21, S_tok=3600,
                   T_c=3, T_o=1, seed=3),
    "recurrent": dict(workload="long-video recurrent mode (rehyat_step), 81 latent frames", B=1, H=12, d=128,
                      F=81, S_tok=1560, T_c=3, T_o=1, seed=2),
}
SWEEP = [(F, tc, to) for (tc, to) in ((2, 1), (3, 1), (5, 2)) for F in (21, 41, 81, 161)]


# --------------------------------------------------------------------------- #
# algorithmic work (FLOPs and bytes the method needs, nothing masked counted)  #
# --------------------------------------------------------------------------- #
def chunks(F, S, Tc, To):
    tc, to = min(Tc, F), min(To, F)
    N, Np = F * S, tc * S
    for t in range(-(-F // tc)):
        q0, q1 = t * Np, min((t + 1) * Np, N)
        yield q0, q1, max(q0 - to * S, 0), q1


def work(c, sets="causal"):
    B, H, d, F, S, Tc, To = (c[k] for k in ("B", "H", "d", "F", "S_tok", "T_c", "T_o"))
    BH, N, D2 = B * H, F * S, 2 * d
    ch = list(chunks(F, S, Tc, To))
    pairs = sum((q1 - q0) * (hi - lo) for q0, q1, lo, hi in ch)
    if sets == "causal":
        n_lin = sum(q1 - q0 for q0, q1, lo, hi in ch if lo > 0)   # queries with a linear term
        folded = max(lo for _, _, lo, _ in ch)                    # keys folded into states
    else:
        n_lin = sum(q1 - q0 for q0, q1, lo, hi in ch if lo > 0 or hi < N)
        folded = N if len(ch) > 1 else 0
    attn_flops = BH * (4 * d * pairs + 2 * D2 * (d + 1) * n_lin)
    state_flops = BH * 2 * D2 * (d + 1) * folded
    attn_bytes = BH * N * d * 2 * 4 + BH * len(ch) * D2 * (d * 4 + 4)     # q,k,v,out + states (hi,lo,z)
    state_bytes = BH * folded * d * 2 * 2 + BH * len(ch) * D2 * (d * 4 + 4)
    # learned feature map, both maps: x [N, d] -> relu(W1 x) [N, 2d] -> phi [N, 2d]
    mlp_flops = 2 * BH * N * 2 * (D2 * d + D2 * D2)
    mlp_bytes = 2 * (BH * N * (d + D2) * 2 + H * (D2 * d + D2 * D2) * 2 + H * 2 * D2 * 4)
    return dict(pairs_per_head=pairs, attn_flops=attn_flops, state_flops=state_flops, attn_bytes=attn_bytes,
                state_bytes=state_bytes, tokens=B * N, mlp_flops=mlp_flops, mlp_bytes=mlp_bytes)


def recurrent_bytes(c):
    """HBM bytes of the recurrent form over one video: every step reads its
    chunk's queries and its whole key/value window (overlap frames again) and
    writes its output (bf16), and reads and writes the fp32 state (S, z)."""
    B, H, d, F, S, Tc, To = (c[k] for k in ("B", "H", "d", "F", "S_tok", "T_c", "T_o"))
    BH, D2 = B * H, 2 * d
    rows = sum(2 * (q1 - q0) + 2 * (hi - lo) for q0, q1, lo, hi in chunks(F, S, Tc, To))
    n_steps = -(-F // min(Tc, F))
    return BH * rows * d * 2 + n_steps * BH * 2 * D2 * (d + 1) * 4


KERNEL_SOURCES = ("tc_kernels.cu", "tc_common.cuh", "ptx.cuh", "kernels.cuh", "geom.cuh")
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "hybrid_chunk_attn_h6_full.md")


def attn_traffic(c):
    """DRAM bytes per full launch from the committed ncu summary, or None if
    the kernel sources changed since it was captured (or the workload differs)."""
    import hashlib
    try:
        csrc = os.path.join(ROOT, "linear_attention_video_chunk_b200", "csrc")
        h = hashlib.sha256(b"".join(open(os.path.join(csrc, f), "rb").read() for f in KERNEL_SOURCES)).hexdigest()
        txt = open(TRAFFIC_PROFILE).read()
        sha = txt.split("- source_sha256:")[1].split()[0]
        nbytes = int(txt.split("- dram_bytes_per_full_launch:")[1].split()[0])
    except Exception:
        return None
    if sha != h or (c["B"], c["H"], c["F"], c["S_tok"]) != (1, 12, 21, 1560):
        return None
    return nbytes


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            j = json.load(fh)
        return j["bf16_tflops"], j.get("bf16_tflops_sustained"), j["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


# --------------------------------------------------------------------------- #
# clocks sampled during the timed region (NVML reads only)                    #
# --------------------------------------------------------------------------- #
class ClockSampler:
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, dev):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:  # NVML enumerates every GPU; match the CUDA device by UUID
                uuid = str(torch.cuda.get_device_properties(dev).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(dev.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv is not None:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.th.join()

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------------------- #
# CPU baseline: the fp64 oracle on bounded row samples                         #
# --------------------------------------------------------------------------- #
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def oracle_sample_rate(c, q, k, v, budget_s):
    """Tokens/s of the oracle: rows (all heads) per second on a row sample
    sized to take about budget_s seconds.  Returns (rate, rows, seconds)."""
    import numpy as np
    import oracle.rehyat_oracle as orc
    N = c["F"] * c["S_tok"]
    rng = np.random.default_rng(7)
    args = (c["F"], c["S_tok"], c["T_c"], c["T_o"])
    # two calibration samples separate the per-call cost (phi of every key)
    # from the per-row cost, so the measured sample lasts about budget_s
    t0 = time.perf_counter()
    orc.oracle_forward(q, k, v, *args, rows=np.sort(rng.choice(N, 8, replace=False)))
    t8 = time.perf_counter() - t0
    t0 = time.perf_counter()
    orc.oracle_forward(q, k, v, *args, rows=np.sort(rng.choice(N, 64, replace=False)))
    t64 = time.perf_counter() - t0
    per_row = max((t64 - t8) / 56, 1e-6)
    fixed = max(t8 - 8 * per_row, 0.0)
    n = int(max(8, min(N, (budget_s - fixed) / per_row)))
    rows = np.sort(rng.choice(N, n, replace=False))
    t0 = time.perf_counter()
    orc.oracle_forward(q, k, v, *args, rows=rows)
    dt = time.perf_counter() - t0
    return n / dt, n, dt


def config_dict(c, world):
    """The workload description both arms print (identical for one workload)."""
    tokens = c["B"] * c["F"] * c["S_tok"]
    return {"workload": c["workload"], "B": c["B"], "H": c["H"], "d": c["d"], "F": c["F"], "S_tok": c["S_tok"],
            "chunk_frames": c["T_c"], "overlap_frames": c["T_o"], "tokens_per_step_per_gpu": tokens,
            "parallelism": f"replicas x{world} (no collective)",
            "l2": "inputs larger than L2: q+k+v = %.0f MB per GPU" % (3 * tokens * c["H"] * c["d"] * 2 / 1e6)}


# --------------------------------------------------------------------------- #
# our arm                                                                      #
# --------------------------------------------------------------------------- #
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_forward_bench(args, c, rank, world, dev):
    import torch
    from linear_attention_video_chunk_b200 import inputs
    from linear_attention_video_chunk_b200 import rehyat as R
    B, H, d, F, S, Tc, To = (c[k] for k in ("B", "H", "d", "F", "S_tok", "T_c", "T_o"))
    N = F * S
    q, k, v = inputs.make_qkv(B, H, N, d, c["seed"] + 1000 * rank, rms_qk=True, pin=True)
    if args.layout == "bnhd":  # heads interleaved per token: [B, N, H, d]
        q, k, v = (x.transpose(1, 2).contiguous().pin_memory() for x in (q, k, v))
    qd, kd, vd = (x.to(dev, non_blocking=True) for x in (q, k, v))
    out = torch.empty_like(qd)
    ws = R.alloc_workspace(R.workspace_bytes(B, H, F, S, d, Tc, To), dev)
    torch.cuda.synchronize()

    mlp = args.phi == "mlp"
    one_call = args.sets != "causal" or args.layout != "bhnd" or mlp
    if mlp:  # learned feature maps: resident weights, phi(q) and phi(k) computed every step
        wq = tuple(t.to(dev) for t in inputs.make_mlp_weights(H, d, c["seed"], "q"))
        wk = tuple(t.to(dev) for t in inputs.make_mlp_weights(H, d, c["seed"], "k"))
        ws = R.alloc_workspace(R.forward_mlp_workspace_bytes(B, H, F, S, d, Tc, To, args.sets), dev)
    elif one_call:  # one call (states + attention) per step
        n = R.ctypes.c_size_t(0)
        R.lib().rehyat_forward_ex_workspace_bytes(B, H, F, S, d, Tc, To, R.SETS[args.sets], R.ctypes.byref(n))
        ws = R.alloc_workspace(n.value, dev)

    def step(e0=None, e1=None, e2=None):
        if e0 is not None:
            e0.record()
        if mlp:
            if e1 is not None:
                e1.record()
            R.forward_mlp(qd, kd, vd, wq, wk, F, S, Tc, To, sets=args.sets, layout=args.layout, out=out,
                          workspace=ws)
        elif one_call:
            if e1 is not None:
                e1.record()
            R.forward_sets(qd, kd, vd, F, S, Tc, To, sets=args.sets, layout=args.layout, out=out, workspace=ws)
        else:
            R.forward_states(kd, vd, F, S, Tc, To, ws)
            if e1 is not None:
                e1.record()
            R.forward_attention(qd, kd, vd, F, S, Tc, To, out, ws)
        if e2 is not None:
            e2.record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        start.record()
        for i in range(K):
            step(*ev[i])
        end.record()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms_step = max_over_ranks(start.elapsed_time(end) / K, world, dev)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    state_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    mlp_ms = None
    if mlp:  # the feature-map kernel alone (one map per launch), for its roofline
        phi_out = torch.empty((B, H, N, 2 * d), dtype=torch.bfloat16, device=dev)
        src = qd
        for _ in range(3):
            R.phi_mlp(src, *wq, layout=args.layout, out=phi_out)
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        Km = max(3, min(K, 50))
        m0.record()
        for _ in range(Km):
            R.phi_mlp(src, *wq, layout=args.layout, out=phi_out)
        m1.record()
        torch.cuda.synchronize()
        mlp_ms = m0.elapsed_time(m1) / Km
        del phi_out

    # end to end through the public API: pinned host inputs -> device ->
    # forward -> result back to pinned host memory, every step
    launches = (4 if mlp else 3) * K
    if args.no_e2e:
        return dict(ms_step=ms_step, attn_ms=attn_ms, state_ms=state_ms, e2e_ms=float("nan"), clocks=clk.summary(),
                    h2d=0, d2h=0, q=q, k=k, v=v, launches=launches, mlp_ms=mlp_ms)
    Ke = max(3, min(K, 20))
    if not mlp:
        # through the C ABI with HOST buffers: every step copies its q, k, v
        # (page-locked) to the device, runs the forward and copies the output
        # back inside rehyat_forward_host; two streams with two device
        # workspaces let one step's copies overlap the other's kernels
        nb = R.forward_host_workspace_bytes(B, H, F, S, d, Tc, To, args.sets)
        streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
        wss = [R.alloc_workspace(nb, dev) for _ in range(2)]
        outs_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]

        def host_step(i):
            R.forward_host(q, k, v, F, S, Tc, To, outs_h[i % 2], wss[i % 2], sets=args.sets, layout=args.layout,
                           stream=streams[i % 2])

        for i in range(4):
            host_step(i)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        s2 = torch.cuda.Event(enable_timing=True)
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        s2.record(streams[0])
        streams[1].wait_event(s2)
        for i in range(Ke):
            host_step(i)
        for j in range(2):
            ends[j].record(streams[j])
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(max(s2.elapsed_time(e) for e in ends) / Ke, world, dev)
        status = R.device_status()
        if status != R.OK:
            raise RuntimeError(f"device status {R.status_string(status)}")
        return dict(ms_step=ms_step, attn_ms=attn_ms, state_ms=state_ms, e2e_ms=e2e_ms, clocks=clk.summary(),
                    h2d=3 * q.numel() * q.element_size(), d2h=out.numel() * out.element_size(), q=q, k=k, v=v,
                    launches=launches, mlp_ms=mlp_ms, e2e_kind="rehyat_forward_host, host buffers, 2 streams")
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

    def fwd(o):  # the public API call a user makes
        if mlp:
            R.forward_mlp(qd, kd, vd, wq, wk, F, S, Tc, To, sets=args.sets, layout=args.layout, out=o,
                          workspace=ws)
        elif args.sets == "causal" and args.layout == "bhnd":
            R.forward(qd, kd, vd, F, S, Tc, To, out=o, workspace=ws)
        else:
            R.forward_sets(qd, kd, vd, F, S, Tc, To, sets=args.sets, layout=args.layout, out=o, workspace=ws)

    for _ in range(2):
        for src, dst in ((q, qd), (k, kd), (v, vd)):
            dst.copy_(src, non_blocking=True)
        fwd(out)
        out_h.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(Ke):
        for src, dst in ((q, qd), (k, kd), (v, vd)):
            dst.copy_(src, non_blocking=True)
        fwd(out)
        out_h.copy_(out, non_blocking=True)
    e2.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(s2.elapsed_time(e2) / Ke, world, dev)
    status = R.device_status()
    if status != R.OK:
        raise RuntimeError(f"device status {R.status_string(status)}")
    return dict(ms_step=ms_step, attn_ms=attn_ms, state_ms=state_ms, e2e_ms=e2e_ms, clocks=clk.summary(),
                h2d=3 * q.numel() * q.element_size(), d2h=out.numel() * out.element_size(), q=q, k=k, v=v,
                launches=launches, mlp_ms=mlp_ms, e2e_kind="forward_mlp after torch copies, one stream")


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    c = dict(CONFIGS[args.config])
    if args.heads:
        c["H"] = args.heads
        c["workload"] += f" (H overridden to {args.heads})"
    if args.config == "recurrent":
        if args.phi != "fixed":
            raise SystemExit("--phi mlp is measured on the parallel form (wan13b, wan14b)")
        res = run_recurrent_bench(args, c, rank, world, dev)
    else:
        res = run_forward_bench(args, c, rank, world, dev)
    w = work(c, args.sets)
    bf16_peak, bf16_sus, hbm, src = peaks()
    tokens = w["tokens"] * world
    if args.sets != "causal":
        c["workload"] += f" ({args.sets} sets)"
    if args.layout != "bhnd":
        c["workload"] += " ([B, N, H, d] layout)"
    if args.phi == "mlp":
        c["workload"] += " (learned phi: 2-layer MLP, degree-2 features)"
    line = {
        "metric": METRIC, "value": tokens / (res["ms_step"] / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) Q/K/V, per-vector RMS-normalised Q/K, bf16 (no latents or weights)",
        "config": config_dict(c, world),
    }
    if args.config != "recurrent" and args.sets == "causal" and args.layout == "bhnd" and args.phi == "fixed":
        achieved = w["attn_flops"] / (res["attn_ms"] / 1e3) / 1e12
        line["roofline"] = {
            "kernel": "hybrid_chunk_attn_kernel", "bound": "tensor", "achieved": achieved, "peak": bf16_peak,
            "unit": "TFLOP/s", "frac": achieved / bf16_peak, "peak_source": f"{src} bf16 dense (burst)",
            "frac_of_sustained": achieved / bf16_sus if bf16_sus else None, "traffic": attn_traffic(c),
            "algorithmic_bytes": w["attn_bytes"],
            "kernel_ms": res["attn_ms"], "flops_per_launch": w["attn_flops"],
            "states_stage_ms": res["state_ms"],
            "path_frac": (w["attn_flops"] + w["state_flops"]) / (res["ms_step"] / 1e3) / 1e12 / bf16_peak,
        }
    line["e2e"] = {"value": tokens / (res["e2e_ms"] / 1e3), "unit": UNIT, "h2d_bytes_per_step": res["h2d"],
                   "d2h_bytes_per_step": res["d2h"], "ms_per_step": res["e2e_ms"]}
    if res.get("e2e_kind"):
        line["e2e"]["how"] = res["e2e_kind"]
    if res.get("eager_ms"):
        line["timing"] = {"timed_as": "one CUDA graph per video (%d steps x 4 kernels)" % (-(-c["F"] // c["T_c"])),
                          "eager_ms_per_video": res["eager_ms"]}
    if args.config == "recurrent":
        # a streamed video does exactly the parallel form's algorithmic work
        # (same pairs, same linear terms, the same keys folded into the state)
        flops = w["attn_flops"] + w["state_flops"]
        achieved = flops / (res["ms_step"] / 1e3) / 1e12
        nbytes = recurrent_bytes(c)
        t_roof = max(flops / (bf16_peak * 1e12), nbytes / (hbm * 1e9)) * 1e3
        line["roofline"] = {
            "kernel": "whole recurrent path (rehyat_step: %d steps x 4 kernels)" % (-(-c["F"] // c["T_c"])),
            "bound": "tensor", "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
            "frac": achieved / bf16_peak, "peak_source": f"{src} bf16 dense (burst)",
            "frac_of_sustained": achieved / bf16_sus if bf16_sus else None, "traffic": None,
            "flops_per_video": flops, "algorithmic_bytes": nbytes, "roofline_ms_per_video": t_roof,
            "ms_per_video": res["ms_step"],
        }
    line["clocks"] = res["clocks"]
    line["gpu_launches"] = res["launches"]
    if args.config != "recurrent" and (args.sets != "causal" or args.layout != "bhnd" or args.phi == "mlp"):
        # one call per step: the whole path's fraction
        flops = w["attn_flops"] + w["state_flops"] + (w["mlp_flops"] if args.phi == "mlp" else 0)
        line["roofline"] = {"kernel": "whole path (%sstates + fused attention)" %
                                      ("phi MLP + " if args.phi == "mlp" else ""), "bound": "tensor",
                            "achieved": flops / (res["ms_step"] / 1e3) / 1e12,
                            "peak": bf16_peak, "unit": "TFLOP/s", "traffic": None,
                            "peak_source": f"{src} bf16 dense (burst)"}
        line["roofline"]["frac"] = line["roofline"]["achieved"] / bf16_peak
    if res.get("mlp_ms"):
        t = res["mlp_ms"] / 1e3
        fl = w["mlp_flops"] / 2 / t / 1e12       # one map per timed launch
        gbs = w["mlp_bytes"] / 2 / t / 1e9
        line["phi_mlp_kernel"] = {"kernel": "phi_mlp_kernel (one map)", "ms": res["mlp_ms"],
                                  "tflops": fl, "frac_tensor": fl / bf16_peak, "gbs": gbs, "frac_hbm": gbs / hbm,
                                  "flops_per_launch": w["mlp_flops"] // 2, "bytes_per_launch": w["mlp_bytes"] // 2}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.config == "wan13b" and not args.heads \
            and args.sets == "causal" and args.layout == "bhnd" and args.phi == "fixed":
        rate, n, dt = oracle_sample_rate(c, res["q"], res["k"], res["v"], args.cpu_budget)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"fp64 explicit-mask oracle on {n} random query rows x all {c['H']} "
                                          f"heads of the same workload ({dt:.1f} s); value = rows/s"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_recurrent_bench(args, c, rank, world, dev):
    """F frames streamed chunk by chunk through rehyat_step; device memory
    must stay flat across steps (state is constant-size)."""
    import torch
    from linear_attention_video_chunk_b200 import inputs
    from linear_attention_video_chunk_b200 import rehyat as R
    B, H, d, F, S, Tc, To = (c[k] for k in ("B", "H", "d", "F", "S_tok", "T_c", "T_o"))
    q, k, v = inputs.make_qkv(B, H, F * S, d, c["seed"] + 1000 * rank, rms_qk=True, pin=True)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    nc = -(-F // Tc)
    slices = []
    for t in range(nc):
        f0, w0, cf, qf, ef = R.step_frames(t, F, Tc, To)
        slices.append((qd[:, :, f0 * S:(f0 + qf) * S].contiguous(), kd[:, :, w0 * S:(f0 + qf) * S].contiguous(),
                       vd[:, :, w0 * S:(f0 + qf) * S].contiguous(), qf, cf, ef))
    Sst = torch.zeros(B, H, 2 * d, d, device=dev)
    zst = torch.zeros(B, H, 2 * d, device=dev)
    ws = R.alloc_workspace(max(R.step_workspace_bytes(B, H, S, d, s[3], s[4], s[5]) for s in slices), dev)
    outs = [torch.empty_like(s[0]) for s in slices]

    def video():
        Sst.zero_()
        zst.zero_()
        for (qc, kc, vc, qf, cf, ef), o in zip(slices, outs):
            R.step(qc, kc, vc, Sst, zst, S, qf, cf, ef, out=o, workspace=ws)

    for _ in range(max(3, args.warmup)):
        video()
    torch.cuda.synchronize()
    # the whole video (27 steps x 4 kernels at 81 frames) as one CUDA graph:
    # the calls take the caller's workspace and allocate nothing, so they
    # capture as they are
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        video()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    K = max(1, args.steps)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    with ClockSampler(dev) as clk:
        ev[0].record()
        for _ in range(K):
            graph.replay()
        ev[1].record()
        torch.cuda.synchronize()
    ms = max_over_ranks(ev[0].elapsed_time(ev[1]) / K, world, dev)
    ev[2].record()
    for _ in range(K):
        video()
    ev[3].record()
    torch.cuda.synchronize()
    eager_ms = ev[2].elapsed_time(ev[3]) / K

    # end to end: every chunk's q, k, v copied in from page-locked host memory
    # and its output copied back, as a streamed video would be
    hs = [(q[:, :, f0 * S:(f0 + qf) * S].contiguous().pin_memory(),
           k[:, :, w0 * S:(f0 + qf) * S].contiguous().pin_memory(),
           v[:, :, w0 * S:(f0 + qf) * S].contiguous().pin_memory())
          for (f0, w0, cf, qf, ef) in (R.step_frames(t, F, Tc, To) for t in range(nc))]
    outs_h = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]

    # three streams: copies in, steps, copies out.  Chunk t's step waits for
    # its own inputs only, so chunk t+1's upload overlaps chunk t's step and
    # chunk t-1's download; across videos, an upload into a chunk's buffers
    # waits for the previous video's step on them, and a step waits for the
    # previous download of its output buffer.
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nc)]
    ev_run = [torch.cuda.Event() for _ in range(nc)]
    ev_out = [torch.cuda.Event() for _ in range(nc)]

    def video_e2e(first):
        for t, ((qh, kh, vh), (qc, kc, vc, qf, cf, ef)) in enumerate(zip(hs, slices)):
            with torch.cuda.stream(s_in):
                if not first:
                    s_in.wait_event(ev_run[t])
                qc.copy_(qh, non_blocking=True)
                kc.copy_(kh, non_blocking=True)
                vc.copy_(vh, non_blocking=True)
                ev_in[t].record(s_in)
        with torch.cuda.stream(s_run):
            Sst.zero_()
            zst.zero_()
            for t, ((qc, kc, vc, qf, cf, ef), o) in enumerate(zip(slices, outs)):
                s_run.wait_event(ev_in[t])
                if not first:
                    s_run.wait_event(ev_out[t])
                R.step(qc, kc, vc, Sst, zst, S, qf, cf, ef, out=o, workspace=ws)
                ev_run[t].record(s_run)
        with torch.cuda.stream(s_out):
            for t, (o, oh) in enumerate(zip(outs, outs_h)):
                s_out.wait_event(ev_run[t])
                oh.copy_(o, non_blocking=True)
                ev_out[t].record(s_out)

    cur = torch.cuda.current_stream(dev)
    for x in (s_in, s_run, s_out):
        x.wait_stream(cur)
    video_e2e(True)
    torch.cuda.synchronize()
    Ke = max(3, min(K, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for x in (s_in, s_run, s_out):
        x.wait_event(e0)
    for _ in range(Ke):
        video_e2e(False)
    for x in (s_in, s_run, s_out):
        cur.wait_stream(x)
    e1.record(cur)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, world, dev)
    h2d = sum(t.numel() * t.element_size() for trip in hs for t in trip)
    d2h = sum(t.numel() * t.element_size() for t in outs_h)
    status = R.device_status()
    if status != R.OK:
        raise RuntimeError(f"device status {R.status_string(status)}")
    return dict(ms_step=ms, eager_ms=eager_ms, e2e_ms=e2e_ms, clocks=clk.summary(), h2d=h2d, d2h=d2h,
                launches=K * nc * 4, q=q, k=k, v=v,
                e2e_kind="rehyat_step per chunk with host copies; copies in, steps and copies out on three streams")


def run_compare_full(args):
    """The hybrid against full bidirectional softmax over the same tokens:
    our fused kernel with one chunk covering every frame (pure softmax), and
    torch's scaled_dot_product_attention as a library reference; FLOPs are
    the algorithmic counts of each computation."""
    import torch
    from linear_attention_video_chunk_b200 import inputs
    from linear_attention_video_chunk_b200 import rehyat as R
    dev = torch.device("cuda", 0)
    bf16_peak, _, _, src = peaks()
    B, H, d, F, S = 1, 12, 128, 21, 1560
    q, k, v = (x.to(dev) for x in inputs.make_qkv(B, H, F * S, d, 1, rms_qk=True))
    out = torch.empty_like(q)

    def timed(fn, K=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    rows = []
    for Tc, To in ((F, 0), (1, 0), (1, 1), (2, 1), (3, 0), (3, 1), (3, 2), (5, 2), (7, 1)):
        ws = R.alloc_workspace(R.workspace_bytes(B, H, F, S, d, Tc, To), dev)
        ms = timed(lambda: R.forward(q, k, v, F, S, Tc, To, out=out, workspace=ws))
        w = work(dict(B=B, H=H, d=d, F=F, S_tok=S, T_c=Tc, T_o=To))
        fl = w["attn_flops"] + w["state_flops"]
        rows.append({"T_c": Tc, "T_o": To, "kind": "full softmax (one chunk)" if Tc >= F else "hybrid",
                     "ms": ms, "tflop": fl / 1e12, "tflops_per_s": fl / (ms / 1e3) / 1e12,
                     "frac_of_peak": fl / (ms / 1e3) / 1e12 / bf16_peak})
    sdpa = torch.nn.functional.scaled_dot_product_attention
    ms = timed(lambda: sdpa(q, k, v))
    fl = B * H * 4 * d * (F * S) ** 2
    rows.append({"kind": "torch scaled_dot_product_attention (library, full softmax)", "ms": ms,
                 "tflop": fl / 1e12, "tflops_per_s": fl / (ms / 1e3) / 1e12})
    full = rows[0]["ms"]
    for r in rows:
        r["speedup_vs_full"] = full / r["ms"]
        print(json.dumps({"compare_full": r, "workload": "Wan2.1-1.3B 480p shape",
                          "peak": f"{bf16_peak} TFLOP/s {src}"}), flush=True)


def run_sweep(args):
    """Every (F, T_c, T_o) point of the scaling sweep (B=2, H=12, d=128, 1560
    tokens a frame): the two stages timed apart with CUDA events over at least
    50 iterations (and at least ~1 s of work), SM clocks sampled over the same
    region, and the roofline fraction of each stage.  The linear fit of time
    against F is given for the raw times and for the times scaled to the
    maximum SM clock (time x median MHz / max MHz), so that a clock drop under
    the power cap can be told apart from a growth of the work per frame."""
    import numpy as np
    import torch
    from linear_attention_video_chunk_b200 import inputs
    from linear_attention_video_chunk_b200 import rehyat as R
    dev = torch.device("cuda", 0)
    bf16_peak, bf16_sus, hbm, src = peaks()
    B, H, d, S = 2, 12, 128, 1560
    res = {}
    for F, Tc, To in SWEEP:
        q, k, v = (x.to(dev) for x in inputs.make_qkv(B, H, F * S, d, 100 + len(res), rms_qk=True))
        out = torch.empty_like(q)
        ws = R.alloc_workspace(R.workspace_bytes(B, H, F, S, d, Tc, To), dev)

        def step(e=None):
            if e is not None:
                e[0].record()
            R.forward_states(k, v, F, S, Tc, To, ws)
            if e is not None:
                e[1].record()
            R.forward_attention(q, k, v, F, S, Tc, To, out, ws)
            if e is not None:
                e[2].record()

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        step()
        torch.cuda.synchronize()
        est = max(time.perf_counter() - t0, 1e-4)
        K = int(min(1000, max(50, 1.0 / est)))
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        with ClockSampler(dev) as clk:
            for i in range(K):
                step(ev[i])
            torch.cuda.synchronize()
        ms = ev[0][0].elapsed_time(ev[-1][2]) / K
        st_ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
        at_ms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
        cl = clk.summary()
        scale = (cl["sm_mhz"] / cl["sm_max_mhz"]) if cl["sm_mhz"] and cl["sm_max_mhz"] else float("nan")
        w = work(dict(B=B, H=H, d=d, F=F, S_tok=S, T_c=Tc, T_o=To))
        res[(F, Tc, To)] = (ms, ms * scale)
        print(json.dumps({
            "sweep_point": {"B": B, "H": H, "F": F, "T_c": Tc, "T_o": To}, "steps": K, "ms": ms,
            "ms_at_max_clock": ms * scale, "ms_per_frame": ms / F, "states_ms": st_ms, "attention_ms": at_ms,
            "tokens_per_s": B * F * S / (ms / 1e3),
            "roofline": {"kernel": "hybrid_chunk_attn_kernel", "bound": "tensor",
                         "achieved": w["attn_flops"] / (at_ms / 1e3) / 1e12, "peak": bf16_peak,
                         "unit": "TFLOP/s", "frac": w["attn_flops"] / (at_ms / 1e3) / 1e12 / bf16_peak,
                         "frac_of_sustained": w["attn_flops"] / (at_ms / 1e3) / 1e12 / bf16_sus if bf16_sus else None,
                         "peak_source": f"{src} bf16 dense (burst)"},
            "states_roofline": {"bound": "hbm", "achieved": w["state_bytes"] / (st_ms / 1e3) / 1e9, "peak": hbm,
                                "unit": "GB/s", "frac": w["state_bytes"] / (st_ms / 1e3) / 1e9 / hbm},
            "path_frac": (w["attn_flops"] + w["state_flops"]) / (ms / 1e3) / 1e12 / bf16_peak,
            "clocks": cl}), flush=True)
        del q, k, v, out, ws
        torch.cuda.empty_cache()
    for Tc, To in ((2, 1), (3, 1), (5, 2)):
        Fs = np.array([F for F, a, b in SWEEP if (a, b) == (Tc, To)], dtype=float)
        A = np.stack([Fs, np.ones_like(Fs)], 1)
        fit = {"T_c": Tc, "T_o": To}
        for i, key in ((0, "raw"), (1, "at_max_clock")):
            ts = np.array([res[(F, Tc, To)][i] for F in Fs.astype(int)])
            coef, *_ = np.linalg.lstsq(A, ts, rcond=None)
            r2 = 1 - ((A @ coef - ts) ** 2).sum() / ((ts - ts.mean()) ** 2).sum()
            fit[key] = {"ms_per_frame": coef[0], "intercept_ms": coef[1], "r2": r2,
                        "ms_per_frame_each_F": [round(t / F, 5) for t, F in zip(ts, Fs)]}
        print(json.dumps({"linear_fit": fit}), flush=True)


# --------------------------------------------------------------------------- #
# reference arm: the fp64 oracle on the host cores                             #
# --------------------------------------------------------------------------- #
def run_reference(args):
    """The fp64 oracle, as it stands, on the host cores: the same workload
    (config, heads override, set mode, feature map) as our arm, each step a
    random query-row sample (all heads) sized so the whole run lasts about
    --ref-budget seconds."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from linear_attention_video_chunk_b200 import inputs
    c = dict(CONFIGS[args.config])
    if args.heads:
        c["H"] = args.heads
        c["workload"] += f" (H overridden to {args.heads})"
    B, H, d, F, S = (c[k] for k in ("B", "H", "d", "F", "S_tok"))
    q, k, v = inputs.make_qkv(B, H, F * S, d, c["seed"], rms_qk=True)
    import numpy as np
    import oracle.rehyat_oracle as orc
    feats = {}
    if args.phi == "mlp":
        # the learned map's features of every token, from the same seeded weights
        for which, x in (("q", q), ("k", k)):
            W1, b1, W2, b2 = (t.float().numpy() for t in inputs.make_mlp_weights(H, d, c["seed"], which))
            xs = x.float().numpy()
            feats["phi_" + which] = np.stack([np.stack([orc.phi_mlp(xs[b, h], W1[h], b1[h], W2[h], b2[h])
                                                        for h in range(H)]) for b in range(B)])
        c["workload"] += " (learned phi: 2-layer MLP, degree-2 features)"
    if args.sets != "causal":
        c["workload"] += f" ({args.sets} sets)"
    if args.layout != "bhnd":
        c["workload"] += " ([B, N, H, d] layout)"

    def call(rows):
        orc.oracle_forward(q, k, v, F, S, c["T_c"], c["T_o"], mode=args.sets, rows=rows, **feats)

    N = F * S
    rng = np.random.default_rng(11)
    per_step_budget = max(0.05, args.ref_budget / max(1, args.steps + args.warmup))
    # size each step's row sample from two calibration calls (per-call cost,
    # phi of every key, and per-row cost)
    t0 = time.perf_counter()
    call(np.arange(4))
    t4 = time.perf_counter() - t0
    t0 = time.perf_counter()
    call(np.arange(36))
    t36 = time.perf_counter() - t0
    per_row = max((t36 - t4) / 32, 1e-6)
    fixed = max(t4 - 4 * per_row, 0.0)
    n = int(max(1, min(N, (per_step_budget - fixed) / per_row)))
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(N, n, replace=False))
        t0 = time.perf_counter()
        call(rows)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    val = B * n / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same generator and seed as the GPU arm)",
        "config": config_dict(c, world),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: fp64 explicit-mask oracle on {n} random query rows x all {H} heads"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", choices=tuple(CONFIGS), default="wan13b")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--compare-full", action="store_true", help="hybrid vs full softmax over (T_c, T_o)")
    ap.add_argument("--sets", choices=("causal", "bidirectional"), default="causal")
    ap.add_argument("--layout", choices=("bhnd", "bnhd"), default="bhnd")
    ap.add_argument("--phi", choices=("fixed", "mlp"), default="fixed",
                    help="feature map: fixed 1+elu features, or the learned two-layer MLP")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--heads", type=int, default=0, help="override H (smaller profiling cases)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=150.0,
                    help="seconds of oracle work for the whole --impl reference run")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} with {world} process(es): run N > 1 as "
                 f"python -m torch.distributed.run --nproc-per-node N bench.py --gpus N")
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.compare_full:
        run_compare_full(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
