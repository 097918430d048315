"""Benchmark of the SDM (Sparse Delta Memory) prefill hot path on B200.

One step = one fresh prefill of the mid-size workload (B=2 sequences, H=4 heads, T=4096
tokens, d_k=128, n=256 sub-keys per half -> N=65,536 slots, d_v=128, k=W=R=32, bf16
q/k/v, fp32 memory): state reset, product-key scoring of the keys (write slots) and the
queries (read slots), the index-only plan and the recurrence row pass.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]

Under torchrun (N > 1) every rank runs its own independent batch (weak scaling, no
collective on the data path); the timed region is bracketed by a barrier and a device
synchronisation, and the reported time is the maximum over ranks.  Rank 0 prints one
JSON line.  `--impl reference` times the CPU oracle on the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SDM prefill tokens·heads/sec and achieved HBM GB/s (% of roofline), config 2"
UNIT = "tokens·heads/s"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2

# DRAM traffic per launch of the recurrence row pass from an ncu capture (bytes), keyed by
# the hash of the kernel sources it was taken with; None when not yet measured for the
# current sources.  Filled by hand from the capture of the row pass on the mid-size workload
# (dram__bytes_read.sum + dram__bytes_write.sum of one launch).
MEASURED_TRAFFIC = {
    # dram read 728.71 MB + write 405.78 MB, taken after the plan's walk moved its occurrence
    # words in 16-byte pieces (the row pass itself unchanged)
    "8251cb32fecc1d0b": 1_134_489_856,
}


def kernel_source_hash() -> str:
    """Hash of the sources that define the recurrence row-pass kernel."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_state_linear_score_b200", "csrc")
    for name in ("common.cuh", "plan.cuh", "recur.cuh", "tc_ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------ workload helpers ---

def workload(name: str):
    import sdm_synth as S
    return S.WORKLOADS[name]


def describe(wl) -> str:
    return (f"{wl.name}: B={wl.B} H={wl.H} T={wl.T} d_k={wl.d_k} n={wl.n_sub} N={wl.N} "
            f"d_v={wl.d_v} k={wl.k_half} W={wl.W} R={wl.R} q/k/v={wl.x_dtype}")


def units_per_step(wl) -> int:
    """tokens x heads processed by one step on one GPU."""
    return wl.B * wl.H * wl.T


def bytes_per_token_head(wl) -> dict:
    """Algorithmic HBM bytes per token.head (no re-reads, no plan records)."""
    xb = 2 if wl.x_dtype == "bf16" else 4
    vb = 2 if wl.v_dtype == "bf16" else 4
    rows = (2 * wl.W + wl.R) * wl.d_v * 4          # W gathers + W scatters + R gathers, fp32 rows
    scoring_io = 2 * wl.d_k * xb + (wl.W + wl.R) * 8  # read q, k; write idx + weights
    recur_io = (wl.W + wl.R) * 8 + wl.d_v * vb + 8 + wl.d_v * 4  # read idx+w, v, alpha+beta; write out
    return {"rows": rows, "scoring_io": scoring_io, "recur_io": recur_io,
            "recurrence_kernel": rows + recur_io, "step": rows + scoring_io + recur_io}


def scoring_flops_per_token_head(wl) -> int:
    return 2 * 2 * wl.n_sub * wl.hd * 2  # two roles x two halves x n x h MACs x 2


def rank_seed(wl, rank: int) -> int:
    """Each rank draws an independent batch of sequences (weak scaling)."""
    return wl.seed + 7919 * rank


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# --------------------------------------------------------------- clocks ---

class ClockSampler:
    """Polls SM clocks and clock-event (throttle) reasons through NVML in a background
    thread while the timed region runs (read-only queries; no setting is changed)."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self._nv = None

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
            self._h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM))
        except Exception as e:  # NVML missing: report it instead of clocks
            self._nv = None
            self.error = repr(e)
            return
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, attr in self.REASONS.items():
                    if bits & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self) -> dict:
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": ["nvml unavailable: " + getattr(self, "error", "")]}
        self._stop.set()
        if self._t:
            self._t.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------- distributed ---

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device) -> float:
    """Maximum of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- GPU arm ---

def run_gpu(args, wl, world, rank, local):
    import torch
    import torch.distributed as dist

    import sdm_synth as S
    import sparse_state_linear_score_b200 as sdm

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    stream = torch.cuda.current_stream()

    inp = S.generate(wl, device=device, seed=rank_seed(wl, rank))
    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                 wl.v_dtype)
    st = sdm.State(d, inp["M0"])
    sel = sdm.selection_buffers(d, device)
    widx, ww, ridx, rw = sel
    out = torch.empty((wl.B, wl.H, wl.T, wl.d_v), dtype=torch.float32, device=device)
    ws = sdm.workspace(d, device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def step(ev=None):
        # ev: (start, after_scoring, before_run, end) events or None
        if ev:
            ev[0].record(stream)
        sdm.state_reset(d, st)
        sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"], (widx, ww, ridx, rw))
        if ev:
            ev[1].record(stream)
        sdm.forward_plan(d, inp["alpha"], inp["beta"], widx, ww, ridx, rw, st, ws)
        if ev:
            ev[2].record(stream)
        sdm.forward_run(d, inp["v"], inp["beta"], widx, ww, ridx, rw, st, out, ws)
        if ev:
            ev[3].record(stream)

    warm = max(3, args.warmup)
    for _ in range(warm):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert sdm.device_error() == 0, "device error during warm-up"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(device.index if "CUDA_VISIBLE_DEVICES" not in os.environ else
                          int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[device.index]))
    clocks.start()
    barrier(device)
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.zero_()  # L2 flush between timed steps, outside the step's events
        step(evs[k])
    torch.cuda.synchronize()
    barrier(device)
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    score_ms = [e[0].elapsed_time(e[1]) for e in evs]
    plan_ms = [e[1].elapsed_time(e[2]) for e in evs]
    run_ms = [e[2].elapsed_time(e[3]) for e in evs]
    total_ms = reduce_max(sum(step_ms), device)
    # reset, score (both roles), plan_local, plan_prefix, plan_pack, run (the per-slot chunk masks
    # fit this workload, so plan_fe and plan_walk are not launched)
    launches_per_step = 6

    # memory-utilisation diagnostics of the write weights (after the timed steps)
    diag = None
    if rank == 0:
        sdm.weight_stats(sel[1])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            g = sdm.weight_stats(sel[1])
        e1.record(stream)
        torch.cuda.synchronize()
        dms = e0.elapsed_time(e1) / 5
        rows = sel[1].numel() // wl.W
        diag = {"kernels": "weight_stats_rows + weight_stats_summary", "rows": rows, "K": wl.W,
                "ms": dms, "mean_eff": float(g["mean_eff"]),
                "quant_eff_p10_p50_p90": [float(x) for x in g["quant"]]}

    # output side of the layer on this step's read output: RMS-norm, swish gate and the
    # head-mixing projection (d_model = 4*H*n) on the tensor cores
    layer = None
    if rank == 0:
        dm = 4 * wl.H * wl.n_sub
        gen = torch.Generator(device=device).manual_seed(wl.seed + 17)
        gate = torch.randn(wl.B, wl.T, wl.H * wl.d_v, device=device, generator=gen).to(torch.bfloat16)
        wn = torch.ones(wl.d_v, device=device)
        Wo_t = (torch.randn(dm, wl.H * wl.d_v, device=device, generator=gen) /
                (wl.H * wl.d_v) ** 0.5).to(torch.bfloat16)
        yb = torch.empty(wl.B, wl.T, dm, device=device)
        lws = torch.empty(max(16, wl.B * wl.T * wl.H * wl.d_v * 2), dtype=torch.uint8, device=device)
        A = torch.randn(wl.B * wl.T, wl.H * wl.d_v, device=device, generator=gen).to(torch.bfloat16)
        Cg = torch.empty(wl.B * wl.T, dm, device=device)
        for _ in range(3):
            sdm.layer_out(d, out, gate, wn, Wo_t, y=yb, ws=lws)
            sdm.gemm_bf16(A, Wo_t, Cg)
        torch.cuda.synchronize()
        res = {}
        for name, fn in (("layer_out", lambda: sdm.layer_out(d, out, gate, wn, Wo_t, y=yb, ws=lws)),
                         ("gemm", lambda: sdm.gemm_bf16(A, Wo_t, Cg))):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(10):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) / 10
        # input side: x [B,T,dm] -> q, k, v, g, alpha, beta (one GEMM with K = dm)
        hs = 2 * wl.d_k + 2 * wl.d_v + 2
        x = torch.randn(wl.B, wl.T, dm, device=device, generator=gen).to(torch.bfloat16)
        Win_t = (torch.randn(wl.H * hs, dm, device=device, generator=gen) / dm ** 0.5).to(torch.bfloat16)
        A_log = torch.zeros(wl.H, device=device)
        dtb = torch.zeros(wl.H, device=device)
        lin = sdm.layer_in(d, x, Win_t, A_log, dtb)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            sdm.layer_in(d, x, Win_t, A_log, dtb, out=lin)
        e1.record(stream)
        torch.cuda.synchronize()
        res["layer_in"] = e0.elapsed_time(e1) / 10
        # the input projection's GEMM alone (x [B*T, dm] x Win^T -> P [B*T, H*hs] fp32)
        x2 = x.view(wl.B * wl.T, dm)
        Pg = torch.empty(wl.B * wl.T, wl.H * hs, device=device)
        sdm.gemm_bf16(x2, Win_t, Pg)
        e0.record(stream)
        for _ in range(10):
            sdm.gemm_bf16(x2, Win_t, Pg)
        e1.record(stream)
        torch.cuda.synchronize()
        res["gemm_in"] = e0.elapsed_time(e1) / 10
        del Pg
        # the output side's RMS-norm and gate fused into the row pass (its read): the row pass
        # with the epilogue, then the projection alone
        abuf = torch.empty(wl.B, wl.T, wl.H * wl.d_v, dtype=torch.bfloat16, device=device)
        gms = []
        for k in range(6):
            sdm.state_reset(d, st)
            sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"], sel)
            sdm.forward_plan(d, inp["alpha"], inp["beta"], widx, ww, ridx, rw, st, ws)
            e0.record(stream)
            sdm.forward_run_gated(d, inp["v"], inp["beta"], widx, ww, ridx, rw, st, gate, wn,
                                  1e-6, out=out, a=abuf, ws=ws)
            e1.record(stream)
            torch.cuda.synchronize()
            if k > 0:
                gms.append(e0.elapsed_time(e1))
        res["run_gated"] = statistics.mean(gms)
        flops = 2.0 * wl.B * wl.T * wl.H * wl.d_v * dm
        tf = flops / (res["gemm"] / 1e3) / 1e12
        tf_in = 2.0 * wl.B * wl.T * wl.H * hs * dm / (res["layer_in"] / 1e3) / 1e12
        tf_gin = 2.0 * wl.B * wl.T * wl.H * hs * dm / (res["gemm_in"] / 1e3) / 1e12
        pk = measured_peaks()["bf16_tflops"]
        st_ms = statistics.mean(step_ms)
        layer = {"d_model": dm, "layer_in_ms": res["layer_in"], "layer_out_ms": res["layer_out"],
                 "layer_forward_ms": res["layer_in"] + st_ms + res["layer_out"],
                 "layer_forward_tokens_per_s": wl.B * wl.T /
                 ((res["layer_in"] + st_ms + res["layer_out"]) / 1e3),
                 "gemm_out": {"M": wl.B * wl.T, "K": wl.H * wl.d_v, "N": dm, "ms": res["gemm"],
                              "tflops": tf, "frac_of_bf16_peak": tf / pk},
                 "fused_into_read": {
                     "run_gated_ms": res["run_gated"], "run_ms": statistics.mean(run_ms),
                     "epilogue_ms": res["run_gated"] - statistics.mean(run_ms),
                     "layer_out_ms": res["run_gated"] - statistics.mean(run_ms) + res["gemm"],
                     "note": "sdm_forward_run_gated: the RMS-norm and gate by the last column "
                             "slice to finish each chunk; then the projection alone"},
                 "gemm_in": {"M": wl.B * wl.T, "K": dm, "N": wl.H * hs, "ms": res["gemm_in"],
                             "tflops": tf_gin, "frac_of_bf16_peak": tf_gin / pk},
                 "gemm_in_with_split": {"M": wl.B * wl.T, "K": dm, "N": wl.H * hs,
                                        "ms": res["layer_in"], "tflops": tf_in,
                                        "frac_of_bf16_peak": tf_in / pk},
                 "note": "bf16 x bf16 -> fp32 on tcgen05 (persistent, warp-specialised: TMA "
                         "producer, MMA issuer, 4 epilogue warps, 4-stage ring, two TMEM "
                         "accumulators); 10 back-to-back calls, no L2 flush (the fp32 outputs "
                         "exceed L2); peak = measured burst bf16; layer_forward = layer_in + "
                         "the timed step + layer_out"}

    # end to end through the public API with host buffers
    e2e = run_e2e(args, wl, d, inp, st, sel, out, ws, device, sdm)
    errs = sdm.device_error()

    # the touched-slots decay variant of the same step, and the decode workload, on rank 0
    touched = run_touched(wl, inp, device, sdm) if rank == 0 else None
    bwd = run_backward(wl, inp, sel, device, sdm) if rank == 0 else None
    dec = run_decode(device, sdm) if rank == 0 and not args.no_decode else None
    extra = {}
    if rank == 0 and args.workloads:
        del inp, st, sel, widx, ww, ridx, rw, out, ws
        torch.cuda.empty_cache()
        for name in [x for x in args.workloads.split(",") if x]:
            extra[name] = run_workload(name, device, sdm,
                                       cpu_seconds=0.0 if args.no_cpu_baseline else 10.0)

    if world > 1:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    if rank != 0:
        return None

    units = units_per_step(wl) * world
    peaks = measured_peaks()
    bpt = bytes_per_token_head(wl)
    run_avg_s = statistics.mean(run_ms) / 1e3
    run_bytes = bpt["recurrence_kernel"] * units_per_step(wl)
    achieved = run_bytes / run_avg_s / 1e9
    step_avg_s = statistics.mean(step_ms) / 1e3
    step_gbs = bpt["step"] * units_per_step(wl) / step_avg_s / 1e9
    score_tflops = (scoring_flops_per_token_head(wl) * units_per_step(wl) /
                    (statistics.mean(score_ms) / 1e3) / 1e12)
    traffic = MEASURED_TRAFFIC.get(kernel_source_hash())
    line = {
        "metric": METRIC,
        "value": units * args.steps / (total_ms / 1e3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": warm,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; shapes and distributions of the mid-size prefill workload)",
        "config": {"workload": describe(wl), "inputs": "bf16 q/k/v and sub-keys, fp32 gates",
                   "state": "fp32 rows, fp64 stamps, reset every step",
                   "l2": "flushed between timed steps (256 MB write outside the step events)",
                   "parallelism": f"dp{world} (independent sequences per rank)"},
        "roofline": {"bound": "hbm", "kernel": "recur_run_kernel (sdm_forward_run)",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": peaks["source"] + " (burst copy)",
                     "algorithmic_bytes_per_launch": run_bytes},
        "step_roofline": {"achieved_gbs": step_gbs, "frac": step_gbs / peaks["hbm_gbs"],
                          "bytes_per_token_head": bpt["step"]},
        "stages_ms": {"reset_and_scoring": statistics.mean(score_ms),
                      "plan": statistics.mean(plan_ms), "run": statistics.mean(run_ms)},
        "scoring": {"tflops": score_tflops, "frac_of_bf16_peak": score_tflops / peaks["bf16_tflops"]},
        "e2e": e2e,
        "diagnostics": diag,
        "layer_out": layer,
        "decode": dec,
        "workloads": extra,
        "touched_decay": touched,
        "backward": bwd,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "device_errors": errs,
    }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    return line


def run_workload(name: str, device, sdm, steps: int = 5, warm: int = 3,
                 cpu_seconds: float = 10.0) -> dict:
    """Another prefill workload at full size on one GPU: the same timed step as the headline
    line (state reset, both scorings in one launch, plan, row pass), `steps` timed steps with
    the L2 flushed between them, each stage timed by CUDA events; then a sampled CPU oracle
    rate on a token prefix of one or two sequences (the full workloads hold 8-34 GB of memory
    tables, and the oracle's rate per token.head does not depend on the number of
    sequences)."""
    import torch

    import sdm_synth as S
    wl = S.WORKLOADS[name]
    stream = torch.cuda.current_stream()
    inp = S.generate(wl, device=device)
    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                 wl.v_dtype)
    st = sdm.State(d, inp["M0"])
    sel = sdm.selection_buffers(d, device)
    widx, ww, ridx, rw = sel
    out = torch.empty((wl.B, wl.H, wl.T, wl.d_v), dtype=torch.float32, device=device)
    ws = sdm.workspace(d, device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        sdm.state_reset(d, st)
        sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"], sel)
        if ev:
            ev[1].record(stream)
        sdm.forward_plan(d, inp["alpha"], inp["beta"], widx, ww, ridx, rw, st, ws)
        if ev:
            ev[2].record(stream)
        sdm.forward_run(d, inp["v"], inp["beta"], widx, ww, ridx, rw, st, out, ws)
        if ev:
            ev[3].record(stream)

    for _ in range(warm):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        step(evs[k])
    torch.cuda.synchronize()
    errs = sdm.device_error()
    step_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in evs)
    score_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    plan_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    run_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    units = units_per_step(wl)
    bpt = bytes_per_token_head(wl)
    peak = measured_peaks()["hbm_gbs"]
    step_gbs = bpt["step"] * units / (step_ms / 1e3) / 1e9
    run_gbs = bpt["recurrence_kernel"] * units / (run_ms / 1e3) / 1e9
    flops = scoring_flops_per_token_head(wl) * units
    res = {"workload": describe(wl), "steps_timed": steps, "ms_per_step": step_ms,
           "token_heads_per_s": units / (step_ms / 1e3),
           "stages_ms": {"reset_and_scoring": score_ms, "plan": plan_ms, "run": run_ms},
           "step_roofline": {"bytes_per_token_head": bpt["step"], "achieved_gbs": step_gbs,
                             "peak": peak, "frac": step_gbs / peak,
                             "roofline_ms": bpt["step"] * units / (peak * 1e9) * 1e3},
           "row_pass": {"algorithmic_bytes": bpt["recurrence_kernel"] * units,
                        "achieved_gbs": run_gbs, "frac": run_gbs / peak},
           "scoring": {"rows": 2 * units, "ms": score_ms,
                       "tflops": flops / (score_ms / 1e3) / 1e12,
                       "path": "tensor cores" if sdm.score_path(d, wl.W) == sdm.SCORE_TC
                       else "CUDA cores"},
           "l2": "flushed between timed steps", "device_errors": errs}
    del inp, st, sel, out, ws, flush
    torch.cuda.empty_cache()
    if cpu_seconds > 0:
        samp = wl.scaled(B=1, H=min(wl.H, 2))
        cb = cpu_baseline(samp, seconds=cpu_seconds)
        cb["sample"] = cb["sample"] + f"; the {wl.name} workload has {wl.B * wl.H} sequences"
        cb["kind"] = "oracle (sampled; rate per token·head extrapolated to the workload)"
        res["cpu_baseline"] = cb
    return res


def run_gemm_only(device, sdm, steps: int = 10, warm: int = 3) -> dict:
    """The layer's two projections (the mid workload's shapes) on their own: the input side's
    GEMM [B*T, d_model] x [H*hs, d_model]^T and the output side's [B*T, H*d_v] x
    [d_model, H*d_v]^T, bf16 in, fp32 out, each timed over `steps` back-to-back calls."""
    import torch

    import sdm_synth as S
    wl = S.MID
    dm = 4 * wl.H * wl.n_sub
    hs = 2 * wl.d_k + 2 * wl.d_v + 2
    gen = torch.Generator(device=device).manual_seed(11)
    res = {}
    pk = measured_peaks()["bf16_tflops"]
    for name, (M, N, K) in (("gemm_in", (wl.B * wl.T, wl.H * hs, dm)),
                            ("gemm_out", (wl.B * wl.T, dm, wl.H * wl.d_v))):
        A = torch.randn(M, K, device=device, generator=gen).to(torch.bfloat16)
        Bt = torch.randn(N, K, device=device, generator=gen).to(torch.bfloat16)
        C = torch.empty(M, N, device=device)
        for _ in range(warm):
            sdm.gemm_bf16(A, Bt, C)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            sdm.gemm_bf16(A, Bt, C)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        tf = 2.0 * M * N * K / (ms / 1e3) / 1e12
        res[name] = {"M": M, "N": N, "K": K, "ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / pk}
        del A, Bt, C
    res["device_errors"] = sdm.device_error()
    return res


def run_score_only(name: str, device, sdm, tokens: int | None = None, steps: int = 5,
                   warm: int = 3) -> dict:
    """Both roles' scoring of one workload (`sdm_score_qk`) on its own: `tokens` replaces the
    workload's T (same d_k, n, k and value distributions), so that a profiler capture of the
    scorer holds a few hundred MB instead of the full workload.  L2 flushed between calls."""
    import torch

    import sdm_synth as S
    wl = S.WORKLOADS[name]
    if tokens:
        wl = wl.scaled(T=tokens, decode_steps=0)
    inp = S.generate(wl, device=device, with_m0=False)
    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                 wl.v_dtype)
    sel = sdm.selection_buffers(d, device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warm):
        flush.zero_()
        sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"], sel)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for e in evs:
        flush.zero_()
        e[0].record(stream)
        sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"], sel)
        e[1].record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    units = units_per_step(wl)
    flops = scoring_flops_per_token_head(wl) * units
    path = {sdm.SCORE_TC: "tensor cores (score_pk_kernel)", sdm.SCORE_ROWS: "row scorer",
            sdm.SCORE_WARP: "one warp per row"}[sdm.score_path(d, wl.W)]
    return {"workload": describe(wl), "calls_timed": steps, "ms": ms, "path": path,
            "rows_per_s": 2 * units / (ms / 1e3),
            "tflops": flops / (ms / 1e3) / 1e12,
            "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / measured_peaks()["bf16_tflops"],
            "device_errors": sdm.device_error()}


def run_decode(device, sdm, steps: int = 64, warm: int = 3, n_sub: int | None = None,
               d_v: int | None = None) -> dict:
    """The decode workload at full size: a 512-token seeded prefill of every (b,h), then
    single-token steps (sdm_decode_step: one scoring launch for both roles and one
    recurrence launch each).  `steps` steps are timed as issued from Python one call at a
    time, and the next `steps` as one CUDA graph of those calls (how a serving loop issues
    them; the headline figure).  The 34 GB state is far larger than L2, and every step
    gathers new random rows of it."""
    import torch

    import sdm_synth as S

    wl = S.DECODE.scaled(decode_steps=warm + 2 * steps)
    if n_sub is not None:  # a smaller table (and state), for captures under a profiler
        wl = wl.scaled(n_sub=n_sub)
    if d_v is not None:  # narrower rows: a smaller state, the same scoring launches
        wl = wl.scaled(d_v=d_v)
    inp = S.generate(wl, device=device)
    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                 wl.v_dtype)
    dd = sdm.Dims(wl.B, wl.H, 1, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                  wl.v_dtype)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    sl = lambda x: x[:, :, :wl.T].contiguous()
    sdm.prefill(d, sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["alpha"]), sl(inp["beta"]),
                inp["skw"], inp["skr"], st)
    qd, kd, vd = (S.decode_layout(inp[k], wl.T) for k in ("q", "k", "v"))
    ad, bd = (S.decode_layout(inp[k], wl.T) for k in ("alpha", "beta"))
    sel = sdm.selection_buffers(dd, device)
    out = torch.empty((wl.B, wl.H, wl.d_v), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    for s in range(warm):
        sdm.decode_step(dd, qd[s], kd[s], vd[s], ad[s], bd[s], inp["skw"], inp["skr"], st,
                        sel=sel, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(warm, warm + steps):
        sdm.decode_step(dd, qd[s], kd[s], vd[s], ad[s], bd[s], inp["skw"], inp["skr"], st,
                        sel=sel, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    us_eager = e0.elapsed_time(e1) * 1e3 / steps
    # the next `steps` tokens as one graph (captured on a side stream, replayed once, timed)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for s in range(warm + steps, warm + 2 * steps):
                sdm.decode_step(dd, qd[s], kd[s], vd[s], ad[s], bd[s], inp["skw"], inp["skr"], st,
                                sel=sel, out=out)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / steps
    del g
    errs = sdm.device_error()
    fused = sdm.decode_path(dd) == sdm.DECODE_FUSED
    rows = wl.B * wl.H
    bpt = bytes_per_token_head(wl)
    step_bytes = (bpt["step"] + (2 * wl.W + wl.R) * 8) * rows  # + stamp reads and writes
    gbs = step_bytes / (us / 1e6) / 1e9
    peak = measured_peaks()["hbm_gbs"]
    res = {"workload": f"decode: B={wl.B} H={wl.H} d_k={wl.d_k} n={wl.n_sub} N={wl.N} "
                       f"d_v={wl.d_v} k={wl.k_half} W={wl.W} R={wl.R} after a {wl.T}-token prefill",
           "steps_timed": steps, "us_per_step": us, "token_heads_per_s": rows / (us / 1e6),
           "us_per_step_issued_one_call_at_a_time": us_eager,
           "gpu_launches_per_step": 1 if fused else 2,
           "path": "one launch (scoring and recurrence steps in clusters of two CTAs)" if fused
                   else "scoring launch + recurrence launch",
           "roofline": {"bound": "hbm", "algorithmic_bytes_per_step": step_bytes,
                        "achieved_gbs": gbs, "peak": peak, "frac": gbs / peak},
           "note": "state 34 GB (fp32 rows) >> L2; each step scores new tokens, so its gathers "
                   "miss L2", "device_errors": errs}
    del inp, st, qd, kd, vd, ad, bd, sel, out
    torch.cuda.empty_cache()
    return res


def run_touched(wl, inp, device, sdm, steps: int = 10, warm: int = 3) -> dict:
    """The same prefill step with touched-slots decay (alpha scales only each token's write
    slots): reset, both scorings, plan, row pass, timed per stage with the L2 flushed
    between steps."""
    import torch

    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                 wl.v_dtype, decay="touched")
    st = sdm.State(d, inp["M0"])
    widx, ww, ridx, rw = sdm.selection_buffers(d, device)
    out = torch.empty((wl.B, wl.H, wl.T, wl.d_v), dtype=torch.float32, device=device)
    ws = sdm.workspace(d, device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        sdm.state_reset(d, st)
        sdm.score_qk(d, inp["q"], inp["k"], inp["skw"], inp["skr"], (widx, ww, ridx, rw))
        if ev:
            ev[1].record(stream)
        sdm.forward_plan(d, inp["alpha"], inp["beta"], widx, ww, ridx, rw, st, ws)
        if ev:
            ev[2].record(stream)
        sdm.forward_run(d, inp["v"], inp["beta"], widx, ww, ridx, rw, st, out, ws)
        if ev:
            ev[3].record(stream)

    for _ in range(warm):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        step(evs[k])
    torch.cuda.synchronize()
    errs = sdm.device_error()
    ms = [statistics.mean(e[a].elapsed_time(e[b]) for e in evs) for a, b in ((0, 3), (0, 1), (1, 2), (2, 3))]
    units = units_per_step(wl)
    run_bytes = bytes_per_token_head(wl)["recurrence_kernel"] * units
    gbs = run_bytes / (ms[3] / 1e3) / 1e9
    peak = measured_peaks()["hbm_gbs"]
    res = {"workload": describe(wl) + ", decay: write slots only", "steps_timed": steps,
           "ms_per_step": ms[0], "token_heads_per_s": units / (ms[0] / 1e3),
           "stages_ms": {"reset_and_scoring": ms[1], "plan": ms[2], "run": ms[3]},
           "row_pass": {"achieved_gbs": gbs, "frac": gbs / peak}, "device_errors": errs}
    del st, out, ws, flush
    torch.cuda.empty_cache()
    return res


def run_backward(wl, inp, sel, device, sdm, reps: int = 2) -> dict:
    """Backward of the recurrence over the whole prefill call (sdm_backward: in-place replay
    with the write-slot log, then the reverse sweep that restores the state), for the step's
    selections and a seeded output gradient, timed with CUDA events."""
    import torch

    d = sdm.Dims(wl.B, wl.H, wl.T, wl.d_k, wl.n_sub, wl.d_v, wl.k_half, wl.W, wl.R, wl.x_dtype,
                 wl.v_dtype)
    st = sdm.State(d, inp["M0"])
    sdm.state_reset(d, st)
    gen = torch.Generator(device=device).manual_seed(wl.seed + 29)
    dout = torch.randn(wl.B, wl.H, wl.T, wl.d_v, device=device, generator=gen)
    ws = torch.empty(max(16, sdm.backward_workspace_bytes(d)), dtype=torch.uint8, device=device)
    widx, ww, ridx, rw = sel
    args = (inp["v"], inp["alpha"], inp["beta"], widx, ww, ridx, rw)
    grads = sdm.backward(d, *args, st, dout, ws=ws)  # warm-up (also the first allocation)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        sdm.backward(d, *args, st, dout, ws=ws, grads=grads)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    # the gradient through both scorings (keys with dww, queries with drw)
    sb = lambda: (sdm.score_backward(d, inp["k"], inp["skw"], wl.W, widx, ww, grads["dww"]),
                  sdm.score_backward(d, inp["q"], inp["skr"], wl.R, ridx, rw, grads["drw"]))
    sb()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        sb()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_score = e0.elapsed_time(e1) / reps
    errs = sdm.device_error()
    units = units_per_step(wl)
    # per token.head: replay 3W rows (gather, log, store); sweep 3R (M, dM in, dM out) and 5W
    # (M_t, log, dM in, dM out, restore) rows of d_v fp32, plus the dense gradient once
    rows = (8 * wl.W + 3 * wl.R) * wl.d_v * 4
    total = rows * units + wl.B * wl.H * wl.N * wl.d_v * 4
    gbs = total / (ms / 1e3) / 1e9
    peak = measured_peaks()["hbm_gbs"]
    res = {"workload": describe(wl) + ", backward of the recurrence (selections fixed)",
           "ms": ms, "token_heads_per_s": units / (ms / 1e3),
           "scoring_backward_ms": ms_score,
           "roofline": {"bound": "hbm", "algorithmic_bytes": total, "achieved_gbs": gbs,
                        "peak": peak, "frac": gbs / peak},
           "note": "tokens one at a time per sequence, one warp per 4-column slice of d_v",
           "device_errors": errs}
    del st, ws, grads, dout
    torch.cuda.empty_cache()
    return res


def run_e2e(args, wl, d, inp, st, sel, out, ws, device, sdm):
    """Same metric through sdm.prefill with pinned host inputs copied in and the output
    copied out inside the timed region, every step.  The copies of step i+1's inputs and of
    step i's output run on their own streams while step i (or i+1) computes, as a serving
    loop would overlap them: inputs and outputs are double-buffered on the device, and
    events order every reuse of a buffer."""
    import torch
    names = ("q", "k", "v", "alpha", "beta")
    host = {n: inp[n].cpu().pin_memory() for n in names}
    dev = [{n: torch.empty_like(inp[n]) for n in names} for _ in range(2)]
    outs = [out, torch.empty_like(out)]
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    comp = torch.cuda.current_stream()
    s_in = torch.cuda.Stream()
    s_out = torch.cuda.Stream()
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = out_h[0].numel() * out_h[0].element_size()
    ev = lambda: torch.cuda.Event()
    in_ready = [ev(), ev()]   # inputs of buffer p copied
    in_free = [ev(), ev()]    # step using input buffer p done
    out_done = [ev(), ev()]   # step writing output buffer p done
    out_free = [ev(), ev()]   # output buffer p copied to the host
    for p in range(2):
        in_free[p].record(comp)
        out_free[p].record(comp)

    def copy_in(i):
        p = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(in_free[p])
            for n in names:
                dev[p][n].copy_(host[n], non_blocking=True)
            in_ready[p].record(s_in)

    def compute(i):
        p = i % 2
        comp.wait_event(in_ready[p])
        comp.wait_event(out_free[p])
        sdm.state_reset(d, st)
        sdm.prefill(d, dev[p]["q"], dev[p]["k"], dev[p]["v"], dev[p]["alpha"],
                    dev[p]["beta"], inp["skw"], inp["skr"], st, sel=sel, out=outs[p], ws=ws)
        in_free[p].record(comp)
        out_done[p].record(comp)

    def copy_out(i):
        p = i % 2
        with torch.cuda.stream(s_out):
            s_out.wait_event(out_done[p])
            out_h[p].copy_(outs[p], non_blocking=True)
            out_free[p].record(s_out)

    def run(steps):
        copy_in(0)
        for i in range(steps):
            if i + 1 < steps:
                copy_in(i + 1)
            compute(i)
            copy_out(i)
        comp.wait_stream(s_out)

    run(3)
    torch.cuda.synchronize()
    steps = max(1, args.steps)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    t0.record(comp)
    s_in.wait_stream(comp)  # the first copy starts inside the timed region
    run(steps)
    t1.record(comp)
    torch.cuda.synchronize()
    barrier(device)
    ms = reduce_max(t0.elapsed_time(t1), device)
    world = dist_world()
    return {"value": units_per_step(wl) * world * steps / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / steps, "overlap": "copies of step i+1 in / step i out overlap compute"}


def dist_world() -> int:
    import torch.distributed as dist
    return dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1


# ------------------------------------------------------------ CPU oracle arm ---

def cpu_baseline(wl, seconds: float = 15.0, seed: int | None = None) -> dict:
    """The CPU oracle (fp64 C, OpenMP over sequences) timed on this host on a bounded
    sample of the same workload: token prefixes of B*H sequences, product-key scoring of
    both roles and the lazy recurrence from M0."""
    import numpy as np

    import oracle
    import sdm_synth as S
    orc = oracle.default()
    cores = orc.max_threads()
    pairs = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    # calibrate on a short prefix
    T_cal = min(wl.T, 64)
    small = S.generate(wl.scaled(T=T_cal), seed=seed)
    arr = {k: v.double().numpy() for k, v in small.items()}
    t0 = time.perf_counter()
    orc.prefill_pairs(arr["q"], arr["k"], arr["v"], arr["alpha"], arr["beta"], arr["skw"],
                      arr["skr"], arr["M0"], wl.k_half, wl.W, wl.R, pairs, nthreads=cores)
    cal = time.perf_counter() - t0
    per_token = cal / T_cal
    T_s = int(max(T_cal, min(wl.T, seconds / max(per_token, 1e-9))))
    samp = S.generate(wl.scaled(T=T_s), seed=seed)
    arr = {k: v.double().numpy() for k, v in samp.items()}
    t0 = time.perf_counter()
    orc.prefill_pairs(arr["q"], arr["k"], arr["v"], arr["alpha"], arr["beta"], arr["skw"],
                      arr["skr"], arr["M0"], wl.k_half, wl.W, wl.R, pairs, nthreads=cores)
    el = time.perf_counter() - t0
    units = len(pairs) * T_s
    return {"value": units / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {T_s} of {wl.T} tokens of all {len(pairs)} (b,h) sequences "
                      f"({units} token.heads, {el:.1f} s, fp64, OpenMP over sequences)"}


def run_reference(args, wl, world, rank):
    """--impl reference: the CPU oracle as it stands, on rank 0 only.  Each step is the whole
    workload (every token of every sequence: product-key scoring of both roles and the lazy
    recurrence from M0) when that takes at most a minute on this host, else a token prefix of
    every sequence, said in `sample`."""
    if rank != 0:
        return None
    import oracle
    import sdm_synth as S
    orc = oracle.default()
    cores = orc.max_threads()
    pairs = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    cal = cpu_baseline(wl, seconds=1.0)  # also the warm-up
    full_s = wl.B * wl.H * wl.T / cal["value"]
    T_s = wl.T if full_s <= 60.0 else max(1, int(wl.T * 60.0 / full_s))
    samp = S.generate(wl.scaled(T=T_s))
    arr = {k: v.double().numpy() for k, v in samp.items()}

    def step():
        orc.prefill_pairs(arr["q"], arr["k"], arr["v"], arr["alpha"], arr["beta"], arr["skw"],
                          arr["skr"], arr["M0"], wl.k_half, wl.W, wl.R, pairs, nthreads=cores)

    for _ in range(max(0, min(args.warmup, 1))):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    el = sum(times)
    units = len(pairs) * T_s
    value = units * len(times) / el
    sample = (f"the whole workload, all {wl.T} tokens of all {len(pairs)} (b,h) sequences "
              f"({units} token.heads per step)" if T_s == wl.T else
              f"first {T_s} of {wl.T} tokens of all {len(pairs)} (b,h) sequences "
              f"({units} token.heads per step)") + ", fp64, OpenMP over sequences"
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * el / max(1, len(times)),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": f"synthetic (seeded; shapes and distributions of the {describe(wl).split(':')[0]} "
                "workload)",
        "config": {"workload": describe(wl), "inputs": "bf16-rounded q/k/v and sub-keys, upcast to fp64",
                   "parallelism": "CPU host cores (OpenMP over sequences)",
                   "tokens_per_step": units},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sdm", "reference"], default="sdm")
    ap.add_argument("--workload", default="mid_prefill")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workloads", default="headline_prefill,long_context",
                    help="other prefill workloads measured after the timed step (rank 0), "
                         "comma-separated; empty for none")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode-workload measurement (rank 0)")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode workload (--steps timed steps after --warmup) and "
                         "print its object")
    ap.add_argument("--decode-n-sub", type=int, default=None,
                    help="sub-keys per half for --decode-only (default: the workload's 256)")
    ap.add_argument("--decode-d-v", type=int, default=None,
                    help="row width for --decode-only (default: the workload's 128)")
    ap.add_argument("--score-only", default=None, metavar="WORKLOAD",
                    help="run only both roles' scoring of WORKLOAD (--steps timed calls after "
                         "--warmup) and print its object")
    ap.add_argument("--score-tokens", type=int, default=None,
                    help="tokens per sequence for --score-only (default: the workload's T)")
    ap.add_argument("--gemm-only", action="store_true",
                    help="run only the layer's two projection GEMMs (--steps timed calls each) "
                         "and print their object")
    args = ap.parse_args(argv)
    if args.gemm_only:
        import torch

        import sparse_state_linear_score_b200 as sdm
        print(json.dumps({"gemm": run_gemm_only(torch.device("cuda", 0), sdm, steps=args.steps,
                                                warm=max(3, args.warmup))}), flush=True)
        return
    if args.score_only:
        import torch

        import sparse_state_linear_score_b200 as sdm
        res = run_score_only(args.score_only, torch.device("cuda", 0), sdm,
                             tokens=args.score_tokens, steps=args.steps,
                             warm=max(3, args.warmup))
        print(json.dumps({"scoring": res}), flush=True)
        return
    if args.decode_only:
        import torch

        import sparse_state_linear_score_b200 as sdm
        res = run_decode(torch.device("cuda", 0), sdm, steps=args.steps,
                         warm=max(3, args.warmup), n_sub=args.decode_n_sub,
                         d_v=args.decode_d_v)
        print(json.dumps({"decode": res}), flush=True)
        return
    world, rank, local = dist_env()
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    wl = workload(args.workload)
    if args.impl == "reference":
        line = run_reference(args, wl, world, rank)
    else:
        line = run_gpu(args, wl, world, rank, local)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
