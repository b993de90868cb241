#!/usr/bin/env python
"""Throughput of the exact RoPE-attention loss + closed-form gradient (forward + backward).

One step = rope_attn_fwd (with the loss) followed by rope_attn_loss_bwd reusing the
forward's workspace, over one batch of the workload: every step of the hot path
(RoPE table, projections + RoPE, attention forward with the loss epilogue, the
tile-wise closed-form backward, inverse RoPE + weight gradients, loss reduction).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

With N > 1 it runs one process per GPU under torch.distributed.run (started by the driver, or
by bench.py itself when WORLD_SIZE is not set; a WORLD_SIZE other than N is an error); every rank runs
its own copy of the workload (the (batch, head) instances are independent, so the work
shards with no collective on the data path) and the reported value is the work of all
ranks divided by the slowest rank's device time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, flop_count, make_inputs, pair_count  # noqa: E402

DEFAULT_WORKLOAD = "b2_h32_n8192_d128_bf16_causal"
METRIC = "RoPE-attention loss+grad fwd+bwd TFLOP/s, % of B200 BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
L2_BYTES = 126 * 2 ** 20
# a timed region at least this long runs under the power cap: its kernels are compared with
# the sustained bf16 peak (a seconds-long loop), shorter ones with the burst peak
SUSTAINED_REGION_MS = 500.0
# B200: 148 SMs x 128 fp32 lanes x 2 flop per FMA at the maximum SM clock
FP32_SIMT_LANES = 148 * 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=250)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-input-grads", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="the backward's fixed-order (bitwise repeatable) mode")
    ap.add_argument("--approx", action="store_true",
                    help="also time the near-linear approximate method (rope_attn_approx_step)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w, n_gpus):
    return {"workload": w.name, "B": w.B, "H": w.H, "n": w.n, "d": w.d, "dtype": w.dtype,
            "causal": w.causal, "rope_base": w.rope_base, "global_batch": w.B * n_gpus,
            "seq_len": w.n, "parallelism": f"replicas{n_gpus}" if n_gpus > 1 else "single",
            "l2": "inputs larger than L2 (%.0f MB of inputs per step vs 126 MB L2)"
                  % (4 * w.B * w.H * w.n * w.d * (2 if w.dtype == "bf16" else 4) / 1e6)}


# ---------------------------------------------------------------------------------------
# multi-rank aggregation (host logic; exercised on CPU with gloo in the tests)
# ---------------------------------------------------------------------------------------
def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Slowest rank's time: every rank contributes its own device-timed milliseconds."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    x = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return float(x.item())


def whole_job_tflops(flops_per_rank_step: float, steps: int, world: int, ms_max: float) -> float:
    """Work of all ranks (weak scaling: each rank runs its own copy) over the slowest time."""
    return world * flops_per_rank_step * steps / (ms_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------------------
# clocks sampled with nvidia-smi during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.gpu_id is not None:
            cmd += ["-i", str(self.gpu_id)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.out.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        hi = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(hi), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


def _gpu_uuid(dev):
    import torch
    try:
        u = torch.cuda.get_device_properties(dev).uuid
        return "GPU-" + str(u)
    except Exception:
        return None


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from loss_closed_form_b200 import rope_attn as ra

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, seed=w.seed + rank)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host = {k: torch.from_numpy(inp[k]).to(tdt).pin_memory()
            for k in ("A1", "A2", "A3", "E", "WQ", "WK", "WV")}
    host["pos"] = torch.from_numpy(inp["pos"]).pin_memory()
    del inp
    t = {k: v.to(dev) for k, v in host.items()}
    det = bool(getattr(args, "deterministic", False))
    m = ra.RopeAttention(t["A1"], t["A2"], t["A3"], t["WQ"], t["WK"], t["WV"], t["E"],
                         t["pos"], w.causal, w.rope_base, deterministic=det)
    stream = torch.cuda.current_stream(dev)
    flops = flop_count(w)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        m.step()
    torch.cuda.synchronize(dev)
    st = ra.last_error()
    if st != ra.RA_OK:
        raise RuntimeError(f"kernel status after warm-up: {ra.status_string(st)}")

    # the dominant kernel: most device time in one more step with events around every launch
    ra.profile_read()
    ra.profile_enable(True)
    m.step()
    torch.cuda.synchronize(dev)
    top_name = max(ra.profile_read().items(), key=lambda kv: kv[1][0])[0]
    ra.profile_enable(False)

    # ---- device-timed region: inputs resident in HBM -------------------------------------
    # CUDA events bracket the dominant kernel's launches only: an event pair between two
    # dependent launches leaves the GPU idle for a few microseconds, which the step would pay.
    clocks = ClockSampler(_gpu_uuid(dev)) if rank == 0 else None
    if clocks:
        clocks.start()
    ra.launch_count()
    ra.profile_only(top_name)
    ra.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        m.step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    launches = ra.launch_count()
    top_rec = ra.profile_read()[top_name]
    ra.profile_enable(False)
    ra.profile_only(None)
    clk = clocks.stop() if clocks else None
    ms = e0.elapsed_time(e1)
    st = ra.last_error()
    if st != ra.RA_OK:
        raise RuntimeError(f"kernel status after timing: {ra.status_string(st)}")
    ms_max = max_over_ranks(ms, world, dev)

    # ---- per-kernel breakdown: the same steps again, events around every launch ----------
    ra.profile_read()
    ra.profile_enable(True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        m.step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    per_kernel = ra.profile_read()
    ra.profile_enable(False)
    ms_events = max_over_ranks(e0.elapsed_time(e1), world, dev)
    st = ra.last_error()
    if st != ra.RA_OK:
        raise RuntimeError(f"kernel status after the per-kernel pass: {ra.status_string(st)}")

    # ---- end to end: pinned host inputs -> device, step, loss + dW back to the host -----
    # Every step copies its own inputs from pinned host memory and reads its loss and weight
    # gradients back.  Two input slots let the next step's host-to-device copy (copy stream)
    # overlap the current step's compute, as a training loop that prefetches would.
    e2e = None
    if not args.no_e2e:
        slots = [(t, m)]
        t2 = {k: torch.empty_like(v) for k, v in t.items()}
        m2 = ra.RopeAttention(t2["A1"], t2["A2"], t2["A3"], t2["WQ"], t2["WK"], t2["WV"],
                              t2["E"], t2["pos"], w.causal, w.rope_base, deterministic=det)
        slots.append((t2, m2))
        out_host = [{"loss": torch.empty((), dtype=torch.float32).pin_memory(),
                     "dWQ": torch.empty_like(m.dWQ, device="cpu").pin_memory(),
                     "dWK": torch.empty_like(m.dWK, device="cpu").pin_memory(),
                     "dWV": torch.empty_like(m.dWV, device="cpu").pin_memory()} for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(v.numel() * v.element_size() for v in out_host[0].values())
        copy_stream = torch.cuda.Stream(dev)
        ready = [torch.cuda.Event() for _ in range(2)]
        free = [torch.cuda.Event() for _ in range(2)]
        for ev in free:
            ev.record(stream)

        def e2e_steps(k_steps):
            for k in range(k_steps):
                s = k % 2
                tk, mk = slots[s]
                with torch.cuda.stream(copy_stream):
                    copy_stream.wait_event(free[s])
                    for key, v in host.items():
                        tk[key].copy_(v, non_blocking=True)
                    ready[s].record(copy_stream)
                stream.wait_event(ready[s])
                mk.step(stream)
                oh = out_host[s]
                oh["loss"].copy_(mk.loss, non_blocking=True)
                oh["dWQ"].copy_(mk.dWQ, non_blocking=True)
                oh["dWK"].copy_(mk.dWK, non_blocking=True)
                oh["dWV"].copy_(mk.dWV, non_blocking=True)
                free[s].record(stream)

        e2e_steps(2)
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        copy_stream.wait_event(e0)
        e2e_steps(args.steps)
        stream.wait_stream(copy_stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)
        if not all(math.isfinite(float(o["loss"])) for o in out_host):
            raise RuntimeError("non-finite loss in the end-to-end run")
        st = ra.last_error()
        if st != ra.RA_OK:
            raise RuntimeError(f"kernel status after the end-to-end run: {ra.status_string(st)}")
        e2e = {"value": round(whole_job_tflops(flops, args.steps, world, ms_e2e), 3),
               "unit": "TFLOP/s", "ms_per_step": round(ms_e2e / args.steps, 4),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipelining": "next step's host-to-device copy overlaps this step's compute"}

    # ---- the input-gradient row (rope_attn_loss_bwd_inputs), timed outside the step -----
    # The metric's step is the forward and the weight-gradient backward; the extra products
    # dA = dX W^T are measured on their own: the backward with input gradients is run a few
    # times with per-kernel events and the input-gradient kernel's average launch is kept.
    input_grads = None
    if not args.no_input_grads:
        m.forward()
        m.backward_inputs(True)
        torch.cuda.synchronize(dev)
        ra.profile_read()
        ra.profile_enable(True)
        reps = 5
        for _ in range(reps):
            m.forward()
            m.backward_inputs(True)
        torch.cuda.synchronize(dev)
        prof_ig = ra.profile_read()
        ra.profile_enable(False)
        st = ra.last_error()
        if st != ra.RA_OK:
            raise RuntimeError(f"kernel status after the input-gradient run: {ra.status_string(st)}")
        for kname in ("input_grads_tc", "input_grads_simt"):
            if kname in prof_ig:
                ms_ig, n_ig = prof_ig[kname]
                input_grads = {"kernel": kname, "avg_launch_ms": round(ms_ig / max(1, n_ig), 4)}

    # ---- the near-linear approximate method (rope_attn_approx_step), timed on its own -----
    approx = None
    if args.approx:
        prob = m.prob
        f32 = dict(dtype=torch.float32, device=dev)
        ao = {"O": torch.empty_like(m.O), "loss": torch.zeros((), **f32),
              **{k: torch.empty_like(m.dWQ) for k in ("dWQ", "dWK", "dWV")}}
        aws = torch.empty(ra.approx_workspace_bytes(prob), dtype=torch.uint8, device=dev)

        def astep():
            ra.approx_step(prob, ao["O"], ao["loss"], ao["dWQ"], ao["dWK"], ao["dWV"], aws)
        astep()
        torch.cuda.synchronize(dev)
        reps = 3
        ra.profile_read()
        ra.profile_enable(True)
        e0.record(stream)
        for _ in range(reps):
            astep()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        prof_ap = ra.profile_read()
        ra.profile_enable(False)
        st = ra.last_error()
        if st != ra.RA_OK:
            raise RuntimeError(f"kernel status after the approximate run: {ra.status_string(st)}")
        approx = {"ms_per_step": round(e0.elapsed_time(e1) / reps, 3),
                  "exact_ms_per_step": round(ms_max / args.steps, 4),
                  "workspace_bytes": int(aws.numel()), "degree": 1,
                  "kernels": {k: round(v[0] / reps, 3) for k, v in
                              sorted(prof_ap.items(), key=lambda kv: -kv[1][0])}}
        del aws

    if rank != 0:
        return None

    # ---- roofline of the dominant kernel ------------------------------------------------
    pk, src = peaks()
    top_ms, top_n = top_rec
    avg_ms = top_ms / max(1, top_n)
    sustained = ms_max >= SUSTAINED_REGION_MS
    roof = roofline(w, top_name, avg_ms, pk, src, sustained, det)
    value = whole_job_tflops(flops, args.steps, world, ms_max)
    total_kernel_ms = sum(v[0] for v in per_kernel.values())
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": dict(workload_config(w, world), **({"deterministic": True} if det else {})),
        "frac_of_bf16_peak": round(value / world / pk["bf16_tflops"], 4),
        "tokens_per_s": round(world * w.B * w.n * args.steps / (ms_max * 1e-3), 1),
        "roofline": roof,
        "kernels": {k: {"ms_per_step": round(v[0] / args.steps, 4),
                        "launches": v[1], "share": round(v[0] / total_kernel_ms, 4)}
                    for k, v in sorted(per_kernel.items(), key=lambda kv: -kv[1][0])},
        "kernel_timing": {
            "timed_region": f"events around {top_name} only",
            "breakdown": "a second pass of the same steps with events around every launch",
            "ms_per_step_with_events": round(ms_events / args.steps, 4)},
        "kernel_rooflines": {k: kernel_roofline(w, k, v[0] / max(1, v[1]), pk, sustained)
                             for k, v in per_kernel.items()
                             if kernel_roofline(w, k, 1.0, pk) is not None},
        "gpu_launches": int(launches),
        "clocks": clk,
        "e2e": e2e,
        "peaks_source": src,
    }
    if approx is not None:
        line["approx"] = approx
    if input_grads is not None:
        line["input_grads"] = dict(input_grads, **(kernel_roofline(
            w, input_grads["kernel"], input_grads["avg_launch_ms"], pk, sustained) or {}))
    return line


def bf16_peak(pk, sustained):
    """The bf16 tensor peak a kernel is compared with: the sustained figure (a seconds-long
    loop under the power cap) for kernels timed inside a long region, else the burst one."""
    if sustained and pk.get("bf16_tflops_sustained"):
        return pk["bf16_tflops_sustained"], "sustained"
    return pk["bf16_tflops"], "burst"


def kernel_roofline(w, kname, avg_ms, pk, sustained=False):
    """Per-kernel roofline of every tensor-core / memory-bound kernel on the path: algorithmic
    flops (tensor) or bytes (HBM) of one launch over its CUDA-event-timed average duration."""
    BH, n, d = w.B * w.H, w.n, w.d
    P = pair_count(n, w.causal)
    act = BH * n * d                     # elements of one [B][H][n][d] tensor
    tensor = {"attn_bwd_tc": 10.0 * d * P * BH, "attn_fwd_tc": 4.0 * d * P * BH}
    # bytes: proj reads A1..A3 and writes Q~, K~, V (bf16); dq_unrotate reads fp32 dQ~ and
    # writes bf16 dQ; dw_tc reads A1..A3 and dQ, dK, dV (bf16); the input gradients read
    # dQ, dK, dV and write dA1..dA3 (bf16).  Tables and weights are L2-resident extras.
    hbm = {"proj_rope_tc": 12.0 * act, "dq_unrotate": 6.0 * act, "dw_tc": 12.0 * act,
           "input_grads_tc": 12.0 * act}
    if kname in tensor:
        ach = tensor[kname] / (avg_ms * 1e-3) / 1e12
        peak, kind = bf16_peak(pk, sustained)
        return {"bound": "tensor", "achieved": round(ach, 3), "peak": peak, "peak_kind": kind,
                "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                "frac_of_burst": round(ach / pk["bf16_tflops"], 4),
                "avg_launch_ms": round(avg_ms, 4)}
    if kname in hbm:
        ach = hbm[kname] / (avg_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4), "avg_launch_ms": round(avg_ms, 4)}
    return None


def roofline(w, kname, avg_ms, pk, src, sustained=False, deterministic=False):
    """Algorithmic work of one launch of the dominant kernel over its measured duration.
    The DRAM traffic is the captured one for the default mode at the bench workload."""
    BH = w.B * w.H
    P = pair_count(w.n, w.causal)
    d, n = w.d, w.n
    tensor_kernels = {"attn_bwd_tc": 10.0 * d * P * BH, "attn_fwd_tc": 4.0 * d * P * BH}
    simt_kernels = {"attn_bwd_simt": 10.0 * d * P * BH, "attn_fwd_simt": 4.0 * d * P * BH,
                    "proj_rope_simt": 6.0 * n * d * d * BH, "dw_partial_simt": 6.0 * n * d * d * BH}
    traffic = (measured_traffic(kname) if w.name == DEFAULT_WORKLOAD and not deterministic
               else None)
    if kname in tensor_kernels:
        flop = tensor_kernels[kname]
        peak, kind = bf16_peak(pk, sustained)
        ach = flop / (avg_ms * 1e-3) / 1e12
        return {"kernel": kname, "bound": "tensor", "achieved": round(ach, 3), "peak": peak,
                "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": traffic,
                "peak_source": f"{src} bf16 dense ({kind}: the timed region is "
                               f"{'at least' if sustained else 'under'} "
                               f"{SUSTAINED_REGION_MS / 1000:.1f} s)",
                "frac_of_burst": round(ach / pk["bf16_tflops"], 4),
                "algorithmic_per_launch": flop, "avg_launch_ms": round(avg_ms, 4)}
    if kname in simt_kernels:
        flop = simt_kernels[kname]
        peak = FP32_SIMT_LANES * 2 * pk.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        ach = flop / (avg_ms * 1e-3) / 1e12
        return {"kernel": kname, "bound": "alu", "achieved": round(ach, 3),
                "peak": round(peak, 2), "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                "traffic": traffic,
                "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 flop x max SM clock",
                "algorithmic_per_launch": flop, "avg_launch_ms": round(avg_ms, 4)}
    # memory-bound kernels: algorithmic bytes are not modelled here
    return {"kernel": kname, "bound": "hbm", "achieved": None, "peak": pk["hbm_gbs"],
            "unit": "GB/s", "frac": None, "traffic": traffic, "avg_launch_ms": round(avg_ms, 4)}


# source files that define each tensor-core kernel; a committed traffic figure counts only
# while these files are unchanged since its ncu capture
KERNEL_SOURCES = {
    "attn_bwd_tc": ("tc_attn_bwd.cuh", "tc_ptx.cuh", "common.cuh"),
    "attn_fwd_tc": ("tc_attn_fwd.cuh", "tc_ptx.cuh", "common.cuh"),
}


def kernel_source_sha(kname):
    import hashlib
    files = KERNEL_SOURCES.get(kname)
    if not files:
        return None
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "loss_closed_form_b200", "csrc")
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kname):
    """DRAM bytes per launch from profiles/traffic.json, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(kname)
    if not ent or ent.get("workload") is None:
        return None
    if ent.get("source_sha") != kernel_source_sha(kname):
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------------------
# the fp64 oracle on the host cores (reference arm and CPU baseline)
# ---------------------------------------------------------------------------------------
def oracle_sample_time(w, instances, seed=0):
    """Run the oracle on `instances` (b, h) instances of workload w; return (seconds, flops)."""
    import oracle
    one = w.with_sizes(B=1, H=1)
    inp = make_inputs(one, seed=seed)
    t0 = time.perf_counter()
    for _ in range(instances):
        oracle.forward_backward(inp, w.causal, w.rope_base)
    dt = time.perf_counter() - t0
    return dt, flop_count(one) * instances


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(w, budget_s=12.0):
    dt, fl = oracle_sample_time(w, 1)
    k = max(1, min(64, int(budget_s / max(dt, 1e-3))))
    if k > 1:
        dt2, fl2 = oracle_sample_time(w, k)
        dt, fl, inst = dt + dt2, fl + fl2, k + 1
    else:
        inst = 1
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": host_cores(),
            "kind": "oracle",
            "sample": f"{inst} (b,h) instance(s) of {w.name} (n={w.n}, d={w.d}, "
                      f"causal={w.causal}), fp64 NumPy, {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    one = w.with_sizes(B=1, H=1)
    # each step: the oracle on a bounded sample of the workload (whole (b,h) instances)
    dt1, _ = oracle_sample_time(w, 1)
    per_step = max(1, min(4, int(4.0 / max(dt1, 1e-3))))
    import oracle
    inp = make_inputs(one)
    times = []
    for i in range(max(3, args.warmup) + args.steps):
        t0 = time.perf_counter()
        for _ in range(per_step):
            oracle.forward_backward(inp, w.causal, w.rope_base)
        if i >= max(3, args.warmup):
            times.append(time.perf_counter() - t0)
    fl = flop_count(one) * per_step
    total = sum(times)
    value = fl * len(times) / total / 1e12
    sample = (f"{per_step} (b,h) instance(s) of {w.name} per step (n={w.n}, d={w.d}, "
              f"causal={w.causal}), fp64 NumPy oracle")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": round(1e3 * total / len(times), 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world), "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": host_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_plan(gpus: int, env, argv, port=None):
    """How to run `bench.py --gpus gpus`: None when this process is already the right rank
    (one GPU, or started by torch.distributed.run with a matching world size), else the
    torch.distributed.run command that starts one rank per GPU on this node.  A world size
    that disagrees with --gpus is an error, not something to run."""
    if gpus < 1:
        raise ValueError(f"--gpus must be >= 1, got {gpus}")
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            raise ValueError(f"launched with WORLD_SIZE={world} but --gpus {gpus}")
        return None
    if gpus == 1:
        return None
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr=127.0.0.1",
            f"--master-port={port if port is not None else _free_port()}",
            os.path.join(ROOT, "bench.py"), *argv]


def main():
    args = parse()
    cmd = launch_plan(args.gpus, os.environ, sys.argv[1:])
    if cmd is not None:
        # one rank per GPU: the ranks print the JSON line (rank 0) and this process relays
        # their exit status
        sys.exit(subprocess.run(cmd, cwd=ROOT).returncode)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(WORKLOADS[args.workload])
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
