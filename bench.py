"""Benchmark of the DCNv3 core on B200: GB/s and Gsamples/s, fraction of HBM peak.

A step is one pass of the whole hot path -- forward (offset/mask staging,
softmax, bilinear gather, weighted sum, store) and backward (recompute,
grad_mask, grad_offset, grad_input scatter) -- over one batch of the
InternImage-L stage-1 shape (fp32, N=32, 96x96, C=160 = 10 groups x 16,
3x3, offset_scale 2.0, softmax mask), inputs drawn from the seeded generator.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--no-sweep] [--no-cpu-baseline] [--no-e2e]

Prints ONE JSON line (rank 0).  Multi-GPU runs (torchrun) are independent
replicas, one per GPU, with no data-path collective (weak scaling); the step
time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DCNv3 core fwd/bwd GB/s and Gsamples/s on 1 B200; fraction of HBM peak"
DEFAULT_WORKLOAD = "internimage_l_stage1_fp32_n32_96x96_c160"
SWEEP = ["internimage_l_stage1_bf16_n64_96x96_c160", "internimage_l_stage2_bf16_n64_48x48_c320",
         "internimage_l_stage3_bf16_n64_24x24_c640", "internimage_l_stage4_bf16_n64_12x12_c1280",
         "internimage_l_stage1_fp16_n64_96x96_c160",
         "internimage_l_stage1_k5_bf16_n16_96x96_c160", "internimage_l_stage1_k7_bf16_n16_96x96_c160",
         "internimage_l_stage1_cg8_bf16_n64_96x96_c160", "internimage_l_stage1_cg32_bf16_n64_96x96_c160",
         "dcnv4_hires_bf16_n2_256x256_c192_s1", "dcnv4_hires_bf16_n2_256x256_c192_s2",
         "dcnv4_hires_bf16_n2_256x256_c192_s1_remove_center",
         "internimage_l_stage2_bwd_fp32_n32_48x48_c320",
         "internimage_l_stage2_bwd_bf16_n32_48x48_c320",
         "internimage_l_stage2_bwd_fp16_n32_48x48_c320"]
# The same backward workloads through dcn_core_backward_deterministic.
DETERMINISTIC_SWEEP = ["internimage_l_stage2_bwd_fp32_n32_48x48_c320",
                       "internimage_l_stage2_bwd_bf16_n32_48x48_c320"]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# Offset / mask projections timed next to the sweep: (workload, query channels).
PROJECTION_SWEEP = [("internimage_l_stage1_fp32_n32_96x96_c160", 160),
                    ("internimage_l_stage1_bf16_n64_96x96_c160", 160),
                    ("internimage_l_stage2_bf16_n64_48x48_c320", 320)]
# guide features (depthwise 3x3 + LayerNorm + GELU) on the stage shapes
GUIDE_SWEEP = ["internimage_l_stage1_fp32_n32_96x96_c160", "internimage_l_stage1_bf16_n64_96x96_c160",
               "internimage_l_stage2_bf16_n64_48x48_c320", "internimage_l_stage3_bf16_n64_24x24_c640",
               "internimage_l_stage4_bf16_n64_12x12_c1280"]
L2_BYTES = 126 * 1024 * 1024
# torch dtype of each storage type name
TORCH_DTYPES = {"f32": "float32", "bf16": "bfloat16", "f16": "float16"}


def bf16_peak():
    """Dense bf16 tensor throughput (TFLOP/s): the burst cuBLAS figure of
    MEASURED_PEAKS.json, for a kernel timed on its own."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources of the kernels the bench step launches: every file under csrc/ except
# those that only define kernels the step never runs.
OTHER_KERNEL_SOURCES = ("dcn_guide.cuh", "dcn_guide_projection.cuh", "dcn_projection.cuh")


def step_kernel_sources_sha() -> str:
    """First 16 hex digits of sha256 over the step kernels' sources (sorted)."""
    import hashlib
    csrc = os.path.join(ROOT, "deformable_convolution_core_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(csrc)):
        if f in OTHER_KERNEL_SOURCES:
            continue
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if the
    kernel sources are unchanged since it was taken (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = step_kernel_sources_sha()
    for line in open(path):
        parts = dict(p.split("=", 1) for p in line.split() if "=" in p)
        if parts.get("kernel") == kernel and parts.get("src_sha") == sha:
            return float(parts["bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.mark = 0

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def begin_region(self):
        self.mark = len(self.lines)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = [r.split(", ") for r in self.lines[self.mark:]] or \
               [r.split(", ") for r in self.lines]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------------------

def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings over the process group (the
    identity at one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif args.impl == "ours":
        torch.cuda.set_device(0)
    return world, rank, local


class Step:
    """Device buffers and the launches of one step of a workload."""

    def __init__(self, wl, inputs, backward: bool, deterministic: bool = False):
        import torch
        import deformable_convolution_core_b200 as dcn
        self.dcn = dcn
        self.wl = wl
        self.backward = backward
        self.deterministic = deterministic
        tdt = getattr(torch, TORCH_DTYPES[wl.dtype])
        self.p = dcn.problem_for(wl)
        dev = torch.device("cuda")
        self.x = torch.from_numpy(inputs["x"]).to(dev).to(tdt)
        self.off = torch.from_numpy(inputs["offset"]).to(dev).to(tdt)
        self.mask = torch.from_numpy(inputs["mask"]).to(dev).to(tdt)
        Ho, Wo = dcn.dcn_core_output_hw(self.p)
        self.out = torch.empty((wl.N, Ho, Wo, wl.C), dtype=tdt, device=dev)
        if backward:
            self.gout = torch.from_numpy(inputs["grad_out"]).to(dev).to(tdt)
            self.gx = torch.empty_like(self.x)
            self.goff = torch.empty_like(self.off)
            self.gm = torch.empty_like(self.mask)
            self.ws_bytes = (dcn.dcn_core_backward_deterministic_workspace(self.p)
                             if deterministic else dcn.dcn_core_backward_workspace(self.p))
            self.ws = (torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
                       if self.ws_bytes else None)
        self.stream = torch.cuda.Stream()
        self.sh = self.stream.cuda_stream

    def fwd(self):
        self.dcn.dcn_core_forward(self.p, self.x, self.off, self.mask, self.out, self.sh)

    def bwd(self):
        call = (self.dcn.dcn_core_backward_deterministic if self.deterministic
                else self.dcn.dcn_core_backward)
        call(self.p, self.x, self.off, self.mask, self.gout, self.gx, self.goff, self.gm,
             self.ws, self.ws_bytes, self.sh)

    def run(self):
        if not (self.wl.backward and self.backward):
            self.fwd()
        if self.backward:
            self.bwd()

    def launches_per_step(self):
        # the deterministic backward is three kernels (bound pre-pass, the
        # backward, the rounding pass) after its zero-fill
        bwd = (3 if self.deterministic else 1) if self.backward else 0
        return (0 if (self.wl.backward and self.backward) else 1) + bwd


def timed(step, steps, warmup, barrier=None, ev_kernels=True):
    """Time `steps` steps on the step's stream; also time each launch with
    events on that stream.  Returns (total_ms, fwd_ms_avg, bwd_ms_avg)."""
    import torch
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    s = step.stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fwd_only = not (step.wl.backward and step.backward)
    torch.cuda.nvtx.range_push(f"dcn {step.wl.name}: {steps} timed steps")
    t0.record(s)
    for i in range(steps):
        ev[i][0].record(s)
        if fwd_only:
            step.fwd()
        ev[i][1].record(s)
        if step.backward:
            step.bwd()
        ev[i][2].record(s)
    t1.record(s)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    total = t0.elapsed_time(t1)
    fw = sum(e[0].elapsed_time(e[1]) for e in ev) / steps if fwd_only else 0.0
    bw = sum(e[1].elapsed_time(e[2]) for e in ev) / steps if step.backward else 0.0
    return total, fw, bw


def run_ours(args, world, rank, local):
    import numpy as np
    import torch
    import gen
    from deformable_convolution_core_b200 import build as lib_build

    lib_build.build()
    wl = gen.WORKLOADS[args.workload]
    backward = wl.backward or wl.dtype == "f32"
    inputs = gen.make_inputs(wl, with_grad_out=backward)
    det = bool(args.deterministic and backward)
    step = Step(wl, inputs, backward, deterministic=det)

    barrier = None
    if world > 1:
        import torch.distributed as dist
        barrier = dist.barrier
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    clocks.begin_region()
    total_ms, fwd_ms, bwd_ms = timed(step, args.steps, args.warmup, barrier)
    time.sleep(0.25)
    clock_summary = clocks.summary()
    total_ms, fwd_ms, bwd_ms = max_over_ranks([total_ms, fwd_ms, bwd_ms], "cuda")
    ms_per_step = total_ms / args.steps

    fwd_bytes = wl.forward_bytes() if not wl.backward else 0
    bwd_bytes = wl.backward_bytes() if backward else 0
    step_bytes = step_bytes_of(wl, backward)
    samples = wl.samples * ((0 if wl.backward else 1) + (1 if backward else 0))
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()

    # dominant launch: the longer of forward and backward
    kernels = []
    if fwd_ms > 0:
        tiled = os.environ.get("DCN_CORE_FORWARD") != "direct"
        if tiled and wl.K == 3 and (wl.Cg == 16 or (wl.Cg == 8 and wl.esize == 2)):
            fname = "dcn_forward_tiled_kernel"
        elif tiled and wl.K in (5, 7) and wl.Cg == 16:
            fname = "dcn_forward_tiled_wide_kernel"
        else:
            fname = "dcn_forward_kernel"
        kernels.append((fname, fwd_bytes, fwd_ms))
    if bwd_ms > 0:
        tiled_bwd = (os.environ.get("DCN_CORE_BACKWARD") != "direct" and wl.K == 3
                     and wl.Cg == 16)
        kernels.append(("dcn_backward_tiled_kernel" if tiled_bwd else "dcn_backward_kernel",
                        bwd_bytes, bwd_ms))
    kname, kbytes, kms = max(kernels, key=lambda k: k[2])
    achieved = kbytes / (kms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                # the recorded DRAM bytes are the default step's (its workload, atomic backward)
                "traffic": (recorded_traffic(kname)
                            if args.workload == DEFAULT_WORKLOAD and not det else None),
                "kernel": kname, "peak_source": peak_kind,
                "algorithmic_bytes_per_launch": kbytes, "avg_launch_ms": round(kms, 4)}

    # end to end through the public API: pinned host inputs -> device, step, results -> host
    e2e = None
    if not args.no_e2e and not det:  # the host entry points run the atomic backward
        e2e = run_e2e(step, inputs, args, barrier, world)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic (seeded counter-based generator)",
        "config": workload_config(wl, backward, world, det),
        "gsamples_per_s": round(world * samples / (ms_per_step * 1e-3) / 1e9, 3),
        "breakdown": {"forward": None if fwd_ms == 0 else {
                          "ms": round(fwd_ms, 4),
                          "GB/s": round(fwd_bytes / (fwd_ms * 1e-3) / 1e9, 1),
                          "Gsamples/s": round(wl.samples / (fwd_ms * 1e-3) / 1e9, 2),
                          "frac_of_hbm": round(fwd_bytes / (fwd_ms * 1e-3) / 1e9 / peak, 4),
                          "frac_of_l1_ceiling": round(
                              wl.samples / (fwd_ms * 1e-3) / 1e9 /
                              l1_ceiling_gsamples(wl, clock_summary.get("sm_mhz")), 4)},
                      "backward": None if bwd_ms == 0 else {
                          "ms": round(bwd_ms, 4),
                          "GB/s": round(bwd_bytes / (bwd_ms * 1e-3) / 1e9, 1),
                          "Gsamples/s": round(wl.samples / (bwd_ms * 1e-3) / 1e9, 2),
                          "frac_of_hbm": round(bwd_bytes / (bwd_ms * 1e-3) / 1e9 / peak, 4),
                          **({"u64_adds_G_per_s": round(red_u64_per_launch(wl) / (bwd_ms * 1e-3) / 1e9, 1),
                              "frac_of_l2_red_ceiling": round(
                                  red_u64_per_launch(wl) / (bwd_ms * 1e-3) / 1e9 / L2_RED_U64_G_PER_S, 4),
                              "l2_red_ceiling": L2_RED_U64_CEILING_NOTE,
                              "note": "deterministic: includes the zero-fill, the bound pre-pass "
                                      "and the rounding pass"} if det else
                           {"red_v4_G_per_s": round(red_v4_per_launch(wl) / (bwd_ms * 1e-3) / 1e9, 1),
                            "frac_of_l2_red_ceiling": round(
                                red_v4_per_launch(wl) / (bwd_ms * 1e-3) / 1e9 / L2_RED_V4_G_PER_S, 4),
                            "l2_red_ceiling": L2_RED_CEILING_NOTE,
                            "note": "includes the zero-fill of grad_input"})}},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": step.launches_per_step() * args.steps,
        "clocks": clock_summary,
    }
    if rank == 0 and world == 1 and not args.no_sweep and args.workload == DEFAULT_WORKLOAD:
        result["sweep"] = run_sweep(gen, peak, clocks)
        result["projection"] = run_projection(gen, peak)
        result["guide"] = run_guide(gen, peak)
        result["block_core_path"] = run_block_core_path(gen)
    clocks.stop()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, inputs, backward)
        result["cpu_baseline_all_cores"] = cpu_baseline_all_cores(wl, inputs, backward)
    if "sweep" in result:
        # last on the line, so that a truncated tail still shows it: the
        # InternImage-L stage forwards (bf16, N=64) against the HBM roofline
        # and the on-chip ceiling
        result["stage_forward_fractions"] = {
            name.split("_bf16")[0].replace("internimage_l_", ""): {
                "frac_of_hbm": result["sweep"][name]["frac_of_hbm"],
                "frac_of_l1_ceiling": result["sweep"][name]["frac_of_l1_ceiling"],
                "ms": result["sweep"][name]["ms"]}
            for name in SWEEP if name.startswith("internimage_l_stage") and "_bf16_" in name
            and "_bwd_" not in name}
    del step
    return result


def run_e2e(step, inputs, args, barrier, world):
    """End to end through the public host entry points: every step copies its
    inputs from pinned host memory and its results back into pinned host
    memory.  Two steps are kept in flight on two streams, each with its own
    device buffers and host result buffers (double buffering), so that one
    step's host-to-device copies overlap the previous step's device-to-host
    copies."""
    import torch
    dcn = step.dcn
    wl = step.wl
    tdt = step.x.dtype
    pin = lambda a: torch.from_numpy(a).to(tdt).pin_memory()
    hx, ho, hm = pin(inputs["x"]), pin(inputs["offset"]), pin(inputs["mask"])
    hg = pin(inputs["grad_out"]) if step.backward else None
    steps = [step, Step(wl, inputs, step.backward, step.deterministic)]

    def host_results(st):
        r = {"out": torch.empty(st.out.shape, dtype=tdt).pin_memory()}
        if st.backward:
            for k, t in (("gx", st.gx), ("goff", st.goff), ("gm", st.gm)):
                r[k] = torch.empty(t.shape, dtype=tdt).pin_memory()
        return r
    outs = [host_results(st) for st in steps]
    h2d = (hx.numel() + ho.numel() + hm.numel()) * hx.element_size()
    d2h = outs[0]["out"].numel() * outs[0]["out"].element_size()
    if step.backward:
        h2d += hg.numel() * hg.element_size()
        d2h += sum(outs[0][k].numel() for k in ("gx", "goff", "gm")) * hx.element_size()
    fwd_only = not wl.backward

    def one(st, r):
        s = st.stream
        if fwd_only:
            dcn.dcn_core_forward_host(st.p, hx, ho, hm, r["out"], st.x, st.off, st.mask, st.out,
                                      st.sh)
        else:
            with torch.cuda.stream(s):
                st.x.copy_(hx, non_blocking=True)
                st.off.copy_(ho, non_blocking=True)
                st.mask.copy_(hm, non_blocking=True)
        if st.backward and not st.deterministic:
            # grad_out in and the three gradients out, chunked and overlapped
            dcn.dcn_core_backward_host(st.p, st.x, st.off, st.mask, hg, r["gx"], r["goff"],
                                       r["gm"], st.gout, st.gx, st.goff, st.gm, st.ws,
                                       st.ws_bytes, st.sh)
        elif st.backward:
            with torch.cuda.stream(s):
                st.gout.copy_(hg, non_blocking=True)
            st.bwd()
            with torch.cuda.stream(s):
                r["gx"].copy_(st.gx, non_blocking=True)
                r["goff"].copy_(st.goff, non_blocking=True)
                r["gm"].copy_(st.gm, non_blocking=True)

    n = max(4, min(args.steps, 20))
    for i in range(2):
        one(steps[i], outs[i])
    torch.cuda.synchronize()
    if barrier:
        barrier()
    sa, sb = steps[0].stream, steps[1].stream
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    join = torch.cuda.Event()
    t0.record(sa)
    sb.wait_event(t0)
    for i in range(n):
        one(steps[i % 2], outs[i % 2])
    join.record(sb)
    sa.wait_event(join)
    t1.record(sa)
    torch.cuda.synchronize()
    ms = max_over_ranks([t0.elapsed_time(t1) / n], "cuda")[0]
    step_bytes = (wl.forward_bytes() if fwd_only else 0) + (wl.backward_bytes() if step.backward else 0)
    del steps[1]
    return {"value": round(world * step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms, 3), "steps": n, "in_flight": 2,
            "note": "every step copies its inputs from pinned host memory and its results back; "
                    "two steps in flight on two streams, each with its own buffers"}


def run_projection(gen, peak, launches=20):
    """dcn_core_offset_mask_projection (tcgen05 GEMM) on the stage shapes:
    bytes = query + weight + bias read, offset + mask written; flops = 2 M N K."""
    import torch
    import deformable_convolution_core_b200 as dcn
    tflops_peak, tf_kind = bf16_peak()
    out = {}
    for name, cq in PROJECTION_SWEEP:
        wl = gen.WORKLOADS[name]
        d = gen.make_projection_inputs(wl, cq)
        p = dcn.problem_for(wl)
        tdt = getattr(torch, TORCH_DTYPES[wl.dtype])
        q = torch.from_numpy(d["query"]).cuda().to(torch.bfloat16)
        w = torch.from_numpy(d["weight"]).cuda().to(torch.bfloat16)
        b = torch.from_numpy(d["bias"]).cuda()
        M = wl.N * wl.Ho * wl.Wo
        nout = wl.G * wl.KK * 3
        off = torch.empty((M, wl.G * wl.KK * 2), dtype=tdt, device="cuda")
        msk = torch.empty((M, wl.G * wl.KK), dtype=tdt, device="cuda")
        s = torch.cuda.Stream()
        for _ in range(3):
            dcn.dcn_core_offset_mask_projection(p, q, cq, w, b, off, msk, s)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(launches):
            dcn.dcn_core_offset_mask_projection(p, q, cq, w, b, off, msk, s)
        e1.record(s)
        torch.cuda.synchronize()
        dcn.dcn_core_sync_status(s)
        ms = e0.elapsed_time(e1) / launches
        nbytes = M * cq * 2 + nout * cq * 2 + nout * 4 + M * nout * wl.esize
        flops = 2.0 * M * nout * cq
        gbs = nbytes / (ms * 1e-3) / 1e9
        tfs = flops / (ms * 1e-3) / 1e12
        out[f"{name} Cq={cq}"] = {
            "ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4),
            "TFLOP/s": round(tfs, 1), "frac_of_bf16_tensor": round(tfs / tflops_peak, 4),
            "bound": "hbm" if nbytes / (peak * 1e9) > flops / (tflops_peak * 1e12) else "tensor",
            "MB": round(nbytes / 1e6, 1), "out_dtype": wl.dtype, "tensor_peak_source": tf_kind}
        del q, w, b, off, msk
        torch.cuda.empty_cache()
    return out


# The backward's binding ceiling: vector fp32 reductions into L2.  A
# microbenchmark on this B200 (16 warps per SM, four lanes per random 64-byte
# chunk, four chunks per step, as the grad_input scatter issues them) sustains
# 331 G red.global.add.v4.f32 per second into an L2-resident buffer (8 or
# 32 MB) and 108 G/s into a 1 GB one.
L2_RED_V4_G_PER_S = 331.0
L2_RED_CEILING_NOTE = ("331 G red.global.add.v4.f32/s: microbenchmark, random 64-byte chunks of "
                       "an L2-resident buffer, 16 warps per SM")


# The deterministic backward's: exact 64-bit fixed-point adds, one per channel
# and corner.  The tiled kernel sends a corner's 16 channels as one 128-byte
# bulk reduction from shared memory (cp.reduce.async.bulk .add.u64); the same
# microbenchmark (random 128-byte corners of an L2-resident buffer, 16 warps
# per SM) sustains 798 G such adds per second.  Scalar red.global.add.u64
# (the direct kernel's form) sustains 466 G/s.
L2_RED_U64_G_PER_S = 798.0
L2_RED_U64_CEILING_NOTE = ("798 G 64-bit adds/s: microbenchmark, random 128-byte bulk reductions "
                           "(cp.reduce.async.bulk .add.u64) into an L2-resident buffer, 16 warps per SM")


def red_u64_per_launch(wl):
    """64-bit reductions the deterministic backward issues: four corners x Cg
    channels per sample."""
    return wl.samples * 4 * wl.Cg


def red_v4_per_launch(wl):
    """Vector reductions the atomic backward issues for grad_input: four
    corners x Cg/4 float4s per sample (16 at Cg = 16)."""
    return wl.samples * 4 * (wl.Cg // 4)


NOMINAL_SM_MHZ = 1965.0


def l1_ceiling_gsamples(wl, sm_mhz=None, sms=148):
    """Samples/s (1e9) if every on-chip byte path delivered 128 B per clock
    per SM and a sample needed only its 2x2 footprint (4 * Cg * size bytes),
    at the SM clock sampled while the passes ran (the nominal maximum when no
    sample was taken)."""
    mhz = sm_mhz if sm_mhz else NOMINAL_SM_MHZ
    return sms * 128.0 * mhz * 1e6 / (4.0 * wl.Cg * wl.esize) / 1e9


def run_guide(gen, peak, launches=20):
    """dcn_core_offset_mask_guide (depthwise 3x3 + LayerNorm + GELU, bf16 query
    out) on the stage shapes: bytes = input read + query written (+ the 12 C
    parameter floats).  Each launch is timed alone after an L2 flush (the
    stage-3 and stage-4 inputs fit in L2); the median is reported."""
    import torch
    import deformable_convolution_core_b200 as dcn
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    out = {}
    for name in GUIDE_SWEEP:
        wl = gen.WORKLOADS[name]
        p = dcn.problem_for(wl)
        tdt = getattr(torch, TORCH_DTYPES[wl.dtype])
        x = torch.from_numpy(gen.make_inputs(wl)["x"]).cuda().to(tdt)
        gp = {k: torch.from_numpy(v).cuda() for k, v in gen.make_guide_params(wl).items()}
        q = torch.empty(x.shape, dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.Stream()

        def call():
            dcn.dcn_core_offset_mask_guide(p, x, gp["dw_weight"], gp["dw_bias"], gp["ln_gamma"],
                                           gp["ln_beta"], 1e-6, q, s)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        ts = []
        for _ in range(launches):
            with torch.cuda.stream(s):
                flush.fill_(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            call()
            e1.record(s)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        dcn.dcn_core_sync_status(s)
        ts.sort()
        ms = ts[len(ts) // 2]
        nbytes = x.numel() * x.element_size() + q.numel() * 2 + 12 * wl.C * 4
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4),
                     "MB": round(nbytes / 1e6, 1), "bound": "hbm",
                     "l2": "flushed before every launch"}
        del x, q, gp
        torch.cuda.empty_cache()
    return out


def run_block_core_path(gen, name="internimage_l_stage1_bf16_n64_96x96_c160", reps=20):
    """The DCNv3 block around the core operator, bf16, four launches on one
    stream: guide features (depthwise 3x3 + LayerNorm + GELU) -> offset/mask
    projection (tensor cores) -> core forward -> output_proj (tensor cores,
    C -> C).  Median per-launch CUDA-event times."""
    import numpy as np
    import torch
    import deformable_convolution_core_b200 as dcn
    wl = gen.WORKLOADS[name]
    d = gen.make_inputs(wl)
    pj = gen.make_projection_inputs(wl, wl.C)
    gp = {k: torch.from_numpy(v).cuda() for k, v in gen.make_guide_params(wl).items()}
    p = dcn.problem_for(wl)
    bf = torch.bfloat16
    x = torch.from_numpy(d["x"]).cuda().to(bf)
    q = torch.empty(x.shape, dtype=bf, device="cuda")  # the guide features
    w = torch.from_numpy(pj["weight"]).cuda().to(bf)
    b = torch.from_numpy(pj["bias"]).cuda()
    w_out = (torch.from_numpy(gen.normal(wl.seed, gen.TID_OUT_WEIGHT, (wl.C, wl.C), 0.0,
                                         wl.C ** -0.5)).cuda().to(bf))
    M = wl.N * wl.Ho * wl.Wo
    off = torch.empty((M, wl.G * wl.KK * 2), dtype=bf, device="cuda")
    msk = torch.empty((M, wl.G * wl.KK), dtype=bf, device="cuda")
    core = torch.empty((M, wl.C), dtype=bf, device="cuda")
    y = torch.empty((M, wl.C), dtype=bf, device="cuda")
    s = torch.cuda.Stream()
    stages = [lambda: dcn.dcn_core_offset_mask_guide(p, x, gp["dw_weight"], gp["dw_bias"],
                                                     gp["ln_gamma"], gp["ln_beta"], 1e-6, q, s),
              lambda: dcn.dcn_core_offset_mask_projection(p, q, wl.C, w, b, off, msk, s),
              lambda: dcn.dcn_core_forward(p, x, off, msk, core, s),
              lambda: dcn.dcn_core_linear_bf16(core, M, wl.C, w_out, wl.C, None, y, "bf16", s)]
    for _ in range(3):
        for f in stages:
            f()
    torch.cuda.synchronize()
    k = len(stages)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(k + 1)] for _ in range(reps)]
    for r in range(reps):
        for i, f in enumerate(stages):
            ev[r][i].record(s)
            f()
        ev[r][k].record(s)
    torch.cuda.synchronize()
    dcn.dcn_core_sync_status(s)
    t = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(k)] for e in ev])
    med = np.median(t, axis=0)
    # the same branch with guide and projection in one kernel (the query stays on chip)
    fused = lambda: dcn.dcn_core_offset_mask_guide_projection(
        p, x, gp["dw_weight"], gp["dw_bias"], gp["ln_gamma"], gp["ln_beta"], 1e-6, w, b, off,
        msk, s)
    fstages = [fused] + stages[2:]
    for _ in range(3):
        for f in fstages:
            f()
    torch.cuda.synchronize()
    fk = len(fstages)
    fev = [[torch.cuda.Event(enable_timing=True) for _ in range(fk + 1)] for _ in range(reps)]
    for r in range(reps):
        for i, f in enumerate(fstages):
            fev[r][i].record(s)
            f()
        fev[r][fk].record(s)
    torch.cuda.synchronize()
    dcn.dcn_core_sync_status(s)
    ft = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(fk)] for e in fev])
    fmed = np.median(ft, axis=0)
    total, ftotal = float(np.median(t.sum(axis=1))), float(np.median(ft.sum(axis=1)))
    return {"workload": name, "guide_ms": round(float(med[0]), 4),
            "projection_ms": round(float(med[1]), 4),
            "core_forward_ms": round(float(med[2]), 4),
            "output_proj_ms": round(float(med[3]), 4),
            "total_ms": round(total, 4),
            "Mpixels/s": round(M / (total * 1e-3) / 1e6, 1),
            "fused_guide_projection_ms": round(float(fmed[0]), 4),
            "fused_total_ms": round(ftotal, 4),
            "fused_Mpixels/s": round(M / (ftotal * 1e-3) / 1e6, 1)}


def run_sweep(gen, peak, clocks=None, reps=30, warmup=3):
    """The other workloads' passes, one launch at a time: L2 is flushed (a
    2 x L2 buffer is written) before every timed launch, and the median and
    the 10th / 90th percentiles of the per-launch CUDA-event times are kept.
    `ms_warm_l2` is the median of the same launches run back to back without
    the flush (inputs partly still in L2: not the row's number, a context).
    The on-chip ceiling of each row uses the median SM clock sampled while
    the sweep ran."""
    import numpy as np
    import torch
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    out = {}
    if clocks is not None:
        clocks.begin_region()
    runs = [(name, False) for name in SWEEP] + [(name, True) for name in DETERMINISTIC_SWEEP]
    for name, det in runs:
        wl = gen.WORKLOADS[name]
        inputs = gen.make_inputs(wl, with_grad_out=wl.backward)
        step = Step(wl, inputs, backward=wl.backward, deterministic=det)
        launch = step.bwd if wl.backward else step.fwd
        for _ in range(warmup):
            launch()
        torch.cuda.synchronize()
        times = []
        torch.cuda.nvtx.range_push(f"dcn sweep {name}{' deterministic' if det else ''}")
        with torch.cuda.stream(step.stream):
            for _ in range(reps):
                flush.fill_(1.0)  # evicts the inputs from L2 (not timed)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(step.stream)
                launch()
                e1.record(step.stream)
                times.append((e0, e1))
        # The same launches back to back, without the flush: the inputs the
        # previous launch left in L2 are reused (reported apart, labelled).
        warm = []
        with torch.cuda.stream(step.stream):
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(step.stream)
                launch()
                e1.record(step.stream)
                warm.append((e0, e1))
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        ms_all = np.array([a.elapsed_time(b) for a, b in times])
        ms = float(np.median(ms_all))
        ms_warm = float(np.median([a.elapsed_time(b) for a, b in warm]))
        b = wl.backward_bytes() if wl.backward else wl.forward_bytes()
        gbs = b / (ms * 1e-3) / 1e9
        gsps = wl.samples / (ms * 1e-3) / 1e9
        key = name + (" deterministic" if det else "")
        out[key] = {"pass": ("deterministic backward" if det else "backward") if wl.backward
                    else "forward", "ms": round(ms, 4),
                    "ms_p10": round(float(np.percentile(ms_all, 10)), 4),
                    "ms_p90": round(float(np.percentile(ms_all, 90)), 4),
                    "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4),
                    "Gsamples/s": round(gsps, 2), "frac_of_l1_ceiling": None,
                    "MB": round(b / 1e6, 1), "l2": "flushed before every launch",
                    "ms_warm_l2": round(ms_warm, 4), "_wl": wl}
        if wl.backward:  # the backward's own ceiling: reductions into L2
            reds, peak_red = ((red_u64_per_launch(wl), L2_RED_U64_G_PER_S) if det
                              else (red_v4_per_launch(wl), L2_RED_V4_G_PER_S))
            out[key]["frac_of_l2_red_ceiling"] = round(reds / (ms * 1e-3) / 1e9 / peak_red, 4)
        del step
        torch.cuda.empty_cache()
    del flush
    sm_mhz = clocks.summary().get("sm_mhz") if clocks is not None else None
    for row in out.values():
        row["frac_of_l1_ceiling"] = round(row["Gsamples/s"] / l1_ceiling_gsamples(row.pop("_wl"),
                                                                                 sm_mhz), 4)
    out["l1_ceiling_sm_mhz"] = sm_mhz if sm_mhz else f"nominal {NOMINAL_SM_MHZ}"
    return out


def cpu_baseline_all_cores(wl, inputs, backward):
    """The same oracle on every host core: images split over threads (the
    oracle's C loops run outside the interpreter lock)."""
    import concurrent.futures
    import oracle
    oracle.build()
    kw = oracle.workload_kwargs(wl)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cores = max(1, min(cores, wl.N))
    bounds = [(i * wl.N // cores, (i + 1) * wl.N // cores) for i in range(cores)]

    def work(lo, hi):
        sl = {k: v[lo:hi] for k, v in inputs.items()}
        if not wl.backward:
            oracle.forward(sl["x"], sl["offset"], sl["mask"], **kw)
        if backward:
            oracle.backward(sl["x"], sl["offset"], sl["mask"], sl["grad_out"], **kw)

    with concurrent.futures.ThreadPoolExecutor(max_workers=cores) as pool:
        t0 = time.perf_counter()
        list(pool.map(lambda b: work(*b), bounds))
        dt = time.perf_counter() - t0
    b = (0 if wl.backward else wl.forward_bytes()) + (wl.backward_bytes() if backward else 0)
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"{wl.N} of {wl.N} images of {wl.name} split over {cores} threads"}


def cpu_baseline(wl, inputs, backward, n_images=None):
    """The CPU oracle, as it stands (single-threaded C, fp64), timed on the host."""
    import oracle
    oracle.build()
    kw = oracle.workload_kwargs(wl)
    n = wl.N if n_images is None else n_images
    sl = {k: v[:n] for k, v in inputs.items()}
    t0 = time.perf_counter()
    if not wl.backward:
        oracle.forward(sl["x"], sl["offset"], sl["mask"], **kw)
    if backward:
        oracle.backward(sl["x"], sl["offset"], sl["mask"], sl["grad_out"], **kw)
    dt = time.perf_counter() - t0
    frac = n / wl.N
    b = ((0 if wl.backward else wl.forward_bytes()) + (wl.backward_bytes() if backward else 0)) * frac
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"{n} of {wl.N} images of {wl.name}, "
                      f"{'forward + backward' if backward and not wl.backward else 'one pass'}, "
                      "including the float64 widening of the inputs"}


def step_bytes_of(wl, backward):
    """Compulsory bytes of one step: the forward (unless the workload is a
    backward-only one) and the backward (if the step runs it)."""
    return (wl.forward_bytes() if not wl.backward else 0) + (wl.backward_bytes() if backward else 0)


def workload_config(wl, backward, world, deterministic=False):
    """The `config` object of the JSON line, the same for both arms: the
    workload, its shape, how grad_input is summed and how the timed steps
    treat L2."""
    return {"workload": wl.name + (" fwd+bwd" if backward and not wl.backward else "")
                        + (" (deterministic grad_input)" if deterministic else ""),
            "N": wl.N, "H": wl.H, "W": wl.W, "G": wl.G, "Cg": wl.Cg, "K": wl.K,
            "stride": wl.stride, "offset_scale": wl.offset_scale, "softmax": wl.softmax,
            "remove_center": wl.remove_center, "per_gpu_batch": wl.N,
            "parallelism": f"replicas x{world} (no collective)",
            "l2": f"inputs larger than L2: {step_bytes_of(wl, backward) / 1e6:.0f} MB touched "
                  "per step, no flush between steps"}


def run_reference(args, world, rank):
    """The oracle as the reference arm: rank 0 only, on host cores, each step a
    bounded sample (one image) of the workload."""
    if rank != 0:
        return None
    import gen
    wl = gen.WORKLOADS[args.workload]
    backward = wl.backward or wl.dtype == "f32"
    inputs = gen.make_inputs(wl, n_images=1, with_grad_out=backward)
    for _ in range(min(args.warmup, 1)):
        cpu_baseline(wl, inputs, backward, n_images=1)
    budget_s = 120.0
    t_all = time.perf_counter()
    vals, secs = [], []
    steps = 0
    for _ in range(args.steps):
        r = cpu_baseline(wl, inputs, backward, n_images=1)
        vals.append(r["value"])
        secs.append(r["seconds"])
        steps += 1
        if time.perf_counter() - t_all > budget_s:
            break
    value = statistics.median(vals)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * statistics.median(secs), 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded counter-based generator)",
            "config": workload_config(wl, backward, world, bool(args.deterministic and backward)),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"1 of {wl.N} images of {wl.name} per step"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="time dcn_core_backward_deterministic as the step's backward")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res = run_ours(args, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
