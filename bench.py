"""Benchmark of the dynamic block-sparse attention hot path on B200.

One step = the whole path on one synthetic 720p-shaped batch (B=1, H=40,
d=128, L=75600, keep=0.1, INT8/FP8): block-mean pooling, scoring + top-k,
INT8/E4M3 quantisation, sparse attention.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank runs its own independent batch (the
path shards by problem; no data-path collective), timing is the max over
ranks, value = effective TFLOP/s of all ranks together.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "720p"
MODE = "int8fp8"
METRIC = "block-sparse attn ms & effective TFLOPS (720p grid, 40\u00d7128, keep 10%)"


def metric_for(workload, H, d, keep):
    """The headline metric's name; other workloads get the same form."""
    if workload == WORKLOAD and H == 40 and d == 128 and abs(keep - 0.1) < 1e-12:
        return METRIC
    return f"block-sparse attn ms & effective TFLOPS ({workload} grid, {H}\u00d7{d}, keep {keep:g})"


# The attention kernel each mode launches and the sources it is built from.
_CSRC = os.path.join(ROOT, "video_dit_dynamic_token_b200", "csrc")
ATTN_KERNEL = {"int8fp8": ("sparse_attn_paired_kernel", ("attn.cuh", "attn_paired.cuh")),
               "bf16": ("sparse_attn_kernel", ("attn.cuh",))}
# DRAM bytes (read + write) of one full-size attention launch, from an ncu
# capture, keyed by the SHA-256 of the kernel sources it was taken on: when
# they change the key no longer matches and the line reports null.
ATTN_DRAM_BYTES = {   # {sha256 of the mode's sources: (bytes per full 720p launch, how it was taken)}
    "879e6bb5ea0b0ae55928d3858cae030564a0462f2718dfe262a4a06f3fecd646":
        (5 * (236.927744e6 + 126.024448e6),
         "ncu dram__bytes_read.sum + dram__bytes_write.sum of the 8-head 720p launch x 5 (traffic grows with the "
         "heads)"),
    "247dd9af093a5ac2507a8ddc7203d69c4d870f132de6b26845a01fc7a98d16dc":
        (5 * (471.053312e6 + 141.109760e6),
         "ncu dram__bytes_read.sum + dram__bytes_write.sum of the 8-head 720p BF16 launch x 5 (traffic grows with "
         "the heads)"),
}

# Dense MACs per clock per SM of one tcgen05 kind::i8 / kind::f8f6f4 M=128 MMA
# stream, measured with back-to-back MMAs on this chip (8170 of 8192).
TC_8BIT_MAC_PER_CLK_SM = 8192
PEAKS_8BIT = os.path.join(ROOT, "MEASURED_PEAKS_8BIT.json")


def attn_source_hash(mode):
    import hashlib
    h = hashlib.sha256()
    for f in ATTN_KERNEL[mode][1]:
        with open(os.path.join(_CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def attn_traffic(mode="int8fp8"):
    try:
        h = attn_source_hash(mode)
    except OSError:
        return None, "kernel source not found"
    if h in ATTN_DRAM_BYTES:
        b, how = ATTN_DRAM_BYTES[h]
        return int(b), how
    return None, "no ncu capture of this kernel source yet"


def reduce_max(x: float, device) -> float:
    """Max of a per-rank float over all ranks (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own batch of `flops_per_rank`."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        out = {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
               "source": "measured"}
    else:
        out = {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}
    # dense 8-bit peaks (cuBLAS int8 and fp8 GEMMs, `bench.py --peaks`); until
    # measured, 2 x the bf16 burst figure (the nominal ratio)
    if os.path.exists(PEAKS_8BIT):
        e = json.load(open(PEAKS_8BIT))
        out["int8"], out["fp8"] = e["int8_tops"], e["fp8_tflops"]
        out["int8_sustained"], out["fp8_sustained"] = e["int8_tops_sustained"], e["fp8_tflops_sustained"]
        out["source_8bit"] = "measured (MEASURED_PEAKS_8BIT.json)"
    else:
        out["int8"] = out["fp8"] = 2.0 * out["bf16"]
        out["int8_sustained"] = out["fp8_sustained"] = 2.0 * out["bf16_sustained"]
        out["source_8bit"] = f"2 x {out['source']} bf16 (nominal ratio)"
    return out


def attn_roofline(flops, ms, peaks, mode, d, sm_mhz=None, sms=148):
    """The attention kernel's effective TFLOP/s against the dense peak of its
    dtype: the 8-bit GEMM burst peak (the larger of int8 and fp8; the kernel
    is timed alone for well under a second) or bf16, plus the sustained
    figure and the tcgen05 MMA rate at the sampled clock as second fields."""
    achieved = flops / (ms * 1e-3) / 1e12
    if mode == "int8fp8":
        peak = max(peaks["int8"], peaks["fp8"])
        sustained = max(peaks["int8_sustained"], peaks["fp8_sustained"])
        note = f"dense 8-bit burst, {peaks['source_8bit']}: int8 {peaks['int8']}, fp8 {peaks['fp8']}"
        mac = TC_8BIT_MAC_PER_CLK_SM
    else:
        peak, sustained = peaks["bf16"], peaks["bf16_sustained"]
        note = f"{peaks['source']} bf16 burst"
        mac = TC_8BIT_MAC_PER_CLK_SM // 2
    out = {"bound": "tensor", "kernel": f"{ATTN_KERNEL[mode][0]}<{d},{mode}>", "achieved": round(achieved, 1),
           "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 3), "peak_note": note,
           "frac_of_sustained": round(achieved / sustained, 3), "sustained_peak": round(sustained, 1)}
    if sm_mhz:
        tc = 2.0 * mac * sms * sm_mhz * 1e6 / 1e12
        out["tcgen05_peak_at_clock"] = round(tc, 1)
        out["frac_of_tcgen05_at_clock"] = round(achieved / tc, 3)
    return out


def measure_8bit_peaks(seconds=4.0, n=8192):
    """Dense int8 (torch._int_mm) and fp8 e4m3 (torch._scaled_mm) GEMM peaks on
    this GPU: the best of 10 single launches (burst) and back-to-back launches
    for `seconds` (sustained), 2*n^3 operations each; nvidia-smi clocks sampled
    during the sustained loops."""
    import torch
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    a8 = torch.randint(-64, 64, (n, n), generator=g, device=dev, dtype=torch.int8)
    b8 = torch.randint(-64, 64, (n, n), generator=g, device=dev, dtype=torch.int8).t()   # column-major B
    af = torch.randn(n, n, generator=g, device=dev).to(torch.float8_e4m3fn)
    bf = torch.randn(n, n, generator=g, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    ops = {"int8": lambda: torch._int_mm(a8, b8),
           "fp8": lambda: torch._scaled_mm(af, bf, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)}
    flop = 2.0 * n ** 3
    res = {}
    for name, f in ops.items():
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            f()
            e.record()
            torch.cuda.synchronize()
            best = min(best, s.elapsed_time(e))
        sampler = ClockSampler(0)
        sampler.start()
        time.sleep(0.2)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(1, int(seconds / (best * 1e-3)))
        s.record()
        for _ in range(reps):
            f()
        e.record()
        torch.cuda.synchronize()
        clk = sampler.stop()
        res[name] = {"burst": flop / (best * 1e-3) / 1e12,
                     "sustained": flop * reps / (s.elapsed_time(e) * 1e-3) / 1e12, "clocks": clk}
    return {"int8_tops": round(res["int8"]["burst"], 1), "int8_tops_sustained": round(res["int8"]["sustained"], 1),
            "fp8_tflops": round(res["fp8"]["burst"], 1), "fp8_tflops_sustained": round(res["fp8"]["sustained"], 1),
            "clocks_int8_sustained": res["int8"]["clocks"], "clocks_fp8_sustained": res["fp8"]["clocks"],
            "gpu_name": torch.cuda.get_device_name(dev), "torch": torch.__version__,
            "how": f"torch._int_mm (int8 x int8 -> int32) and torch._scaled_mm (e4m3 x e4m3 -> bf16, unit scales), "
                   f"{n}^3, 2*n^3 operations: best of 10 single launches (burst) and back to back for "
                   f"{seconds:g} s (sustained)"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except FileNotFoundError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import video_dit_dynamic_token_b200 as lx
    from video_dit_dynamic_token_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    B, H, d, L = w.B, args.heads or w.H, w.d, w.L
    keep = args.keep if args.keep else w.keep
    mode = args.mode
    nB = math.ceil(L / 64)
    Q, K, V = synth.make_qkv(B, H, d, w.grid, seed=rank, device=dev)
    k, _, _, plan_ws_bytes = lx.lx_plan_size(B, H, L, d, keep)
    plan = lx.empty_plan(B, H, L, d, keep, dev)
    plan_ws = torch.empty(plan_ws_bytes, dtype=torch.uint8, device=dev)
    # planner workspace: [means of Q | means of K | scores], 256-byte aligned
    means = (4 * B * H * nB * d + 255) // 256 * 256
    mq = plan_ws[:means][: 4 * B * H * nB * d].view(torch.float32).view(B, H, nB, d)
    mk = plan_ws[means:2 * means][: 4 * B * H * nB * d].view(torch.float32).view(B, H, nB, d)
    score_ws = plan_ws[2 * means:]
    qc = torch.empty((B, H, L, d), dtype=torch.int8, device=dev)
    kc = torch.empty_like(qc)
    vc = torch.empty((B, H, L, d), dtype=torch.uint8, device=dev)
    qs = torch.empty((B, H, nB), dtype=torch.float32, device=dev)
    ks = torch.empty_like(qs)
    vs = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    amax = torch.empty((B, H, d), dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    stream = torch.cuda.current_stream(dev)
    flops = lx.effective_flops(B, H, L, d, keep)
    if mode == "int8fp8":
        # Q/K block pass (means + INT8 codes), score GEMM, top-k, V absmax, V codes, attention
        launches_per_step = 6
        names = ["pool_quant_qk", "score_topk", "quant_v", "attn"]
        if args.prologue:
            names[0] = "qk_prologue"
        elif args.smooth_k:
            # K channel means (two launches), then the Q/K pass with K smoothed
            launches_per_step = 8
            names = ["k_mean", "pool_quant_qk_smooth", "score_topk", "quant_v", "attn"]
    else:
        launches_per_step = 4  # pool, score GEMM, top-k, attention
        names = ["pool", "score_topk", "attn"]

    # --prologue: the Q/K pass also applies per-head RMSNorm and the 3D RoPE of
    # the workload's grid (random per-head weights; the table is built once)
    pro = None
    if args.prologue and mode == "int8fp8":
        g = torch.Generator(device="cpu").manual_seed(1234 + rank)
        wq = (1.0 + 0.2 * torch.randn(H, d, generator=g)).float().to(dev)
        wk = (1.0 + 0.2 * torch.randn(H, d, generator=g)).float().to(dev)
        pro = dict(wq=wq, wk=wk, table=lx.lx_rope3d_table(w.grid, d, device=dev))

    km_buf = km_ws = None
    if args.smooth_k and mode == "int8fp8":
        km_buf = torch.empty((B, H, d), dtype=torch.float32, device=dev)
        km_ws = torch.empty(8 * B * H * ((L + 511) // 512) * d, dtype=torch.uint8, device=dev)

    def step(ev=None):
        marks = iter(range(len(names) + 1))
        def mark():
            i = next(marks)
            if ev is not None:
                ev[i].record(stream)
        mark()
        if args.smooth_k and mode == "int8fp8":
            lx.lx_k_channel_mean(K, out=km_buf, ws=km_ws)
            mark()
            lx.lx_pool_quantize_qk_smooth(Q, K, km_buf, (mq, mk, qc, qs, kc, ks))
        elif pro is not None:
            lx.lx_qk_prologue_into(Q, K, pro["wq"], pro["wk"], 1e-6, w.grid, pro["table"], mq, mk, qc, qs, kc, ks)
        elif mode == "int8fp8":
            lx.lx_pool_quantize_qk(Q, K, out=(mq, mk, qc, qs, kc, ks))
        else:
            lx.lx_pool_means(Q, K, out=(mq, mk))
        mark()
        lx.lx_score_topk(mq, mk, L, keep, plan=plan, ws=score_ws)
        mark()
        if mode == "int8fp8":
            lx.lx_quantize_v(V, out=(vc, vs), amax_ws=amax)
            mark()
            lx.lx_attn_int8fp8(qc, qs, kc, ks, vc, vs, plan, out=O)
        else:
            lx.lx_attn_bf16(Q, K, V, plan, out=O)
        mark()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = lx.lx_last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = t0.elapsed_time(t1)
    per = {n: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j, n in enumerate(names)}
    if lx.lx_last_device_status() != 0:
        raise RuntimeError("device status error in timed region")

    total_ms = reduce_max(total_ms, dev)
    ms_step = total_ms / args.steps
    value = job_tflops(world, flops, ms_step)

    # ---- the planner alone (a1 + a2: block means, scores, top-k) as a user
    # calls it, for its HBM roofline: Q and K read once, the plan written once
    pl_ms = None
    if args.planner_steps > 0:
        for _ in range(2):
            lx.lx_sparse_attn_plan(Q, K, keep, plan=plan, ws=plan_ws)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.planner_steps):
            lx.lx_sparse_attn_plan(Q, K, keep, plan=plan, ws=plan_ws)
        b.record(stream)
        torch.cuda.synchronize()
        pl_ms = reduce_max(a.elapsed_time(b) / args.planner_steps, dev)
        if lx.lx_last_device_status() != 0:
            raise RuntimeError("device status error in the planner leg")

    # ---- end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        from video_dit_dynamic_token_b200.pipeline import HostPipeline
        hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        # the public host-to-host path: head chunks with copies and kernels overlapped
        pipe = HostPipeline(B, H, L, d, keep, mode, heads_per_chunk=args.e2e_heads_per_chunk, device=dev)

        def e2e_step():
            pipe.run(hQ, hK, hV, hO, stream=stream)

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = reduce_max(a.elapsed_time(b) / args.e2e_steps, dev)
        e2e = {"value": job_tflops(world, flops, e_ms), "unit": "TFLOP/s", "ms_per_step": e_ms,
               "path": f"pinned host Q/K/V -> device -> pinned host O through HostPipeline, chunks of "
                       f"{args.e2e_heads_per_chunk} heads with copies and kernels overlapped",
               "h2d_bytes_per_step": 3 * Q.numel() * 2, "d2h_bytes_per_step": O.numel() * 2}

    if rank != 0:
        return None
    peaks = _peaks()
    attn_ms = per["attn"]
    achieved = flops / (attn_ms * 1e-3) / 1e12
    # algorithmic HBM bytes of the phases before attention (each tensor once per
    # pass that must touch it; the block means and scores are small or L2-sized)
    N = B * H * L * d
    means_b = 2 * B * H * nB * d * 4
    plan_out_b = B * H * nB * k * 4 + B * H * nB * ((nB + 31) // 32) * 4
    phase_bytes = {"score_topk": means_b + plan_out_b}
    if mode == "int8fp8":
        qk_name = "pool_quant_qk_smooth" if args.smooth_k else names[0]
        phase_bytes[qk_name] = 2 * N * 2 + 2 * N + means_b + 2 * B * H * nB * 4
        if args.smooth_k:
            phase_bytes["k_mean"] = N * 2 + B * H * d * 4  # K read once
        phase_bytes["quant_v"] = 2 * N * 2 + N + B * H * d * 4  # V read twice: the channel scale needs all of V
    else:
        phase_bytes["pool"] = 2 * N * 2 + means_b
    phases = {n: {"ms": round(per[n], 4), "algorithmic_mb": round(b / 1e6, 1),
                  "gbs": round(b / (per[n] * 1e-3) / 1e9, 1),
                  "hbm_frac": round(b / (per[n] * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)} for n, b in phase_bytes.items()}
    if pl_ms is not None:
        # the planner's algorithmic bytes: Q and K read once, idx and mask written once
        pb = 2 * N * 2 + plan_out_b
        phases["planner"] = {"ms": round(pl_ms, 4), "algorithmic_mb": round(pb / 1e6, 1),
                             "gbs": round(pb / (pl_ms * 1e-3) / 1e9, 1),
                             "hbm_frac": round(pb / (pl_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
                             "call": "lx_sparse_attn_plan (block means, score GEMM, top-k), timed alone",
                             "of_8tbs_spec": round(pb / (pl_ms * 1e-3) / 1e9 / 8000.0, 3)}
    # Q/K/V (codes or bf16) read once, O written once (bf16), kept ids
    esz = 1 if mode == "int8fp8" else 2
    attn_bytes = 3 * B * H * L * d * esz + B * H * L * d * 2 + B * H * nB * k * 4
    roof = attn_roofline(flops, attn_ms, peaks, mode, d, (clocks or {}).get("sm_mhz"))
    traffic, traffic_note = attn_traffic(mode)
    if args.heads or args.workload != WORKLOAD or args.keep:
        traffic, traffic_note = None, "captured for the 720p headline launch only"
    roof.update({"traffic": traffic, "traffic_note": traffic_note, "algorithmic_bytes": int(attn_bytes)})
    out = {
        "metric": metric_for(args.workload, H, d, keep), "value": round(value, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": mode, "data": "synthetic (smooth coarsened N(0,1) field + noise, seeded)",
        "config": {"workload": f"{args.workload}-shaped B={B} H={H} d={d} L={L} keep={keep} mode={mode}", "k": k,
                   "nB": nB,
                   "effective_tflop_per_step": round(flops / 1e12, 3), "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (2.3 GB of Q/K/V per step)"},
        "breakdown_ms": {n: round(v, 4) for n, v in per.items()},
        "attn_ms": round(attn_ms, 4), "attn_effective_tflops": round(achieved, 1),
        "phases": phases,
        "roofline": roof,
        "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_note": f"{launches_per_step} library kernels per step; the planner leg and e2e are timed "
                             "separately",
        "clocks": clocks,
        "e2e": e2e,
    }
    return out


# ------------------------------------------------------------------ Light-Ulysses share
def ulysses_cpu_sample(N, B, H, d, L, flops, sample_tokens=256, attn=None):
    """The oracle on a bounded sample of one rank's share: the exchange steps
    (pack/unpack of the Q/K/V payload and of the output) on `sample_tokens` of
    the shard's tokens, scaled to the shard, plus the attention at the oracle's
    sampled rate (cpu_oracle_sample, or `attn` when given)."""
    import numpy as np

    import oracle
    Hr, Lr = H // N, L // N
    rng = np.random.default_rng(0)
    ts = min(sample_tokens, Lr)
    q, k, v = (rng.standard_normal((B, ts, H, d)).astype(np.float32) for _ in range(3))
    o = rng.standard_normal((B, Hr, N * ts, d)).astype(np.float32)
    t0 = time.perf_counter()
    c, sc = oracle.pack_qkv_ref(q, k, v, N)
    oracle.unpack_qkv_ref(c, sc)            # the send buffer stands in for the received one
    oc, osc = oracle.pack_o_ref(o, N)
    oracle.unpack_o_ref(oc, osc)
    t_x = (time.perf_counter() - t0) * (Lr / ts)
    attn = attn or cpu_oracle_sample()
    t_attn = flops / (attn["value"] * 1e12)
    return {"value": flops / (t_attn + t_x) / 1e12, "unit": "TFLOP/s", "cores": attn["cores"], "kind": "oracle",
            "sample": f"exchange steps on {ts} of the shard's {Lr} tokens ({t_x * ts / Lr:.2f} s, scaled x{Lr / ts:.0f}); "
                      f"attention at the oracle's sampled rate ({attn['sample']})"}


def run_ulysses_share(args):
    """One rank's share of an N-GPU Light-Ulysses step at the workload's grid,
    timed on one GPU: pack this rank's token shard (all heads) into the FP8
    payload, unpack a payload of the same layout (the send buffer stands in for
    the received one: with one GPU there is no exchange), the attention of the
    H/N heads over all tokens, then the output's pack and unpack.  Reports each
    exchange kernel against the HBM roofline; the all-to-all itself is not
    timed."""
    import torch

    import video_dit_dynamic_token_b200 as lx
    from video_dit_dynamic_token_b200 import synth, ulysses

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    N = args.ulysses
    B, H, d, L = w.B, w.H, w.d, w.L
    if H % N or L % N:
        raise SystemExit("heads and tokens must divide by N")
    Hr, Lr = H // N, L // N
    keep = args.keep if args.keep else w.keep
    g = torch.Generator(device=dev).manual_seed(0)
    q, k, v = ((torch.randn(B, Lr, H, d, generator=g, device=dev)).to(torch.bfloat16) for _ in range(3))
    qv, kv, vv = (x.permute(0, 2, 1, 3) for x in (q, k, v))
    pay = ulysses.new_payload(N, B, Hr, Lr, d, 3, dev)
    qh, kh, vh = (torch.empty((B, Hr, L, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    pay_o = ulysses.new_payload(N, B, Hr, Lr, d, 1, dev)
    out = torch.empty_like(q)
    ws = torch.empty(lx.lx_sparse_attn_ws_size(qh, keep, args.mode), dtype=torch.uint8, device=dev)
    oh = torch.empty_like(qh)
    names = ["pack_qkv", "unpack_qkv", "attn", "pack_o", "unpack_o"]

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record()
        mark(0)
        ulysses.pack_qkv(qv, kv, vv, N, 0, Hr, pay)
        mark(1)
        ulysses.unpack_qkv(pay, N, qh, kh, vh)
        mark(2)
        lx.lx_sparse_attn(qh, kh, vh, keep, args.mode, out=oh, ws=ws)
        mark(3)
        ulysses.pack_o(oh, N, pay_o)
        mark(4)
        ulysses.unpack_o(pay_o, N, 0, Hr, out.permute(0, 2, 1, 3))
        mark(5)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(0)
    sampler.start()
    t0.record()
    for i in range(args.steps):
        step(evs[i])
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if lx.lx_last_device_status() != 0:
        raise RuntimeError("device status error")
    ms = t0.elapsed_time(t1) / args.steps
    per = {n: sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j, n in enumerate(names)}
    peaks = _peaks()
    rows_qkv, rows_o = 3 * B * H * Lr, B * H * Lr     # one rank's payload rows (all destinations)
    byt = {"pack_qkv": rows_qkv * (2 * d + d + 4), "unpack_qkv": rows_qkv * (d + 4 + 2 * d),
           "pack_o": rows_o * (2 * d + d + 4), "unpack_o": rows_o * (d + 4 + 2 * d)}
    phases = {n: {"ms": round(per[n], 4), "algorithmic_mb": round(b / 1e6, 1),
                  "gbs": round(b / (per[n] * 1e-3) / 1e9, 1),
                  "hbm_frac": round(b / (per[n] * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)} for n, b in byt.items()}
    flops = lx.effective_flops(B, Hr, L, d, keep)
    return {"metric": f"Light-Ulysses one-rank share of an N={N} step ({args.workload} grid, {H}x{d}, keep {keep})",
            "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "dtype": args.mode,
            "data": "synthetic N(0,1) shards", "config": {"workload": f"{args.workload} B={B} H={H} d={d} L={L} N={N}",
                                                          "shard_tokens": Lr, "heads_after_exchange": Hr},
            "breakdown_ms": {n: round(v, 4) for n, v in per.items()}, "phases": phases,
            "roofline": attn_roofline(flops, per["attn"], peaks, args.mode, d, (clocks or {}).get("sm_mhz")),
            "gpu_launches": (10 if args.mode == "int8fp8" else 8) * args.steps, "clocks": clocks, "e2e": None,
            "cpu_baseline": (None if args.no_cpu_baseline else ulysses_cpu_sample(N, B, H, d, L, flops)),
            "note": "the all-to-all is not timed (one GPU); the send buffer stands in for the received one"}


# ------------------------------------------------------------------ NVFP4 linear
GEMM_WORKLOAD = "Wan2.2-A14B fused QKV projection, 720p grid: M=75600 tokens, K=5120, N=15360, fp32 bias"


def nvfp4_cpu_sample(M, N, K, rows=32):
    """The oracle (quantisation + fp64 GEMM) on `rows` rows of the workload."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(0)
    t0 = time.perf_counter()
    X = rng.standard_normal((rows, K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    t1 = time.perf_counter()
    xq = oracle.quant_nvfp4_ref(X)
    wq = oracle.quant_nvfp4_ref(W)
    oracle.gemm_nvfp4_ref(xq, wq, np.zeros(N, np.float32))
    dt = time.perf_counter() - t1
    flops = 2.0 * rows * N * K
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{rows} of the {M} rows (weights quantised in the sample too), {dt:.1f} s",
            "setup_s": round(t1 - t0, 1)}


def run_nvfp4_gemm(args):
    """One step = one NVFP4 linear layer: quantise the bf16 activations (amax
    pass, global scale, quantiser) and run the block-scaled GEMM with the column
    bias; the weights are quantised once, before timing, as a deployed model's
    would be.  X (774 MB) is larger than L2, so no flush is needed."""
    import torch

    import video_dit_dynamic_token_b200 as lx

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M, N, K = (args.gemm_m or 75600), (args.gemm_n or 15360), (args.gemm_k or 5120)
    g = torch.Generator(device=dev).manual_seed(0)
    X = torch.randn((M, K), generator=g, device=dev).to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    bias = torch.randn(N, generator=g, device=dev) * 0.1
    wq = lx.lx_nvfp4_quantize(W)
    xq = lx.lx_nvfp4_quantize(X)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        lx.lx_nvfp4_quantize(X, out=xq)
        if ev is not None:
            ev[1].record(stream)
        lx.lx_nvfp4_gemm(xq, wq, bias, out=Y)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0)
    clocks.start()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if lx.lx_last_device_status() != 0:
        raise RuntimeError("device status error")
    ms = t0.elapsed_time(t1) / args.steps
    q_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    g_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    flops = lx.nvfp4_gemm_flops(M, N, K)
    peaks = _peaks()
    fp4_peak = 4.0 * peaks["bf16"]   # dense fp4 : bf16 = 9 : 2.25 PFLOP/s nominal
    q_bytes = 2 * (M * K * 2) + M * K // 2 + M * K // 16   # two reads of X (amax, quantiser), codes + scales
    g_bytes = M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + M * N * 2 + N * 4
    out = {"metric": "NVFP4 linear (activation quantisation + block-scaled GEMM + bias) TFLOP/s",
           "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
           "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3/16 scales, f32 accumulate, bf16 out)",
           "data": "synthetic: X ~ N(0,1), W ~ N(0, 0.02^2), bias ~ N(0, 0.01)",
           "config": {"workload": GEMM_WORKLOAD if (M, N, K) == (75600, 15360, 5120)
                      else f"NVFP4 linear layer, M={M}, K={K}, N={N}",
                      "M": M, "N": N, "K": K, "l2": f"inputs larger than L2 (X {M * K * 2 / 1e6:.0f} MB)"},
           "breakdown_ms": {"quantise_x": round(q_ms, 4), "gemm": round(g_ms, 4)},
           "roofline": {"bound": "tensor", "achieved": round(flops / (g_ms * 1e-3) / 1e12, 1),
                        "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                        "frac": round(flops / (g_ms * 1e-3) / 1e12 / fp4_peak, 3), "traffic": None,
                        "peak_source": f"{peaks['source']} bf16 burst x 4 (nominal dense fp4/bf16 ratio)",
                        "kernel": "nvfp4_gemm_kernel"},
           "phases": {"quantise_x": {"ms": round(q_ms, 4), "algorithmic_mb": round(q_bytes / 1e6, 1),
                                     "gbs": round(q_bytes / (q_ms * 1e-3) / 1e9, 1),
                                     "hbm_frac": round(q_bytes / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)},
                      "gemm": {"ms": round(g_ms, 4), "algorithmic_mb": round(g_bytes / 1e6, 1),
                               "hbm_frac_of_time": round(g_bytes / (g_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}},
           "gpu_launches": 4 * args.steps, "clocks": clk, "e2e": None,
           "note": "sub-benchmark of the NVFP4 projection kernel; the headline line (no flags) carries e2e"}
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = nvfp4_cpu_sample(M, N, K)
    if (M, N, K) != (75600, 15360, 5120):
        out["note"] = "another shape: a characterisation or profiling case, not the benchmark"
    return out

# ------------------------------------------------------------------ CPU oracle timing
def cpu_oracle_sample(seconds_target=12.0):
    """Time the oracle (as it stands) on one head of the workload: planner and
    quantisers for that head, INT8/FP8 attention for a bounded number of its
    query blocks; returns effective TFLOP/s of the sampled work."""
    import numpy as np

    import oracle
    from video_dit_dynamic_token_b200 import synth

    w = synth.WORKLOADS[WORKLOAD]
    d, L, keep = w.d, w.L, w.keep
    Q, K, V = synth.make_qkv(1, 1, d, w.grid, seed=0)
    t0 = time.perf_counter()
    p = oracle.plan_ref(Q, K, keep)
    qc, sq = oracle.quant_qk_ref(Q)
    kc, sk = oracle.quant_qk_ref(K)
    vc, sv = oracle.quant_v_ref(V)
    t_head = time.perf_counter() - t0
    nB, k = p["nB"], p["k"]
    rng = np.random.default_rng(0)
    order = rng.permutation(nB)
    t1 = time.perf_counter()
    done = 0
    while done < nB and time.perf_counter() - t1 < seconds_target:
        oracle.attn_int8fp8_from_codes(qc, sq, kc, sk, vc, sv, p["idx"], L, blocks=[(0, 0, int(order[done]))])
        done += 1
    t_attn = time.perf_counter() - t1
    # the head's planner + quantisers amortised over the head's nB query blocks
    t_total = t_attn + t_head * done / nB
    flops = 4.0 * (64 * done) * (k * 64) * d
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = 1
    return {"value": flops / t_total / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"1 of 40 heads at 720p: planner + quantisers on the full head ({t_head:.1f} s, "
                      f"amortised by {done}/{nB} blocks) and INT8/FP8 attention on {done} random query blocks "
                      f"({t_attn:.1f} s); numpy fp64"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    times = []
    vals = []
    cb = None
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        cb = cpu_oracle_sample(seconds_target=4.0)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
            vals.append(cb["value"])
    v = sum(vals) / len(vals)
    return {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"720p-shaped B=1 H=40 d=128 L=75600 keep=0.1 mode={MODE} (bounded sample)"},
            "impl": "reference", "cpu_baseline": {**cb, "value": v},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-heads-per-chunk", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--planner-steps", type=int, default=10, help="timed calls of the planner alone")
    ap.add_argument("--peaks", action="store_true",
                    help="measure the dense int8 and fp8 GEMM peaks (cuBLAS) and print them as JSON")
    ap.add_argument("--heads", type=int, default=0, help="fewer heads: a smaller case for profiling only")
    ap.add_argument("--workload", default=WORKLOAD, choices=["480p", "720p", "long"],
                    help="grid shape (the headline is 720p; the others are characterisation runs)")
    ap.add_argument("--mode", default=MODE, choices=["int8fp8", "bf16"])
    ap.add_argument("--keep", type=float, default=0.0, help="override the workload's keep ratio (sweeps)")
    ap.add_argument("--smooth-k", action="store_true",
                    help="int8fp8: K smoothing (channel means of K subtracted before its INT8 codes)")
    ap.add_argument("--ulysses", type=int, default=0,
                    help="time one rank's share of an N-GPU Light-Ulysses step instead (exchange kernels + attention)")
    ap.add_argument("--prologue", action="store_true",
                    help="int8fp8: the Q/K pass also applies per-head RMSNorm and 3D RoPE (lx_qk_prologue)")
    ap.add_argument("--gemm", action="store_true",
                    help="time one NVFP4 linear layer (the 720p fused QKV projection) instead")
    ap.add_argument("--gemm-m", type=int, default=0, help="--gemm with another token count (profiling)")
    ap.add_argument("--gemm-n", type=int, default=0, help="--gemm with another output width (characterisation)")
    ap.add_argument("--gemm-k", type=int, default=0, help="--gemm with another input width (characterisation)")
    args = ap.parse_args()
    if args.peaks:
        print(json.dumps(measure_8bit_peaks()))
        return
    if args.gemm:
        print(json.dumps(run_nvfp4_gemm(args)))
        return
    if args.ulysses:
        print(json.dumps(run_ulysses_share(args)))
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out))
        return

    import datetime

    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=__import__("torch").device("cuda", local_rank))
    cpu = None
    if (rank == 0 and world == 1 and not args.no_cpu_baseline and not args.heads and args.workload == WORKLOAD
            and args.mode == MODE and not args.keep):
        cpu = cpu_oracle_sample()
    out = run_ours(args, rank, world, local_rank)
    if world > 1:
        dist.destroy_process_group()
    if out is not None:
        out["cpu_baseline"] = cpu
        print(json.dumps(out))


if __name__ == "__main__":
    main()
