"""Benchmark: NVFP4 W4A4 routed-expert MoE layer on B200.

One step = one pass of the hot path over one batch: gather + per-expert
dynamic NVFP4 quantize of the routed activations -> block-scaled FP4 grouped
gate_up GEMM -> SwiGLU + per-expert requantize -> grouped down GEMM, for the
MoE layer with 512 experts, top-10 routing, 8192 tokens, hidden 4096, expert
intermediate 1024 (weights resident in HBM as NVFP4).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs its own replica (independent batch, its own
experts): weak scaling, no collective in the data path; timing is the max
over ranks.  Rank 0 prints one JSON line.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 W4A4 expert GEMM TFLOPS & % FP4 peak; quantize GB/s & % HBM"
WORKLOAD = "moe_routed_experts_e512_top10_t8192_h4096_i1024"
CFG = dict(E=512, topk=10, T=8192, H=4096, I=1024, seed=0)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 9.0 / 2.25      # nominal dense ratio (4x)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def moe_flops(R, H, I):
    return 2.0 * R * (2 * I * H + H * I)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return out
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        out.update(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=max(mx) if mx else None,
                   reasons=reasons, samples=len(rows))
        return out


# --------------------------------------------------------------------------- setup
def setup_moe(device, seed):
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L

    E, k, T, H, I = CFG["E"], CFG["topk"], CFG["T"], CFG["H"], CFG["I"]
    r = synthetic.route_topk_softmax(seed, T, E, k)
    R = len(r["row_index"])
    ws = L.workspace(E, device)
    # weights: N(0, 0.02^2) bf16 generated on the device, quantized statically
    # (one global scale per expert and projection) by the same library.
    packs = []
    for name, rows_per, K in (("w_gate_up", 2 * I, H), ("w_down", H, I)):
        w = sc.gaussian_bf16(seed, synthetic.STREAMS[name], (E * rows_per, K), sigma=0.02)
        offs = torch.arange(0, (E + 1) * rows_per, rows_per, dtype=torch.int32, device=device)
        p = L.quantize(w, None, offs, E, layout=1, ws=ws)
        p.offsets, p.num_groups, p.rows = None, 1, E * rows_per
        packs.append(p)
        del w
    torch.cuda.synchronize()
    x = sc.gaussian_bf16(seed, synthetic.STREAMS["x"], (T, H))
    moe = L.MoEExperts(packs[0], packs[1], E, H, I, max_rows=R, out_dtype=1, mid_dtype=1, device=device)
    ri = torch.from_numpy(r["row_index"]).to(device)
    off = torch.from_numpy(r["offsets"]).to(device)
    return moe, x, ri, off, r, R


def gemm_bytes(R, E_touched, N, K, out_bytes=2):
    """Algorithmic bytes of one grouped GEMM: touched expert weights + packed
    activations, each read once, plus the output written once."""
    w = E_touched * N * K * 0.5625
    a = R * K * 0.5625
    return w + a + R * N * out_bytes


def run_ours(args, rank, world, device):
    import torch
    import torch.distributed as dist

    peaks, peaks_kind = load_peaks()
    moe, x, ri, off, r, R = setup_moe(device, CFG["seed"] + rank)
    E, H, I = CFG["E"], CFG["H"], CFG["I"]
    flops = moe_flops(R, H, I)
    e_touched = int((np.diff(r["offsets"]) > 0).sum())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step():
        return moe.forward(x, ri, off)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # timed region: per-step events, L2 flushed between steps (outside the events)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        s0, g0, g1, s1 = ev[i]
        s0.record(stream)
        a1 = L.quantize(x, ri, off, E, layout=1, out=moe.a1, ws=moe.ws, rows=R)
        g0.record(stream)
        L.grouped_gemm(a1, moe.w_gate_up, 2 * I, moe.mid_dtype, y=moe.y1[:R])
        g1.record(stream)
        a2, _ = L.swiglu_quantize(moe.y1[:R], off, E, layout=1, out=moe.a2, h=moe.h[:R], ws=moe.ws)
        L.grouped_gemm(a2, moe.w_down, H, moe.out_dtype, y=moe.y2[:R])
        s1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    gemm_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = sum(step_ms)
    t = torch.tensor([total_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * flops * args.steps / (total_ms * 1e-3) / 1e12

    # e2e through the public API with host buffers: H2D inputs, D2H result
    x_host = x.cpu().pin_memory()
    ri_host = ri.cpu().pin_memory()
    off_host = off.cpu().pin_memory()
    y_host = torch.empty((R, H), dtype=torch.bfloat16).pin_memory()
    x_d = torch.empty_like(x)
    ri_d = torch.empty_like(ri)
    off_d = torch.empty_like(off)
    e2e_steps = max(2, min(args.steps, 5))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        x_d.copy_(x_host, non_blocking=True)
        ri_d.copy_(ri_host, non_blocking=True)
        off_d.copy_(off_host, non_blocking=True)
        y = moe.forward(x_d, ri_d, off_d)
        y_host.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    t = torch.tensor([e2e_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_ms = float(t.item())
    h2d = x.numel() * 2 + ri.numel() * 4 + off.numel() * 4
    d2h = R * H * 2

    # roofline of the dominant kernel (gate_up grouped GEMM), HBM-bound at this shape
    gemm_avg_s = statistics.mean(gemm_ms) * 1e-3
    gbytes = gemm_bytes(R, e_touched, 2 * I, H, out_bytes=2)
    g_flops = 2.0 * R * 2 * I * H
    fp4_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP4_OVER_BF16
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    roof = {"bound": "hbm", "kernel": "nvfp4::gemm::grouped_gemm_kernel (gate_up)",
            "achieved": round(gbytes / gemm_avg_s / 1e9, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(gbytes / gemm_avg_s / 1e9 / hbm_peak, 4), "traffic": None,
            "peak_source": f"{peaks_kind} hbm_gbs",
            "tensor_tflops": round(g_flops / gemm_avg_s / 1e12, 1),
            "pct_fp4_peak": round(100 * g_flops / gemm_avg_s / 1e12 / fp4_peak, 2),
            "fp4_peak_tflops": round(fp4_peak, 1),
            "algorithmic_bytes_per_launch": int(gbytes), "gemm_ms": round(1e3 * gemm_avg_s, 4)}

    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales) -> fp32 accum, bf16 io",
        "data": "synthetic (seeded SplitMix64 / Irwin-Hall N(0,1) activations, N(0,0.02^2) weights, softmax top-10 routing)",
        "config": {"workload": WORKLOAD, "experts": E, "topk": CFG["topk"], "tokens": CFG["T"], "hidden": H,
                   "intermediate": I, "routed_rows": R, "experts_touched": e_touched,
                   "flops_per_step": flops, "l2": "flushed between steps (256 MB write)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roof,
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_ms, 3)},
        "gpu_launches": 8 * args.steps,
        "clocks": clk,
    }
    return out


# --------------------------------------------------------------------------- CPU oracle baseline
_SAMPLE_INPUTS = {}


def oracle_sample(seconds: float, seed: int = 0):
    """Time the oracle on a bounded sample of the same workload: whole experts
    (their routed rows) through gather-quantize, fp64 gate_up, SwiGLU,
    requantize and fp64 down, until ``seconds`` of CPU work.  Returns
    (TFLOP/s, experts done, rows done, threads)."""
    import oracle
    import synthetic

    E, k, T, H, I = CFG["E"], CFG["topk"], CFG["T"], CFG["H"], CFG["I"]
    if seed not in _SAMPLE_INPUTS:
        _SAMPLE_INPUTS[seed] = (synthetic.route_topk_softmax(seed, T, E, k),
                                synthetic.gaussian_bf16(seed, synthetic.STREAMS["x"], (T, H)))
    r, x = _SAMPLE_INPUTS[seed]
    done_flops, experts, rows = 0.0, 0, 0
    t_work = 0.0
    for e in range(E):
        r0, r1 = int(r["offsets"][e]), int(r["offsets"][e + 1])
        m = r1 - r0
        if m == 0:
            continue
        wgu = synthetic.gaussian_bf16(seed, synthetic.STREAMS["w_gate_up"], (2 * I, H), sigma=0.02,
                                      start=e * 2 * I * H)
        wd = synthetic.gaussian_bf16(seed, synthetic.STREAMS["w_down"], (H, I), sigma=0.02, start=e * H * I)
        t0 = time.perf_counter()
        qg, sg, gg, _ = oracle.quantize(wgu)
        qd, sd, gd, _ = oracle.quantize(wd)
        q1, s1, g1, _ = oracle.quantize(x, r["row_index"][r0:r1])
        a1 = oracle.dequantize_f64(q1, s1, np.full(m, g1[0], np.float32))
        y1, _ = oracle.gemm_f64(a1, oracle.dequantize_f64(qg, sg, np.full(2 * I, gg[0], np.float32)))
        h = oracle.swiglu(y1.astype(np.float32))
        q2, s2, g2, _ = oracle.quantize(h)
        a2 = oracle.dequantize_f64(q2, s2, np.full(m, g2[0], np.float32))
        oracle.gemm_f64(a2, oracle.dequantize_f64(qd, sd, np.full(H, gd[0], np.float32)))
        t_work += time.perf_counter() - t0
        done_flops += 2.0 * m * (2 * I * H + H * I)
        experts += 1
        rows += m
        if t_work >= seconds:
            break
    return done_flops / t_work / 1e12, experts, rows, t_work


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, rank, world):
    """The oracle as the reference arm (host cores), each step a bounded sample."""
    import oracle
    oracle.build()
    secs = []
    vals = []
    for _ in range(max(1, args.warmup if args.warmup < 2 else 1)):
        oracle_sample(0.5)
    for _ in range(args.steps):
        v, ne, nr, t = oracle_sample(2.0)
        vals.append(v)
        secs.append(t)
    value = statistics.mean(vals)
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(secs), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic", "config": {"workload": WORKLOAD},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"whole experts of the same MoE layer until ~2 s of CPU work per step "
                                   f"(last step: {ne} experts, {nr} routed rows)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    import torch
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    from nvfp4_w4a4_quantized_04_b200 import build as nvbuild
    nvbuild.build()
    import synthetic.cuda as sc
    sc.build()

    out = run_ours(args, rank, world, device)
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        v, ne, nr, t = oracle_sample(12.0)
        out["cpu_baseline"] = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                               "sample": f"{ne} whole experts ({nr} routed rows) of the same layer, "
                                         f"{t:.1f} s of CPU work"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
