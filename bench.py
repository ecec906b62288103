"""Benchmark: NVFP4 W4A4 routed-expert path on B200.

Headline step = one pass of the hot path over one batch of the MoE layer
with 512 experts, top-10 routing, 8192 tokens, hidden 4096, expert
intermediate 1024: gather + per-expert dynamic NVFP4 quantize of the routed
activations -> block-scaled FP4 grouped gate_up GEMM -> SwiGLU + per-expert
requantize -> grouped down GEMM (weights resident in HBM as NVFP4).

The other rows of the path are measured in the same run as "components":
the dense MLP (4096 tokens, 5120 -> 2x17408 -> 5120), the decode MoE (384
experts, 64 tokens, Zipf routing, MXFP4 weights remapped to NVFP4), the
NVFP4 KV cache (4 heads x 256 x 262144 tokens, K and V), the activation
quantize sweep [T, 5120], the MXFP4 -> NVFP4 remap of 2^28 elements, the
W4A16 decode layer, the MXFP4 encoder and GEMM, the whole MoE block (route,
experts, combine), and the smallest GEMM [128 x 256 x 512] in microseconds.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--experts E --tokens T] [--components all|none|<name,...>] [--no-cpu-baseline]
Under torchrun each rank runs its own replica (its own batch and experts):
weak scaling, no collective in the data path; timing is the max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
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
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 9.0 / 2.25      # nominal dense FP4 / BF16 tensor ratio
L2_BYTES = 126 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p)), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


PEAKS, PEAKS_KIND = load_peaks()
HBM_PEAK = PEAKS.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
# DRAM traffic / algorithmic bytes of the gate_up + SwiGLU grouped GEMM launch
# (dram__bytes_read.sum + dram__bytes_write.sum over the bench's algorithmic
# bytes), from one ncu capture at 128 experts / 2048 tokens of the kernel built
# from the sources whose digest is recorded beside it.  Once those sources
# change the figure no longer describes the kernel that runs, and the bench
# reports the traffic as null until a new capture is recorded here.
GATE_UP_TRAFFIC = {"ratio": 701062144 / 693108736, "capture": "128 experts, 2048 tokens",
                   "sources_sha256": "1ecd55039044bcf7f7e965a332b7a652fb0369c560eedf0b0033c60da57a8f6d"}
GEMM_KERNEL_SOURCES = ("gemm.cu", "gemm_w2.cu", "gemm_common.cuh", "common.cuh")


def gemm_sources_digest() -> str:
    h = hashlib.sha256()
    for name in GEMM_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "nvfp4_w4a4_quantized_04_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gate_up_traffic_ratio():
    """The recorded DRAM/algorithmic ratio, or None when the kernel changed since its capture."""
    if GATE_UP_TRAFFIC["ratio"] is None:
        return None
    return GATE_UP_TRAFFIC["ratio"] if gemm_sources_digest() == GATE_UP_TRAFFIC["sources_sha256"] else None


def grouped_gemm_kernel_name(R, E, N, K, bf16_out, swiglu):
    """The kernel nvfp4_grouped_gemm's automatic choice launches for this
    problem (its rule, restated for the bench line's label only)."""
    tag = "<swiglu>" if swiglu else ""
    if N % 256 == 0 and bf16_out and K >= 1024:
        return f"nvfp4::gemm::w2::grouped_gemm_w2_kernel{tag} (two weight blocks per tile)"
    if K % 512 != 0:
        return f"nvfp4::gemm::grouped_gemm_kernel{tag}"
    return f"nvfp4::gemm::grouped_gemm_k512_kernel{tag}" + (" (deep ring)" if R <= 16 * E else "")
FP4_PEAK = PEAKS.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP4_OVER_BF16


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx, self.proc, self.path = gpu_index, None, None

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
        rows = [[p.strip() for p in line.split(",")] for line in open(self.path)]
        rows = [r for r in rows if len(r) >= 9]
        os.unlink(self.path)
        if not rows:
            return out

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        out.update(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=max(mx) if mx else None,
                   reasons=reasons, samples=len(rows), power_w_max=max(pw) if pw else None)
        return out


# --------------------------------------------------------------------------- timing helpers
def timed(fn, iters, warmup, flush=None):
    """Median device time (ms) of fn() over iters, CUDA events on the current
    stream; L2 flushed between iterations (outside the events) when given."""
    import torch
    s = torch.cuda.current_stream()
    for _ in range(max(3, warmup)):
        fn()
    ts = []
    for i in range(iters):
        if flush is not None:
            flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        fn()
        b.record(s)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def max_over_ranks(value, world, device="cpu"):
    """Largest per-rank value over all ranks of the process group (its own
    backend: NCCL with CUDA tensors, gloo with CPU tensors); the value itself
    when there is one rank."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, world, steps, total_ms):
    """Units per second of the whole job: every rank processes its own
    units_per_rank_step each step (weak scaling), timed by the slowest rank."""
    return world * units_per_rank_step * steps / (total_ms * 1e-3)


def gbs(nbytes, ms):
    return nbytes / (ms * 1e-3) / 1e9


def moe_flops(R, H, I):
    return 2.0 * R * (2 * I * H + H * I)


def gemm_bytes(R, e_touched, N, K, out_bytes=2):
    """Algorithmic bytes of one grouped GEMM launch: the touched experts'
    packed weights (0.5625 B/element) and the packed activations, each read
    once, and the output written once."""
    return e_touched * N * K * 0.5625 + R * K * 0.5625 + R * N * out_bytes


# --------------------------------------------------------------------------- headline: MoE layer
def setup_moe(device, seed, E, T, H, I, topk, fused=True):
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L

    r = synthetic.route_topk_softmax(seed, T, E, topk)
    R = len(r["row_index"])
    ws = L.workspace(E, device)
    packs = []
    for name, rows_per, K in (("w_gate_up", 2 * I, H), ("w_down", H, I)):
        w = sc.gaussian_bf16(seed, synthetic.STREAMS[name], (E * rows_per, K), sigma=0.02)
        ri = L.gate_up_interleave_index(E, I, device) if (fused and name == "w_gate_up") else None
        packs.append(L.pack_weights(w, E, rows_per, ri, ws))
        del w
    torch.cuda.synchronize()
    x = sc.gaussian_bf16(seed, synthetic.STREAMS["x"], (T, H))
    moe = L.MoEExperts(packs[0], packs[1], E, H, I, max_rows=R, out_dtype=1, mid_dtype=1, device=device,
                       fused_swiglu=fused)
    ri = torch.from_numpy(r["row_index"]).to(device)
    off = torch.from_numpy(r["offsets"]).to(device)
    r["slot_dev"] = torch.from_numpy(r["slot"].astype(np.int32)).to(device)
    return moe, x, ri, off, r, R


def run_headline(args, rank, world, device):
    import torch
    import torch.distributed as dist
    from nvfp4_w4a4_quantized_04_b200 import layer as L

    E, T, H, I, k = args.experts, args.tokens, 4096, 1024, 10
    fused = not args.unfused
    moe, x, ri, off, r, R = setup_moe(device, rank, E, T, H, I, k, fused=fused)
    sl = r["slot_dev"]
    flops = moe_flops(R, H, I)
    e_touched = int((np.diff(r["offsets"]) > 0).sum())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    from nvfp4_w4a4_quantized_04_b200 import GS_AMAX_GIVEN, nvfp4_quantize

    def stages(evs=None):
        rec = (lambda i: evs[i].record(stream)) if evs else (lambda i: None)
        rec(0)
        a1 = L.moe_quantize(x, sl, off, E, layout=1, out=moe.a1, ws=moe.ws, rows=R)
        rec(1)
        if fused:
            h, amax = L.grouped_gemm_swiglu(a1, moe.w_gate_up, 2 * I, h=moe.h[:R], amax=moe.amax)
            rec(2)
            a2 = moe.a2
            a2.offsets, a2.num_groups, a2.rows, a2.gs = off, E, R, amax
            nvfp4_quantize(h, R, I, I, None, off, E, GS_AMAX_GIVEN, amax, a2.q, a2.sf, 1, moe.ws)
        else:
            L.grouped_gemm(a1, moe.w_gate_up, 2 * I, moe.mid_dtype, y=moe.y1[:R])
            rec(2)
            a2, _ = L.swiglu_quantize(moe.y1[:R], off, E, layout=1, out=moe.a2, h=moe.h[:R], ws=moe.ws)
        rec(3)
        L.grouped_gemm(a2, moe.w_down, H, moe.out_dtype, y=moe.y2[:R])
        rec(4)

    for _ in range(max(3, args.warmup)):
        stages()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.25)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)               # L2 flush between steps, outside the events
        stages(evs[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    time.sleep(0.15)
    clk = clocks.stop()
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])
    step_ms = per.sum(axis=1)
    total_ms = max_over_ranks(float(step_ms.sum()), world, device)
    value = whole_job_rate(flops, world, args.steps, total_ms) / 1e12

    # e2e through the public API a user calls for the block, MoELayer.forward
    # (routing order from the router's top-k ids, the same NVFP4 experts, the
    # weighted combine back to [T, H]), with host buffers.  Every step's pinned
    # H2D copy of its inputs (x, top-k ids and weights) and D2H copy of the
    # block's output are inside the timed region; as a server would, the
    # copies run on their own streams (PCIe is full duplex), so step i+1's
    # inputs go up and step i-1's output comes down while step i computes.
    # Inputs and outputs are double-buffered and ordered by events.
    layers = [L.MoELayer(moe, T, k, device) for _ in range(2)]
    ids_host = torch.from_numpy(r["experts"].astype(np.int32)).pin_memory()
    w_host = torch.from_numpy(r["weights"].astype(np.float32)).pin_memory()
    x_host = x.cpu().pin_memory()
    out_host = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(x) for _ in range(2)]
    ids_d = [torch.empty_like(ids_host, device=device) for _ in range(2)]
    w_d = [torch.empty_like(w_host, device=device) for _ in range(2)]
    for lay in layers:                      # the block's own warm-up (routing and combine kernels)
        lay.forward(x, ids_host.to(device), w_host.to(device))
    torch.cuda.synchronize()
    s_up, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    n_e2e = max(4, min(6 * args.steps, 60))       # long enough that pipeline fill and drain amortise
    up_done = [torch.cuda.Event() for _ in range(n_e2e)]
    comp_done = [torch.cuda.Event() for _ in range(n_e2e)]
    down_done = [torch.cuda.Event() for _ in range(n_e2e)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(n_e2e):
        b = i & 1
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(comp_done[i - 2])          # buffer b's last reader is done
            x_d[b].copy_(x_host, non_blocking=True)
            ids_d[b].copy_(ids_host, non_blocking=True)
            w_d[b].copy_(w_host, non_blocking=True)
            up_done[i].record(s_up)
        stream.wait_event(up_done[i])
        if i >= 2:
            stream.wait_event(down_done[i - 2])            # output b has been read back
        out = layers[b].forward(x_d[b], ids_d[b], w_d[b])
        comp_done[i].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[i])
            out_host[b].copy_(out, non_blocking=True)
            down_done[i].record(s_down)
    s_down.wait_event(down_done[n_e2e - 1])
    e1.record(s_down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, device)
    # the floor the copies set alone: the same uploads and read-backs on the same
    # two streams, concurrently, with no compute between them
    out_d = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    down_end = torch.cuda.Event()
    torch.cuda.synchronize()
    c0.record(s_up)
    s_down.wait_event(c0)
    for i in range(n_e2e):
        b = i & 1
        with torch.cuda.stream(s_up):
            x_d[b].copy_(x_host, non_blocking=True)
            ids_d[b].copy_(ids_host, non_blocking=True)
            w_d[b].copy_(w_host, non_blocking=True)
        with torch.cuda.stream(s_down):
            out_host[b].copy_(out_d, non_blocking=True)
    down_end.record(s_down)
    s_up.wait_event(down_end)
    c1.record(s_up)
    torch.cuda.synchronize()
    copies_ms = max_over_ranks(c0.elapsed_time(c1) / n_e2e, world, device)

    h2d = x.numel() * 2 + ids_host.numel() * 4 + w_host.numel() * 4
    d2h = T * H * 2

    med = np.median(per, axis=0)
    g1_ms, g2_ms = float(np.mean(per[:, 1])), float(np.mean(per[:, 3]))
    g1_bytes = gemm_bytes(R, e_touched, 2 * I, H)
    if fused:
        g1_bytes += R * I * 2 - R * 2 * I * 2          # the fused launch writes h [R, I], not [R, 2I]
    g1_flops = 2.0 * R * 2 * I * H
    g2_bytes = gemm_bytes(R, e_touched, H, I)
    g2_flops = 2.0 * R * H * I
    # the other two stages: x read once and R packed rows written; h read and
    # its packed copy written
    q1_bytes = T * H * 2 + R * H * (0.5 + 1 / 16)
    q2_bytes = R * I * 2 + R * I * (0.5 + 1 / 16)
    q1_ms, q2_ms = float(np.mean(per[:, 0])), float(np.mean(per[:, 2]))
    traffic_ratio = gate_up_traffic_ratio()
    kname = grouped_gemm_kernel_name(R, E, 2 * I, H, fused or moe.mid_dtype == 1, fused)
    roof = {"bound": "hbm", "kernel": kname + (": gate_up + SwiGLU epilogue launch" if fused else ": gate_up launch"),
            "achieved": round(gbs(g1_bytes, g1_ms), 1), "peak": HBM_PEAK, "unit": "GB/s",
            "frac": round(gbs(g1_bytes, g1_ms) / HBM_PEAK, 4),
            "traffic": (int(traffic_ratio * g1_bytes) if fused and traffic_ratio else None),
            "traffic_source": (("ncu dram__bytes_read.sum + dram__bytes_write.sum of the gate_up + SwiGLU launch at "
                                f"{GATE_UP_TRAFFIC['capture']}, ratio to algorithmic bytes {traffic_ratio:.3f}, "
                                "scaled by the units processed") if fused and traffic_ratio else
                               "null: no ncu capture of the kernel as built" if fused else None),
            "peak_source": f"{PEAKS_KIND} hbm_gbs (burst copy)",
            "algorithmic_bytes_per_launch": int(g1_bytes), "avg_launch_ms": round(g1_ms, 4),
            "tensor_tflops": round(g1_flops / (g1_ms * 1e-3) / 1e12, 1),
            "pct_fp4_peak": round(100 * g1_flops / (g1_ms * 1e-3) / 1e12 / FP4_PEAK, 2),
            "fp4_peak_tflops": round(FP4_PEAK, 1),
            "fp4_peak_source": f"{PEAKS_KIND} bf16_tflops x 4 (nominal fp4/bf16 ratio)"}
    breakdown = {
        "pipeline": "gate_up GEMM with SwiGLU epilogue" if fused else "gate_up GEMM, then SwiGLU + requantize",
        "dispatch_quantize_ms": round(float(med[0]), 4),
        "dispatch_quantize_gbs": round(gbs(q1_bytes, q1_ms), 1),
        ("gate_up_swiglu_gemm_ms" if fused else "gate_up_gemm_ms"): round(float(med[1]), 4),
        ("requantize_ms" if fused else "swiglu_requantize_ms"): round(float(med[2]), 4),
        "requantize_gbs": round(gbs(q2_bytes, q2_ms), 1),
        "down_gemm_ms": round(float(med[3]), 4),
        "gate_up_gbs": round(gbs(g1_bytes, g1_ms), 1), "gate_up_tflops": round(g1_flops / (g1_ms * 1e-3) / 1e12, 1),
        "down_gbs": round(gbs(g2_bytes, g2_ms), 1), "down_tflops": round(g2_flops / (g2_ms * 1e-3) / 1e12, 1),
        "layer_roofline_ms": round(1e3 * max((q1_bytes + g1_bytes + q2_bytes + g2_bytes) / (HBM_PEAK * 1e9),
                                             flops / (FP4_PEAK * 1e12)), 4),
    }
    workload = f"moe_routed_experts_e{E}_top{k}_t{T}_h{H}_i{I}"
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 e2m1 x e2m1 (e4m3 block scales), fp32 accumulate, bf16 io",
        "data": "synthetic: seeded SplitMix64 / Irwin-Hall N(0,1) activations, N(0,0.02^2) weights, softmax top-10 routing",
        "config": {"workload": workload, "experts": E, "topk": k, "tokens": T, "hidden": H, "intermediate": I,
                   "routed_rows": R, "experts_touched": e_touched, "flops_per_step": flops,
                   "l2": "flushed between steps (256 MB write, outside the timed events)",
                   "parallelism": f"{world} independent replicas" if world > 1 else "single GPU"},
        "roofline": roof,
        "breakdown": breakdown,
        "e2e": {"value": round(whole_job_rate(flops, world, 1, e2e_ms) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_ms, 3),
                "api": "MoELayer.forward: routing order, the NVFP4 experts, weighted combine to [T, H]",
                "steps": n_e2e, "copies": "own streams, overlapping the neighbouring steps' compute",
                "copies_only_ms_per_step": round(copies_ms, 3),
                "copies_only_note": "the same H2D and D2H copies alone, concurrently on the same streams: "
                                    "the floor PCIe sets for ms_per_step"},
        # per step: dispatch (amax, finalize + tables, encode), gate_up, then either
        # requantize (finalize, encode) or SwiGLU + quantize (amax, finalize, encode), down
        "gpu_launches": (7 if fused else 8) * args.steps,
        "clocks": clk,
    }


# --------------------------------------------------------------------------- components
def comp_dense_mlp(device, iters, warmup, flush):
    """Dense MLP of the 64-layer hybrid model, one layer: 4096 tokens, hidden
    5120, intermediate 17408, X with 0.1% outliers x50.  The same stages as the
    MoE layer with one group: quantize X -> gate_up GEMM with the SwiGLU
    epilogue (bf16 h and its amax) -> requantize h with that amax -> down."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import GS_AMAX_GIVEN, nvfp4_quantize
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    M, H, I = 4096, 5120, 17408
    ws = L.workspace(1, device)
    wgu = L.pack_weights(sc.gaussian_bf16(0, synthetic.STREAMS["w_gate_up"], (2 * I, H), sigma=0.02), 1, 2 * I,
                         L.gate_up_interleave_index(1, I, device), ws)
    wd = L.pack_weights(sc.gaussian_bf16(0, synthetic.STREAMS["w_down"], (H, I), sigma=0.02), 1, H, None, ws)
    xb = synthetic.gaussian_bf16(0, synthetic.STREAMS["x"], (M, H), outlier_frac=0.001)
    x = torch.from_numpy(xb.view(np.int16)).to(device).view(torch.bfloat16)
    a1 = L.empty_packed(M, H, 1, None, 1, device)
    a2 = L.empty_packed(M, I, 1, None, 1, device)
    h = torch.empty((M, I), dtype=torch.bfloat16, device=device)
    amax = torch.empty(1, dtype=torch.float32, device=device)
    a2.gs = amax                         # AMAX_GIVEN turns the amax into h's global scale in place
    y2 = torch.empty((M, H), dtype=torch.bfloat16, device=device)
    t = {}

    def q():
        L.quantize(x, layout=1, out=a1, ws=ws)

    def g1():
        L.grouped_gemm_swiglu(a1, wgu, 2 * I, h=h, amax=amax)

    def sq():
        nvfp4_quantize(h, M, I, I, None, None, 1, GS_AMAX_GIVEN, amax, a2.q, a2.sf, 1, ws)

    def g2():
        L.grouped_gemm(a2, wd, H, 1, y=y2)

    def layer():
        q(); g1(); sq(); g2()
    for name, fn in (("quantize", q), ("down", g2), ("layer", layer)):
        t[name] = timed(fn, iters, warmup, flush)
    t["gate_up"] = timed(g1, iters, warmup, flush)
    g1()
    t["requantize"] = timed(sq, iters, warmup, flush)      # sq turns amax into s_g: time it after a fresh g1
    f1, f2 = 2.0 * M * 2 * I * H, 2.0 * M * H * I
    tf = (f1 + f2) / (t["layer"] * 1e-3) / 1e12
    return {"workload": "dense_mlp_t4096_h5120_i17408", "pipeline": "gate_up GEMM with SwiGLU epilogue",
            "layer_ms": round(t["layer"], 4),
            "layer_tflops": round(tf, 1), "pct_fp4_peak": round(100 * tf / FP4_PEAK, 2),
            "gate_up_swiglu_ms": round(t["gate_up"], 4),
            "gate_up_tflops": round(f1 / (t["gate_up"] * 1e-3) / 1e12, 1),
            "gate_up_pct_fp4_peak": round(100 * f1 / (t["gate_up"] * 1e-3) / 1e12 / FP4_PEAK, 2),
            "down_ms": round(t["down"], 4), "down_tflops": round(f2 / (t["down"] * 1e-3) / 1e12, 1),
            "quantize_ms": round(t["quantize"], 4), "requantize_ms": round(t["requantize"], 4),
            "roofline": {"bound": "tensor", "peak_tflops": round(FP4_PEAK, 1),
                         "frac": round(tf / FP4_PEAK, 4)}}


def comp_moe_static_h(device, iters, warmup, flush):
    """The headline MoE layer with a calibrated (given) global for the down
    projection's input: dispatch quantize -> gate_up whose SwiGLU epilogue
    writes NVFP4 h -> down.  The scale comes from one dynamic forward."""
    import torch

    from nvfp4_w4a4_quantized_04_b200 import layer as L
    E, T, H, I, k = 512, 8192, 4096, 1024, 10
    moe, x, ri, off, r, R = setup_moe(device, 0, E, T, H, I, k)
    sl = r["slot_dev"]
    L.calibrate_h_scale(moe, x, ri, off, slot=sl)
    ms = timed(lambda: moe.forward(x, ri, off, slot=sl), iters, warmup, flush)
    a1 = L.moe_quantize(x, sl, off, E, out=moe.a1, ws=moe.ws, rows=R)
    g1 = timed(lambda: L.grouped_gemm_swiglu_nvfp4(a1, moe.w_gate_up, 2 * I, moe.h_scale, out=moe.a2), iters,
               warmup, flush)
    flops = moe_flops(R, H, I)
    e_t = int((np.diff(r["offsets"]) > 0).sum())
    g1_bytes = gemm_bytes(R, e_t, 2 * I, H) - R * 2 * I * 2 + R * I * (0.5 + 1 / 16)
    moe.h_scale = None
    return {"workload": f"moe_routed_experts_e{E}_top{k}_t{T}_h{H}_i{I}_given_down_input_scale",
            "layer_ms": round(ms, 4), "layer_tflops": round(flops / (ms * 1e-3) / 1e12, 1),
            "gate_up_swiglu_nvfp4_ms": round(g1, 4), "gate_up_gbs": round(gbs(g1_bytes, g1), 1),
            "gate_up_frac_hbm": round(gbs(g1_bytes, g1) / HBM_PEAK, 4)}


def comp_decode_moe(device, iters, warmup, flush):
    """Decode MoE: 384 experts, 64 tokens, top-10 Zipf(1.1) routing (seed 7),
    hidden 7168, intermediate 2048, weights generated as MXFP4 and remapped."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    E, T, H, I, k = 384, 64, 7168, 2048, 10
    r = synthetic.route_zipf_gumbel(7, T, E, k)
    R = len(r["row_index"])
    ws = L.workspace(2 * E, device)
    packs, remap_ms, remap_bytes = [], 0.0, 0.0
    for name, rows_per, K in (("gate_up", 2 * I, H), ("down", H, I)):
        n = E * rows_per * K
        q = sc.mxfp4_codes(7, synthetic.STREAMS["mx_codes_" + name], n // 2).view(E * rows_per, K // 2)
        e8 = sc.mxfp4_exponents(7, synthetic.STREAMS["mx_exp_" + name], n // 32, lo=-10)
        if name == "gate_up":
            # checkpoint rows put in the SwiGLU epilogue's gate/up interleaved order
            perm = L.gate_up_interleave_index(E, I, device).long()
            q = q[perm].contiguous()
            e8 = e8.view(E * rows_per, K // 32)[perm].reshape(-1).contiguous()
        qn = torch.empty_like(q)
        sf = torch.empty(n // 16, dtype=torch.uint8, device=device)
        gs = torch.empty(E, dtype=torch.float32, device=device)
        st = torch.zeros(1, dtype=torch.int32, device=device)
        from nvfp4_w4a4_quantized_04_b200 import mxfp4_to_nvfp4

        def remap():
            mxfp4_to_nvfp4(q, e8, E, rows_per, K, qn, sf, 1, gs, ws, st)
        remap_ms += timed(remap, max(2, iters // 2), 1, flush)
        remap_bytes += n * (0.5 + 1 / 32) + n * (0.5 + 1 / 16)
        assert int(st.item()) == 0
        packs.append(L.Packed(qn, sf, gs, E * rows_per, K, 1))
        del q, e8
    xb = sc.gaussian_bf16(7, synthetic.STREAMS["x"], (T, H))
    moe = L.MoEExperts(packs[0], packs[1], E, H, I, max_rows=R, out_dtype=1, mid_dtype=1, device=device,
                       fused_swiglu=True)
    ri = torch.from_numpy(r["row_index"]).to(device)
    off = torch.from_numpy(r["offsets"]).to(device)
    ms = timed(lambda: moe.forward(xb, ri, off), iters, warmup, flush)
    # the activation quantize on its own: the most that folding it into the
    # GEMM's prologue could save
    q_ms = timed(lambda: moe._quantize_input(xb, ri, off, None, None), iters, warmup, flush)
    touched = int((np.diff(r["offsets"]) > 0).sum())
    wbytes = touched * (2 * I * H + H * I) * 0.5625
    # the whole decode block (routing order, experts, weighted combine) through
    # MoELayer, launched eagerly and as one captured CUDA graph
    block = L.MoELayer(moe, T, k, device)
    ids = torch.from_numpy(r["experts"].astype(np.int32)).to(device)
    wts = torch.from_numpy(r["weights"].astype(np.float32)).to(device)
    block_ms = timed(lambda: block.forward(xb, ids, wts), iters, warmup, flush)
    graph, _ = block.capture(xb, ids, wts)
    graph_ms = timed(graph.replay, iters, warmup, flush)
    del graph
    return {"workload": "decode_moe_e384_top10_zipf1.1_t64_h7168_i2048", "experts_touched": touched,
            "routed_rows": R, "layer_ms": round(ms, 4), "activation_quantize_ms": round(q_ms, 4),
            "touched_weight_gbs": round(gbs(wbytes, ms), 1),
            "roofline": {"bound": "hbm", "frac": round(gbs(wbytes, ms) / HBM_PEAK, 4), "peak": HBM_PEAK},
            "block_ms": round(block_ms, 4), "block_graph_ms": round(graph_ms, 4),
            "remap_ms": round(remap_ms, 4), "remap_gbs": round(gbs(remap_bytes, remap_ms), 1)}


def comp_decode_w4a16(device, iters, warmup, flush):
    """W4A16 (NVFP4 weights, bf16 activations) experts at decode size: 384
    experts, 64 tokens, top-10 Zipf(1.1) routing (seed 7), hidden 7168,
    intermediate 2048; gate_up with the SwiGLU epilogue, then down."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    from nvfp4_w4a4_quantized_04_b200 import mxfp4_to_nvfp4
    E, T, H, I, k = 384, 64, 7168, 2048, 10
    r = synthetic.route_zipf_gumbel(7, T, E, k)
    R = len(r["row_index"])
    ws = L.workspace(2 * E, device)
    packs = []
    for name, rows_per, K in (("gate_up", 2 * I, H), ("down", H, I)):
        n = E * rows_per * K
        q = sc.mxfp4_codes(7, synthetic.STREAMS["mx_codes_" + name], n // 2).view(E * rows_per, K // 2)
        e8 = sc.mxfp4_exponents(7, synthetic.STREAMS["mx_exp_" + name], n // 32, lo=-10)
        qn = torch.empty_like(q)
        sf = torch.empty(n // 16, dtype=torch.uint8, device=device)
        gs = torch.empty(E, dtype=torch.float32, device=device)
        st = torch.zeros(1, dtype=torch.int32, device=device)
        mxfp4_to_nvfp4(q, e8, E, rows_per, K, qn, sf, 0, gs, ws, st)   # row-major scales
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        packs.append(L.Packed(qn, sf, gs, E * rows_per, K, 0))
        del q, e8
    xb = sc.gaussian_bf16(7, synthetic.STREAMS["x"], (T, H))
    ri = torch.from_numpy(r["row_index"]).to(device)
    off = torch.from_numpy(r["offsets"]).to(device)
    h = torch.empty((R, I), dtype=torch.bfloat16, device=device)
    y = torch.empty((R, H), dtype=torch.bfloat16, device=device)

    ws = L.w4a16_workspace(R, E, max(H, I), device)

    def layer():
        L.grouped_gemm_w4a16(xb, packs[0], 2 * I, ri, off, E, rows=R, out_dtype=1, swiglu=True, y=h, ws=ws)
        L.grouped_gemm_w4a16(h, packs[1], H, None, off, E, rows=R, out_dtype=1, y=y, ws=ws)
    ms = timed(layer, iters, warmup, flush)
    t_gu = timed(lambda: L.grouped_gemm_w4a16(xb, packs[0], 2 * I, ri, off, E, rows=R, out_dtype=1, swiglu=True,
                                             y=h, ws=ws), iters, warmup, flush)
    touched = int((np.diff(r["offsets"]) > 0).sum())
    wbytes = touched * (2 * I * H + H * I) * 0.5625
    gu_bytes = touched * 2 * I * H * 0.5625
    del packs, ws, h, y
    # Larger groups, where the automatic choice takes the tcgen05 kernel: the
    # same gate_up shape for 64 experts, 2048 tokens top-8 (about 256 tokens
    # per expert), timed on both kernels.
    from nvfp4_w4a4_quantized_04_b200 import nvfp4_w4a16_select_kernel
    nvtx = getattr(torch.cuda, "nvtx", None)
    if nvtx is not None:
        nvtx.range_push("w4a16_groups256")
    E2, T2, k2 = 64, 2048, 8
    r2 = synthetic.route_topk_softmax(5, T2, E2, k2)
    R2 = len(r2["row_index"])
    w2 = sc.gaussian_bf16(5, synthetic.STREAMS["w_gate_up"], (E2 * 2 * I, H), sigma=0.02)
    offs2 = torch.arange(0, (E2 + 1) * 2 * I, 2 * I, dtype=torch.int32, device=device)
    wp2 = L.quantize(w2, None, offs2, E2, 0)
    wp2.offsets, wp2.num_groups, wp2.rows = None, 1, E2 * 2 * I
    del w2
    x2 = sc.gaussian_bf16(5, synthetic.STREAMS["x"], (T2, H))
    ri2 = torch.from_numpy(r2["row_index"]).to(device)
    off2 = torch.from_numpy(r2["offsets"]).to(device)
    h2 = torch.empty((R2, I), dtype=torch.bfloat16, device=device)
    ws2 = L.w4a16_workspace(R2, E2, H, device)
    big = {}
    for mode, name in ((2, "tcgen05"), (1, "warp_mma")):
        nvfp4_w4a16_select_kernel(mode)
        t = timed(lambda: L.grouped_gemm_w4a16(x2, wp2, 2 * I, ri2, off2, E2, rows=R2, out_dtype=1, swiglu=True,
                                               y=h2, ws=ws2), iters, warmup, flush)
        big[name + "_ms"] = round(t, 4)
        big[name + "_tflops"] = round(2.0 * R2 * 2 * I * H / (t * 1e-3) / 1e12, 1)
    nvfp4_w4a16_select_kernel(0)
    if nvtx is not None:
        nvtx.range_pop()
    return {"workload": "decode_w4a16_experts_e384_top10_zipf1.1_t64_h7168_i2048", "experts_touched": touched,
            "routed_rows": R, "layer_ms": round(ms, 4), "touched_weight_gbs": round(gbs(wbytes, ms), 1),
            "gate_up_swiglu_ms": round(t_gu, 4), "gate_up_gbs": round(gbs(gu_bytes, t_gu), 1),
            "kernel": "warp-MMA (automatic choice: at most 16 rows per expert)",
            "roofline": {"bound": "hbm", "frac": round(gbs(wbytes, ms) / HBM_PEAK, 4), "peak": HBM_PEAK},
            "groups256_gate_up": dict(workload="w4a16_gate_up_e64_top8_t2048_h7168_i2048", rows=R2, **big)}


def comp_kv(device, iters, warmup, flush):
    """NVFP4 KV cache for one full-attention layer: K, V [262144 tokens, 4, 256]."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L, nvfp4_kv_dequantize, nvfp4_kv_quantize
    T, Hh, D = 262144, 4, 256
    n = T * Hh * D
    k = sc.gaussian_bf16(0, synthetic.STREAMS["kv_k"], (T * Hh, D))
    v = sc.gaussian_bf16(0, synthetic.STREAMS["kv_v"], (T * Hh, D))
    kq, vq = (torch.empty((T * Hh, D // 2), dtype=torch.uint8, device=device) for _ in range(2))
    ks, vs = (torch.empty(n // 16, dtype=torch.uint8, device=device) for _ in range(2))
    kg, vg = (torch.empty(1, dtype=torch.float32, device=device) for _ in range(2))
    ko, vo = torch.empty_like(k), torch.empty_like(v)
    ws = L.workspace(2, device)
    nvfp4_kv_quantize(k, v, T, Hh, D, 0, kg, vg, kq, ks, vq, vs, ws)
    t_amax = timed(lambda: nvfp4_kv_quantize(k, v, T, Hh, D, 0, kg, vg, kq, ks, vq, vs, ws), iters, warmup, flush)
    t_given = timed(lambda: nvfp4_kv_quantize(k, v, T, Hh, D, 1, kg, vg, kq, ks, vq, vs, ws), iters, warmup, flush)
    t_dq = timed(lambda: nvfp4_kv_dequantize(kq, ks, kg, vq, vs, vg, T, Hh, D, ko, vo), iters, warmup, flush)
    b_given = 2 * n * (2 + 0.5625)
    b_amax = 2 * n * (2 + 2 + 0.5625)
    b_dq = 2 * n * (0.5625 + 2)
    return {"workload": "kv_cache_t262144_h4_d256_k_and_v",
            "quantize_given_scale_ms": round(t_given, 4), "quantize_given_scale_gbs": round(gbs(b_given, t_given), 1),
            "quantize_given_scale_frac_hbm": round(gbs(b_given, t_given) / HBM_PEAK, 4),
            "quantize_amax_ms": round(t_amax, 4), "quantize_amax_gbs": round(gbs(b_amax, t_amax), 1),
            "quantize_amax_frac_hbm": round(gbs(b_amax, t_amax) / HBM_PEAK, 4),
            "dequantize_ms": round(t_dq, 4), "dequantize_gbs": round(gbs(b_dq, t_dq), 1),
            "dequantize_frac_hbm": round(gbs(b_dq, t_dq) / HBM_PEAK, 4)}


def comp_act_sweep(device, iters, warmup, flush):
    """Standalone dynamic activation quantize on [T, 5120] bf16."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    out = {}
    H = 5120
    ws = L.workspace(1, device)
    for T in (1, 64, 1024, 16384, 131072):
        x = sc.gaussian_bf16(0, synthetic.STREAMS["x_sweep"], (T, H))
        p = L.empty_packed(T, H, 1, None, 1, device)
        ms = timed(lambda: L.quantize(x, layout=1, out=p, ws=ws), iters, warmup, flush)
        per_el = 2.5625 if T * H * 2 <= L2_BYTES // 2 else 4.5625
        b = T * H * per_el
        out[f"T{T}"] = {"us": round(ms * 1e3, 2), "gbs": round(gbs(b, ms), 1),
                        "frac_hbm": round(gbs(b, ms) / HBM_PEAK, 4), "bytes_per_element": per_el}
        del x, p
    return out


def comp_gemm_small(device, iters, warmup, flush):
    """The smallest GEMM case, X [128, 512] x W [256, 512] -> fp32 [128, 256]:
    launch- and latency-bound, reported in microseconds (dynamic quantize of X,
    the GEMM, and both back to back)."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    M, N, K = 128, 256, 512
    ws = L.workspace(1, device)
    w = L.pack_weights(sc.gaussian_bf16(0, synthetic.STREAMS["w_gate_up"], (N, K), sigma=0.02), 1, N, None, ws)
    x = sc.gaussian_bf16(0, synthetic.STREAMS["x"], (M, K))
    a = L.empty_packed(M, K, 1, None, 1, device)
    y = torch.empty((M, N), dtype=torch.float32, device=device)
    t_q = timed(lambda: L.quantize(x, layout=1, out=a, ws=ws), iters, warmup, flush)
    t_g = timed(lambda: L.grouped_gemm(a, w, N, 0, y=y), iters, warmup, flush)

    def both():
        L.quantize(x, layout=1, out=a, ws=ws)
        L.grouped_gemm(a, w, N, 0, y=y)
    t_b = timed(both, iters, warmup, flush)
    # the floor of this measurement: a one-element fill timed the same way
    z = torch.empty(1, dtype=torch.float32, device=device)
    t_0 = timed(lambda: z.fill_(1.0), iters, warmup, flush)
    flop = 2.0 * M * N * K
    return {"workload": "gemm_m128_n256_k512_fp32_out", "quantize_us": round(t_q * 1e3, 2),
            "gemm_us": round(t_g * 1e3, 2), "quantize_and_gemm_us": round(t_b * 1e3, 2),
            "one_element_fill_us": round(t_0 * 1e3, 2),
            "gemm_tflops": round(flop / (t_g * 1e-3) / 1e12, 3), "bound": "launch latency"}


def comp_remap(device, iters, warmup, flush):
    """MXFP4 -> NVFP4 remap of 2^28 elements as 1024 tensors of [512, 512]."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L, mxfp4_to_nvfp4
    nt, rows, K = 1024, 512, 512
    n = nt * rows * K
    q = sc.mxfp4_codes(0, synthetic.STREAMS["mx_codes"], n // 2).view(nt * rows, K // 2)
    e8 = sc.mxfp4_exponents(0, synthetic.STREAMS["mx_exp"], n // 32)
    qn = torch.empty_like(q)
    sf = torch.empty(n // 16, dtype=torch.uint8, device=device)
    gs = torch.empty(nt, dtype=torch.float32, device=device)
    ws = L.workspace(nt, device)
    ms = timed(lambda: mxfp4_to_nvfp4(q, e8, nt, rows, K, qn, sf, 1, gs, ws), iters, warmup, flush)
    b = n * (0.5 + 1 / 32) + n * (0.5 + 1 / 16)
    return {"workload": "remap_2^28_as_1024x512x512", "ms": round(ms, 4), "gbs": round(gbs(b, ms), 1),
            "frac_hbm": round(gbs(b, ms) / HBM_PEAK, 4)}


def comp_mxfp4_encode(device, iters, warmup, flush):
    """MXFP4 encode (one UE8M0 scale per 32 elements) of 2^28 bf16 elements as
    [65536, 4096], tensor-core scale layout."""
    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    rows, K = 65536, 4096
    x = sc.gaussian_bf16(0, synthetic.STREAMS["x_sweep"], (rows, K))
    q, e8 = L.mxfp4_quantize(x, layout=1)
    ms = timed(lambda: L.mxfp4_quantize(x, layout=1), iters, warmup, flush)
    n = rows * K
    b = n * (2 + 0.5 + 1 / 32)
    return {"workload": "mxfp4_encode_2^28_as_65536x4096", "ms": round(ms, 4), "gbs": round(gbs(b, ms), 1),
            "frac_hbm": round(gbs(b, ms) / HBM_PEAK, 4), "bytes_per_element": 2 + 0.5 + 1 / 32}


def comp_mx_gemm_routes(device, iters, warmup, flush):
    """MXFP4 weights two ways on the headline gate_up GEMM (512 experts, 81,920
    routed rows, N = 2048, K = 4096): the direct kind::mxf4 grouped GEMM on
    MXFP4 activations, and the NVFP4 grouped GEMM on the losslessly remapped
    weights with NVFP4 activations.  Operands are prepared outside the events;
    only the GEMM launches are timed."""
    import torch

    import synthetic
    import synthetic.cuda as sc
    from nvfp4_w4a4_quantized_04_b200 import layer as L, nvfp4_padded_rows_bound
    E, T, k, N, K = 512, 8192, 10, 2048, 4096
    r = synthetic.route_topk_softmax(0, T, E, k)
    R = len(r["row_index"])
    off = torch.from_numpy(r["offsets"]).to(device)
    bound = nvfp4_padded_rows_bound(R, E)
    # activations already in their 128-aligned expert slots (padding rows hold data too)
    xs = sc.gaussian_bf16(0, synthetic.STREAMS["x"], (bound, K))
    w = sc.gaussian_bf16(0, synthetic.STREAMS["w_gate_up"], (E * N, K), sigma=0.02)
    wq, we_tiled = L.mxfp4_quantize(w, layout=1)
    _, we_rm = L.mxfp4_quantize(w, layout=0)
    del w
    xq, xe = L.mxfp4_quantize(xs, layout=1)
    ws = L.workspace(E, device)
    w_nv = L.remap_mxfp4(wq, we_rm, E, N, K, layout=1, ws=ws)
    a_nv = L.quantize(xs, layout=1, ws=ws)
    a_nv = L.Packed(a_nv.q, a_nv.sf, a_nv.gs.repeat(E), R, K, 1, off, E)
    w_nv = L.Packed(w_nv.q, w_nv.sf, w_nv.gs, E * N, K, 1)
    del xs
    y = torch.empty((R, N), dtype=torch.bfloat16, device=device)
    t_mx = timed(lambda: L.mx_grouped_gemm(xq, xe, wq, we_tiled, N, K, R, off, E, out_dtype=1, y=y),
                 iters, warmup, flush)
    t_nv = timed(lambda: L.grouped_gemm(a_nv, w_nv, N, 1, y=y), iters, warmup, flush)
    touched = int((np.diff(r["offsets"]) > 0).sum())
    w_mx_bytes = touched * N * K * (0.5 + 1 / 32)
    w_nv_bytes = touched * N * K * (0.5 + 1 / 16)
    a_mx, a_nvb = R * K * (0.5 + 1 / 32), R * K * (0.5 + 1 / 16)
    out_b = R * N * 2
    flops = 2.0 * R * N * K
    b_mx, b_nv = w_mx_bytes + a_mx + out_b, w_nv_bytes + a_nvb + out_b
    return {"workload": f"gate_up_e{E}_top{k}_t{T}_n{N}_k{K}",
            "mxfp4_gemm_ms": round(t_mx, 4), "mxfp4_gbs": round(gbs(b_mx, t_mx), 1),
            "mxfp4_frac_hbm": round(gbs(b_mx, t_mx) / HBM_PEAK, 4),
            "mxfp4_tflops": round(flops / (t_mx * 1e-3) / 1e12, 1),
            "remap_nvfp4_gemm_ms": round(t_nv, 4), "remap_nvfp4_gbs": round(gbs(b_nv, t_nv), 1),
            "remap_nvfp4_frac_hbm": round(gbs(b_nv, t_nv) / HBM_PEAK, 4),
            "remap_nvfp4_tflops": round(flops / (t_nv * 1e-3) / 1e12, 1)}


def comp_moe_full(device, iters, warmup, flush):
    """The whole routed-expert block of the headline layer: on-device routing
    order from the router's top-10 ids, the NVFP4 experts, and the weighted
    combine back to [8192, 4096]."""
    import torch

    import synthetic
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    E, T, H, I, k = 512, 8192, 4096, 1024, 10
    moe, x, ri, off, r, R = setup_moe(device, 0, E, T, H, I, k)
    full = L.MoELayer(moe, T, k, device)
    ids = torch.from_numpy(r["experts"].astype(np.int32)).to(device)
    w = torch.from_numpy(r["weights"].astype(np.float32)).to(device)
    t_route = timed(lambda: L.route(ids, E), iters, warmup, flush)
    y2 = moe.forward(x, ri, off)
    sl = r["slot_dev"]                     # the slot map of the routing that ordered y2's rows
    t_comb = timed(lambda: L.combine(y2, sl, w, out_dtype=1, out=full.out[:T]), iters, warmup, flush)
    full.forward(x, ids, w)
    t_full = timed(lambda: full.forward(x, ids, w), iters, warmup, flush)
    flops = moe_flops(R, H, I)
    comb_bytes = R * H * 2 + T * H * 2
    return {"workload": f"moe_block_e{E}_top{k}_t{T}_h{H}_i{I}_route_experts_combine",
            "block_ms": round(t_full, 4), "block_tflops": round(flops / (t_full * 1e-3) / 1e12, 1),
            "route_ms": round(t_route, 4), "combine_ms": round(t_comb, 4),
            "combine_gbs": round(gbs(comb_bytes, t_comb), 1),
            "combine_frac_hbm": round(gbs(comb_bytes, t_comb) / HBM_PEAK, 4)}


COMPONENTS = {"moe_full": comp_moe_full, "moe_static_h": comp_moe_static_h, "dense_mlp": comp_dense_mlp,
              "decode_moe": comp_decode_moe,
              "decode_w4a16": comp_decode_w4a16, "kv_cache": comp_kv,
              "act_quant_sweep": comp_act_sweep, "remap": comp_remap, "mxfp4_encode": comp_mxfp4_encode,
              "mx_gemm_routes": comp_mx_gemm_routes, "gemm_small": comp_gemm_small}


# --------------------------------------------------------------------------- CPU oracle baseline
_SAMPLE_INPUTS = {}


def oracle_sample(seconds: float, seed: int = 0, E=512, T=8192, H=4096, I=1024, k=10):
    """Time the oracle on a bounded sample of the headline workload: whole
    experts (their routed rows) through gather-quantize, fp64 gate_up,
    SwiGLU, requantize and fp64 down, until ``seconds`` of CPU work.
    Returns (TFLOP/s, experts done, rows done, seconds of work)."""
    import oracle
    import synthetic

    key = (seed, E, T, H)
    if key not in _SAMPLE_INPUTS:
        _SAMPLE_INPUTS[key] = (synthetic.route_topk_softmax(seed, T, E, k),
                               synthetic.gaussian_bf16(seed, synthetic.STREAMS["x"], (T, H)))
    r, x = _SAMPLE_INPUTS[key]
    done_flops, experts, rows, t_work = 0.0, 0, 0, 0.0
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


def run_reference(args, world):
    """The oracle as the reference arm (host cores); each step a bounded sample."""
    import oracle
    oracle.build()
    oracle_sample(0.5, E=args.experts, T=args.tokens)
    vals, secs, ne, nr = [], [], 0, 0
    for _ in range(args.steps):
        v, ne, nr, t = oracle_sample(2.0, E=args.experts, T=args.tokens)
        vals.append(v)
        secs.append(t)
    value = statistics.mean(vals)
    workload = f"moe_routed_experts_e{args.experts}_top10_t{args.tokens}_h4096_i1024"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(secs), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic", "config": {"workload": workload},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"whole experts of the same MoE layer until ~2 s of CPU work per step "
                                   f"(last step: {ne} experts, {nr} routed rows)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--experts", type=int, default=512)
    ap.add_argument("--tokens", type=int, default=8192)
    ap.add_argument("--components", default="auto")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="run SwiGLU + requantize as separate kernels instead of the GEMM epilogue")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return

    import torch
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    from nvfp4_w4a4_quantized_04_b200 import build as nvbuild
    nvbuild.build()
    import synthetic.cuda as sc
    sc.build()

    out = run_headline(args, rank, world, device)
    torch.cuda.empty_cache()

    comps = args.components
    if comps == "auto":
        comps = "all" if world == 1 else "none"
    names = list(COMPONENTS) if comps == "all" else ([] if comps == "none" else comps.split(","))
    if names:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        out["components"] = {}
        for n in names:
            # an NVTX range per component, so a profiler can select one
            # component's launches (ncu --nvtx --nvtx-include "<name>/")
            nvtx = getattr(torch.cuda, "nvtx", None)
            try:
                nvtx.range_push(n)
            except Exception:
                nvtx = None
            out["components"][n] = COMPONENTS[n](device, 7, 3, flush)
            if nvtx is not None:
                nvtx.range_pop()
            torch.cuda.empty_cache()

    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        v, ne, nr, t = oracle_sample(12.0, E=args.experts, T=args.tokens)
        out["cpu_baseline"] = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                               "sample": f"{ne} whole experts ({nr} routed rows) of the same layer, "
                                         f"{t:.1f} s of CPU work (gather-quantize, fp64 gate_up, SwiGLU, "
                                         f"requantize, fp64 down)"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
