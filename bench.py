"""Benchmark of the quantized MoE FFN layer forward on B200.

Contract workload: the large-expert layer (H=12288, F=14336, E=128, top-2;
gate/up 4-bit, down 2-bit, group 32 with fp16 scales; 32.4 GB packed) run as
prefill of T=8192 tokens, the largest configuration of the workload set.  One
step = one full layer forward (router, top-k, permute, gather, gate/up GEMM +
SwiGLU, down GEMM, combine) over one batch.  Every other layer and batch of the
set (tiny T=16; Mixtral-like T=1/8/64/2048; hot/cold T=32/4096; NVFP4
T=16/8192; large T=64; graded T=32/4096) is reported under "runs".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (the plain C reference) on the host
cores on a bounded sample of the same workload.  Multi-GPU (torchrun) runs
independent replicas: each rank runs its own batch, no data-path collective.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen.workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
CSRC = os.path.join(ROOT, "mixed_precision_quantized_fp32_b200", "csrc")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def workload_desc(L: W.Layer, T: int, mode: str) -> str:
    f = L.fmt[0]
    return (f"{L.name} layer {mode} T={T} (H={L.H}, F={L.F}, E={L.E}, top-{L.k}, "
            f"gate/up/down {int(f[0])}/{int(f[1])}/{int(f[2])}-bit group-32 fp16 scales)")


def peaks():
    if os.path.exists(PEAKS_FILE):
        d = json.load(open(PEAKS_FILE))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


TRAFFIC_SOURCES = ("expert_gemm_tc.cu", "tc_ptx.cuh", "moe_common.cuh")


def _code_only(src: str) -> str:
    """C/C++ source without comments and with whitespace runs collapsed."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return re.sub(r"\s+", " ", src).strip()


def csrc_hash() -> str:
    """Hash of the code (comments and layout ignored) of the sources that define the
    dominant kernel (the tcgen05 expert GEMM)."""
    h = hashlib.sha256()
    for fn in TRAFFIC_SOURCES:
        h.update(_code_only(open(os.path.join(CSRC, fn)).read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, or None if the
    summary is missing or was taken on different kernel sources."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    if d.get("csrc_hash") != csrc_hash():
        return None
    v = d.get("kernels", {}).get(kernel_key)
    return None if v is None else v.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ replicas (N > 1)
def replica_seed(rank: int) -> int:
    """Seed of rank `rank`'s tokens: every replica runs its own batch of the same layer."""
    return rank


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Max over ranks of a per-rank duration; every rank calls it at the same point."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ CUDA-graph replay
def graph_step_ms(forward, flush, n: int) -> float:
    """Median device time of one forward replayed from a CUDA graph (no host launch
    cost), with L2 flushed before each replay (outside the timed interval)."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        forward()  # first call outside the capture (sets kernel attributes)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        forward()
    torch.cuda.synchronize()
    ts = []
    for _ in range(n + 2):
        if flush is not None:
            flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    del g
    return float(np.median(ts[2:]))


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            self.sel = str(device_index)

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.sel, f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
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
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ our arm
HEADLINE = ("large", 8192)
# (layer, batch, activation format of NVFP4 layers: 0 per-token FP8, 1 NVFP4)
RUNS = [("tiny", 16, 0), ("mixtral", 1, 0), ("mixtral", 8, 0), ("mixtral", 64, 0), ("mixtral", 2048, 0),
        ("hotcold", 32, 0), ("hotcold", 4096, 0), ("nvfp4", 16, 0), ("nvfp4", 8192, 0), ("nvfp4", 16, 1),
        ("nvfp4", 8192, 1), ("large", 64, 0), ("graded", 32, 0), ("graded", 4096, 0)]
FP4_PER_BF16 = 4.0  # dense FP4 / dense bf16 tensor rate (9 / 2.25 PFLOP/s nominal)
STAGES = ["router_topk", "permute", "gather", "gateup", "h_quant", "down", "combine"]


def matrix_bytes(L: W.Layer, e: int, p: int) -> float:
    """Packed bytes (codes + scales) of matrix p of expert e."""
    f = int(L.fmt[e, p])
    n = L.F * L.H
    return n * (4 if f == 16 else f) / 8 + n / 16


def launches_per_forward(L: W.Layer, T: int) -> int:
    """Kernels one forward launches on the prefill (tcgen05) path: router (split of the fp32
    weights + GEMM when T > 64 and E > 32, else one kernel) + top-k, permutation (one kernel
    when T*k <= 1024, else three), activation gather (NVFP4: quantize + gather), gate/up,
    h quantization (NVFP4), down, combine."""
    router = 2 if (T > 64 and L.E > 32) else 1
    perm = 1 if T * L.k <= 1024 else 3
    return router + 1 + perm + (2 if L.fp4 else 1) + 1 + (1 if L.fp4 else 0) + 1 + 1


def gpu_pack(L: W.Layer, moe, dev):
    """Quantize and pack the layer on the GPU through the C ABI, a few experts at a time."""
    import torch
    fmt = np.ascontiguousarray(L.fmt.reshape(-1))
    packed = moe.alloc_packed(moe.pack_layout(L.E, L.H, L.F, fmt)[0], dev)
    per = max(1, min(L.E, (1 << 31) // (3 * L.H * L.F * 4)))
    stage = torch.empty((per, 3, L.H * L.F), dtype=torch.float32, device=dev)
    for e0 in range(0, L.E, per):
        ne = min(per, L.E - e0)
        moe.moe_pack(W.device_expert_weights(L, e0, ne, out=stage[:ne]), e0, L.E, L.H, L.F, fmt, packed)
    torch.cuda.synchronize()
    del stage
    return moe.PackedLayer(L.E, L.H, L.F, fmt, packed)


def measure_batch(L: W.Layer, layer, T: int, moe, dev, pk, flush, n: int, seed: int = 0, act: int = 0):
    """One layer / batch: event-timed forwards (L2 flushed before each decode step) and the
    roofline of its gate/up and down kernels.  Decode batches add CUDA-graph replay.
    act = 1 runs an NVFP4 layer with NVFP4 activations (block-scaled FP4 MMA in prefill)."""
    import torch
    decode = T in L.decode_T
    if act:
        layer = moe.PackedLayer(layer.E, layer.H, layer.F, layer.fmt, layer.packed, act)
    nev = moe.MOE_STAGE_EVENTS
    Wr, b = W.device_router(L)
    x = torch.empty((T, L.H), dtype=torch.bfloat16, device=dev)
    W.fill_device_bf16(x, seed, W.TID_X, 1.0)
    ws = moe.alloc_packed(moe.workspace_bytes(layer, T, L.k), dev)
    y = torch.empty_like(x)
    cnt = torch.zeros(L.E, dtype=torch.int32, device=dev)
    moe.moe_layer_forward(x, Wr, b, layer, L.k, y=y, ws=ws, debug={"counts": cnt})
    torch.cuda.synchronize()
    active = np.nonzero(cnt.cpu().numpy())[0]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(n)]
    for row in ev:
        for e_ in row:
            e_.record()
    for _ in range(3):
        moe.moe_layer_forward(x, Wr, b, layer, L.k, y=y, ws=ws)
    for i in range(n):
        if decode:
            flush.zero_()
        moe.moe_layer_forward(x, Wr, b, layer, L.k, y=y, ws=ws, stage_events=ev[i])
    torch.cuda.synchronize()
    st = np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(nev - 1)] for i in range(n)]).mean(0)
    step = float(np.mean([ev[i][0].elapsed_time(ev[i][-1]) for i in range(n)]))
    gu, dn = float(st[3]), float(st[5])
    mode = "decode" if decode else "prefill"
    desc = workload_desc(L, T, mode) + (", NVFP4 activations" if act else ", FP8 activations" if L.fp4 else "")
    out = {"workload": desc, "layer": L.name, "T": T, "mode": mode, "act": "nvfp4" if act else "fp8" if L.fp4 else None,
           "tokens_per_s": round(T / step * 1e3, 1), "ms_per_step": round(step, 4),
           "active_experts": int(len(active)),
           "stages_ms": dict(zip(STAGES, [round(float(v), 4) for v in st]))}
    if decode:
        gms = graph_step_ms(lambda: moe.moe_layer_forward(x, Wr, b, layer, L.k, y=y, ws=ws), flush, n)
        out["graph_tokens_per_s"] = round(T / gms * 1e3, 1)
        out["graph_ms_per_step"] = round(gms, 4)
        bg = sum(matrix_bytes(L, int(e), 0) + matrix_bytes(L, int(e), 1) for e in active)
        bd = sum(matrix_bytes(L, int(e), 2) for e in active)
        for key, by, t in (("gateup", bg, gu), ("down", bd, dn)):
            out[key] = {"bound": "hbm", "achieved": round(by / t / 1e6, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": round(by / t / 1e6 / pk["hbm_gbs"], 4), "algorithmic_bytes_per_launch": by,
                        "avg_launch_ms": round(t, 4)}
    else:
        fl = 2.0 * T * L.k * L.H * L.F
        peak = pk["bf16_tflops"] * (FP4_PER_BF16 if act else 1.0)
        for key, f, t in (("gateup", 2 * fl, gu), ("down", fl, dn)):
            out[key] = {"bound": "tensor", "achieved": round(f / t / 1e9, 1), "peak": round(peak, 1),
                        "unit": "TFLOP/s", "frac": round(f / t / 1e9 / peak, 4),
                        "algorithmic_flops_per_launch": f, "avg_launch_ms": round(t, 4)}
            if pk.get("bf16_tflops_sustained"):  # the same against the sustained (power-capped) peak
                ps = pk["bf16_tflops_sustained"] * (FP4_PER_BF16 if act else 1.0)
                out[key]["frac_sustained"] = round(f / t / 1e9 / ps, 4)
            if act:
                out[key]["peak_source"] = "measured dense bf16 burst x 4 (nominal FP4/bf16 ratio)"
    del ws, x, y
    return out


def run_ours(args, rank, world, local_rank):
    import torch

    import mixed_precision_quantized_fp32_b200 as moe

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    name, T = HEADLINE
    L = W.layer(name)
    layer = gpu_pack(L, moe, dev)
    x = torch.empty((T, L.H), dtype=torch.bfloat16, device=dev)
    W.fill_device_bf16(x, replica_seed(rank), W.TID_X, 1.0)   # each replica its own tokens
    Wr, b = W.device_router(L)
    ws = moe.alloc_packed(moe.workspace_bytes(layer, T, L.k), dev)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    nev = moe.MOE_STAGE_EVENTS

    def forward(ev=None, xx=x, yy=y):
        return moe.moe_layer_forward(xx, Wr, b, layer, L.k, y=yy, ws=ws, stage_events=ev)

    # ---- device-resident timing
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record()
    for _ in range(args.warmup):
        forward()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.6)  # let the sampler take its first reading before the timed region
    torch.cuda.synchronize()
    for s in range(args.steps):
        forward(evs[s])
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    step_ms = [evs[s][0].elapsed_time(evs[s][-1]) for s in range(args.steps)]
    stage_ms = np.array([[evs[s][i].elapsed_time(evs[s][i + 1]) for i in range(nev - 1)]
                         for s in range(args.steps)])
    total_ms = max_over_ranks(float(sum(step_ms)), world, dev)
    value = job_tokens_per_s(T, args.steps, world, total_ms)

    # ---- end to end through the public API with host buffers (pinned).  Every step
    # copies its own input in and its result out; copy streams (one per direction)
    # overlap step i+1's input copy and step i's output copy with compute, through
    # two device buffers (the usual double-buffered serving loop).
    x_host = [x.cpu().pin_memory(), x.cpu().pin_memory()]
    y_host = [torch.empty_like(x_host[0]).pin_memory(), torch.empty_like(x_host[0]).pin_memory()]
    x_dev = [torch.empty_like(x), torch.empty_like(x)]
    y_dev = [torch.empty_like(x), torch.empty_like(x)]
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e_steps(n):
        done = [None, None]   # compute of the step that last used buffer i
        out_done = [None, None]  # output copy of that step
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(h2d):
                if done[j] is not None:
                    h2d.wait_event(done[j])  # buffer j's previous step has finished reading x
                x_dev[j].copy_(x_host[j], non_blocking=True)
                x_in = torch.cuda.Event()
                x_in.record(h2d)
            stream.wait_event(x_in)
            if out_done[j] is not None:
                stream.wait_event(out_done[j])  # y_dev[j] was copied out before it is overwritten
            forward(xx=x_dev[j], yy=y_dev[j])
            done[j] = torch.cuda.Event()
            done[j].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done[j])
                y_host[j].copy_(y_dev[j], non_blocking=True)
                out_done[j] = torch.cuda.Event()
                out_done[j].record(d2h)
        for ev in out_done:
            if ev is not None:
                stream.wait_event(ev)

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_steps(args.steps)
    e1.record(stream)  # after the last output copy (the compute stream waited for it)
    torch.cuda.synchronize()
    assert torch.equal(y_host[(args.steps - 1) % 2].view(torch.int16), y.cpu().view(torch.int16))
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_tokens_per_s(T, args.steps, world, e2e_ms)

    # ---- roofline of the dominant kernel (gate/up GEMM with the SwiGLU epilogue)
    pk, pk_kind = peaks()
    gateup_ms = float(stage_ms[:, 3].mean())
    down_ms = float(stage_ms[:, 5].mean())
    flops_gateup = 2.0 * T * L.k * 2 * L.H * L.F
    flops_down = 2.0 * T * L.k * L.H * L.F
    achieved = flops_gateup / (gateup_ms / 1e3) / 1e12
    achieved_down = flops_down / (down_ms / 1e3) / 1e12
    # The GEMMs run inside back-to-back steps of tens of milliseconds of tensor-core
    # work, under the 1 kW power cap: the sustained GEMM peak is their denominator
    # (the burst figure is kept beside it).
    sustained = pk.get("bf16_tflops_sustained")
    peak = sustained or pk["bf16_tflops"]
    roofline = {"bound": "tensor", "kernel": "expert GEMM gate/up + SwiGLU (tcgen05, fp16 operands)",
                "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": ncu_traffic(f"gateup_prefill_{name}"),
                "peak_source": (f"{pk_kind} dense bf16 (= fp16) GEMM, sustained (back to back under the power "
                                f"cap), MEASURED_PEAKS.json" if sustained else
                                f"{pk_kind} dense bf16 (= fp16) burst" if pk_kind == "measured"
                                else "fallback 1.59 PFLOP/s"),
                "peak_burst": pk["bf16_tflops"], "frac_burst": round(achieved / pk["bf16_tflops"], 4),
                "algorithmic_flops_per_launch": flops_gateup, "avg_launch_ms": round(gateup_ms, 4),
                "down": {"achieved": round(achieved_down, 2), "frac": round(achieved_down / peak, 4),
                         "frac_burst": round(achieved_down / pk["bf16_tflops"], 4),
                         "avg_launch_ms": round(down_ms, 4),
                         "traffic": ncu_traffic(f"down_prefill_{name}")}}
    stages = dict(zip(STAGES, [round(float(v), 4) for v in stage_ms.mean(0)]))
    del ws, x_dev, y_dev, layer
    torch.cuda.empty_cache()

    # ---- every other layer and batch of the workload set
    runs = []
    if not args.no_runs:
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        done = {}
        for rn, rT, ract in RUNS:
            if rn not in done:
                done.clear()
                torch.cuda.empty_cache()
                done[rn] = gpu_pack(W.layer(rn), moe, dev)
            runs.append(measure_batch(W.layer(rn), done[rn], rT, moe, dev, pk, flush, max(args.steps // 2, 10),
                                      seed=replica_seed(rank), act=ract))
        done.clear()
        del flush
        torch.cuda.empty_cache()

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": {"workload": workload_desc(L, T, "prefill"), "global_batch": T * world,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (32.4 GB packed weights streamed per step)"},
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x.numel() * 2), "d2h_bytes_per_step": int(y.numel() * 2),
                "overlap": "double-buffered: copy streams move step i+1's input and step i-1's output while "
                           "step i computes"},
        "gpu_launches": launches_per_forward(L, T) * args.steps,
        "clocks": clk, "stages_ms": stages, "runs": runs,
    }
    return out


# ------------------------------------------------------------------ all layers (report)
def run_suite(args):
    """Every batch of the named layers: tokens/s and the roofline of the gate/up and down
    kernels, one JSON line per batch."""
    import torch

    import mixed_precision_quantized_fp32_b200 as moe
    dev = torch.device("cuda", 0)
    pk, _ = peaks()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for name in args.suite.split(","):
        L = W.layer(name)
        layer = gpu_pack(L, moe, dev)
        for T in list(L.decode_T) + list(L.prefill_T):
            if args.batch and T != args.batch:
                continue
            act = 1 if (args.act == "nvfp4" and L.fp4) else 0
            if act:
                layer = moe.PackedLayer(layer.E, layer.H, layer.F, layer.fmt, layer.packed, moe.ACT_NVFP4)
            print(json.dumps(measure_batch(L, layer, T, moe, dev, pk, flush, 10, act=act)), flush=True)
        del layer
        torch.cuda.empty_cache()


# ------------------------------------------------------------------ oracle (CPU) timing
class OracleSample:
    """The CPU oracle on a bounded sample (the first n tokens) of a batch."""

    def __init__(self, L: W.Layer, T_full: int, x_seed: int = 0):
        import oracle as orc
        self.orc, self.L, self.T_full = orc, L, T_full
        self.Wr = W.router_w(L.E, L.H)
        self.x_all = W.x_bf16_bits(T_full, L.H, seed=x_seed)
        self.buf = None
        self.packed = set()

    def _prepare(self, n: int):
        orc, L = self.orc, self.L
        xs = np.ascontiguousarray(self.x_all[:n])
        idx = orc.topk_softmax(orc.router(xs, self.Wr, L.bias), L.k)[0]
        for e in sorted(set(np.unique(idx).tolist()) - self.packed):   # oracle packing, untimed
            self.buf = orc.pack_layer(W.expert_w(e, L.H, L.F)[None], e, L.E, L.H, L.F, L.fmt.reshape(-1),
                                      out=self.buf)
            self.packed.add(e)
        return xs

    def step(self, n: int) -> float:
        """Seconds for one oracle forward over the first n tokens."""
        xs = self._prepare(n)
        t0 = time.perf_counter()
        self.orc.moe_forward(self.buf, xs, self.Wr, self.L.bias, self.L.k)
        return time.perf_counter() - t0

    def calibrate(self, budget_s: float) -> int:
        """Smallest doubling of n whose forward takes about budget_s (capped at the batch)."""
        n = 2
        while True:
            dt = self.step(n)
            if dt >= budget_s or n >= self.T_full:
                return n
            n = min(self.T_full, max(n + 1, int(n * min(4.0, 0.9 * budget_s / dt))))

    def describe(self, n: int) -> str:
        return (f"first {n} of {self.T_full} tokens of the same batch, {len(self.packed)} of {self.L.E} experts "
                f"active (oracle packing untimed; the oracle decodes each active expert's rows once per call, "
                f"so with fewer rows per expert than the full batch this rate is a lower bound of its "
                f"full-batch rate)")


def oracle_time(L: W.Layer, T_full: int, budget_s: float, x_seed: int = 0):
    """(tokens/s, sample description, threads) of the oracle on a sample taking ~budget_s."""
    s = OracleSample(L, T_full, x_seed)
    n = s.calibrate(budget_s)
    dt = s.step(n)
    return n / dt, s.describe(n), s.orc.num_threads()


def run_reference(args, rank, world):
    if rank != 0:
        return None
    name, T = HEADLINE
    L = W.layer(name)
    s = OracleSample(L, T)
    n = s.calibrate(max(2.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        s.step(n)
    times = [s.step(n) for _ in range(args.steps)]
    value = n * args.steps / sum(times)
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * sum(times) / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(L, T, "prefill"), "parallelism": "CPU oracle",
                       "step": f"one oracle forward over the {s.describe(n)}"},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": s.orc.num_threads(),
                             "kind": "oracle", "sample": s.describe(n)},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-runs", action="store_true", help="skip the other layers and batches (\"runs\")")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--suite", default="", help="comma-separated layers to report instead of the contract line "
                                                "(tiny,mixtral,hotcold,nvfp4,large,graded)")
    ap.add_argument("--batch", type=int, default=0, help="with --suite: only this batch size")
    ap.add_argument("--act", choices=["fp8", "nvfp4"], default="fp8",
                    help="with --suite: activation format of NVFP4 layers")
    args = ap.parse_args()
    if args.suite:
        run_suite(args)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            v, sample, cores = oracle_time(W.layer(HEADLINE[0]), HEADLINE[1], args.cpu_budget)
            out["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                   "sample": sample}
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
