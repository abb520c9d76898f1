#!/usr/bin/env python
"""Benchmark of the routed-expert MoE layer on B200.

Default workload: one GLM-5.2-shaped MoE layer in decode (H=6144, 256 routed
experts of SwiGLU intermediate 2048 + 1 shared, top-8 softmax routing, batch 1,
all 257 int4 gs64 experts resident in HBM).  A step is one moe_layer_forward
(router + top-k + bucket, fused gate/up + SwiGLU + requant, down + combine) on
one token drawn from a pool of 64 seeded hidden states, so the routed union
varies from step to step.

Metric: expert-weight GB/s of the layer = (|union| + 1) * 20,054,016 bytes per
step / device time of the step (plus us per token-layer and the per-kernel
roofline).  L2 is flushed (256 MiB write) before every timed step, outside the
step's CUDA events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of
the layer on its own tokens (the path has no cross-token exchange), timing is
the max over ranks, value = bytes all ranks streamed / that time ("weak").
--impl reference times the CPU oracle (single thread, plain C) on a bounded
sample of the same workload on this machine's host cores.
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

import torch  # noqa: E402

import moe_inputs as mi  # noqa: E402

METRIC = "MoE layer µs/token & expert-weight GB/s vs HBM peak; prefill int8 TOPS"
POOL = 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 50; tiered: 462 timed tokens, the rest of a 512-token sequence)")
    ap.add_argument("--warmup", type=int, default=None, help="untimed steps (default 5; tiered: 50)")
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "stacked", "tiered"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="oracle sample budget")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--experts", type=int, default=None,
                    help="routed experts per layer (profiling: a small pool, same per-step work)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per layer call: decode 1-16 (default 1), prefill (default 2048)")
    ap.add_argument("--chain", action="store_true",
                    help="stacked workload: each layer's input from the previous layer's output "
                         "(default: hidden states drawn independently per layer and step)")
    ap.add_argument("--path", choices=["auto", "decode"], default="auto",
                    help="decode line: the library's choice (fused kernel) or MOE_PATH_DECODE (union kernels)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="default workload: leave out the prefill sub-object of the line")
    args = ap.parse_args()
    tiered = args.workload == "tiered"
    if args.steps is None:
        args.steps = 462 if tiered else 50
    if args.warmup is None:
        args.warmup = 50 if tiered else 5
    if args.workload == "decode" and args.tokens is not None and not 1 <= args.tokens <= 16:
        ap.error("--tokens: the decode line takes 1 to 16 tokens per call")
    return args


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def profiled_traffic(name: str, source: str):
    """DRAM bytes per launch of a kernel from its committed ncu summary
    (profiles/<name>.md), or None once the kernel's source has changed since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", name + ".md")
    if not os.path.exists(p):
        return None
    traffic, sha = None, None
    for line in open(p):
        if line.startswith("traffic_bytes_per_launch:"):
            traffic = int(line.split(":")[1])
        if line.startswith("source:") and "sha256[:16]" in line:
            sha = line.split()[-1]
    cur = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()[:16]
    return traffic if sha == cur else None


def tensor_peak():
    """Dense fp16/bf16 tensor TFLOP/s (burst) of this machine's B200s: the prefill
    GEMM issues tcgen05.mma kind::f16, so this is its own dtype's peak."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        for k in ("bf16_tflops", "bf16_tflops_burst"):
            if k in d:
                return float(d[k]), "measured"
    return 1590.0, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None

    def __enter__(self):
        try:
            self.f = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- distributed
def dist_setup(backend: str = "nccl"):
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE from the launcher).
    The bench uses NCCL; the CPU tests of this plumbing use gloo."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return ws, rank, local


def rank_seed(w: mi.Workload, rank: int) -> int:
    """Seed of a rank's replica: every rank draws its own router, experts and tokens
    (independent problems; no data-path collective)."""
    return w.seed + 1000 * rank


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(v: float, ws: int, op: str) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def allreduce_max(v: float, ws: int) -> float:
    return _reduce(v, ws, "max")


def allreduce_sum(v: float, ws: int) -> float:
    return _reduce(v, ws, "sum")


def aggregate(my_units: float, my_ms: float, ws: int):
    """Whole-job totals: the units all ranks processed and the slowest rank's
    device time (ms); the job's throughput is their ratio."""
    return allreduce_sum(float(my_units), ws), allreduce_max(float(my_ms), ws)


# ----------------------------------------------------------------- oracle timing
def host_cpu() -> dict:
    """The host the oracle baseline ran on: CPU model and logical CPU count."""
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def decode_config(w: mi.Workload, ws_n: int, path: str = "auto") -> dict:
    """The decode workload's config record (the native and the reference arm print the same)."""
    c = {"workload": f"decode: one GLM-5.2-shaped MoE layer, H={w.H}, {w.E} routed experts x "
                     f"SwiGLU I={w.I} + 1 shared, top-{w.k} softmax, batch {w.T}, all experts resident",
         "H": w.H, "I": w.I, "E": w.E, "k": w.k, "T": w.T, "global_batch": w.T * ws_n,
         "parallelism": f"replicas x{ws_n}", "l2": "flushed (256 MiB write) before each step",
         "x_pool": POOL}
    if path != "auto":
        c["path"] = ("MOE_PATH_DECODE (routing, gate/up and down kernels over the batch union)" if w.T > 1
                     else "MOE_PATH_DECODE (one token: the fused kernel, as on every path)")
    return c


def prefill_config(w: mi.Workload, ws_n: int) -> dict:
    return {"workload": "prefill: one GLM-5.2-shaped MoE layer, 2048 tokens, router biased to Zipf(1.1) "
                        "expert popularity, grouped GEMM over the union",
            "H": w.H, "I": w.I, "E": w.E, "k": w.k, "T": w.T, "global_batch": w.T * ws_n,
            "parallelism": f"replicas x{ws_n}", "l2": "flushed (256 MiB write) before each step"}


def oracle_sample(w: mi.Workload, x_pool, Wr_h, blob_fn, budget_s: float, max_tokens: int):
    """Times the CPU oracle token-layer by token-layer until the budget is spent.
    Returns (bytes, seconds, tokens)."""
    import numpy as np

    import oracle as orc
    blob_bytes = w.blob_bytes
    total_b, total_s, n = 0, 0.0, 0
    cache = {}
    for i in range(max_tokens):
        xt = x_pool[i % len(x_pool)].reshape(1, -1)
        lg = orc.router_logits(xt, Wr_h)
        idx, _ = orc.topk_softmax(lg, w.k)
        need = sorted(set(idx.reshape(-1).tolist()) | {w.E})
        for e in need:
            if e not in cache:
                cache[e] = blob_fn(e)
        dummy = np.zeros(16, np.uint8)
        blist = [cache.get(e, dummy) for e in range(w.E + 1)]
        t0 = time.perf_counter()
        orc.moe_layer(xt, Wr_h, blist, w.H, w.I, w.E, w.k)
        dt = time.perf_counter() - t0
        total_b += len(need) * blob_bytes
        total_s += dt
        n += 1
        if total_s >= budget_s:
            break
    return total_b, total_s, n


# ----------------------------------------------------------------- native arm
def run_native(args, ws_n, rank, local):
    import int4_routed_expert_softmax_b200 as moe

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = mi.WORKLOADS[args.workload]
    if args.experts:
        w = mi.shrink(w, E=args.experts)
    if args.tokens:
        w = mi.shrink(w, T=args.tokens)
    seed = rank_seed(w, rank)
    wl = mi.shrink(w, seed=seed)
    T = w.T
    Wr = mi.make_router(w.E, w.H, mi.sub_seed(seed, 0, 2), dev)
    blobs = mi.make_blobs(w.H, w.I, w.E + 1, mi.sub_seed(seed, 0, 3), dev)
    xpool = mi.make_x(POOL * T, w.H, mi.sub_seed(seed, 0, 1), dev).view(POOL, T, w.H)
    d = moe.dims(w.H, w.I, w.E, w.k)
    path = moe.MOE_PATH_DECODE if args.path == "decode" else moe.MOE_PATH_AUTO
    ws = moe.alloc_workspace(d, T, dev, path=path)
    table = moe.expert_table(blobs)
    out = torch.empty((T, w.H), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    view = moe.moe_workspace_view(d, T, ws)
    nuni_t = moe.ws_slice(ws, view.n_uni, (1,), torch.int32)
    status_t = moe.ws_slice(ws, view.status, (4,), torch.int32)
    blob_b = w.blob_bytes
    gu_b = 2 * mi.matrix_bytes(w.I, w.H)
    dn_b = mi.matrix_bytes(w.H, w.I)
    router_b = w.E * w.H * 4
    stream = torch.cuda.current_stream()

    def step(i):
        moe.moe_layer_forward(d, xpool[i % POOL], Wr, table, out, ws, path=path)

    moe.moe_profile_enable(True)
    for i in range(args.warmup):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    if int(status_t[0].item()) != 0:
        raise RuntimeError(f"device status {status_t.tolist()}")

    K = args.steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    # each step's union size is copied on the device after the step's end
    # event; the host never waits inside the loop
    nuni_hist = torch.zeros(K, dtype=torch.int32, device=dev)
    layer_ms = []
    moe.moe_profile_enable(True)                      # fresh per-call history
    barrier(ws_n)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.zero_()
            ev0[i].record(stream)
            step(args.warmup + i)
            ev1[i].record(stream)
            nuni_hist[i:i + 1].copy_(nuni_t)
        torch.cuda.synchronize()
    barrier(ws_n)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    for i in range(K):
        layer_ms.append(ev0[i].elapsed_time(ev1[i]))
    prof = moe.moe_profile_read(K)
    moe.moe_profile_enable(False)
    nuni = [int(u) for u in nuni_hist.tolist()]
    if len(prof) != K:
        raise RuntimeError(f"profiled {len(prof)} of {K} calls")
    if int(status_t[0].item()) != 0:
        raise RuntimeError(f"device status {status_t.tolist()}")

    my_bytes = sum((u + 1) * blob_b for u in nuni)
    my_ms = sum(layer_ms)
    all_bytes, max_ms = aggregate(my_bytes, my_ms, ws_n)
    value = all_bytes / (max_ms * 1e-3) / 1e9
    ms_per_step = max_ms / K

    launches = moe.moe_layer_launches(d, T, path)
    fused = launches == 1
    rt_ms = sum(p[0] for p in prof)
    gu_ms = sum(p[1] for p in prof)
    dn_ms = sum(p[2] for p in prof)
    call_ms = sum(p[3] for p in prof)
    gu_bytes = sum((u + 1) * gu_b for u in nuni)
    dn_bytes = sum((u + 1) * dn_b for u in nuni)
    x_b = T * w.H * 4
    peak, peak_src = peaks()
    gbs = lambda b, ms: b / (ms * 1e-3) / 1e9
    # the expert FFN span: from routing's end (the union known) to the last output
    ffn_ms = call_ms - rt_ms
    ffn = {"bytes_per_launch": round(my_bytes / K), "us": round(ffn_ms / K * 1e3, 2),
           "achieved": round(gbs(my_bytes, ffn_ms), 1), "frac": round(gbs(my_bytes, ffn_ms) / peak, 4),
           "what": "expert bytes ((|U|+1) blobs) / device time from the union known to the last output"}
    if fused:
        # one token: k_decode_fused1; 2-16 tokens: k_decode_fused, which streams
        # each token's k + 1 blobs in turn (the algorithmic bytes count every
        # union expert once, as the union kernels read it)
        kname = "k_decode_fused1" if T == 1 else "k_decode_fused"
        launch_b = my_bytes + K * (router_b + x_b)
        roofline = {"bound": "hbm", "kernel": kname, "achieved": round(gbs(launch_b, call_ms), 1),
                    "peak": peak, "unit": "GB/s", "frac": round(gbs(launch_b, call_ms) / peak, 4),
                    "peak_source": peak_src,
                    "traffic": profiled_traffic(f"{kname}_glm_T{T}",
                                                "int4_routed_expert_softmax_b200/csrc/moe_fused.cu"),
                    "bytes_per_launch": round(launch_b / K), "us_per_launch": round(call_ms / K * 1e3, 2),
                    "bytes_what": "(|U|+1) x 20,054,016 expert bytes + E x H x 4 router bytes + x",
                    "ffn": ffn}
        if T > 1:
            roofline["streamed_bytes_per_launch"] = T * (w.k + 1) * blob_b + router_b + x_b
        kernels = {
            kname: {"us": round(call_ms / K * 1e3, 2), "GB/s": round(gbs(launch_b, call_ms), 1)},
            "phases_us": {"routing": round(rt_ms / K * 1e3, 2), "gate_up": round(gu_ms / K * 1e3, 2),
                          "down": round(dn_ms / K * 1e3, 2)},
            "timing": "device %globaltimer stamps per phase of the one kernel (first CTA start, last CTA end): "
                      "routing to the union known, gate/up stages, down stages and combine",
        }
    else:
        roofline = {"bound": "hbm", "kernel": "k_gateup_decode", "achieved": round(gbs(gu_bytes, gu_ms), 1),
                    "peak": peak, "unit": "GB/s", "frac": round(gbs(gu_bytes, gu_ms) / peak, 4),
                    "peak_source": peak_src,
                    "traffic": profiled_traffic(f"k_gateup_decode_glm_T{T}",
                                                "int4_routed_expert_softmax_b200/csrc/moe_decode.cu"),
                    "bytes_per_launch": round(gu_bytes / K), "us_per_launch": round(gu_ms / K * 1e3, 2),
                    "down": {"achieved": round(gbs(dn_bytes, dn_ms), 1),
                             "frac": round(gbs(dn_bytes, dn_ms) / peak, 4)},
                    "ffn": ffn}
        kernels = {
            "k_route_decode": {"us": round(rt_ms / K * 1e3, 2), "GB/s": round(gbs(router_b * K, rt_ms), 1)},
            "k_gateup_decode": {"us": round(gu_ms / K * 1e3, 2), "GB/s": round(gbs(gu_bytes, gu_ms), 1)},
            "k_down_decode": {"us": round(dn_ms / K * 1e3, 2), "GB/s": round(gbs(dn_bytes, dn_ms), 1)},
            "call_span": {"us": round(call_ms / K * 1e3, 2)},
            "timing": "device %globaltimer stamps per kernel phase (first CTA start, last CTA end); "
                      "gate/up from its dependency wait, down from its first CTA (overlaps gate/up's tail)",
        }

    # ---- end to end: host buffers through moe_layer_forward_host
    e2e = None
    if not args.no_e2e:
        xh = xpool.cpu().pin_memory()
        oh = torch.empty((T, w.H), dtype=torch.float32).pin_memory()
        for i in range(args.warmup):
            moe.moe_layer_forward_host(d, xh[i % POOL], Wr, table, oh, ws, path=path)
        torch.cuda.synchronize()
        e_ms, e_bytes = 0.0, 0
        barrier(ws_n)
        torch.cuda.synchronize()
        for i in range(K):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            moe.moe_layer_forward_host(d, xh[(args.warmup + i) % POOL], Wr, table, oh, ws, path=path)
            b.record(stream)
            b.synchronize()
            e_ms += a.elapsed_time(b)
            e_bytes += (int(nuni_t.item()) + 1) * blob_b
        barrier(ws_n)
        e_max = allreduce_max(e_ms, ws_n)
        e_all = allreduce_sum(float(e_bytes), ws_n)
        e2e = {"value": round(e_all / (e_max * 1e-3) / 1e9, 1), "unit": "GB/s",
               "h2d_bytes_per_step": T * w.H * 4, "d2h_bytes_per_step": T * w.H * 4,
               "us_per_token_layer": round(e_max / K / T * 1e3, 2)}

    # ---- CPU oracle baseline (rank 0, single GPU only)
    cpu = None
    if rank == 0 and ws_n == 1 and not args.no_cpu:
        xh = xpool.cpu().numpy()
        Wr_h = Wr.cpu().numpy()
        nb, ns, nt = oracle_sample(w, xh.reshape(POOL * T, w.H), Wr_h,
                                   lambda e: blobs[e].cpu().numpy(), args.cpu_seconds, 64)
        cpu = {"value": round(nb / ns / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", **host_cpu(),
               "us_per_token_layer": round(ns / nt * 1e6, 1),
               "sample": f"{nt} token-layers of the decode workload (pool draws 0..{nt - 1}), "
                         f"single-threaded C oracle"}

    clocks = clk.summary()
    return dict(
        metric=METRIC, value=round(value, 1), unit="GB/s", n_gpus=ws_n, steps=K, warmup=args.warmup,
        ms_per_step=round(ms_per_step, 5), higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype="int4xint8->fp32", data="synthetic",
        config=decode_config(w, ws_n, args.path),
        us_per_token_layer=round(ms_per_step / T * 1e3, 2),
        union_mean=round(sum(nuni) / len(nuni), 2),
        roofline=roofline, kernels=kernels, e2e=e2e, cpu_baseline=cpu, clocks=clocks,
        gpu_launches=launches * K, wall_s=round(wall, 3))


# ----------------------------------------------------------------- prefill
def prefill_ops(w: mi.Workload, T: int) -> float:
    """Algorithmic int8 multiply-adds x 2 of one prefill layer: every (token,
    slot) pair, routed and shared, through gate, up and down."""
    return 2.0 * T * (w.k + 1) * 3 * w.H * w.I


def attainable(ops: float, n_union: int, blob_bytes: int, hbm_gbs: float, fp16_tflops: float,
               ms_per_layer: float) -> dict:
    """The prefill layer's attainable floor: the slower of its expert bytes (the
    union plus the shared expert, each read once) at the HBM copy peak and its
    int8 operations at the int8 peak, taken as twice the fp16/bf16 peak (the
    nominal dense ratio); and the measured layer time as a fraction of it."""
    hbm_us = (n_union + 1) * blob_bytes / (hbm_gbs * 1e9) * 1e6
    int8_us = ops / (2.0 * fp16_tflops * 1e12) * 1e6
    floor = max(hbm_us, int8_us)
    return {"floor_us": round(floor, 1), "hbm_floor_us": round(hbm_us, 1), "int8_floor_us": round(int8_us, 1),
            "bound": "hbm" if hbm_us >= int8_us else "tensor", "frac": round(floor / (ms_per_layer * 1e3), 4)}


def run_prefill(args, ws_n, rank, local):
    import int4_routed_expert_softmax_b200 as moe

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = mi.WORKLOADS["prefill"]
    if args.experts:
        w = mi.shrink(w, E=args.experts)
    seed = rank_seed(w, rank)
    T = args.tokens or w.T
    x = mi.make_x(T, w.H, mi.sub_seed(seed, 0, 1), dev, zipf=True)
    Wr = mi.make_router(w.E, w.H, mi.sub_seed(seed, 0, 2), dev, zipf_s=w.zipf_s)
    blobs = mi.make_blobs(w.H, w.I, w.E + 1, mi.sub_seed(seed, 0, 3), dev)
    d = moe.dims(w.H, w.I, w.E, w.k)
    ws = moe.alloc_workspace(d, T, dev, path=moe.MOE_PATH_PREFILL)
    table = moe.expert_table(blobs)
    out = torch.empty((T, w.H), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    view = moe.moe_workspace_view(d, T, ws)
    nuni_t = moe.ws_slice(ws, view.n_uni, (1,), torch.int32)
    status_t = moe.ws_slice(ws, view.status, (4,), torch.int32)
    stream = torch.cuda.current_stream()
    PF = moe.MOE_PATH_PREFILL

    def step():
        moe.moe_layer_forward(d, x, Wr, table, out, ws, path=PF)

    moe.moe_profile_enable(True)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if int(status_t[0].item()) != 0:
        raise RuntimeError(f"device status {status_t.tolist()}")
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    moe.moe_profile_enable(True)                      # fresh per-call history
    barrier(ws_n)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(ws_n)
    prof = moe.moe_profile_read(K)
    moe.moe_profile_enable(False)
    if len(prof) != K:
        raise RuntimeError(f"profiled {len(prof)} of {K} calls")
    if int(status_t[0].item()) != 0:
        raise RuntimeError(f"device status {status_t.tolist()}")
    my_ms = sum(a.elapsed_time(b) for a, b in ev)
    max_ms = allreduce_max(my_ms, ws_n)
    ops = prefill_ops(w, T)
    value = ops * K * ws_n / (max_ms * 1e-3) / 1e12
    rt_ms = sum(p[0] for p in prof) / K
    gu_ms = sum(p[1] for p in prof) / K
    dn_ms = sum(p[2] for p in prof) / K
    peak, src = tensor_peak()
    gu_ops = 2.0 * T * (w.k + 1) * 2 * w.H * w.I
    gu_tflops = gu_ops / (gu_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "k_gemm_pf<0> (gate/up)", "achieved": round(gu_tflops, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(gu_tflops / peak, 4), "peak_source": src,
                "peak_dtype": "fp16/bf16 dense (the kernel's tcgen05 kind::f16)",
                "frac_of_int8_peak": round(gu_tflops / (2 * peak), 4), "traffic": None,
                "ops_per_launch": gu_ops, "us_per_launch": round(gu_ms * 1e3, 1)}
    kernels = {"route+bucket+gathers": {"us": round(rt_ms * 1e3, 1)},
               "k_gemm_pf<0> gate/up": {"us": round(gu_ms * 1e3, 1), "TFLOP/s": round(gu_tflops, 2)},
               "k_gemm_pf<1> down + combine": {"us": round(dn_ms * 1e3, 1),
                                               "TFLOP/s": round(2.0 * T * (w.k + 1) * w.H * w.I / (dn_ms * 1e-3) / 1e12, 2)}}
    e2e = None
    if not args.no_e2e:
        xh = x.cpu().pin_memory()
        oh = torch.empty((T, w.H), dtype=torch.float32).pin_memory()
        for _ in range(min(2, args.warmup)):
            moe.moe_layer_forward_host(d, xh, Wr, table, oh, ws, path=PF)
        torch.cuda.synchronize()
        e_ms = 0.0
        barrier(ws_n)
        for _ in range(K):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            moe.moe_layer_forward_host(d, xh, Wr, table, oh, ws, path=PF)
            b.record(stream)
            b.synchronize()
            e_ms += a.elapsed_time(b)
        e_max = allreduce_max(e_ms, ws_n)
        e2e = {"value": round(ops * K * ws_n / (e_max * 1e-3) / 1e12, 2), "unit": "TOPS",
               "h2d_bytes_per_step": T * w.H * 4, "d2h_bytes_per_step": T * w.H * 4}
    cpu = None
    if rank == 0 and ws_n == 1 and not args.no_cpu:
        cpu = oracle_prefill_sample(w, x.cpu().numpy(), Wr.cpu().numpy(), lambda e: blobs[e].cpu().numpy(),
                                    args.cpu_seconds)
    n_u = int(nuni_t.item())
    cnt = moe.ws_slice(ws, view.cnt, (w.E,), torch.int32).cpu()
    nz = cnt[cnt > 0]
    counts = {"union": n_u, "top": int(nz.max()), "median": float(nz.float().median()), "min": int(nz.min()),
              "rows": int(nz.sum()) + T}
    return dict(
        metric=METRIC, value=round(value, 2), unit="TOPS", n_gpus=ws_n, steps=K, warmup=args.warmup,
        ms_per_step=round(max_ms / K, 4), higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype="int4xint8->fp32 (tensor cores: int4 weights exact in fp16 x an fp16 hi/lo split of the "
              "dequantised int8 activations, fp32 accumulation)", data="synthetic",
        config=prefill_config(w, ws_n),
        union=n_u, routing_counts=counts, us_per_token_layer=round(max_ms / K / T * 1e3, 3),
        attainable=attainable(ops, n_u, w.blob_bytes, peaks()[0], peak, max_ms / K),
        roofline=roofline, kernels=kernels, e2e=e2e, cpu_baseline=cpu, clocks=clk.summary(),
        gpu_launches=moe.moe_layer_launches(d, T, PF) * K)


def prefill_summary(args, rank, local) -> dict:
    """The prefill layer (2048 tokens, Zipf(1.1) routing) as a sub-object of the
    default line: a short run of its own (3 warm-up, 5 timed steps), with the
    oracle timed on sampled tokens."""
    a = argparse.Namespace(**vars(args))
    a.workload, a.steps, a.warmup, a.experts, a.tokens = "prefill", 5, 3, None, None
    a.cpu_seconds = min(args.cpu_seconds, 10.0)
    r = run_prefill(a, 1, rank, local)
    peak, _ = tensor_peak()
    return {"metric": "prefill layer int8-equivalent TOPS", "value": r["value"], "unit": "TOPS",
            "ms_per_step": r["ms_per_step"], "steps": a.steps, "warmup": a.warmup,
            "frac_of_fp16_peak": round(r["value"] / peak, 4), "frac_of_int8_peak": round(r["value"] / (2 * peak), 4),
            "peak_tflops_fp16": peak, "attainable": r["attainable"], "roofline": r["roofline"],
            "kernels": r["kernels"], "e2e": r["e2e"], "cpu_baseline": r["cpu_baseline"], "dtype": r["dtype"],
            "config": r["config"], "union": r["union"], "routing_counts": r["routing_counts"],
            "clocks": r["clocks"], "gpu_launches": r["gpu_launches"]}


def oracle_prefill_sample(w, x_h, Wr_h, blob_fn, budget_s: float, tokens_max: int = 64):
    """The oracle on sampled tokens of the prefill batch, until the budget is
    spent; returns the cpu_baseline record in TOPS (same op count per token)."""
    import numpy as np

    import oracle as orc
    lg = orc.router_logits(x_h[:tokens_max], Wr_h)
    idx, _ = orc.topk_softmax(lg, w.k)
    cache = {}
    spent, n = 0.0, 0
    for t in range(tokens_max):
        need = sorted(set(idx[t].tolist()) | {w.E})
        for e in need:
            if e not in cache:
                cache[e] = blob_fn(e)
        dummy = np.zeros(16, np.uint8)
        blist = [cache.get(e, dummy) for e in range(w.E + 1)]
        t0 = time.perf_counter()
        orc.moe_layer_tokens(x_h, Wr_h, blist, w.H, w.I, w.E, w.k, [t])
        spent += time.perf_counter() - t0
        n += 1
        if spent >= budget_s:
            break
    return {"value": round(prefill_ops(w, n) / spent / 1e12, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
            **host_cpu(), "sample": f"{n} tokens of the prefill batch (tokens 0..{n - 1}), single-threaded C oracle, "
                      f"{spent:.1f} s"}


# ----------------------------------------------------------------- stacked and tiered
def chain_next_dev(x: torch.Tensor, out: torch.Tensor, gamma: float = 0.5, zipf: bool = False) -> torch.Tensor:
    """Input of the next layer (workload glue between layers, outside every
    timed region): v = x + gamma * out / rms(out); x' = v / rms(v)."""
    ro = out.double().pow(2).mean(-1, keepdim=True).sqrt().float()
    ro = torch.where(ro > 0, ro, torch.ones_like(ro))
    v = x + gamma * out / ro
    nx = v / (v.double().pow(2).mean(-1, keepdim=True) + 1e-12).sqrt().float()
    if zipf:
        nx[..., 0] = 1.0
    return nx.contiguous()


def run_stacked(args, ws_n, rank, local):
    """8 stacked GLM-5.2-shaped layers resident in HBM; batches of 1, 2, 3, 4 and
    16 tokens (2-3: draft-verification sizes) with hidden states N(0, 1) drawn
    independently per layer and step (so the union per layer spans 8 to 128),
    or with --chain each layer's input made from the previous layer's output;
    per-layer us and union-weighted expert GB/s."""
    import int4_routed_expert_softmax_b200 as moe
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = mi.WORKLOADS["stacked"]
    seed = rank_seed(w, rank)
    L = w.layers
    routers = [mi.make_router(w.E, w.H, mi.sub_seed(seed, l, 2), dev) for l in range(L)]
    blobs = [mi.make_blobs(w.H, w.I, w.E + 1, mi.sub_seed(seed, l, 3), dev) for l in range(L)]
    tables = [moe.expert_table(b) for b in blobs]
    d = moe.dims(w.H, w.I, w.E, w.k)
    stream = torch.cuda.current_stream()
    res, tot_b, tot_ms = {}, 0.0, 0.0
    with ClockSampler(local) as clk:
        for T in w.T_list:
            ws = moe.alloc_workspace(d, T, dev)
            view = moe.moe_workspace_view(d, T, ws)
            nuni_t = moe.ws_slice(ws, view.n_uni, (1,), torch.int32)
            x_bufs = [mi.make_x(T, w.H, mi.sub_seed(seed, 100, 1 + l), dev).clone() for l in range(L)]
            outs = [torch.empty((T, w.H), dtype=torch.float32, device=dev) for _ in range(L)]
            layer_ms, layer_b = [], []
            # One step (the L layers, with --chain the glue between them, a copy
            # of each layer's union size) is one CUDA graph, with an event pair
            # around every layer call: Python between the layers would otherwise
            # leave the GPU waiting for the host.  Read once per step.
            nuni_hist = torch.zeros(L, dtype=torch.int32, device=dev)
            evs = [(torch.cuda.Event(enable_timing=True, external=True),
                    torch.cuda.Event(enable_timing=True, external=True)) for _ in range(L)]
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):  # the library's one-time setup, outside the capture
                moe.moe_layer_forward(d, x_bufs[0], routers[0], tables[0], outs[0], ws)
            stream.wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                gs = torch.cuda.current_stream()
                x = x_bufs[0]
                for l in range(L):
                    if not args.chain:
                        x = x_bufs[l]
                    evs[l][0].record(gs)
                    moe.moe_layer_forward(d, x, routers[l], tables[l], outs[l], ws)
                    evs[l][1].record(gs)
                    nuni_hist[l:l + 1].copy_(nuni_t)
                    if args.chain:
                        x = chain_next_dev(x, outs[l])
            for it in range(args.warmup + args.steps):
                for l in range(1 if args.chain else L):
                    x_bufs[l].copy_(mi.make_x(T, w.H, mi.sub_seed(seed, 100 + it, 1 + l), dev))
                graph.replay()
                torch.cuda.synchronize()
                if it >= args.warmup:
                    for a, b in evs:
                        layer_ms.append(a.elapsed_time(b))
                    layer_b.extend((int(u) + 1) * w.blob_bytes for u in nuni_hist.tolist())
            del graph
            ms = allreduce_max(sum(layer_ms), ws_n)
            bts = allreduce_sum(float(sum(layer_b)), ws_n)
            res[f"T={T}"] = {"us_per_layer": round(ms / len(layer_ms) * 1e3, 2),
                             "us_per_token_layer": round(ms / len(layer_ms) / T * 1e3, 2),
                             "union_mean": round(sum(layer_b) / len(layer_b) / w.blob_bytes - 1, 1),
                             "GB/s": round(bts / (ms * 1e-3) / 1e9, 1)}
            tot_b += bts
            tot_ms += ms
    value = tot_b / (tot_ms * 1e-3) / 1e9
    return dict(metric=METRIC, value=round(value, 1), unit="GB/s", n_gpus=ws_n, steps=args.steps,
                warmup=args.warmup, ms_per_step=round(tot_ms / args.steps, 4), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="int4xint8->fp32", data="synthetic",
                config={"workload": "stacked: 8 GLM-5.2-shaped layers resident in HBM (41.2 GB), batches of "
                                    + ", ".join(str(t) for t in w.T_list) + " tokens, "
                                    + ("layers chained (each layer's input from the previous output)" if args.chain
                                       else "hidden states N(0,1) drawn independently per layer and step"),
                        "layers": L, "T_list": list(w.T_list),
                        "parallelism": f"replicas x{ws_n}", "l2": "each layer streams its own experts (> L2)",
                        "timing": "one CUDA graph per step (layers, glue if chained, union-size copies), "
                                  "CUDA events around each layer call inside it"},
                by_batch=res, clocks=clk.summary(),
                gpu_launches=sum(moe.moe_layer_launches(d, T) for T in w.T_list) * L * args.steps)


def run_tiered(args, ws_n, rank, local):
    """16 GLM-5.2-shaped layers in pinned host memory, 20 GB HBM expert cache
    (LRU + pins learned from route counts + one-layer-ahead prefetch), 512
    decode tokens with Zipf(1.1) routing persisting token to token."""
    import numpy as np  # noqa: F401

    import int4_routed_expert_softmax_b200 as moe
    from int4_routed_expert_softmax_b200 import _cache as C
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = mi.WORKLOADS["tiered"]
    seed = rank_seed(w, rank)
    L, E1 = w.layers, w.E + 1
    n_tok = args.steps
    host = torch.empty((L, E1, w.blob_bytes), dtype=torch.uint8, pin_memory=True)
    for l in range(L):
        host[l].copy_(mi.make_blobs(w.H, w.I, E1, mi.sub_seed(seed, l, 3), dev), non_blocking=False)
    routers = [mi.make_router(w.E, w.H, mi.sub_seed(seed, l, 2), dev, zipf_s=w.zipf_s) for l in range(L)]
    torch.cuda.synchronize()
    d = moe.dims(w.H, w.I, w.E, w.k)
    cache = C.ExpertCache(d, L, [[host[l, e] for e in range(E1)] for l in range(L)], w.cache_bytes)
    ws = moe.alloc_workspace(d, 1, dev)
    ws_pred = moe.alloc_workspace(d, 1, dev)
    out = torch.empty((1, w.H), dtype=torch.float32, device=dev)
    counts = [torch.zeros(w.E, dtype=torch.int32, device=dev) for _ in range(L)]
    side = torch.cuda.Stream(device=dev)
    stream = torch.cuda.current_stream()
    xs = mi.make_x(args.warmup + n_tok, w.H, mi.sub_seed(seed, 0, 1), dev, zipf=True, rho=w.rho)
    # the glue between layers (x_{l+1} = RMS-normalised x_l + gamma out_l, not
    # part of the MoE layer) as one CUDA graph on fixed buffers, so that its
    # launches cost one replay per layer
    x_buf = xs[0:1].clone()
    for _ in range(2):
        x_buf.copy_(chain_next_dev(x_buf, out, zipf=True))
    torch.cuda.synchronize()
    glue = torch.cuda.CUDAGraph()
    with torch.cuda.graph(glue):
        x_buf.copy_(chain_next_dev(x_buf, out, zipf=True))
    host_s = {"layer_call": 0.0, "glue": 0.0}

    def token(t, timed=False):
        x_buf.copy_(xs[t:t + 1])
        for l in range(L):
            h0 = time.perf_counter()
            cache.tiered_layer_forward(l, x_buf, routers[l], out, ws, ws_pred=ws_pred,
                                       Wr_next=routers[l + 1] if l + 1 < L else None,
                                       route_counts=counts[l], side_stream=side)
            h1 = time.perf_counter()
            glue.replay()
            if timed:
                host_s["layer_call"] += h1 - h0
                host_s["glue"] += time.perf_counter() - h1

    for t in range(args.warmup):
        token(t)
    # pins learned from the warm-up's route counts
    n_pin = max(0, min(cache.stats()["slots_per_layer"] - (w.k + 1) - 8, w.E // 4))
    for l in range(L):
        cache.learn_pins(l, counts[l].cpu().tolist(), n_pin)
    torch.cuda.synchronize()
    s0 = cache.stats()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    moe.moe_profile_enable(True)   # per layer call: routing, gate/up, down, first start to last end
    barrier(ws_n)
    with ClockSampler(local) as clk:
        a.record(stream)
        for t in range(args.warmup, args.warmup + n_tok):
            token(t, timed=True)
        b.record(stream)
        torch.cuda.synchronize()
    ms = allreduce_max(a.elapsed_time(b), ws_n)
    prof = moe.moe_profile_read(1024)
    moe.moe_profile_enable(False)
    device_us = {name: round(sum(p[i] for p in prof) / max(1, len(prof)) * 1e3, 2)
                 for i, name in enumerate(("routing", "gate_up", "down", "call_span"))}
    s1 = cache.stats()
    dd = {k: s1[k] - s0[k] for k in ("hits", "misses", "prefetches", "prefetch_hits", "bytes_h2d", "evictions")}
    # host link alone: one 20 MB blob copy, pinned host -> HBM
    blob_dev = torch.empty(w.blob_bytes, dtype=torch.uint8, device=dev)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(20):
        blob_dev.copy_(host[0, 0], non_blocking=True)
    c1.record(stream)
    torch.cuda.synchronize()
    link = 20 * w.blob_bytes / (c0.elapsed_time(c1) * 1e-3) / 1e9
    tok_s = n_tok * ws_n / (ms * 1e-3)
    lookups = dd["hits"] + dd["misses"]
    cache.close()
    return dict(metric=METRIC, value=round(tok_s, 2), unit="tok/s", n_gpus=ws_n, steps=n_tok,
                warmup=args.warmup, ms_per_step=round(ms / n_tok, 3), higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="int4xint8->fp32", data="synthetic",
                config={"workload": "tiered: 16 GLM-5.2-shaped layers (82.5 GB) in pinned host memory, HBM cache "
                                    "20 GB, LRU + learned pins + one-layer-ahead prefetch, decode tokens with "
                                    "Zipf(1.1) routing persisting token to token (rho 0.9)",
                        "layers": L, "cache_bytes": w.cache_bytes, "tokens_timed": n_tok,
                        "pins_per_layer": n_pin, "parallelism": f"replicas x{ws_n}"},
                hit_rate=round(dd["hits"] / max(1, lookups), 4),
                prefetch_accuracy=round(dd["prefetch_hits"] / max(1, dd["prefetches"]), 4),
                host_link_GBps={"during_run": round(dd["bytes_h2d"] / (ms * 1e-3) / 1e9, 2),
                                "single_copy": round(link, 2)},
                cache_delta=dd, us_per_token_layer=round(ms / n_tok / L * 1e3, 2),
                host_us_per_layer={k: round(v / (n_tok * L) * 1e6, 1) for k, v in host_s.items()},
                device_us_per_layer=dict(device_us, calls=len(prof),
                                         what="device stamps: routing kernel, gate/up, down, and the "
                                              "span from routing's first CTA to down's last (misses' "
                                              "copies and the host's acquire fall inside it); the first "
                                              "layer calls of the timed region, up to the ring's 1024"),
                clocks=clk.summary(),
                # per token: every layer's routing, gate/up and down kernels, plus the
                # next layer's prediction router for all but the last layer
                gpu_launches=n_tok * (3 * L + (L - 1)))


# ----------------------------------------------------------------- reference arm
def run_reference(args, ws_n, rank):
    """The CPU oracle on a bounded sample of the same workload (rank 0 only)."""
    if rank != 0:
        return None
    import numpy as np  # noqa: F401

    import oracle as orc  # noqa: F401
    if args.workload == "prefill":
        return run_reference_prefill(args, ws_n)
    w = mi.WORKLOADS[args.workload]
    if args.workload == "decode":
        # the native line's --experts / --tokens, so that both arms name one config
        if args.experts:
            w = mi.shrink(w, E=args.experts)
        if args.tokens:
            w = mi.shrink(w, T=args.tokens)
    seed = w.seed
    Wr = mi.make_router(w.E, w.H, mi.sub_seed(seed, 0, 2), "cpu").numpy()
    xpool = mi.make_x(POOL * w.T, w.H, mi.sub_seed(seed, 0, 1), "cpu").numpy()
    cache = {}

    def blob_fn(e):
        if e not in cache:
            b = torch.empty(w.blob_bytes, dtype=torch.uint8)
            mi.fill_blob(b, w.H, w.I, mi.blob_seed(mi.sub_seed(seed, 0, 3), e))
            cache[e] = b.numpy()
        return cache[e]

    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    mi_ = 0
    for _ in range(args.warmup):
        oracle_sample(w, xpool[mi_:mi_ + 1], Wr, blob_fn, 0.0, 1)
        mi_ += 1
    tb, ts, tn = 0, 0.0, 0
    for i in range(args.steps):
        b, s, n = oracle_sample(w, xpool[(mi_ + i) % POOL:(mi_ + i) % POOL + 1], Wr, blob_fn, per_step, 1)
        tb, ts, tn = tb + b, ts + s, tn + n
    value = tb / ts / 1e9
    cpu = {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", **host_cpu(),
           "sample": f"{tn} token-layers of the decode workload, single-threaded C oracle"}
    return dict(
        impl="reference", metric=METRIC, value=round(value, 4), unit="GB/s", n_gpus=ws_n,
        steps=args.steps, warmup=args.warmup, ms_per_step=round(ts / max(1, tn) * 1e3, 3),
        higher_is_better=True, scaling="weak", vs_baseline=None, dtype="int4xint8->fp32",
        data="synthetic",
        config=decode_config(w, ws_n, args.path),
        us_per_token_layer=round(ts / max(1, tn) * 1e6, 1), cpu_baseline=cpu,
        e2e={"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})


def run_reference_prefill(args, ws_n):
    w = mi.WORKLOADS["prefill"]
    x = mi.make_x(w.T, w.H, mi.sub_seed(w.seed, 0, 1), "cpu", zipf=True).numpy()
    Wr = mi.make_router(w.E, w.H, mi.sub_seed(w.seed, 0, 2), "cpu", zipf_s=w.zipf_s).numpy()
    cache = {}

    def blob_fn(e):
        if e not in cache:
            b = torch.empty(w.blob_bytes, dtype=torch.uint8)
            mi.fill_blob(b, w.H, w.I, mi.blob_seed(mi.sub_seed(w.seed, 0, 3), e))
            cache[e] = b.numpy()
        return cache[e]

    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    oracle_prefill_sample(w, x, Wr, blob_fn, 0.0, 1)  # warm-up: one token
    recs = [oracle_prefill_sample(w, x, Wr, blob_fn, per_step, 16) for _ in range(args.steps)]
    value = sum(r["value"] for r in recs) / len(recs)
    cpu = {"value": round(value, 6), "unit": "TOPS", "cores": 1, "kind": "oracle", **host_cpu(),
           "sample": recs[0]["sample"] + f"; {len(recs)} steps"}
    return dict(
        impl="reference", metric=METRIC, value=round(value, 6), unit="TOPS", n_gpus=ws_n, steps=args.steps,
        warmup=args.warmup, higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype="int4xint8->fp32", data="synthetic",
        config=prefill_config(w, ws_n),
        cpu_baseline=cpu,
        e2e={"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})


def main():
    args = parse()
    if args.impl == "reference":
        ws_n = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, ws_n, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    ws_n, rank, local = dist_setup()
    try:
        fn = {"prefill": run_prefill, "stacked": run_stacked, "tiered": run_tiered}.get(args.workload, run_native)
        res = fn(args, ws_n, rank, local)
        if args.workload == "decode" and ws_n == 1 and not args.no_prefill:
            res["prefill"] = prefill_summary(args, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if ws_n > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
