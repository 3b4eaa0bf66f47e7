#!/usr/bin/env python
"""Benchmark of the quantized MoE expert step on B200 (one JSON line on rank 0).

Workloads (seeded synthetic inputs, shapes from the pages; see workloads/):
  decode  (default) hidden 2048, 512 experts + 1 shared, top-10, 4-bit blocks,
          1 token per step; steps rotate over --layers copies of the layer so
          the weights streamed per step come from HBM, not L2
  verify  same layer with 2-bit blocks, Zipf-skewed router bias, a window of
          --window tokens per step
  prefill same layer as decode, --chunk tokens per step (tensor-core path)
  paging  24,576 two-bit experts in page-locked host memory, 2048 HBM slots,
          Gumbel-top-10 routing over drifting Zipf popularity, 1 token per step

A step is one pass of the whole step (route -> permute -> expert FFN ->
combine; paging adds the cache) over one batch.  The timed region is a CUDA
graph replay of exactly --steps steps (paging: an eager loop, since every
step synchronises with the host), bracketed by a barrier and
torch.cuda.synchronize(); multi-GPU runs are replicas (weak scaling) timed as
the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores instead (each
step a bounded sample of the same workload).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "MoE-layer tokens/s and expert weight GB/s vs HBM peak (decode, prefill, paging)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- helpers
def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={device_index}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.25)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in Path(self.f.name).read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), util=float(parts[4]),
                                 hw=parts[6], hwt=parts[7], swt=parts[8], swp=parts[9]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return None
        load = [r for r in rows if r["util"] >= 50] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


def src_hash(*names):
    """Hash of the named kernel sources plus every header they can include
    (the library's internal headers and the C ABI header), so a change to any
    of them marks recorded DRAM counters as stale."""
    csrc = ROOT / "quantized_expert_ffn_route_b200" / "csrc"
    files = [csrc / n for n in names]
    files += sorted(p for p in csrc.iterdir() if p.suffix in (".cuh", ".h"))
    files.append(ROOT / "include" / "moe.h")
    h = hashlib.sha256()
    for f in files:
        h.update(f.name.encode())
        h.update(f.read_bytes())
    return h.hexdigest()[:16]


def fp32_peak_tflops(sm_mhz, sms=148):
    """FP32 FMA roof derived from unit counts: SMs x 128 FP32 lanes x 2 FLOP
    per FMA x SM clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def layer_roofline(kind, fused, H, I, E, k, T, n_act, blob, ms_launch, pk, sm_mhz):
    """Roofline object of one expert-step launch.  Algorithmic bytes: the
    distinct expert blobs + x read once + y written once (+ the router rows
    and logits when the launch also routes); intermediates (x_perm, h, y_perm)
    are not credited.  Algorithmic FLOPs: 2*3*H*I per (token, expert)
    assignment including the shared expert (+ 2*H*E per token for a routing
    launch)."""
    if fused:
        nbytes = (k + 1) * blob + E * H * 2 + H * 2 + E * 4 + H * 4
        flops = 2 * 3 * H * I * (k + 1) + 2 * H * E
    else:
        nbytes = (n_act + 1) * blob + T * H * 2 + T * H * 4
        flops = 2 * 3 * H * I * T * (k + 1)
    sec = ms_launch / 1e3
    gbs = nbytes / sec / 1e9
    hbm = pk["hbm_gbs"]
    if kind == "prefill":
        peak_tf = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        tf = flops / sec / 1e12
        if flops / nbytes > peak_tf * 1e12 / (hbm * 1e9):
            roof = {"bound": "tensor", "achieved": round(tf, 2), "peak": peak_tf, "unit": "TFLOP/s",
                    "frac": round(tf / peak_tf, 4)}
        else:
            roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(gbs / hbm, 4)}
        roof["fp16_tensor_tflops_achieved"] = round(tf, 2)
    else:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(gbs / hbm, 4)}
        if kind == "verify":
            # the binding roof is the slower of the HBM and the FP32 ALU time
            alu_peak = fp32_peak_tflops(sm_mhz)
            tf = flops / sec / 1e12
            t_hbm, t_alu = nbytes / (hbm * 1e9), flops / (alu_peak * 1e12)
            roof["hbm_frac"] = round(gbs / hbm, 4)
            roof["alu_achieved_tflops"] = round(tf, 3)
            roof["alu_peak_tflops"] = round(alu_peak, 2)
            roof["alu_frac"] = round(tf / alu_peak, 4)
            roof["alu_peak_source"] = f"derived: 148 SMs x 128 FP32 lanes x 2 FLOP x {sm_mhz:.0f} MHz"
            if t_alu > t_hbm:
                roof.update({"bound": "alu", "achieved": round(tf, 3), "peak": round(alu_peak, 2),
                             "unit": "TFLOP/s", "frac": round(tf / alu_peak, 4)})
            roof["binding_roof_time_us"] = round(max(t_hbm, t_alu) * 1e6, 3)
    roof["algorithmic_bytes_per_launch"] = int(nbytes)
    roof["algorithmic_flops_per_launch"] = int(flops)
    return roof


def traffic_from_profiles(key: str, sha: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on this kernel source."""
    p = ROOT / "profiles" / "traffic.txt"
    if not p.exists():
        return None
    for line in p.read_text().splitlines():
        f = line.split()
        if len(f) >= 3 and f[0] == key and f[1] == sha:
            return float(f[2])
    return None


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def _reduce(v: float, world: int, op: str) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(v: float, world: int) -> float:
    return _reduce(v, world, "max")


def sum_over_ranks(v: float, world: int) -> float:
    return _reduce(v, world, "sum")


def job_rate(units: float, ms: float, world: int) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's device time (ms)."""
    total = sum_over_ranks(units, world)
    return total / (max_over_ranks(ms, world) / 1e3)


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------- workloads
def build_layer(kind):
    import workloads as W
    if kind == "verify":
        return W.verify_layer()
    c = W.DECODE
    return W.make_layer(W.SEED["decode"], 4, c["H"], c["I"], c["E"], c["k"], shared=True, w_dtype="bf16")


def gpu_copies(layer, n):
    import quantized_expert_ffn_route_b200 as M
    base = M.MoELayer(layer.bits, layer.H, layer.I, layer.E, layer.k, layer.blobs, layer.shared, layer.w_router,
                      layer.w_dtype, layer.bias)
    return [base] + [base.clone() for _ in range(n - 1)]


def timed_oracle(step, seconds, min_n):
    """Calls step(i) for i = 0, 1, ... until `seconds` have passed and at least
    min_n calls have run; returns (calls, seconds)."""
    t0, n = time.perf_counter(), 0
    while time.perf_counter() - t0 < seconds or n < min_n:
        step(n)
        n += 1
    return n, time.perf_counter() - t0


def oracle_baseline(step, seconds, min_n, tokens_per_call, what):
    """The oracle, as it stands, on a bounded sample: on all host cores, then
    on one thread (a shorter sample), each as tokens/s."""
    import oracle
    cores = host_cores()
    oracle.set_threads(cores)
    n, dt = timed_oracle(step, seconds, min_n)
    oracle.set_threads(1)
    n1, dt1 = timed_oracle(step, max(2.0, seconds / 3), min_n)
    oracle.set_threads(cores)
    return {"value": round(n * tokens_per_call / dt, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} {what} through the fp64 oracle on {cores} threads, {dt:.1f} s",
            "one_thread": {"value": round(n1 * tokens_per_call / dt1, 4), "unit": "tokens/s", "cores": 1,
                           "sample": f"{n1} {what} on 1 thread, {dt1:.1f} s"}}


def layer_oracle_step(layer, tokens, T_batch=8):
    """One call of the oracle's layer on the next batch of T_batch tokens."""
    import oracle

    def step(n):
        i = n % max(1, tokens.shape[0] // T_batch)
        oracle.moe_layer(layer.bits, tokens[i * T_batch:(i + 1) * T_batch], "bf16", layer.blobs, k=layer.k,
                         H=layer.H, I=layer.I, E=layer.E, w_router=layer.w_router, w_dtype="bf16", bias=layer.bias,
                         shared_blob=layer.shared)
    return step


def graph_upload(graph):
    """Uploads an instantiated CUDA graph to the device (cuGraphUpload) so
    that its first replay runs only its work.  A graph whose replay changes
    state (the expert cache of the paging workloads) cannot be replayed once
    beforehand just to upload it."""
    import ctypes
    import torch
    drv = ctypes.CDLL("libcuda.so.1")
    drv.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    rc = drv.cuGraphUpload(ctypes.c_void_p(graph.raw_cuda_graph_exec()),
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != 0:
        raise RuntimeError(f"cuGraphUpload failed ({rc})")


def run_graph_steps(step_fn, first, count, time_ffn=True):
    """Captures `count` steps in one CUDA graph; returns (graph, ffn event pairs)."""
    import torch
    g = torch.cuda.CUDAGraph()
    pairs = []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(first, first + count):
                if time_ffn:
                    e0 = torch.cuda.Event(enable_timing=True, external=True)
                    e1 = torch.cuda.Event(enable_timing=True, external=True)
                    step_fn(i, e0, e1)
                    pairs.append((e0, e1))
                else:
                    step_fn(i, None, None)
    torch.cuda.current_stream().wait_stream(s)
    return g, pairs


def bench_layer(args, world, rank, pk):
    """decode / verify / prefill: resident layer, graph-replayed steps."""
    import torch
    import quantized_expert_ffn_route_b200 as M
    import workloads as W

    kind = args.workload
    layer = build_layer(kind)
    H, I, E, k, bits = layer.H, layer.I, layer.E, layer.k, layer.bits
    one_kernel = getattr(args, "decode_one_kernel", False)
    if one_kernel:
        M.moe_test_hook(M.MOE_HOOK_DECODE_ONE_KERNEL, 1)
    T = {"decode": 1, "verify": args.window, "prefill": args.chunk}[kind]
    n_layers, mode, fused = workload_shape(kind, args)
    blob = M.moe_expert_blob_bytes(bits, H, I)
    # layer copies at distinct addresses: the steps of one sweep touch far more
    # than the 126 MB L2 (decode: 16 x 908 MB), so weights come from HBM
    copies = gpu_copies(layer, n_layers)
    n_steps = args.warmup + args.steps
    seed = W.SEED[kind] + 7919 * rank
    x_host = W.make_tokens(seed, n_steps * T if kind != "prefill" else 2 * T, H, "bf16")
    xs = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).cuda()
    bufs = copies[0].buffers(T, mode)

    def x_of(i):
        if kind == "prefill":
            j = i % 2
            return xs[j * T:(j + 1) * T]
        return xs[i * T:(i + 1) * T]

    dbuf = copies[0].decode_buffers() if fused else None

    def step(i, e0=None, e1=None):
        L = copies[i % n_layers]
        if fused:                                      # the whole step in one kernel
            if e0 is not None:
                e0.record()
            L.forward_decode(x_of(i), M.MOE_BF16, bufs=dbuf)
            if e1 is not None:
                e1.record()
            return
        b = bufs
        x = x_of(i)
        M.moe_route_topk(x, M.MOE_BF16, L.w_router, L.w_dtype, None, L.bias, T, H, E, k, b.ids, b.w, b.logits,
                         b.ws_route, b.sizes["route"])
        M.moe_permute(b.ids, T, k, E, b.offsets, b.perm_src, b.perm_dst, b.active, b.ws_perm, b.sizes["perm"])
        ffn = M.moe_expert_ffn_q4 if bits == 4 else M.moe_expert_ffn_q2
        if e0 is not None:
            e0.record()
        ffn(L.table, b.offsets, b.active, b.perm_src, x, M.MOE_BF16, T, k, H, I, E, L.shared, b.y_perm, b.y_shared,
            mode, b.ws_ffn, b.sizes["ffn"])
        if e1 is not None:
            e1.record()
        M.moe_combine(b.y_perm, b.perm_dst, b.w, b.y_shared, T, k, H, b.y)

    def ffn_only(i):
        L = copies[i % n_layers]
        if fused:
            L.forward_decode(x_of(i), M.MOE_BF16, bufs=dbuf)
            return
        b = bufs
        ffn = M.moe_expert_ffn_q4 if bits == 4 else M.moe_expert_ffn_q2
        ffn(L.table, b.offsets, b.active, b.perm_src, x_of(i), M.MOE_BF16, T, k, H, I, E, L.shared, b.y_perm,
            b.y_shared, mode, b.ws_ffn, b.sizes["ffn"])

    for i in range(args.warmup):                      # eager warm-up
        step(i)
    torch.cuda.synchronize()
    assert M.moe_device_error() == 0
    n0 = M.moe_kernel_launches()
    # the timed graph holds the K steps and nothing else: an event recorded
    # inside a graph costs a few microseconds per node, which would be timed
    # as part of the step
    graph, _ = run_graph_steps(step, args.warmup, args.steps, time_ffn=False)
    launches = M.moe_kernel_launches() - n0
    graph.replay()                                     # first replay uploads the graph
    torch.cuda.synchronize()

    clocks = ClockSampler(torch.cuda.current_device())
    # keep the GPU busy long enough for the clock sampler to see it under load
    t_end = time.perf_counter() + 1.0
    while time.perf_counter() < t_end:
        graph.replay()
        torch.cuda.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    graph.replay()
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world)
    if fused:
        # the step is the one call: its average duration is the timed region
        # over K (conservative: the gaps between calls are included)
        ffn_ms = [ms / args.steps]
        ffn_timing = ("timed region / K: the timed graph is K moe_layer_decode calls and nothing else, bracketed by "
                      "one event pair on the launching stream")
    else:
        # a graph of the same K expert-FFN calls alone (same inputs and
        # buffers as the timed steps), bracketed by one event pair
        torch.cuda.synchronize()
        g2, _ = run_graph_steps(lambda i, e0, e1: ffn_only(i), args.warmup, args.steps, time_ffn=False)
        g2.replay()
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g2.replay()
        z.record()
        torch.cuda.synchronize()
        ffn_ms = [a.elapsed_time(z) / args.steps]
        ffn_timing = ("graph of the K expert-FFN calls alone (the timed steps' inputs and routing), one event pair "
                      "on the launching stream / K")
    ffn_avg_ms = float(np.mean(ffn_ms))
    assert M.moe_device_error() == 0

    # distinct routed experts per launch: k for one token; for windows the
    # mean over the windows that routing_stats reads back; for prefill the
    # last chunk's active count
    routing = routing_stats(step, bufs, T, k, n_steps) if kind == "verify" else None
    if fused or kind == "decode":
        n_act = k
    elif routing and "distinct_experts_per_step" in routing:
        n_act = routing["distinct_experts_per_step"]
    else:
        n_act = int(bufs.active[0].item())
    tokens_total = sum_over_ranks(args.steps * T, world)
    value = tokens_total / (ms_max / 1e3)

    sm_mhz = (clk or {}).get("sm_mhz") or 1965.0
    roof = layer_roofline(kind, fused, H, I, E, k, T, n_act, blob, ffn_avg_ms, pk, sm_mhz)
    sha = src_hash(*(("decode.cu", "decode_step.cu") if fused else (("gemv.cu",) if kind != "prefill" else ("gemm_tc.cu",))))
    roof["traffic"] = traffic_from_profiles("k_decode" if fused else f"expert_ffn_{kind}_{T}", sha)
    if fused and one_kernel:
        roof["kernel"] = "moe_layer_decode (k_dec_step: one persistent kernel, one CTA per SM, two grid barriers)"
    elif fused:
        roof["kernel"] = ("moe_layer_decode (k_dec_route -> k_dec_gateup -> k_dec_down, chained by programmatic "
                          "dependent launch; one call)")
    else:
        roof["kernel"] = "moe_expert_ffn (gate/up + down kernels)"
    roof["ms_per_launch"] = round(ffn_avg_ms, 5)
    roof["timing"] = ffn_timing
    roof["peak_source"] = pk["source"]

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        n_e2e = min(args.steps, args.e2e_steps)
        xh = torch.from_numpy(x_host[: max(T, n_e2e * T if kind != "prefill" else T)].view(np.int16)).view(
            torch.bfloat16).pin_memory()
        yh = torch.empty(T * H, dtype=torch.float32).pin_memory()
        xd = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.current_stream()
        # one prepared moe_layer_decode call per layer copy (its arguments
        # marshalled once); a recorded decode session (MoELayer.decode_session)
        # measured slower here: ~48 us per token against ~44
        prepared = [c.prepare_decode(xd, M.MOE_BF16, stream=s, bufs=dbuf) for c in copies] if fused else None
        for i in range(3):
            xd.copy_(xh[:T], non_blocking=True)
            if fused:
                prepared[i % n_layers]()
                yh.copy_(dbuf["y"][:H], non_blocking=True)
            else:
                copies[i % n_layers].forward(xd, M.MOE_BF16, T=T, mode=mode, bufs=bufs)
                yh.copy_(bufs.y[:T * H], non_blocking=True)
            s.synchronize()
        barrier(world)
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(n_e2e):
            j = i * T if kind != "prefill" else 0
            xd.copy_(xh[j:j + T], non_blocking=True)
            if fused:
                prepared[i % n_layers]()
                yh.copy_(dbuf["y"][:H], non_blocking=True)
            else:
                copies[i % n_layers].forward(xd, M.MOE_BF16, T=T, mode=mode, bufs=bufs)
                yh.copy_(bufs.y[:T * H], non_blocking=True)
            s.synchronize()
        b2.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b2), world)
        e2e = {"value": round(sum_over_ranks(n_e2e * T, world) / (e_ms / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 4, "steps": n_e2e,
               "note": ("MoELayer.prepare_decode (one moe_layer_decode call per step)" if fused
                        else "MoELayer.forward") +
                       " via the C ABI; pinned host x in, fp32 y out, stream sync every step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(layer_oracle_step(layer, x_host, 8), args.cpu_seconds, 1, 8,
                              f"batches of 8 tokens of the {kind} workload")

    cfg = layer_config(kind, H, E, k, I, bits, T, n_layers, blob, mode, fused, world)
    return dict(value=value, ms=ms_max, steps=args.steps, roofline=roof, e2e=e2e, cpu=cpu, clocks=clk,
                launches=launches, config=cfg, routing=routing, dtype="fp32 (CUDA-core FMA on 4-bit codes)" if kind == "decode"
                else ("fp32 (CUDA-core FMA on 2-bit codes)" if kind == "verify" else "fp16 tensor cores, fp32 accum"))


def require_host_memory(what, need, spare=16 << 30):
    """Stops with a message (not a failed allocation) when the host cannot
    page-lock `need` bytes and keep `spare` free."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        return
    if avail < need + spare:
        raise SystemExit(f"{what}: {need / 2**30:.1f} GiB of page-locked host memory needed, "
                         f"{avail / 2**30:.1f} GiB available")


def host_link_gbs(nbytes=1 << 30):
    """Pinned host -> device copy bandwidth (best of 3)."""
    import torch
    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    best = 0.0
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        d.copy_(h, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) / 1e3) / 1e9)
    del h, d
    return best


def bench_paging(args, world, rank, pk):
    """24,576 two-bit experts paged from pinned host memory into 2048 HBM slots."""
    import torch
    import quantized_expert_ffn_route_b200 as M
    import workloads as W
    c = W.PAGING
    E, k, H, I, cap = c["E"], c["k"], c["H"], c["I"], c["capacity"]
    base = W.make_layer(W.SEED["paging"], 2, H, I, 512, k, shared=False, w_dtype="bf16")
    nb = M.moe_expert_blob_bytes(2, H, I)
    stride = (nb + 255) // 256 * 256
    link = host_link_gbs()
    # page-locked pool of all experts (512 distinct blobs repeated: only bytes moved matter here)
    need = E * stride
    require_host_memory("paging", need)
    pool = torch.empty(need, dtype=torch.uint8, pin_memory=True)
    pv = pool.view(E, stride)
    bt = torch.from_numpy(base.blobs)
    for e0 in range(0, E, 512):
        pv[e0:e0 + 512, :nb].copy_(bt)
    slab = torch.empty(cap * stride, dtype=torch.uint8, device="cuda")
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    dev_mode = args.device_staging
    if dev_mode:                                         # policy and copies on the device (devcache_*)
        from quantized_expert_ffn_route_b200.paged import DevicePagedExpertStack
        stack = DevicePagedExpertStack(1, E, 2, H, I, k, pool, slab, table, cap, nb, stride, decay_period=256,
                                       admit_min=args.admit_min)
        cache = stack.cache
    else:
        cache = M.ExpCache(E, cap, nb, stride, pool, slab, table, decay_period=256)
    n_steps = args.warmup + args.steps
    # untimed steps after the timed ones: 64 for the overlap pass, then the end-to-end steps
    n_more = 64 + (0 if args.no_e2e else min(args.steps, args.e2e_steps))
    trace = np.stack(list(W.paging_trace(W.SEED["paging"] + 17 * rank, E, k, n_steps + n_more, s=c["zipf_s"],
                                         drift_every=c["drift_every"], drift_prob=c["drift_prob"],
                                         hot=c["hot"])))
    logits = torch.from_numpy(trace).cuda()
    x_host = W.make_tokens(W.SEED["paging"] + 1, n_steps + n_more, H, "bf16")
    xs = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).cuda()
    b = stack.b if dev_mode else M.alloc_step_buffers(1, H, I, E, k, 2, M.MOE_MODE_GEMV, torch.device("cuda"),
                                                         False)
    ids_h = torch.empty(k, dtype=torch.int32).pin_memory()
    # expert lists of the two FFN calls of a step: [count, ids...] for the
    # hits (resident: computed at once) and for the misses (after their copies)
    act_h = torch.zeros(64, dtype=torch.int32).pin_memory()
    act_d = torch.zeros(64, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    misses_per_step = []
    ev_hit = [None, None]

    def step(i, x=None):
        if dev_mode:
            stack.layer_step(0, xs[i] if x is None else x, M.MOE_BF16, logits[i])
            return
        M.moe_route_topk(None, 0, None, 0, logits[i], None, 1, H, E, k, b.ids, b.w, None, b.ws_route,
                         b.sizes["route"])
        M.moe_permute(b.ids, 1, k, E, b.offsets, b.perm_src, b.perm_dst, b.active, b.ws_perm, b.sizes["perm"])
        ids_h.copy_(b.ids[:k], non_blocking=True)
        s.synchronize()                                  # the ids cross to the host
        ids = ids_h.numpy().copy()
        hit, _, _ = cache.stage(ids)
        hits, miss = np.sort(ids[hit == 1]), np.sort(ids[hit == 0])
        misses_per_step.append(int(miss.size))
        a = act_h.numpy()
        a[0], a[1:1 + hits.size] = hits.size, hits
        a[32], a[33:33 + miss.size] = miss.size, miss
        act_d.copy_(act_h, non_blocking=True)
        xi = xs[i] if x is None else x
        ffn = M.moe_expert_ffn_q2
        if ev_hit[0] is not None:
            ev_hit[0].record()
        if hits.size:                                    # resident experts: at once, overlapping the copies
            ffn(table, b.offsets, act_d[0:], b.perm_src, xi, M.MOE_BF16, 1, k, H, I, E, None, b.y_perm, None,
                M.MOE_MODE_GEMV, b.ws_ffn, b.sizes["ffn"])
        if ev_hit[1] is not None:
            ev_hit[1].record()
        cache.join()                                     # the rest waits for its copies + table patch
        if miss.size:
            ffn(table, b.offsets, act_d[32:], b.perm_src, xi, M.MOE_BF16, 1, k, H, I, E, None, b.y_perm, None,
                M.MOE_MODE_GEMV, b.ws_ffn, b.sizes["ffn"])
        M.moe_combine(b.y_perm, b.perm_dst, b.w, None, 1, k, H, b.y)

    def overlap_pass(first, n):
        """Untimed pass over n more steps: the share of each step's copy time
        (first copy issued -> table patched) during which the hit experts'
        FFN ran on the compute stream."""
        ref = torch.cuda.Event(enable_timing=True)
        ev_hit[0], ev_hit[1] = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ref.record()
        copy_ms = hidden_ms = 0.0
        for i in range(first, first + n):
            m0 = len(misses_per_step)
            step(i)
            torch.cuda.synchronize()
            if misses_per_step[m0] == 0:
                continue
            c0, c1 = cache.copy_times(ref)
            h0, h1 = ref.elapsed_time(ev_hit[0]), ref.elapsed_time(ev_hit[1])
            copy_ms += c1 - c0
            hidden_ms += max(0.0, min(c1, h1) - max(c0, h0))
        ev_hit[0] = ev_hit[1] = None
        return (hidden_ms / copy_ms if copy_ms > 0 else None), copy_ms

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    graph = None
    if dev_mode:
        # nothing in a device-staged step waits for the host: the K steps are
        # one CUDA graph, uploaded before the timed region and replayed once
        nc0 = M.moe_kernel_launches()
        graph, _ = run_graph_steps(lambda i, e0, e1: step(i), args.warmup, args.steps, time_ffn=False)
        graph_launches = M.moe_kernel_launches() - nc0
        graph_upload(graph)                              # the timed replay is the steps' only run
        torch.cuda.synchronize()
    st0 = cache.stats()
    n0 = M.moe_kernel_launches()
    clocks = ClockSampler(torch.cuda.current_device())
    barrier(world)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.warmup, n_steps):
            step(i)
    z.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    launches = graph_launches if graph is not None else M.moe_kernel_launches() - n0
    assert M.moe_device_error() == 0
    ms = max_over_ranks(a.elapsed_time(z), world)
    st1 = cache.stats()
    value = sum_over_ranks(args.steps, world) / (ms / 1e3)
    if dev_mode:
        in_place = st1["in_place"] - st0["in_place"]
        staged = st1["bytes_copied"] - st0["bytes_copied"] + in_place * nb     # every byte over the link
        mps = [(st1["misses"] - st0["misses"]) / args.steps]
        overlap = None
    else:
        mps = misses_per_step[args.warmup:n_steps]
        overlap, copy_ms = overlap_pass(n_steps, min(200, 64))
        staged = st1["bytes_staged"] - st0["bytes_staged"]
    link_ach = staged / (ms / 1e3) / 1e9
    steady = mps[500:] if len(mps) > 600 else mps
    roof = {"bound": "host_link", "achieved": round(link_ach, 2), "peak": round(link, 2), "unit": "GB/s",
            "frac": round(link_ach / link, 4), "traffic": None,
            "kernel": ("devcache_stage (policy kernel on the device; copy kernel of SM loads from the mapped pinned "
                       "pool; no host synchronisation per step)" if dev_mode
                       else "expcache_stage copies (cudaMemcpyAsync pinned host -> HBM slot)"),
            "peak_source": "pinned 1 GiB host->device copy measured in this run",
            "misses_per_step": round(float(np.mean(mps)), 3),
            "misses_per_step_steady": round(float(np.mean(steady)), 3),
            "hbm_bytes_per_step": k * nb,
            "overlap": None if overlap is None else round(overlap, 4),
            "overlap_definition": ("share of each step's copy interval (first copy issued -> device table "
                                   "patched) during which the resident experts' FFN ran on the compute stream, "
                                   "from CUDA events over an untimed pass of 64 further steps; not measured "
                                   "with device staging, whose copies run in a kernel beside the hits' FFN")}
    if dev_mode:
        roof["in_place_per_step"] = round(in_place / args.steps, 3)
        roof["admit_min"] = args.admit_min
    else:
        cache.wait(30_000_000)
        bins, nh = cache.copy_histogram()
        roof["copy_time_histogram"] = {"bins_log2_us": bins.tolist(), "steps": int(nh),
                                       "definition": "steps whose copies (first issued -> table patched) took "
                                                     "[2^i, 2^(i+1)) microseconds, all steps of this run"}

    e2e = None
    if not args.no_e2e:
        n_e2e = min(args.steps, args.e2e_steps)
        xh = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
        yh = torch.empty(H, dtype=torch.float32).pin_memory()
        xd = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
        barrier(world)
        a.record()
        for j in range(n_e2e):
            i = n_steps + 64 + j                         # the trace goes on: fresh steps, as in the timed region
            xd.copy_(xh[i:i + 1], non_blocking=True)
            step(i, xd)
            yh.copy_(b.y[:H], non_blocking=True)
            s.synchronize()
        z.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(z), world)
        e2e = {"value": round(sum_over_ranks(n_e2e, world) / (e_ms / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": H * 2, "d2h_bytes_per_step": H * 4 + k * 4, "steps": n_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        blob_list = [pv[e, :nb].numpy() for e in range(E)]

        def step(n):
            i = n % n_steps
            oracle.moe_layer(2, x_host[i:i + 1], "bf16", blob_list, k=k, H=H, I=I, E=E, logits_in=trace[i:i + 1])
        cpu = oracle_baseline(step, args.cpu_seconds, 2, 1, "paging steps (1 token, 10 of 24,576 experts)")
    cache.close()
    cfg = paging_config(E, k, nb, cap, c, world)
    if dev_mode:
        cfg["staging"] = "device-initiated" + (f", admit_min {args.admit_min}" if args.admit_min > 1 else "")
    roof["cache"] = {"misses": st1["misses"] - st0["misses"], "hits": st1["hits"] - st0["hits"]}
    return dict(value=value, ms=ms, steps=args.steps, roofline=roof, e2e=e2e, cpu=cpu, clocks=clk,
                launches=launches, config=cfg, dtype="fp32 (CUDA-core FMA on 2-bit codes)")


def paging_ssd_config(E, k, nb, c, world):
    """The `config` object of the three-tier workload (both arms print it)."""
    return {"workload": f"paging_ssd: {E} experts (2-bit, {nb} B each, {E * nb / 1e9:.1f} GB) in a file read with "
                        f"O_DIRECT into {c['ram_slots']} page-locked RAM slots, {c['hbm_slots']} HBM slots, "
                        f"top-{k}, Zipf s={c['zipf_s']} with drift every {c['drift_every']} steps",
            "tokens_per_step": 1, "l2": "weights paged from the drive and host RAM; HBM slots > L2",
            "parallelism": f"replicas x{world}"}


def bench_paging_ssd(args, world, rank, pk):
    """Three tiers: the experts in a file on the local drive (read with
    O_DIRECT by the store's I/O threads), a page-locked RAM tier, HBM slots."""
    import tempfile
    import torch
    import quantized_expert_ffn_route_b200 as M
    import workloads as W
    from quantized_expert_ffn_route_b200.paged import PagedExpertStack
    c = W.PAGING_SSD
    E, k, H, I, cap, rs = c["E"], c["k"], c["H"], c["I"], c["hbm_slots"], c["ram_slots"]
    base = W.make_layer(W.SEED["paging_ssd"], 2, H, I, 512, k, shared=False, w_dtype="bf16")
    nb = M.moe_expert_blob_bytes(2, H, I)
    stride = (nb + 4095) // 4096 * 4096
    link = host_link_gbs()
    fd, path = tempfile.mkstemp(prefix=f"moe_experts_r{rank}_", suffix=".bin", dir=args.ssd_dir)
    try:
        chunk = np.zeros((512, stride), np.uint8)
        chunk[:, :nb] = base.blobs                       # 512 distinct blobs, repeated: only bytes moved matter
        with os.fdopen(fd, "wb") as f:
            for _ in range(E // 512):
                f.write(chunk.tobytes())
            f.flush()
            os.fsync(f.fileno())
        raw = torch.zeros(rs * stride + 4096, dtype=torch.uint8, pin_memory=True)
        off = (-raw.data_ptr()) % 4096
        ram = raw[off:off + rs * stride]
        # the drive's own rate for this access pattern: 32 random experts per
        # batch into an empty store of 32 slots, same threads, O_DIRECT
        probe_ram = raw[off:off + 32 * stride]
        probe = M.ExpStore(path, E, nb, stride, 32, probe_ram, io_threads=c["io_threads"], use_direct=True)
        rng = np.random.default_rng(7)
        t0 = time.perf_counter()
        nbat = 16
        for _ in range(nbat):
            probe.fetch(rng.choice(E, 32, replace=False))
        drive = nbat * 32 * stride / (time.perf_counter() - t0) / 1e9
        probe.close()
        store = M.ExpStore(path, E, nb, stride, rs, ram, io_threads=c["io_threads"], use_direct=True)
        slab = torch.empty(cap * stride, dtype=torch.uint8, device="cuda")
        table = torch.zeros(E, dtype=torch.int64, device="cuda")
        stack = PagedExpertStack(1, E, 2, H, I, k, ram, slab, table, cap, nb, stride, decay_period=256, prefetch=0,
                                 store=store)
        n_steps = args.warmup + args.steps
        n_more = max(64, 0 if args.no_e2e else min(args.steps, args.e2e_steps))
        trace = np.stack(list(W.paging_trace(W.SEED["paging_ssd"] + 17 * rank, E, k, n_steps + n_more,
                                             s=c["zipf_s"], drift_every=c["drift_every"],
                                             drift_prob=c["drift_prob"], hot=c["hot"])))
        logits = torch.from_numpy(trace).cuda()
        x_host = W.make_tokens(W.SEED["paging_ssd"] + 1, n_steps + n_more, H, "bf16")
        xs = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).cuda()

        def step(i, x=None):
            return stack.layer_step(0, xs[i:i + 1] if x is None else x, M.MOE_BF16, logits[i])

        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        st0, ss0 = stack.cache.stats(), store.stats()
        n0 = M.moe_kernel_launches()
        clocks = ClockSampler(torch.cuda.current_device())
        barrier(world)
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(args.warmup, n_steps):
            step(i)
        z.record()
        torch.cuda.synchronize()
        barrier(world)
        clk = clocks.stop()
        launches = M.moe_kernel_launches() - n0
        assert M.moe_device_error() == 0
        ms = max_over_ranks(a.elapsed_time(z), world)
        st1, ss1 = stack.cache.stats(), store.stats()
        value = sum_over_ranks(args.steps, world) / (ms / 1e3)
        read = ss1["bytes_read"] - ss0["bytes_read"]
        hbm_miss = st1["misses"] - st0["misses"]
        ram_hit = ss1["hits"] - ss0["hits"]
        drive_ach = read / (ms / 1e3) / 1e9
        roof = {"bound": "drive", "achieved": round(drive_ach, 3), "peak": round(drive, 3), "unit": "GB/s",
                "frac": round(drive_ach / drive, 4), "traffic": None,
                "kernel": "expstore_fetch (O_DIRECT preads by 8 threads into the RAM tier) + expcache_stage_from",
                "peak_source": "O_DIRECT reads of 32 random experts per batch by the same threads, this run",
                "host_link_gbs": round(link, 2),
                "hbm_misses_per_step": round(hbm_miss / args.steps, 3),
                "ram_hits_per_step": round(ram_hit / args.steps, 3),
                "drive_reads_per_step": round((ss1["reads"] - ss0["reads"]) / args.steps, 3),
                "read_wait_ms_per_step": round((ss1["read_seconds"] - ss0["read_seconds"]) * 1e3 / args.steps, 4)}
        e2e = None
        if not args.no_e2e:
            n_e2e = min(args.steps, args.e2e_steps)
            xh = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
            yh = torch.empty(H, dtype=torch.float32).pin_memory()
            xd = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
            s = torch.cuda.current_stream()
            barrier(world)
            a.record()
            for j in range(n_e2e):
                i = n_steps + j
                xd.copy_(xh[i:i + 1], non_blocking=True)
                y = step(i, xd)
                yh.copy_(y[:H], non_blocking=True)
                s.synchronize()
            z.record()
            torch.cuda.synchronize()
            e_ms = max_over_ranks(a.elapsed_time(z), world)
            e2e = {"value": round(sum_over_ranks(n_e2e, world) / (e_ms / 1e3), 1), "unit": "tokens/s",
                   "h2d_bytes_per_step": H * 2, "d2h_bytes_per_step": H * 4 + k * 4, "steps": n_e2e}
        stack.close()
        store.close()
    finally:
        os.unlink(path)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        blob_list = [base.blobs[e % 512] for e in range(E)]

        def ostep(n):
            i = n % n_steps
            oracle.moe_layer(2, x_host[i:i + 1], "bf16", blob_list, k=k, H=H, I=I, E=E, logits_in=trace[i:i + 1])
        cpu = oracle_baseline(ostep, args.cpu_seconds, 2, 1, f"paging steps (1 token, 10 of {E} experts)")
    cfg = paging_ssd_config(E, k, nb, c, world)
    return dict(value=value, ms=ms, steps=args.steps, roofline=roof, e2e=e2e, cpu=cpu, clocks=clk,
                launches=launches, config=cfg, dtype="fp32 (CUDA-core FMA on 2-bit codes)")


def bench_paging48(args, world, rank, pk):
    """48 layers x 512 two-bit experts = the 24,576-expert pool in page-locked
    host memory, one cache of 2048 HBM slots, 10 experts per layer per token,
    the next layer's most used experts prefetched while a layer computes."""
    import torch
    import quantized_expert_ffn_route_b200 as M
    import workloads as W
    from quantized_expert_ffn_route_b200.paged import PagedExpertStack
    c = W.PAGING48
    L, El, k, H, I, cap = c["layers"], c["experts_per_layer"], c["k"], c["H"], c["I"], c["capacity"]
    E = L * El
    pf_n = c["prefetch"] if args.prefetch < 0 else args.prefetch
    base = W.make_layer(W.SEED["paging48"], 2, H, I, El, k, shared=False, w_dtype="bf16")
    nb = M.moe_expert_blob_bytes(2, H, I)
    stride = (nb + 255) // 256 * 256
    link = host_link_gbs()
    require_host_memory("paging48", E * stride)
    pool = torch.empty(E * stride, dtype=torch.uint8, pin_memory=True)
    pv = pool.view(E, stride)
    bt = torch.from_numpy(base.blobs)
    for l in range(L):                                   # every layer's blobs (bytes moved are what matter here)
        pv[l * El:(l + 1) * El, :nb].copy_(bt)
    slab = torch.empty(cap * stride, dtype=torch.uint8, device="cuda")
    table = torch.zeros(E, dtype=torch.int64, device="cuda")
    dev_mode = args.device_staging
    if dev_mode:                                         # policy and copies on the device; no prefetch
        from quantized_expert_ffn_route_b200.paged import DevicePagedExpertStack
        pf_n = 0
        stack = DevicePagedExpertStack(L, El, 2, H, I, k, pool, slab, table, cap, nb, stride, decay_period=256,
                                       admit_min=args.admit_min)
    else:
        stack = PagedExpertStack(L, El, 2, H, I, k, pool, slab, table, cap, nb, stride, decay_period=256,
                                 prefetch=pf_n)
    tokens_w, tokens_t = max(1, args.warmup // 3), min(args.steps, c["tokens"])
    n_tok = tokens_w + tokens_t + 16
    trace = np.stack(list(W.paging48_trace(W.SEED["paging48"] + 17 * rank, L, El, n_tok, s=c["zipf_s"],
                                           drift_every=c["drift_every"], drift_prob=c["drift_prob"],
                                           hot=c["hot_per_layer"])))
    logits = torch.from_numpy(trace).cuda()
    x_host = W.make_tokens(W.SEED["paging48"] + 1, n_tok, H, "bf16")
    xs = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).cuda()

    def token(t, x=None):
        for l in range(L):
            y = stack.layer_step(l, xs[t:t + 1] if x is None else x, M.MOE_BF16, logits[t, l])
        return y

    for t in range(tokens_w):
        token(t)
    torch.cuda.synchronize()
    graph = None
    if dev_mode:
        # no layer waits for the host: the timed tokens are one CUDA graph
        nc0 = M.moe_kernel_launches()
        graph, _ = run_graph_steps(lambda t, e0, e1: token(t), tokens_w, tokens_t, time_ffn=False)
        graph_launches = M.moe_kernel_launches() - nc0
        graph_upload(graph)                              # the timed replay is the tokens' only run
        torch.cuda.synchronize()
    st0 = stack.cache.stats()
    stack.record, stack.events = True, []
    n0 = M.moe_kernel_launches()
    clocks = ClockSampler(torch.cuda.current_device())
    barrier(world)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    if graph is not None:
        graph.replay()
    else:
        for t in range(tokens_w, tokens_w + tokens_t):
            token(t)
    z.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    stack.record = False
    launches = graph_launches if graph is not None else M.moe_kernel_launches() - n0
    assert M.moe_device_error() == 0
    ms = max_over_ranks(a.elapsed_time(z), world)
    st1 = stack.cache.stats()
    misses = st1["misses"] - st0["misses"]
    if dev_mode:
        in_place = st1["in_place"] - st0["in_place"]
        staged = st1["bytes_copied"] - st0["bytes_copied"] + in_place * nb     # every byte over the link
        prefetched = 0
    else:
        staged = st1["bytes_staged"] - st0["bytes_staged"]
        prefetched = st1["prefetched"] - st0["prefetched"]
    # prefetched experts that a later stage found resident before they were evicted
    pending, useful = set(), 0
    for gids, hit, _, victim, pf, pf_slot, pf_victim in (() if dev_mode else stack.events):
        for e, h in zip(gids.tolist(), hit.tolist()):
            if h and e in pending:
                useful += 1
                pending.discard(e)
        pending.difference_update(v for v in victim.tolist() if v >= 0)
        pending.difference_update(v for v in pf_victim.tolist() if v >= 0)
        pending.update(e for e, sl in zip(pf.tolist(), pf_slot.tolist()) if sl >= 0)
    value = sum_over_ranks(tokens_t, world) / (ms / 1e3)
    link_ach = staged / (ms / 1e3) / 1e9
    roof = {"bound": "host_link", "achieved": round(link_ach, 2), "peak": round(link, 2), "unit": "GB/s",
            "frac": round(link_ach / link, 4), "traffic": None,
            "kernel": ("devcache_stage (policy kernel on the device; copy kernel of SM loads from the mapped pinned "
                       "pool; no host synchronisation per layer)" if dev_mode
                       else "expcache_stage + expcache_prefetch copies (cudaMemcpyAsync pinned host -> HBM slot)"),
            "peak_source": "pinned 1 GiB host->device copy measured in this run",
            "misses_per_token": round(misses / tokens_t, 2),
            "prefetched_per_token": round(prefetched / tokens_t, 2),
            "prefetched_used_share": round(useful / prefetched, 4) if prefetched else None,
            "expert_accesses_per_token": L * k, "hbm_bytes_per_token": L * k * nb}

    e2e = None
    if not args.no_e2e:
        n_e2e = min(tokens_t, 16)
        xh = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
        yh = torch.empty(H, dtype=torch.float32).pin_memory()
        xd = torch.empty(1, H, dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.current_stream()
        barrier(world)
        a.record()
        for j in range(n_e2e):
            t = tokens_w + tokens_t + (j % 16)
            xd.copy_(xh[t:t + 1], non_blocking=True)
            y = token(t, xd)
            yh.copy_(y[:H], non_blocking=True)
            s.synchronize()
        z.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(z), world)
        e2e = {"value": round(sum_over_ranks(n_e2e, world) / (e_ms / 1e3), 2), "unit": "tokens/s",
               "h2d_bytes_per_step": H * 2, "d2h_bytes_per_step": H * 4 + L * k * 4, "steps": n_e2e,
               "note": "one token through 48 layers per step; x copied in from page-locked host memory, the last "
                       "layer's y read back"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        blob_list = [pv[e % El, :nb].numpy() for e in range(El)]

        def step(n):
            t, l = (n // L) % n_tok, n % L
            oracle.moe_layer(2, x_host[t:t + 1], "bf16", blob_list, k=k, H=H, I=I, E=El, logits_in=trace[t, l][None])
        cpu = oracle_baseline(step, args.cpu_seconds, L, 1.0 / L, "layer steps (1 token through 1 of 48 layers)")
    stack.close()
    cfg = paging48_config(L, El, k, nb, cap, c, pf_n, world)
    if dev_mode:
        cfg["staging"] = "device-initiated" + (f", admit_min {args.admit_min}" if args.admit_min > 1 else "")
    return dict(value=value, ms=ms, steps=tokens_t, roofline=roof, e2e=e2e, cpu=cpu, clocks=clk,
                launches=launches, config=cfg, dtype="fp32 (CUDA-core FMA on 2-bit codes)")


def paging48_config(L, El, k, nb, cap, c, pf_n, world):
    """The `config` object of the model-scale paging workload (both arms print it)."""
    return {"workload": f"paging48: {L} layers x {El} experts (2-bit, {nb} B each, {L * El * nb / 1e9:.1f} GB pinned "
                        f"host), {cap} HBM slots, top-{k} per layer, Zipf s={c['zipf_s']} per layer with drift every "
                        f"{c['drift_every']} tokens, prefetch of the next layer's {pf_n} most used experts",
            "tokens_per_step": 1, "layers_per_token": L, "l2": "weights paged from host; HBM slots 2 GB > L2",
            "parallelism": f"replicas x{world}"}


def expert_stats(ids_per_step, hot=42):
    """Routing of some steps (one int array of selected ids per step): mean
    distinct experts per step and the share of selections that fall on the
    `hot` most often selected experts."""
    distinct = [len(np.unique(a)) for a in ids_per_step]
    allids = np.concatenate([np.asarray(a).ravel() for a in ids_per_step])
    counts = np.sort(np.bincount(allids))[::-1]
    return {"distinct_experts_per_step": round(float(np.mean(distinct)), 2),
            f"top{hot}_share": round(float(counts[:hot].sum() / max(1, allids.size)), 4),
            "steps": len(ids_per_step)}


def routing_stats(step, bufs, T, k, n_steps, n=64):
    """Runs n steps eagerly and reads the selected ids back (verify windows)."""
    import torch
    try:
        got = []
        for i in range(min(n, n_steps)):
            step(i)
            torch.cuda.synchronize()
            got.append(bufs.ids[:T * k].cpu().numpy())
        return expert_stats(got)
    except Exception as e:                             # a statistic only: never lose the bench line
        return {"error": str(e)[:200]}


def layer_config(kind, H, E, k, I, bits, T, n_layers, blob, mode, fused, world):
    """The `config` object of a resident-layer workload (both arms print it)."""
    return {"workload": workload_name(kind, H, E, k, I, bits, T),
            "tokens_per_step": T, "layer_copies": n_layers,
            "l2": f"inputs larger than L2: {n_layers} layer copies x {E + 1} experts x {blob} B rotate per step",
            "mode": "fused decode kernel" if fused else {0: "auto", 1: "gemv", 2: "gemm"}[mode],
            "parallelism": f"replicas x{world}"}


def paging_config(E, k, nb, cap, c, world):
    """The `config` object of the paging workload (both arms print it)."""
    return {"workload": f"paging: {E} experts (2-bit, {nb} B each, {E * nb / 1e9:.1f} GB pinned host), "
                        f"{cap} HBM slots, top-{k}, Zipf s={c['zipf_s']} with drift every {c['drift_every']} steps",
            "tokens_per_step": 1, "l2": "weights paged from host; HBM slots 2 GB > L2",
            "parallelism": f"replicas x{world}"}


def workload_shape(kind, args):
    """(layer copies, FFN mode, fused) of a resident-layer workload as bench_layer runs it."""
    n_layers = args.layers or (2 if kind == "prefill" else 16)
    mode = {"gemv": 1, "gemm": 2}.get(getattr(args, "ffn_mode", "auto"), 2 if kind == "prefill" else 0)
    fused = kind == "decode" and not args.unfused
    return n_layers, mode, fused


def workload_name(kind, H, E, k, I, bits, T):
    return (f"{kind}: hidden {H}, {E} experts + 1 shared, top-{k}, intermediate {I}, "
            f"{bits}-bit blocks of 32 + fp16 scale, {T} token(s)/step")


def bench_reference(args, world, rank):
    """The oracle on the host cores, as it stands; each step is a bounded
    sample of the workload: one token (decode, verify, prefill) or one paging
    step, so K steps take about K x 25-50 ms on 16 cores."""
    import oracle
    import workloads as W
    if rank != 0:
        return None
    oracle.set_threads(host_cores())
    kind = args.workload
    n = args.warmup + args.steps
    if kind == "paging48":
        c = W.PAGING48
        L, El, k, H, I, cap = c["layers"], c["experts_per_layer"], c["k"], c["H"], c["I"], c["capacity"]
        base = W.make_layer(W.SEED["paging48"], 2, H, I, El, k, shared=False, w_dtype="bf16")
        n_tok = n // L + 2
        trace = np.stack(list(W.paging48_trace(W.SEED["paging48"], L, El, n_tok, s=c["zipf_s"],
                                               drift_every=c["drift_every"], drift_prob=c["drift_prob"],
                                               hot=c["hot_per_layer"])))
        x = W.make_tokens(W.SEED["paging48"] + 1, n_tok, H, "bf16")

        def one(i):
            t, l = i // L, i % L
            oracle.moe_layer(2, x[t:t + 1], "bf16", base.blobs, k=k, H=H, I=I, E=El, logits_in=trace[t, l][None])
        pf_n = c["prefetch"] if getattr(args, "prefetch", -1) < 0 else args.prefetch
        cfg = paging48_config(L, El, k, oracle.blob_bytes(2, H, I), cap, c, pf_n, world)
        sample = "1 layer step of a token (10 of 512 experts of one of 48 layers); tokens/s = steps / 48 / time"
        for i in range(args.warmup):
            one(i)
        t0 = time.perf_counter()
        for i in range(args.warmup, n):
            one(i)
        dt = time.perf_counter() - t0
        return dict(value=args.steps / L / dt, ms=dt * 1e3, config=cfg, sample=sample)
    if kind == "paging_ssd":
        c = W.PAGING_SSD
        E, k, H, I = c["E"], c["k"], c["H"], c["I"]
        base = W.make_layer(W.SEED["paging_ssd"], 2, H, I, 512, k, shared=False, w_dtype="bf16")
        blob_list = [base.blobs[e % 512] for e in range(E)]
        trace = np.stack(list(W.paging_trace(W.SEED["paging_ssd"], E, k, n, s=c["zipf_s"],
                                             drift_every=c["drift_every"], drift_prob=c["drift_prob"],
                                             hot=c["hot"])))
        x = W.make_tokens(W.SEED["paging_ssd"] + 1, n, H, "bf16")

        def one(i):
            oracle.moe_layer(2, x[i:i + 1], "bf16", blob_list, k=k, H=H, I=I, E=E, logits_in=trace[i:i + 1])
        cfg = paging_ssd_config(E, k, oracle.blob_bytes(2, H, I), c, world)
        sample = f"1 paging step (1 token, 10 of {E} experts)"
    elif kind == "paging":
        c = W.PAGING
        E, k, H, I, cap = c["E"], c["k"], c["H"], c["I"], c["capacity"]
        base = W.make_layer(W.SEED["paging"], 2, H, I, 512, k, shared=False, w_dtype="bf16")
        blob_list = [base.blobs[e % 512] for e in range(E)]     # the pool repeats 512 distinct blobs
        trace = np.stack(list(W.paging_trace(W.SEED["paging"], E, k, n, s=c["zipf_s"],
                                             drift_every=c["drift_every"], drift_prob=c["drift_prob"],
                                             hot=c["hot"])))
        x = W.make_tokens(W.SEED["paging"] + 1, n, H, "bf16")

        def one(i):
            oracle.moe_layer(2, x[i:i + 1], "bf16", blob_list, k=k, H=H, I=I, E=E, logits_in=trace[i:i + 1])
        cfg = paging_config(E, k, oracle.blob_bytes(2, H, I), cap, c, world)
        sample = "1 paging step (1 token, 10 of 24,576 experts)"
    else:
        layer = build_layer(kind)
        x = W.make_tokens(W.SEED[kind], n, layer.H, "bf16")

        def one(i):
            oracle.moe_layer(layer.bits, x[i:i + 1], "bf16", layer.blobs, k=layer.k, H=layer.H, I=layer.I,
                             E=layer.E, w_router=layer.w_router, w_dtype="bf16", bias=layer.bias,
                             shared_blob=layer.shared)
        Tw = {"decode": 1, "verify": args.window, "prefill": args.chunk}[kind]
        n_layers, mode, fused = workload_shape(kind, args)
        cfg = layer_config(kind, layer.H, layer.E, layer.k, layer.I, layer.bits, Tw, n_layers,
                           oracle.blob_bytes(layer.bits, layer.H, layer.I), mode, fused, world)
        sample = f"1 token of the {kind} workload"
    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.warmup, n):
        one(i)
    dt = time.perf_counter() - t0
    return dict(value=args.steps / dt, ms=dt * 1e3, config=cfg, sample=sample)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "verify", "prefill", "paging", "paging48", "paging_ssd"])
    ap.add_argument("--ssd-dir", default=None, help="paging_ssd: directory of the expert file (default: the temp dir)")
    ap.add_argument("--prefetch", type=int, default=-1, help="paging48: experts prefetched per layer (-1: config)")
    ap.add_argument("--ffn-mode", default="auto", choices=["auto", "gemv", "gemm"],
                    help="verify/prefill: the expert FFN mode (auto: GEMV up to 16 tokens, else the grouped GEMM)")
    ap.add_argument("--device-staging", action="store_true",
                    help="paging, paging48: the cache policy and copies on the device (devcache_*)")
    ap.add_argument("--admit-min", type=int, default=0,
                    help="device staging: misses used fewer times are computed in place, not admitted")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--window", type=int, default=16)
    ap.add_argument("--chunk", type=int, default=8192)
    ap.add_argument("--layers", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--unfused", action="store_true", help="decode through the four separate calls")
    ap.add_argument("--decode-one-kernel", action="store_true",
                    help="fused decode through the one-kernel persistent step instead of the three-kernel chain")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    pk = peaks()

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        r = bench_reference(args, world, rank)
        if r is None:
            return
        line = {"metric": METRIC, "value": round(r["value"], 4), "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms"] / args.steps, 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded)", "impl": "reference",
                "config": r["config"],
                "cpu_baseline": {"value": round(r["value"], 4), "unit": "tokens/s", "cores": host_cores(),
                                 "kind": "oracle",
                                 "sample": f"{args.steps} steps, each {r['sample']}"},
                "e2e": {"value": round(r["value"], 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    world, rank, local = dist_setup(args.gpus)
    if args.workload == "paging":
        r = bench_paging(args, world, rank, pk)
    elif args.workload == "paging48":
        r = bench_paging48(args, world, rank, pk)
    elif args.workload == "paging_ssd":
        r = bench_paging_ssd(args, world, rank, pk)
    else:
        r = bench_layer(args, world, rank, pk)
    if rank == 0:
        line = {"metric": METRIC, "value": round(r["value"], 2), "unit": "tokens/s", "n_gpus": world,
                "steps": r["steps"], "warmup": args.warmup, "ms_per_step": round(r["ms"] / r["steps"], 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": r["dtype"],
                "data": "synthetic (seeded generators; no weights or datasets)", "config": r["config"],
                "roofline": r["roofline"], "cpu_baseline": r["cpu"], "e2e": r["e2e"],
                "gpu_launches": int(r["launches"]), "clocks": r["clocks"]}
        if r.get("routing"):
            line["routing"] = r["routing"]
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
