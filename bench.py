"""Benchmark of the grouped 4-bit MoE matmul library on B200.

Headline (one JSON line on rank 0): the Qwen3-30B-A3B-shaped NF4 decode
layer -- one token routed to 8 of 128 experts, gate_up (N=1536, K=2048) then
down (N=2048, K=768) through the bandwidth GEMV -- as HBM GB/s of
algorithmic bytes (packed codes + scales of the active experts + x + out).
A step is one such layer.  Consecutive steps rotate over 16 disjoint expert
sets, so a step never finds its 21 MB of weights in the 126 MB L2 (340 MB are
cycled).  Steps run as CUDA-graph replays.

Also measured on one GPU and reported under "secondary": Qwen3 prefill
(32768 routed rows) and the NF4 training dgrad on the tensor-core path,
gpt-oss-20b MXFP4 at 2048 tokens (tensor cores) and at one token (GEMV).

--impl reference times the CPU oracle (the plain fp64 definition) on the same
decode workload on the host cores.
Multi-GPU (torchrun): every rank runs an independent replica of the same
workload (the layer has no exchange step); value = all ranks' bytes / the
slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "grouped 4-bit MoE GEMM TFLOP/s (prefill) and decode GB/s, % of B200 roofline"
WORKLOAD = ("qwen3_30b_a3b_nf4_decode: E=128, top-8, 1 token; gate_up N=1536 K=2048 "
            "then down N=2048 K=768; weights N(0,0.02) NF4-packed, x N(0,1) bf16")
N_SETS = 16  # disjoint 8-expert sets cycled by consecutive steps
GRAPH_CHUNK = 1024  # layers per captured graph (a multiple of N_SETS)
GU_CHAIN = 256      # gate_up launches per graph when timing that kernel alone


def bench_config(world):
    """The workload description both arms print (identical dicts)."""
    return {"workload": WORKLOAD, "weights": "nf4 (absmax fp32 per 64)",
            "activations": "bf16", "experts_cycled": f"{N_SETS} disjoint sets of 8",
            "l2": "inputs larger than L2: 340 MB of packed weights cycled, 21 MB per step",
            "path": "bandwidth GEMV (GBW_MODE_AUTO picks it for P <= 4 E)",
            "parallelism": f"replicas x{world}"}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p["bf16_tflops_sustained"]), "measured")
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- units

def gemv_bytes(fmt, P, N, K, T_rows):
    """Algorithmic bytes of one grouped GEMV launch: the active experts'
    packed codes and scales (P rows, one per expert), x read once, out."""
    codes = P * N * K // 2
    scales = P * N * (K // 64) * 4 if fmt == "nf4" else P * N * (K // 32)
    return codes + scales + T_rows * K * 2 + P * N * 2


def gemm_flops(P, N, K):
    return 2.0 * P * N * K


# ---------------------------------------------------------------- ranks

def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank times its own replica on its own
    device; the job takes as long as the slowest one (a MAX all-reduce of
    one number, on the process group's backend: NCCL on GPUs, gloo in the
    CPU tests)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(bytes_per_rank_step: float, steps: int, world: int, ms_max: float,
             scale: float = 1e9) -> float:
    """Whole-job throughput: every rank processed `steps` steps of
    `bytes_per_rank_step`, all done when the slowest rank is."""
    return world * bytes_per_rank_step * steps / (ms_max * 1e-3) / scale


# ---------------------------------------------------------------- clocks

class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *a):
        self.rows = []
        if self.p is None:
            return
        time.sleep(0.25)
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except Exception:
            self.p.kill()
            out = ""
        for line in out.strip().splitlines():
            f = [s.strip() for s in line.split(",")]
            if len(f) >= 8:
                self.rows.append(f)

    def summary(self):
        rows = getattr(self, "rows", [])
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        pw = [num(r[2]) for r in rows if num(r[2]) is not None]
        busy = [s for s, p in zip(sm, pw) if p is not None and p > 250] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v == "Active"})
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max((num(r[1]) or 0) for r in rows),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------- GPU side

def make_nf4(torch, gbw, E, N, K, std, gen, dev):
    codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=dev)
    scale = torch.empty((E, N, K // 64), dtype=torch.float32, device=dev)
    for e in range(E):  # one expert at a time keeps the fp32 staging small
        w = torch.randn((N, K), generator=gen, device=dev) * std
        c, s = gbw.gnf4_quantize(w)
        codes[e].copy_(c)
        scale[e].copy_(s)
    return codes, scale


def make_mxfp4(torch, gbw, E, N, K, std, gen, dev):
    codes = torch.empty((E, N, K // 32, 16), dtype=torch.uint8, device=dev)
    scale = torch.empty((E, N, K // 32), dtype=torch.uint8, device=dev)
    for e in range(E):
        w = torch.randn((N, K), generator=gen, device=dev) * std
        c, s = gbw.gmxfp4_quantize(w)
        codes[e].copy_(c)
        scale[e].copy_(s)
    return codes, scale


def graph_upload(g, stream):
    """Uploads a captured graph's executable on `stream` (driver
    cuGraphUpload: runs nothing, moves the upload out of the first replay)."""
    import ctypes
    drv = ctypes.CDLL("libcuda.so.1")
    drv.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    rc = drv.cuGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                           ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"cuGraphUpload failed: {rc}")


def event_time_ms(torch, fn, iters, stream):
    """Average device time of fn() over iters calls, CUDA events on the
    launching stream, synchronised on both sides."""
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(iters):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def decode_routing(E, k, n_sets, seed):
    """Disjoint expert sets; set j routes one token to experts perm[k*j:k*(j+1)]."""
    import synth
    perm = np.random.default_rng(seed).permutation(E)
    return [synth.decode_routing(E, k, 0, experts=np.sort(perm[k * j:k * (j + 1)]))
            for j in range(n_sets)]


def run_ours(args, rank, world, dev):
    import torch
    import grouped_bit_weight_b200 as gbw
    import synth

    hbm, bf16, bf16_sus, peak_kind = peaks()
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + rank)
    launches = {"n": 0}

    # ---- the decode layer (headline) ----
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    wgu = make_nf4(torch, gbw, GU.E, GU.N, GU.K, GU.w_std, gen, dev)
    wdn = make_nf4(torch, gbw, DN.E, DN.N, DN.K, DN.w_std, gen, dev)
    sets = decode_routing(GU.E, 8, N_SETS, seed=5)
    offs = [torch.from_numpy(o).to(dev) for o, _ in sets]
    r2ts = [torch.from_numpy(r).to(dev) for _, r in sets]
    x_gu = (torch.randn((1, GU.K), generator=gen, device=dev)).to(torch.bfloat16)
    x_dn = (torch.randn((8, DN.K), generator=gen, device=dev)).to(torch.bfloat16)
    out_gu = torch.empty((8, GU.N), dtype=torch.bfloat16, device=dev)
    out_dn = torch.empty((8, DN.N), dtype=torch.bfloat16, device=dev)

    # The expert weights and the routing are written once, before the timed
    # loop, so every call may overlap the kernel before it (the library reads
    # x and writes out only after that kernel has finished).
    def step(j):
        gbw.gnf4_grouped_gemm(x_gu, wgu[0], wgu[1], offs[j], r2ts[j], out=out_gu,
                              overlap_prev=True)
        gbw.gnf4_grouped_gemm(x_dn, wdn[0], wdn[1], offs[j], None, out=out_dn,
                              overlap_prev=True)

    bytes_gu = gemv_bytes("nf4", 8, GU.N, GU.K, 1)
    bytes_dn = gemv_bytes("nf4", 8, DN.N, DN.K, 8)
    bytes_step = bytes_gu + bytes_dn

    for j in range(N_SETS):  # eager warm-up of every kernel / attribute
        step(j)
    torch.cuda.synchronize()
    assert gbw.device_status(dev) == 0

    # Exactly `n` layers, cycling the expert sets, as CUDA graphs of at most
    # GRAPH_CHUNK layers (a multiple of N_SETS, so replays continue the
    # cycle): the timed region is one graph launch for any --steps up to
    # GRAPH_CHUNK, and the step count does not change the per-step cost.
    def graphs_for(n):
        out = []
        for cnt, reps in ((GRAPH_CHUNK, n // GRAPH_CHUNK), (n % GRAPH_CHUNK, 1)):
            if cnt and reps:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for j in range(cnt):
                        step(j % N_SETS)
                out.append((g, reps))
        return out

    warm_graphs = graphs_for(args.warmup)
    timed_graphs = graphs_for(args.steps)
    for g, _ in timed_graphs:  # upload now: a first replay would pay it in the timed region
        graph_upload(g, stream)

    def run_graphs(gs):
        for g, reps in gs:
            for _ in range(reps):
                g.replay()

    # The clock sampler starts before the warm-up (it needs a moment to come
    # up), so the warm-up runs right before the timed region and the GPU is
    # not left idle between them.
    with Clocks(dev.index if dev.index is not None else 0) as clk:
        run_graphs(warm_graphs)
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        # a ~100 us device-side delay ahead of the start event keeps the GPU
        # busy while the host enqueues the event and the timed graphs, so the
        # region starts with the first kernel, not with the host's launch
        # latency (which is tens of microseconds against a 20-step region of
        # a few hundred)
        torch.cuda._sleep(200_000)
        t0.record(stream)
        run_graphs(timed_graphs)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    launches["n"] += 2 * args.steps
    ms_per_step = ms / args.steps
    value = job_rate(bytes_step, args.steps, world, ms)

    # dominant kernel: the gate_up GEMV alone, back to back in a graph of
    # one launch per expert set; average device time per launch
    gu_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gu_graph):
        for j in range(GU_CHAIN):
            gbw.gnf4_grouped_gemm(x_gu, wgu[0], wgu[1], offs[j % N_SETS], r2ts[j % N_SETS],
                                  out=out_gu, overlap_prev=True)
    gu_graph.replay()
    gu_ms = event_time_ms(torch, gu_graph.replay, 4, stream) / GU_CHAIN
    launches["n"] += 0  # the roofline loop runs outside the timed region
    achieved = bytes_gu / (gu_ms * 1e-3) / 1e9
    traffic = load_traffic("gemv_nf4_qwen3_decode_gate_up")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "traffic": traffic, "kernel": "gemv_kernel<NF4> (gate_up)",
                "timing": f"graph of {GU_CHAIN} back-to-back launches cycling the 16 expert sets, "
                          "replayed 4 times, CUDA events; per-launch mean",
                "algorithmic_bytes_per_launch": bytes_gu,
                "launch_ms": round(gu_ms, 5), "peak_source": peak_kind}

    # e2e: host buffers, copies inside the timed region, public API calls
    e2e = measure_e2e(torch, gbw, args, dev, stream, wgu, wdn, sets, bytes_step, world)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": bench_config(world),
        "timing": ("exactly --steps layers captured as CUDA graphs of up to "
                   f"{GRAPH_CHUNK} layers, CUDA events on the launching stream"),
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches["n"],
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_secondary:
        result["secondary"] = secondary(torch, gbw, synth, gen, dev, stream, hbm, bf16, peak_kind)
        for e in result["secondary"]:  # the decode comparator against this layer's packed path
            if e["workload"].startswith("comparator: dequantise-then-GEMM qwen3 decode layer"):
                e["packed_ms"] = round(ms_per_step, 6)
                e["packed_speedup"] = round(e["value"] / ms_per_step, 3)
        result["gpu_launches"] = launches["n"]
    return result


def load_traffic(name):
    """DRAM bytes per launch of `name` from the committed ncu summary
    (profiles/traffic.json), or None when absent or when the kernel sources
    have changed since the capture (their sha256 no longer matches)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            ent = json.load(f)[name]
        d = hashlib.sha256()
        for rel in ent["sources"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                d.update(f.read())
        return ent["bytes"] if d.hexdigest() == ent["source_sha256"] else None
    except Exception:
        return None


def measure_e2e(torch, gbw, args, dev, stream, wgu, wdn, sets, bytes_step, world=1):
    """Same decode layer through the public API with host buffers.  Every
    step writes its inputs (x for both projections, the step's expert
    offsets and row map) into one pinned staging buffer, copies it to the
    device in one transfer, makes the two library calls on views of it, and
    reads both outputs back in one transfer; one synchronisation per step.
    value: the step's copies and library calls captured once as a CUDA graph
    (as a decode loop runs them) and replayed each step after the host has
    written that step's routing; eager_value: the same steps issued call by
    call from Python."""
    import synth
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN

    def layout(parts):  # (name, bytes) -> 16-byte aligned offsets, total
        offs, at = {}, 0
        for name, nb in parts:
            offs[name] = (at, nb)
            at += (nb + 15) // 16 * 16
        return offs, at

    nxg, nxd = GU.K * 2, 8 * DN.K * 2
    noff, nr2t = sets[0][0].nbytes, sets[0][1].nbytes
    lin, nin = layout([("xg", nxg), ("xd", nxd), ("off", noff), ("r2t", nr2t)])
    lout, nout = layout([("og", 8 * GU.N * 2), ("od", 8 * DN.N * 2)])
    h_in = torch.zeros(nin, dtype=torch.uint8).pin_memory()
    h_out = torch.empty(nout, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(nin, dtype=torch.uint8, device=dev)
    d_out = torch.empty(nout, dtype=torch.uint8, device=dev)

    def view(buf, lay, name, dtype, shape):
        a, nb = lay[name]
        return buf[a:a + nb].view(dtype).view(shape)

    h_in_np = h_in.numpy()
    xg = torch.randn((1, GU.K)).to(torch.bfloat16)
    xd = torch.randn((8, DN.K)).to(torch.bfloat16)
    view(h_in, lin, "xg", torch.bfloat16, (1, GU.K)).copy_(xg)
    view(h_in, lin, "xd", torch.bfloat16, (8, DN.K)).copy_(xd)
    d_xgu = view(d_in, lin, "xg", torch.bfloat16, (1, GU.K))
    d_xdn = view(d_in, lin, "xd", torch.bfloat16, (8, DN.K))
    d_off = view(d_in, lin, "off", torch.int32, (GU.E + 1,))
    d_r2t = view(d_in, lin, "r2t", torch.int32, (8,))
    d_ogu = view(d_out, lout, "og", torch.bfloat16, (8, GU.N))
    d_odn = view(d_out, lout, "od", torch.bfloat16, (8, DN.N))
    raw = [(np.ascontiguousarray(o).view(np.uint8), np.ascontiguousarray(r).view(np.uint8))
           for o, r in sets]
    (ao, _), (ar, _) = lin["off"], lin["r2t"]
    bi, bo = nin, nout                     # bytes of the two transfers (incl. 16-byte padding)

    def one(j):
        o, r = raw[j]
        h_in_np[ao:ao + noff] = o          # this step's routing, host side
        h_in_np[ar:ar + nr2t] = r
        d_in.copy_(h_in, non_blocking=True)
        gbw.gnf4_grouped_gemm(d_xgu, wgu[0], wgu[1], d_off, d_r2t, out=d_ogu)
        gbw.gnf4_grouped_gemm(d_xdn, wdn[0], wdn[1], d_off, None, out=d_odn)
        h_out.copy_(d_out, non_blocking=True)
        stream.synchronize()

    def device_part():
        d_in.copy_(h_in, non_blocking=True)
        gbw.gnf4_grouped_gemm(d_xgu, wgu[0], wgu[1], d_off, d_r2t, out=d_ogu)
        gbw.gnf4_grouped_gemm(d_xdn, wdn[0], wdn[1], d_off, None, out=d_odn)
        h_out.copy_(d_out, non_blocking=True)

    o, r = raw[0]  # a valid routing before the first call (the buffer starts zeroed)
    h_in_np[ao:ao + noff] = o
    h_in_np[ar:ar + nr2t] = r
    device_part()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        device_part()
    graph_upload(g, stream)

    def one_graph(j):
        o, r = raw[j]
        h_in_np[ao:ao + noff] = o
        h_in_np[ar:ar + nr2t] = r
        g.replay()
        stream.synchronize()

    n = max(16, min(args.steps, 2000))

    def timed(fn):
        for j in range(32):
            fn(j % N_SETS)
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        t = time.perf_counter()
        for i in range(n):
            fn(i % N_SETS)
        return max_over_ranks((time.perf_counter() - t) * 1e3, world, dev)

    ms_graph = timed(one_graph)
    from_graph = h_out.clone()  # the last step's outputs, from the replayed graph
    ms_eager = timed(one)       # ends with the same step's routing
    assert torch.equal(from_graph, h_out), "graph replay and eager calls disagree"
    assert gbw.device_status(dev) == 0, "device error during the end-to-end steps"
    del g
    return {"value": round(job_rate(bytes_step, n, world, ms_graph), 2), "unit": "GB/s",
            "eager_value": round(job_rate(bytes_step, n, world, ms_eager), 2),
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": n,
            "timing": "host wall clock around steps that each write their routing into "
                      "pinned memory, copy the inputs in and the outputs out (one transfer "
                      "each way) and end in a stream sync; value replays the step captured "
                      "as a CUDA graph, eager_value issues it call by call; max over ranks"}


def secondary(torch, gbw, synth, gen, dev, stream, hbm, bf16, peak_kind):
    out = []

    def tc_entry(name, flops, fn, iters=20):
        for _ in range(3):
            fn()
        ms = event_time_ms(torch, fn, iters, stream)
        tf = flops / (ms * 1e-3) / 1e12
        return {"workload": name, "value": round(tf, 1), "unit": "TFLOP/s",
                "ms": round(ms, 4),
                "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                             "peak": bf16, "unit": "TFLOP/s",
                             "frac": round(tf / bf16, 4), "peak_source": peak_kind}}

    def hbm_entry(name, nbytes, ms, extra=None):
        gbs = nbytes / (ms * 1e-3) / 1e9
        e = {"workload": name, "value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 5),
             "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                          "unit": "GB/s", "frac": round(gbs / hbm, 4), "peak_source": peak_kind}}
        if extra:
            e.update(extra)
        return e

    def graph_ms(fn, n_inner, replays=20):
        """Device time of fn() captured n_inner times in one CUDA graph, per
        inner call (CUDA events around `replays` replays)."""
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n_inner):
                fn()
        g.replay()
        return event_time_ms(torch, g.replay, replays, stream) / n_inner

    # Qwen3-30B-A3B prefill, NF4, tensor cores
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    off, r2t = synth.prefill_routing()
    P = int(off[-1])
    d_off = torch.from_numpy(off).to(dev)
    d_r2t = torch.from_numpy(r2t).to(dev)
    wgu = make_nf4(torch, gbw, GU.E, GU.N, GU.K, GU.w_std, gen, dev)
    wdn = make_nf4(torch, gbw, DN.E, DN.N, DN.K, DN.w_std, gen, dev)
    x = torch.randn((4096, GU.K), generator=gen, device=dev).to(torch.bfloat16)
    o = torch.empty((P, GU.N), dtype=torch.bfloat16, device=dev)
    gu_prefill = tc_entry("qwen3 prefill gate_up NF4 (P=32768, N=1536, K=2048)",
                          gemm_flops(P, GU.N, GU.K),
                          lambda: gbw.gnf4_grouped_gemm(x, wgu[0], wgu[1], d_off, d_r2t, out=o))
    out.append(gu_prefill)
    dy = (torch.randn((P, GU.N), generator=gen, device=dev) * 1e-2).to(torch.bfloat16)
    dx = torch.empty((P, GU.K), dtype=torch.bfloat16, device=dev)
    out.append(tc_entry("qwen3 dgrad gate_up NF4 (P=32768, N=1536, K=2048)",
                        gemm_flops(P, GU.N, GU.K),
                        lambda: gbw.gnf4_grouped_dgrad(dy, wgu[0], wgu[1], d_off, out=dx)))
    del dy, dx
    xd = torch.randn((P, DN.K), generator=gen, device=dev).to(torch.bfloat16)
    od = torch.empty((P, DN.N), dtype=torch.bfloat16, device=dev)
    dn_prefill = tc_entry("qwen3 prefill down NF4 (P=32768, N=2048, K=768)",
                          gemm_flops(P, DN.N, DN.K),
                          lambda: gbw.gnf4_grouped_gemm(xd, wdn[0], wdn[1], d_off, None, out=od))
    out.append(dn_prefill)
    dyd = (torch.randn((P, DN.N), generator=gen, device=dev) * 1e-2).to(torch.bfloat16)
    dxd = torch.empty((P, DN.K), dtype=torch.bfloat16, device=dev)
    out.append(tc_entry("qwen3 dgrad down NF4 (P=32768, N=2048, K=768)",
                        gemm_flops(P, DN.N, DN.K),
                        lambda: gbw.gnf4_grouped_dgrad(dyd, wdn[0], wdn[1], d_off, out=dxd)))
    del dyd, dxd

    # fused expert pass: gate_up with the SwiGLU epilogue, then down over h
    hbuf = torch.empty((P, DN.K), dtype=torch.bfloat16, device=dev)
    of = torch.empty((P, DN.N), dtype=torch.bfloat16, device=dev)
    out.append(tc_entry("qwen3 prefill fused expert pass NF4 (gate_up + SwiGLU + down, P=32768)",
                        gemm_flops(P, GU.N, GU.K) + gemm_flops(P, DN.N, DN.K),
                        lambda: gbw.gnf4_grouped_expert_mlp(x, wgu[0], wgu[1], wdn[0], wdn[1], d_off,
                                                            d_r2t, h=hbuf, out=of)))
    sets = decode_routing(GU.E, 8, N_SETS, seed=5)
    offs = [torch.from_numpy(a).to(dev) for a, _ in sets]
    r2ts = [torch.from_numpy(b).to(dev) for _, b in sets]
    x1 = torch.randn((1, GU.K), generator=gen, device=dev).to(torch.bfloat16)
    h1 = torch.empty((8, DN.K), dtype=torch.bfloat16, device=dev)
    o1 = torch.empty((8, DN.N), dtype=torch.bfloat16, device=dev)
    it = {"j": 0}

    def fused_decode():
        j = it["j"] % N_SETS
        it["j"] += 1
        gbw.gnf4_grouped_expert_mlp(x1, wgu[0], wgu[1], wdn[0], wdn[1], offs[j], r2ts[j],
                                    h=h1, out=o1)
    ms = graph_ms(fused_decode, N_SETS)
    out.append(hbm_entry("qwen3 decode fused expert pass NF4 (1 token, 8 experts; gate_up with "
                         "SwiGLU then down, both on the bandwidth GEMV)",
                         gemv_bytes("nf4", 8, GU.N, GU.K, 1) + gemv_bytes("nf4", 8, DN.N, DN.K, 8), ms))

    # a decode batch of 4 tokens (top-8: 32 routed rows, some experts with
    # 2-3): AUTO takes the GEMV; an expert's rows are consecutive, so its
    # weights come from HBM once and from L2 for its other rows.  bytes = the
    # active experts' codes and scales once + x + out
    bsets = [synth.uniform_routing(4, GU.E, 8, seed=200 + j) for j in range(N_SETS)]
    boffs = [torch.from_numpy(a).to(dev) for a, _ in bsets]
    br2ts = [torch.from_numpy(b).to(dev) for _, b in bsets]
    xb = torch.randn((4, GU.K), generator=gen, device=dev).to(torch.bfloat16)
    ob = torch.empty((32, GU.N), dtype=torch.bfloat16, device=dev)
    it["j"] = 0

    def batch_step():
        j = it["j"] % N_SETS
        it["j"] += 1
        gbw.gnf4_grouped_gemm(xb, wgu[0], wgu[1], boffs[j], br2ts[j], out=ob, overlap_prev=True)
    ms = graph_ms(batch_step, N_SETS)
    act = float(np.mean([(np.diff(a) > 0).sum() for a, _ in bsets]))
    nbytes = act * (GU.N * GU.K // 2 + GU.N * (GU.K // 64) * 4) + 4 * GU.K * 2 + 32 * GU.N * 2
    out.append(hbm_entry(f"qwen3 decode batch of 4 tokens gate_up NF4 (32 routed rows over "
                         f"{act:.1f} active experts; bytes count each expert's weights once)", nbytes, ms))

    # dequantise-then-GEMM comparator: decode the weights to bf16 in HBM
    # (the library's bit-exact decoder), then cuBLAS bf16 matmuls per expert
    out += dequant_comparator(torch, gbw, x, xd, wgu, wdn, off, r2t, d_r2t, sets, gu_prefill,
                              dn_prefill, graph_ms, dev)
    del wgu, wdn, x, o, xd, od, hbuf, of
    torch.cuda.empty_cache()

    # gpt-oss-20b MXFP4: 2048 tokens (tensor cores) and 1 token (GEMV)
    for L in (synth.GPTOSS_GATE_UP, synth.GPTOSS_DOWN):
        w = make_mxfp4(torch, gbw, L.E, L.N, L.K, L.w_std, gen, dev)
        off, r2t = synth.uniform_routing(2048, L.E, 4, seed=7)
        P = int(off[-1])
        d_off, d_r2t = torch.from_numpy(off).to(dev), torch.from_numpy(r2t).to(dev)
        x = torch.randn((2048, L.K), generator=gen, device=dev).to(torch.bfloat16)
        o = torch.empty((P, L.N), dtype=torch.bfloat16, device=dev)
        packed = tc_entry(f"gpt-oss-20b {L.name.split('_')[-1]} MXFP4 batch 2048 (P=8192, N={L.N}, K={L.K})",
                          gemm_flops(P, L.N, L.K),
                          lambda: gbw.gmxfp4_grouped_gemm(x, w[0], w[1], d_off, d_r2t, out=o))
        out.append(packed)
        out.append(comparator_prefill(torch, gbw.gmxfp4_dequant, w, L, x, off, d_r2t, packed,
                                      graph_ms, dev, "gpt-oss-20b batch 2048"))
        dyg = (torch.randn((P, L.N), generator=gen, device=dev) * 1e-2).to(torch.bfloat16)
        dxg = torch.empty((P, L.K), dtype=torch.bfloat16, device=dev)
        out.append(tc_entry(f"gpt-oss-20b {L.name.split('_')[-1]} MXFP4 dgrad batch 2048 (P=8192, N={L.N}, K={L.K})",
                            gemm_flops(P, L.N, L.K),
                            lambda: gbw.gmxfp4_grouped_dgrad(dyg, w[0], w[1], d_off, out=dxg)))
        del dyg, dxg
        sets = decode_routing(L.E, 4, 8, seed=9)
        offs = [torch.from_numpy(a).to(dev) for a, _ in sets]
        r2ts = [torch.from_numpy(b).to(dev) for _, b in sets]
        x1 = torch.randn((1, L.K), generator=gen, device=dev).to(torch.bfloat16)
        o1 = torch.empty((4, L.N), dtype=torch.bfloat16, device=dev)
        for j in range(8):
            gbw.gmxfp4_grouped_gemm(x1, w[0], w[1], offs[j], r2ts[j], out=o1)
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1):
            for j in range(8):
                gbw.gmxfp4_grouped_gemm(x1, w[0], w[1], offs[j], r2ts[j], out=o1)
        ms = event_time_ms(torch, g1.replay, 40, stream) / 8
        nbytes = gemv_bytes("mxfp4", 4, L.N, L.K, 1)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out.append({"workload": f"gpt-oss-20b {L.name.split('_')[-1]} MXFP4 batch 1 (P=4, N={L.N}, K={L.K}), 8 expert sets cycled",
                    "value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 5),
                    "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                                 "unit": "GB/s", "frac": round(gbs / hbm, 4),
                                 "peak_source": peak_kind}})
        del w, x, o
        torch.cuda.empty_cache()
    torch.cuda.synchronize()
    assert gbw.device_status(dev) == 0
    return out


def comparator_prefill(torch, dequant, w, L, xin, off, d_r2t, packed, graph_ms, dev, what):
    """Dequantise-then-GEMM for one projection of a large batch: every
    expert of the layer decoded to bf16 in one launch, the routed rows
    gathered (index_select through row_to_token, when given), one cuBLAS
    bf16 matmul per expert with rows; one CUDA graph, timed by replays."""
    live = [int(e) for e in np.nonzero(np.diff(off))[0]]
    P = int(off[-1])
    wbf = torch.empty((L.E, L.N, L.K), dtype=torch.bfloat16, device=dev)
    xg = torch.empty((P, L.K), dtype=torch.bfloat16, device=dev) if d_r2t is not None else None
    ob = torch.empty((P, L.N), dtype=torch.bfloat16, device=dev)
    r2t_long = d_r2t.long() if d_r2t is not None else None

    def step():
        dequant(w[0], w[1], out=wbf)
        src = xin
        if r2t_long is not None:
            torch.index_select(xin, 0, r2t_long, out=xg)
            src = xg
        for e in live:
            a, b = int(off[e]), int(off[e + 1])
            torch.mm(src[a:b], wbf[e].t(), out=ob[a:b])
    ms = graph_ms(step, 1, replays=10)
    del wbf, xg, ob
    return {"workload": f"comparator: dequantise-then-GEMM {what} {L.name.split('_')[-1]} "
                        f"({dequant.__name__} of all {L.E} experts + {len(live)} cuBLAS bf16 "
                        f"matmuls)",
            "value": round(ms, 4), "unit": "ms", "higher_is_better": False,
            "packed_ms": packed["ms"], "packed_speedup": round(ms / packed["ms"], 3)}


def dequant_comparator(torch, gbw, x, xd, wgu, wdn, off, r2t, d_r2t, sets, gu_prefill,
                       dn_prefill, graph_ms, dev):
    """The pages' control experiment ("dequant tax"): the same projections
    computed by first decoding the packed weights to bf16 in HBM
    (gnf4_dequant or gmxfp4_dequant, bit-exact), then bf16 matmuls by cuBLAS (torch.mm per
    expert with routed rows, captured in one CUDA graph).  Reported next to
    the packed path as time and the packed path's speedup."""
    import synth
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    res = [comparator_prefill(torch, gbw.gnf4_dequant, w, L, xin, off, rows, packed, graph_ms,
                              dev, "qwen3 prefill")
           for L, w, xin, rows, packed in ((GU, wgu, x, d_r2t, gu_prefill),
                                           (DN, wdn, xd, None, dn_prefill))]
    # decode layer: dequantise the 8 active experts of each projection, then
    # batched matmuls (one token for gate_up, one row per expert for down)
    wg8 = torch.empty((8, GU.N, GU.K), dtype=torch.bfloat16, device=dev)
    wd8 = torch.empty((8, DN.N, DN.K), dtype=torch.bfloat16, device=dev)
    x1 = torch.randn((1, 1, GU.K), device=dev).to(torch.bfloat16).expand(8, 1, GU.K)
    xd8 = torch.randn((8, 1, DN.K), device=dev).to(torch.bfloat16)
    og8 = torch.empty((8, 1, GU.N), dtype=torch.bfloat16, device=dev)
    od8 = torch.empty((8, 1, DN.N), dtype=torch.bfloat16, device=dev)
    experts = [[int(e) for e in np.nonzero(np.diff(o))[0]] for o, _ in sets]
    it = {"j": 0}

    def layer():
        ex = experts[it["j"] % len(experts)]
        it["j"] += 1
        for i, e in enumerate(ex):
            gbw.gnf4_dequant(wgu[0][e], wgu[1][e], out=wg8[i])
            gbw.gnf4_dequant(wdn[0][e], wdn[1][e], out=wd8[i])
        torch.bmm(x1, wg8.transpose(1, 2), out=og8)
        torch.bmm(xd8, wd8.transpose(1, 2), out=od8)
    ms = graph_ms(layer, len(experts))
    res.append({"workload": "comparator: dequantise-then-GEMM qwen3 decode layer (16 gnf4_dequant "
                            "launches for the 8 active experts of both projections + 2 cuBLAS "
                            "batched bf16 matmuls)",
                "value": round(ms, 5), "unit": "ms", "higher_is_better": False})
    return res


# ---------------------------------------------------------------- single cases

def run_case(args, dev):
    """One kernel on one workload, `--warmup` then `--steps` launches, for
    profiling (ncu -k / -s / -c pick launches out of this command)."""
    import torch
    import grouped_bit_weight_b200 as gbw
    import synth
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)
    c = args.case
    if c in ("decode_gate_up", "decode_down"):
        L = synth.QWEN_GATE_UP if c == "decode_gate_up" else synth.QWEN_DOWN
        w = make_nf4(torch, gbw, L.E, L.N, L.K, L.w_std, gen, dev)
        sets = decode_routing(L.E, 8, N_SETS, seed=5)
        offs = [torch.from_numpy(o).to(dev) for o, _ in sets]
        r2ts = [torch.from_numpy(r).to(dev) for _, r in sets]
        T = 1 if L is synth.QWEN_GATE_UP else 8
        x = torch.randn((T, L.K), generator=gen, device=dev).to(torch.bfloat16)
        o = torch.empty((8, L.N), dtype=torch.bfloat16, device=dev)
        it = {"i": 0}
        def fn():
            j = it["i"] % N_SETS
            it["i"] += 1
            gbw.gnf4_grouped_gemm(x, w[0], w[1], offs[j], r2ts[j] if T == 1 else None, out=o)
        nbytes, unit = gemv_bytes("nf4", 8, L.N, L.K, T), "GB/s"
    elif c in ("prefill_gate_up", "prefill_down", "dgrad_gate_up", "dgrad_down"):
        L = synth.QWEN_GATE_UP if c.endswith("gate_up") else synth.QWEN_DOWN
        off, r2t = synth.prefill_routing()
        P = int(off[-1])
        d_off, d_r2t = torch.from_numpy(off).to(dev), torch.from_numpy(r2t).to(dev)
        w = make_nf4(torch, gbw, L.E, L.N, L.K, L.w_std, gen, dev)
        if c.startswith("prefill"):
            T = 4096 if L is synth.QWEN_GATE_UP else P
            x = torch.randn((T, L.K), generator=gen, device=dev).to(torch.bfloat16)
            o = torch.empty((P, L.N), dtype=torch.bfloat16, device=dev)
            rt = d_r2t if T == 4096 else None
            fn = lambda: gbw.gnf4_grouped_gemm(x, w[0], w[1], d_off, rt, out=o)
        else:
            dy = (torch.randn((P, L.N), generator=gen, device=dev) * 1e-2).to(torch.bfloat16)
            o = torch.empty((P, L.K), dtype=torch.bfloat16, device=dev)
            fn = lambda: gbw.gnf4_grouped_dgrad(dy, w[0], w[1], d_off, out=o)
        nbytes, unit = gemm_flops(P, L.N, L.K), "TFLOP/s"
    elif c in ("mxfp4_2048_gate_up", "mxfp4_2048_down", "mxfp4_1_gate_up", "mxfp4_1_down"):
        L = synth.GPTOSS_GATE_UP if c.endswith("gate_up") else synth.GPTOSS_DOWN
        w = make_mxfp4(torch, gbw, L.E, L.N, L.K, L.w_std, gen, dev)
        T = 2048 if "_2048_" in c else 1
        off, r2t = (synth.uniform_routing(T, L.E, 4, seed=7) if T > 1
                    else synth.decode_routing(L.E, 4, 0))
        P = int(off[-1])
        d_off, d_r2t = torch.from_numpy(off).to(dev), torch.from_numpy(r2t).to(dev)
        x = torch.randn((T, L.K), generator=gen, device=dev).to(torch.bfloat16)
        o = torch.empty((P, L.N), dtype=torch.bfloat16, device=dev)
        fn = lambda: gbw.gmxfp4_grouped_gemm(x, w[0], w[1], d_off, d_r2t, out=o)
        nbytes, unit = ((gemm_flops(P, L.N, L.K), "TFLOP/s") if T > 1
                        else (gemv_bytes("mxfp4", P, L.N, L.K, 1), "GB/s"))
    elif c == "decode_batch4_gate_up":
        L = synth.QWEN_GATE_UP
        w = make_nf4(torch, gbw, L.E, L.N, L.K, L.w_std, gen, dev)
        sets = [synth.uniform_routing(4, L.E, 8, seed=200 + j) for j in range(N_SETS)]
        offs = [torch.from_numpy(o).to(dev) for o, _ in sets]
        r2ts = [torch.from_numpy(r).to(dev) for _, r in sets]
        x = torch.randn((4, L.K), generator=gen, device=dev).to(torch.bfloat16)
        o = torch.empty((32, L.N), dtype=torch.bfloat16, device=dev)
        it = {"i": 0}
        def fn():
            j = it["i"] % N_SETS
            it["i"] += 1
            gbw.gnf4_grouped_gemm(x, w[0], w[1], offs[j], r2ts[j], out=o)
        act = float(np.mean([(np.diff(a) > 0).sum() for a, _ in sets]))
        nbytes, unit = act * (L.N * L.K // 2 + L.N * (L.K // 64) * 4) + 4 * L.K * 2 + 32 * L.N * 2, "GB/s"
    elif c in ("mxfp4_dgrad_gate_up", "mxfp4_dgrad_down"):
        L = synth.GPTOSS_GATE_UP if c.endswith("gate_up") else synth.GPTOSS_DOWN
        w = make_mxfp4(torch, gbw, L.E, L.N, L.K, L.w_std, gen, dev)
        off, _ = synth.uniform_routing(2048, L.E, 4, seed=7)
        P = int(off[-1])
        d_off = torch.from_numpy(off).to(dev)
        dy = (torch.randn((P, L.N), generator=gen, device=dev) * 1e-2).to(torch.bfloat16)
        o = torch.empty((P, L.K), dtype=torch.bfloat16, device=dev)
        fn = lambda: gbw.gmxfp4_grouped_dgrad(dy, w[0], w[1], d_off, out=o)
        nbytes, unit = gemm_flops(P, L.N, L.K), "TFLOP/s"
    elif c in ("fused_prefill", "fused_decode"):
        GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
        wgu = make_nf4(torch, gbw, GU.E, GU.N, GU.K, GU.w_std, gen, dev)
        wdn = make_nf4(torch, gbw, DN.E, DN.N, DN.K, DN.w_std, gen, dev)
        if c == "fused_prefill":
            off, r2t = synth.prefill_routing()
            T = 4096
        else:
            off, r2t = synth.decode_routing(GU.E, 8, 0)
            T = 1
        P = int(off[-1])
        d_off, d_r2t = torch.from_numpy(off).to(dev), torch.from_numpy(r2t).to(dev)
        x = torch.randn((T, GU.K), generator=gen, device=dev).to(torch.bfloat16)
        h = torch.empty((P, DN.K), dtype=torch.bfloat16, device=dev)
        o = torch.empty((P, DN.N), dtype=torch.bfloat16, device=dev)
        fn = lambda: gbw.gnf4_grouped_expert_mlp(x, wgu[0], wgu[1], wdn[0], wdn[1], d_off, d_r2t,
                                                 h=h, out=o)
        if T > 1:
            nbytes, unit = gemm_flops(P, GU.N, GU.K) + gemm_flops(P, DN.N, DN.K), "TFLOP/s"
        else:
            nbytes, unit = gemv_bytes("nf4", 8, GU.N, GU.K, 1) + gemv_bytes("nf4", 8, DN.N, DN.K, 8), "GB/s"
    else:
        raise SystemExit(f"unknown case {c}")
    for _ in range(args.warmup):
        fn()
    ms = event_time_ms(torch, fn, args.steps, stream)
    assert gbw.device_status(dev) == 0
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    print(json.dumps({"case": c, "ms": round(ms, 5), "launches": args.steps,
                      "value": round(nbytes / (ms * 1e-3) / scale, 2), "unit": unit}))


# ---------------------------------------------------------------- oracle side

def oracle_decode_step_fn():
    """One decode layer by the CPU oracle: decode the 8 active experts'
    weights, then the fp64 grouped matmuls (inputs drawn on the CPU)."""
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import oracle as orc
    import synth
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    pg = orc.nf4_pack(synth.normal((8, GU.N, GU.K), 31, GU.w_std))
    pd = orc.nf4_pack(synth.normal((8, DN.N, DN.K), 32, DN.w_std))
    xg = synth.to_bf16_bits(synth.normal((1, GU.K), 33))
    xd = synth.to_bf16_bits(synth.normal((8, DN.K), 34))
    off = np.arange(9, dtype=np.int32)        # one row per active expert
    r2t = np.zeros(8, np.int32)

    def step():
        wg = orc.nf4_decode(pg[0], pg[1], GU.K, bf16=True)
        orc.grouped_forward(xg, wg, off, r2t)
        wd = orc.nf4_decode(pd[0], pd[1], DN.K, bf16=True)
        orc.grouped_forward(xd, wd, off, None)
    return step, orc.num_threads()


def run_reference(args):
    import synth
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    step, cores = oracle_decode_step_fn()
    nbytes = gemv_bytes("nf4", 8, GU.N, GU.K, 1) + gemv_bytes("nf4", 8, DN.N, DN.K, 8)
    for _ in range(max(1, min(args.warmup, 3))):
        step()
    n = max(1, min(args.steps, 40))
    t = time.perf_counter()
    for _ in range(n):
        step()
    dt = time.perf_counter() - t
    v = nbytes * n / dt / 1e9
    sample = f"{n} full decode layers (8 experts x gate_up + down), fp64 oracle"
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
            "n_gpus": 1, "steps": n, "warmup": args.warmup,
            "ms_per_step": round(dt / n * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def cpu_baseline():
    """The oracle, as it stands, on ~10-30 s of the decode workload; plus the
    tiny NF4 config on one thread (a 1-core figure)."""
    import synth
    GU, DN = synth.QWEN_GATE_UP, synth.QWEN_DOWN
    step, cores = oracle_decode_step_fn()
    nbytes = gemv_bytes("nf4", 8, GU.N, GU.K, 1) + gemv_bytes("nf4", 8, DN.N, DN.K, 8)
    step()
    n, t = 0, time.perf_counter()
    while time.perf_counter() - t < 10.0 and n < 20000:
        step()
        n += 1
    dt = time.perf_counter() - t
    return {"value": round(nbytes * n / dt / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{n} full decode layers (8 experts, gate_up + down) in {dt:.1f} s",
            "tiny_single_thread": oracle_tiny_single_thread()}


def oracle_tiny_single_thread():
    """Config 1 (E=8, N=256, K=512, 64 tokens top-2 -> 128 routed rows) by
    the oracle on one thread: NF4 decode of the 8 experts + fp64 grouped
    forward, in GFLOP/s of 2*P*N*K."""
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import oracle as orc
    import synth
    off, r2t = synth.tiny_routing(0)
    codes, absmax = orc.nf4_pack(synth.normal((8, 256, 512), 1))
    x = synth.to_bf16_bits(synth.normal((64, 512), 2))
    prev = orc.num_threads()
    orc.set_num_threads(1)
    try:
        def one():
            w = orc.nf4_decode(codes, absmax, 512, bf16=True)
            orc.grouped_forward(x, w, off, r2t)
        one()
        n, t = 0, time.perf_counter()
        while time.perf_counter() - t < 2.0:
            one()
            n += 1
        dt = time.perf_counter() - t
    finally:
        orc.set_num_threads(prev)
    flops = gemm_flops(int(off[-1]), 256, 512)
    return {"value": round(flops * n / dt / 1e9, 4), "unit": "GFLOP/s", "cores": 1,
            "ms_per_call": round(dt / n * 1e3, 3),
            "sample": f"{n} calls of decode + grouped forward, tiny NF4 config"}


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=3200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None,
                    help="time one kernel on one workload (profiling helper)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    dev = torch.device("cuda", local)
    if args.case:
        run_case(args, dev)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(dev)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    res = run_ours(args, rank, world, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
