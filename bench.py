"""Benchmark of the routed MXFP4 MoE layer on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                [--extra NAMES | --no-extra]

One step = one pass of the whole layer (route, permute, routed experts, gated
shared expert, combine) over one batch of synthetic input, weights resident in
HBM. Each timed step is a CUDA-graph replay of moe_layer, bracketed by CUDA
events on the launching stream; L2 is flushed before every
step, outside the events. With N > 1 (torchrun) every rank runs an independent
replica of the layer (the layer does not shard: no collective on the data
path); timing is the max over ranks and ``value`` counts the tokens of all
ranks ("scaling": "weak").

Activations: decode workloads keep bf16 activations (exact f16 operand of the
grouped GEMVs); prefill workloads quantise them to MXFP4 for the tcgen05
block-scaled GEMMs (``--act`` overrides).

The printed line is the decode1 workload (T=1 H=8192 I=2048 E=512 k=10,
I_shared=2048); by default the same measurement of decode32, latent16 and
prefill4096 rides in the same line under ``workloads`` (``--extra`` /
``--no-extra`` change that; extras time min(steps, 10) steps).

Extra keys: ``roofline`` for the routed-expert call (moe_expert_ffn), timed
alone in its own loop with the same flushing, against HBM bandwidth or, when
its FLOPs take longer than its bytes at peak, the FP4 tensor peak;
``cpu_baseline`` (the C++ fp64 oracle on the host cores, all threads and one
thread, rank 0 only); ``e2e`` (the same metric through moe_layer with the
step's x copied in from pinned host memory and y copied back, inside the
timed region); ``clocks`` (nvidia-smi samples taken during the timed region).
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

METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill MXF4 TFLOPS as % of roofline"
DATA = ("synthetic, seeded: x ~ N(0,1) and bf16 weights ~ N(0,0.02) rounded to bf16; routed "
        "MXFP4 codes uniform over 0..15, E8M0 scale codes uniform over 120..127; skewed routing "
        "(decode32: 60% of tokens Zipf(1.1) over a hot set of 64; prefill: Zipf(1.1) over all "
        "experts); random-init weights, no checkpoint")
EXTRA_DEFAULT = ("decode32", "latent16", "prefill4096")
EXPERT_BYTES_PER_ROW_BLOCK = 17   # 16 packed bytes + 1 E8M0 code per 32 weights


def workload_label(w):
    lat = f" L={w.L}" if w.L else ""
    return (f"{w.name}: T={w.T} H={w.H} I={w.I} E={w.E} k={w.k} I_shared={w.I_shared}{lat}"
            f" skew={w.skew}")


def expert_bytes(w):
    """HBM bytes of one routed expert (gate + up + down, codes + scales)."""
    per_matrix = w.I * w.W // 32 * EXPERT_BYTES_PER_ROW_BLOCK
    return 3 * per_matrix


def dense_bytes(w):
    b = 2 * (w.E * w.H + 3 * w.I_shared * w.H + w.H)
    if w.L:
        b += 2 * 2 * w.L * w.H
    return b


def layer_bytes(w, n_active):
    """Algorithmic bytes of one layer pass: every weight read once plus x in and y out."""
    return n_active * expert_bytes(w) + dense_bytes(w) + w.T * w.H * 2 + w.T * w.H * 4


def ffn_bytes(w, n_active, act="bf16"):
    """Algorithmic bytes of one moe_expert_ffn call: the active experts' weights
    read once, the activation operand read once (bf16 rows, or MXFP4 codes +
    scales per (token, slot) row), and the routed output at its algorithmic
    size T x W fp32. Intermediates this implementation chose (per-slot fp32
    y_perm rows, h written by gate/up and read by down) are not counted; see
    ffn_intermediate_bytes."""
    R = w.T * w.k
    x_op = R * w.W * 17 // 32 if act == "mxfp4" else w.T * w.W * 2
    return n_active * expert_bytes(w) + x_op + w.T * w.W * 4


def ffn_intermediate_bytes(w, act="bf16"):
    """DRAM bytes of this implementation's intermediates per call (not in the
    roofline): y_perm rows [T*k, W] fp32 written (the per-slot output beyond
    the T x W counted above) and h written + read (fp32 in bf16 mode, MXFP4 in
    MXFP4 mode)."""
    R = w.T * w.k
    h = 2 * R * w.I * (17 / 32 if act == "mxfp4" else 4)
    return int((R - w.T) * w.W * 4 + h)


def ffn_flops(w):
    """Multiply-adds x 2 of the routed experts: gate, up and down for every (token, slot)."""
    return 2 * w.T * w.k * 3 * w.I * w.W


def layer_flops(w):
    R = w.T * w.k
    f = 2 * R * 3 * w.I * w.W + 2 * w.T * (3 * w.I_shared * w.H + w.H) + 2 * w.T * w.E * w.H
    if w.L:
        f += 2 * 2 * w.T * w.L * w.H
    return f


# sources of the single-token expert kernel whose DRAM counters profiles/traffic.json holds
TRAFFIC_SOURCES = ("gemv_fma.cu", "common.cuh", "tc05.cuh")


def _csrc_digest(files=TRAFFIC_SOURCES):
    import hashlib
    d = os.path.join(ROOT, "mxfp4_routed_expert_04_b200", "csrc")
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def _traffic(workload):
    """DRAM bytes per moe_expert_ffn call from the committed ncu summary, if it
    was taken on the current sources of those kernels (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        if t.get("csrc_sha") == _csrc_digest() and workload in t.get("bytes_per_call", {}):
            return t["bytes_per_call"][workload]
    except Exception:
        pass
    return None


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


FP4_PER_BF16 = 4.0      # nominal dense ratio: 9 PFLOP/s FP4 / 2.25 PFLOP/s bf16


def _fp4_peak_tflops():
    """FP4 dense tensor peak = measured cuBLAS bf16 burst x the nominal ratio."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]) * FP4_PER_BF16, "measured bf16 burst x 4 (nominal fp4/bf16)"
    except Exception:
        return 1590.0 * FP4_PER_BF16, "fallback bf16 x 4 (nominal fp4/bf16)"


def default_act(w):
    """Prefill-sized batches quantise activations to MXFP4 for the tcgen05 block-scaled
    MMA; decode keeps bf16 activations (f16 operand, exact)."""
    return "mxfp4" if w.name.startswith("prefill") else "bf16"


class ClockSampler:
    """nvidia-smi samples (200 ms) during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:6]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist_env():
    n = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), n


def max_over_ranks(value, world, device):
    """The largest of the ranks' values (every rank calls this in the same
    order; world == 1: the value itself)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank, world, step_ms):
    """Whole-job throughput of N replicas: every rank's tokens over the slowest
    rank's step time."""
    return tokens_per_rank * world / (step_ms * 1e-3)


def measure(args, w, steps, rank, local_rank, world, act=None):
    """Time one workload on this rank (every rank runs the same collective
    steps in the same order); returns the workload's result dict on rank 0,
    None elsewhere."""
    import torch
    import torch.distributed as dist

    import mxfp4_routed_expert_04_b200 as M
    import synth

    dev = synth.to_device(w)
    act = act or default_act(w)
    dims = M.MoeDims.of(w, M.ACT_MXFP4 if act == "mxfp4" else M.ACT_BF16)
    layer = M.MoeLayer(dims, {k: v for k, v in dev.items() if k != "x"})
    x = dev["x"]
    stream = torch.cuda.Stream()
    # L2 flush outside the timed region: write 512 MiB, then read another
    # 512 MiB so the written lines are evicted (written back) before the events
    # start and no write-back of the flush itself lands inside a timed step
    flush_w = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(128 << 20, dtype=torch.float32, device="cuda")
    flush_sink = torch.empty((), dtype=torch.float32, device="cuda")

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    def barrier():
        if world > 1:
            dist.barrier()

    # warm up eagerly (first call also does the per-device set-up), then capture
    with torch.cuda.stream(stream):
        for _ in range(2):
            layer(x, stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        layer(x, stream)
    torch.cuda.synchronize()
    n_active = int((layer.counts > 0).sum())

    # kernels enqueued by one moe_layer call: router 2 (logits, top-k), permute 2
    # (dispatch, activation operand), combine 1; shared expert 3 (gate/up,
    # SwiGLU finaliser, down), or 2 for one token on the row GEMV and for 128+
    # tokens (SwiGLU in the GEMM epilogue); routed experts 4 or 5 (bf16: two
    # GEMV pairs; 1 for one token, whose experts all have a single token and
    # run both projections in one launch) or 3
    # (mxfp4: tile list + two tcgen05 GEMMs); latent projections 3 (the down
    # projection rides with the router rows; its bf16 rounding, the routed sum
    # at width L, the up-projection GEMM)
    rows_k = (1024, 2048, 4096, 8192)
    rows_path = w.T == 1 and w.H in rows_k and w.I_shared in rows_k
    # (many tokens: the sigmoid-gate row rides with the router rows as well)
    shared = 2 if (rows_path or w.T >= 128) else 3
    # (one token, no latent projection: the combine runs in the shared down
    # launch)
    fused_combine = rows_path and not w.L
    # (several tokens, W and I multiples of 512: gate/up, h row scales, down on
    # the TMA-ring kernels beside the two CUDA-core GEMVs)
    routed_multi = 5 if (w.W % 512 == 0 and w.I % 512 == 0) else 4
    # (one token, bf16 activations, no latent projection: the top-k launch also
    # writes the dispatch and the activation operand)
    fused_dispatch = w.T == 1 and act == "bf16" and not w.L
    launches_per_step = (5 - (1 if fused_combine else 0) - (2 if fused_dispatch else 0) + shared
                         + (3 if act == "mxfp4" else (1 if w.T == 1 else routed_multi)) + (3 if w.L else 0))

    def timed(fn, steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        with torch.cuda.stream(stream):
            for a, b in evs:
                flush()
                a.record(stream)
                fn()
                b.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush()
            graph.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    def soak(seconds):
        # the same flushed step, untimed, so the clock samples see the timed region's load
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            with torch.cuda.stream(stream):
                for _ in range(50):
                    flush()
                    graph.replay()
            torch.cuda.synchronize()

    with ClockSampler(local_rank) as clk:
        soak(0.7)
        ms = timed(graph.replay, steps)
        soak(0.7)
    torch.cuda.synchronize()
    barrier()
    step_ms = max_over_ranks(sum(ms) / len(ms), world, "cuda")

    # dominant call alone: moe_expert_ffn on the routing of the captured step
    lw = layer.w      # the layer's weights (tiled scales for mxfp4 activations)

    def ffn():
        M.moe_expert_ffn(dims, layer.x_op, layer.offsets, layer.expert_list, layer.row_token, lw["wg_q"],
                         lw["wg_s"], lw["wu_q"], lw["wu_s"], lw["wd_q"], lw["wd_s"],
                         layer.y_perm, layer.ws, stream)
    # (an NVTX range, so that a profiler can pick out these launches)
    torch.cuda.nvtx.range_push("ffn_alone")
    timed(ffn, 3)
    ffn_ms = statistics.mean(timed(ffn, max(5, steps)))
    torch.cuda.nvtx.range_pop()

    # end to end through moe_layer with host buffers
    x_host = x.cpu().pin_memory()
    y_host = torch.empty(w.T, w.H, dtype=torch.float32).pin_memory()

    def e2e_step():
        x.copy_(x_host, non_blocking=True)
        graph.replay()
        y_host.copy_(layer.y, non_blocking=True)
    timed(e2e_step, 3)
    e2e_ms = max_over_ranks(statistics.mean(timed(e2e_step, steps)), world, "cuda")
    clocks = clk.summary()
    del graph
    if rank != 0:
        return None
    peak, peak_kind = _peaks()
    fb = ffn_bytes(w, n_active, act)
    lb = layer_bytes(w, n_active)
    ff = ffn_flops(w)
    hbm_gbs = fb / (ffn_ms * 1e-3) / 1e9
    if act == "mxfp4":
        tpeak, tkind = _fp4_peak_tflops()
        tflops = ff / (ffn_ms * 1e-3) / 1e12
        t_mem, t_tc = fb / (peak * 1e9), ff / (tpeak * 1e12)
        kernel = "moe_expert_ffn (k_tile_list + k_mxf4_gemm<gate/up> + k_mxf4_gemm<down>)"
        if t_tc > t_mem:
            roof = {"bound": "tensor", "achieved": tflops, "peak": tpeak, "unit": "TFLOP/s",
                    "frac": tflops / tpeak, "peak_kind": tkind}
        else:
            roof = {"bound": "hbm", "achieved": hbm_gbs, "peak": peak, "unit": "GB/s",
                    "frac": hbm_gbs / peak, "peak_kind": peak_kind}
        roof.update({"hbm_frac": hbm_gbs / peak, "tensor_frac": tflops / tpeak,
                     "tensor_tflops": tflops, "fp4_peak_tflops": tpeak,
                     "roofline_ms": max(t_mem, t_tc) * 1e3,
                     "frac_of_roofline_time": max(t_mem, t_tc) / (ffn_ms * 1e-3)})
    else:
        # single-token experts on the CUDA-core GEMV pair; experts with 2+
        # tokens on the TMA-fed mma.sync pair (whole 512-element slices) or,
        # for other widths, on the per-warp GEMV pair
        multi = ("k_mma_gateup" if w.W % 512 == 0 else "k_gateup_mxfp4",
                 "k_mma_down" if w.I % 512 == 0 else "k_down_mxfp4")
        kernel = ("moe_expert_ffn (k_fma_routed1: gate/up and down in one launch)" if w.T == 1
                  else "moe_expert_ffn (k_fma_gemv + %s + %s)" % multi)
        roof = {"bound": "hbm", "achieved": hbm_gbs, "peak": peak, "unit": "GB/s",
                "frac": hbm_gbs / peak, "peak_kind": peak_kind}
    roof = dict({"kernel": kernel}, **roof)
    roof.update({"bytes_per_launch": fb, "flops_per_launch": ff, "ms_per_launch": ffn_ms,
                 "intermediate_bytes_per_launch": ffn_intermediate_bytes(w, act),
                 "bytes_rule": "active experts' weights once + activation operand once + "
                               "routed output T x W fp32",
                 "traffic": _traffic(w.name)})
    out = {
        "value": job_tokens_per_s(w.T, world, step_ms),
        "unit": "tokens/s",
        "steps": steps,
        "ms_per_step": step_ms,
        "dtype": ("mxfp4 weights x mxfp4 activations (tcgen05 kind::mxf4), fp32 accumulate"
                  if act == "mxfp4" else "mxfp4 weights x f16 activations, fp32 accumulate"),
        "data": DATA,
        "config": {"workload": workload_label(w), "parallelism": f"replicas x{world}",
                   "l2": "flushed before every step (512 MiB write, then 512 MiB read of another "
                         "buffer, outside the events)",
                   "act_mode": act, "active_experts": n_active},
        "layer": {"algorithmic_bytes": lb, "hbm_gbs": lb / (step_ms * 1e-3) / 1e9,
                  "hbm_frac": lb / (step_ms * 1e-3) / 1e9 / peak,
                  "tflops": layer_flops(w) / (step_ms * 1e-3) / 1e12},
        "roofline": roof,
        "gpu_launches": launches_per_step * steps,
        "e2e": {"value": job_tokens_per_s(w.T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": w.T * w.H * 2, "d2h_bytes_per_step": w.T * w.H * 4,
                "ms_per_step": e2e_ms},
        "clocks": clocks,
        "clocks_note": "nvidia-smi every 200 ms over the timed steps plus 0.7 s of the same "
                       "flushed step on either side",
    }
    return out


def measure_streamed(args, base, tokens=16, slots=128):
    """Decode with the routed experts streamed from host memory through the
    expert cache (moe_expert_ffn_streamed): the layer of `base` (weights
    seeded as that workload) with every expert in page-locked host memory, a
    cache of `slots` experts on the device, and a fresh token each step (the
    cache starts empty). One step = route, dispatch, read the expert list
    back, the streamed routed experts, combine; CUDA events around it on the
    launching stream. The bound is the host link: the same bytes copied
    host -> device alone (pinned, one copy) give the peak."""
    import dataclasses

    import torch

    import mxfp4_routed_expert_04_b200 as M
    import synth

    w = dataclasses.replace(base, T=1)
    wt = dataclasses.replace(base, T=tokens)                 # the token rows, same weights
    dense = synth.dense_inputs(w)
    xs = synth.dense_inputs(wt)["x"]
    dev = {n: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
           for n, a in dense.items() if n != "x"}
    (Ng, Kg), (Nd, Kd) = synth.expert_shapes(w)
    shp = {"wg_q": (Ng, Kg // 2), "wg_s": (Ng, Kg // 32), "wu_q": (Ng, Kg // 2),
           "wu_s": (Ng, Kg // 32), "wd_q": (Nd, Kd // 2), "wd_s": (Nd, Kd // 32)}
    host = {n: torch.empty((w.E,) + s, dtype=torch.uint8, pin_memory=True) for n, s in shp.items()}
    for e0 in range(0, w.E, 32):
        ids = list(range(e0, min(w.E, e0 + 32)))
        ex = synth.expert_weights(w, ids)
        for n in shp:
            host[n][e0:e0 + len(ids)].copy_(torch.from_numpy(ex[n]))
    names = ("wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s")
    dims = M.MoeDims.of(w)
    # the layer's buffers; no routed expert is resident (the step calls used
    # here never read the routed weights of the layer)
    layer = M.MoeLayer(dims, dict(dev, wg_q=None, wg_s=None, wu_q=None, wu_s=None, wd_q=None,
                                  wd_s=None))
    cache = M.ExpertCache(dims, slots, [tuple(host[n][e] for n in names) for e in range(w.E)])
    x = torch.empty(1, w.H, dtype=torch.int16, device="cuda")
    xs_dev = torch.from_numpy(xs.view(np.int16)).cuda()
    stream = torch.cuda.current_stream()
    L = layer

    def step(t):
        x.copy_(xs_dev[t:t + 1])
        M.moe_route(dims, x, dev["w_router"], L.topk_idx, L.topk_w, None, L.ws)
        M.moe_permute(dims, L.topk_idx, x, L.counts, L.offsets, L.expert_list, L.row_token,
                      L.row_slot, L.slot_row, L.x_op, L.ws)
        lst = L.expert_list[:1 + w.k].cpu().tolist()      # the dispatch read back (a sync)
        cache.ffn(lst[1:1 + lst[0]], L.x_op, L.offsets, L.row_token, L.y_perm, L.ws)
        M.moe_combine(dims, L.y_perm, L.slot_row, L.topk_w, x, dev["w_sgate"], dev["ws_gate"],
                      dev["ws_up"], dev["ws_down"], None, L.y, L.ws)

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(tokens)]
    torch.cuda.synchronize()
    for t in range(tokens):
        a, b = evs[t]
        a.record(stream)
        step(t)
        b.record(stream)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    st = cache.stats()
    cache.close()
    # the host link alone: one pinned copy of the same number of bytes
    nbytes = max(st["bytes_copied"], 1 << 20)
    src = host["wg_q"].view(-1)[: min(nbytes, host["wg_q"].numel())]
    dst = torch.empty_like(src, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dst.copy_(src, non_blocking=True)
    a.record(stream)
    dst.copy_(src, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize()
    link_gbs = src.numel() / (a.elapsed_time(b) * 1e-3) / 1e9
    total_s = sum(ms) * 1e-3
    h2d_gbs = st["bytes_copied"] / total_s / 1e9
    return {"value": tokens / total_s, "unit": "tokens/s", "steps": tokens,
            "ms_per_step": sum(ms) / tokens,
            "config": {"workload": workload_label(w) + f", experts in host memory, {slots}-slot "
                                                      f"device cache (LRU), {tokens} distinct tokens",
                       "act_mode": "bf16"},
            "cache": st, "hit_rate": st["hits"] / max(1, st["hits"] + st["misses"]),
            "roofline": {"bound": "host link", "achieved": h2d_gbs, "peak": link_gbs,
                         "unit": "GB/s", "frac": h2d_gbs / link_gbs,
                         "peak_kind": "measured in this run: one pinned host-to-device copy"}}


def run_ours(args, w):
    """The headline workload plus the extra workloads, one after the other on
    the same GPU(s); rank 0 returns the JSON line's dict."""
    import gc

    import torch
    import torch.distributed as dist

    import synth

    rank, local_rank, world = _dist_env()
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    head = measure(args, w, args.steps, rank, local_rank, world, args.act)
    extras = {}
    for name in args.extra:
        if name == w.name:
            continue
        gc.collect()
        torch.cuda.empty_cache()
        r = measure(args, synth.WORKLOADS[name], min(args.steps, 10), rank, local_rank, world)
        if r is not None:
            extras[name] = r
    if args.streamed:
        gc.collect()
        torch.cuda.empty_cache()
        r = measure_streamed(args, w)
        if rank == 0:
            extras["decode1_streamed"] = r
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    out = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None}
    out.update({k: v for k, v in head.items() if k not in out and k != "steps"})
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, act=args.act or default_act(w))
    if extras:
        out["workloads"] = extras
    return out


def _oracle_getter(w):
    import synth
    (Ng, Kg), (Nd, Kd) = synth.expert_shapes(w)
    cache = {}

    def get(e):
        # regenerated from the seed once per expert (weights resident, as on the GPU)
        if e not in cache:
            cache[e] = (synth.expert_matrix(w.seed, "gate", e, Ng, Kg)
                        + synth.expert_matrix(w.seed, "up", e, Ng, Kg)
                        + synth.expert_matrix(w.seed, "down", e, Nd, Kd))
        return cache[e]
    return get


def _oracle_token_pass(w, t, dense, getter, act="bf16"):
    """One token of the batch through the oracle's whole layer (moe_o_layer)."""
    import oracle as O
    sub = dict(dense, x=dense["x"][t:t + 1])
    return O.moe_layer(sub, w.k, getter, act="mxfp4" if act == "mxfp4" else "exact")


def _time_tokens(w, dense, getter, act, budget_s, first=0):
    """Single-token layer passes until about budget_s seconds (at least one);
    each token's experts are generated before its timed pass."""
    import oracle as O
    n, total = 0, 0.0
    while n < w.T and (n == 0 or total < budget_s):
        t = (first + n) % w.T
        sel = O.topk_route(O.router_logits(dense["x"][t:t + 1], dense["w_router"]), w.k)[0]
        for e in np.unique(sel):
            getter(int(e))
        t0 = time.perf_counter()
        _oracle_token_pass(w, t, dense, getter, act)
        total += time.perf_counter() - t0
        n += 1
    return n, total


def cpu_baseline(w, budget_s: float = 12.0, act: str = "bf16"):
    """The C++ fp64 oracle, as it stands, on a bounded sample of the workload:
    whole tokens of the same batch through the whole layer, one at a time,
    with all host threads and then with one thread. Weight generation is not
    timed (the weights are resident, as on the GPU)."""
    import oracle as O
    import synth

    dense = synth.dense_inputs(w)
    getter = _oracle_getter(w)
    O.set_threads(0)
    cores = O.threads()
    n, dt = _time_tokens(w, dense, getter, act, budget_s)
    O.set_threads(1)
    try:
        n1, dt1 = _time_tokens(w, dense, getter, act, budget_s)
    finally:
        O.set_threads(0)
    return {"value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "single_thread": {"value": n1 / dt1, "unit": "tokens/s", "cores": 1,
                              "sample": f"{n1} token(s), {dt1:.1f} s"},
            "sample": f"{n} token(s) of {w.name}, each a full layer pass of the C++ oracle "
                      f"(routing, its k experts decoded to fp64, shared expert, combine) on "
                      f"{cores} threads, {dt:.1f} s"}


def run_reference(args, w):
    """The reference arm: the C++ fp64 oracle on the host cores (rank 0 only)."""
    rank, _, world = _dist_env()
    if rank != 0:
        return None
    import oracle as O
    import synth

    dense = synth.dense_inputs(w)
    getter = _oracle_getter(w)
    act = args.act or default_act(w)
    O.set_threads(0)
    cores = O.threads()
    # each step is one token's full layer pass; keep the whole run within a few minutes
    warmup = max(1, args.warmup)
    _, per = _time_tokens(w, dense, getter, act, 0.0)   # the first warm-up pass sizes the run
    for i in range(1, warmup):
        _time_tokens(w, dense, getter, act, 0.0, first=i)
    steps = max(1, min(args.steps, int(150.0 / max(per, 1e-3))))
    times = []
    for i in range(steps):
        _, dt = _time_tokens(w, dense, getter, act, 0.0, first=i)
        times.append(dt)
    step = statistics.mean(times)
    v = 1.0 / step
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": DATA,
        "config": {"workload": workload_label(w), "parallelism": "host cores, rank 0",
                   "act_mode": act, "step": "one token of the batch through the whole layer"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{steps} single-token layer passes of {w.name} through "
                                   f"the C++ oracle on {cores} threads (steps capped so the "
                                   f"run stays near 150 s; weight generation untimed)"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode1")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra", default=None,
                    help="comma-separated workloads measured after the headline one and "
                         "reported under 'workloads' (default with the decode1 headline: "
                         + ",".join(EXTRA_DEFAULT) + ")")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-streamed", dest="streamed", action="store_false",
                    help="skip the decode measurement with experts streamed from host memory")
    ap.add_argument("--act", choices=["bf16", "mxfp4"], default=None,
                    help="activation operand of the routed experts (default: mxfp4 for "
                         "prefill workloads, bf16 otherwise)")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling case: keep only this many experts resident (same shapes "
                         "and top-k); the line is then not the workload's metric")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling case: this many tokens instead of the workload's T")
    args = ap.parse_args()
    import dataclasses

    import synth
    w = synth.WORKLOADS[args.workload]
    if args.experts:
        w = dataclasses.replace(w, E=args.experts, name=f"{w.name}-E{args.experts}")
    if args.tokens:
        w = dataclasses.replace(w, T=args.tokens, name=f"{w.name}-T{args.tokens}")
    if args.workload != "decode1":
        args.streamed = False
    if args.no_extra or args.experts or args.tokens:
        args.extra = []
        args.streamed = False
    elif args.extra is None:
        args.extra = list(EXTRA_DEFAULT) if args.workload == "decode1" else []
    else:
        args.extra = [n for n in args.extra.split(",") if n]
        for n in args.extra:
            if n not in synth.WORKLOADS:
                ap.error(f"unknown workload {n}")
    res = run_reference(args, w) if args.impl == "reference" else run_ours(args, w)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
