#!/usr/bin/env python
"""Benchmark of the Beam-style sparse MoE layer forward (libbeam_moe) on B200 GPUs.

One step = one whole layer forward (router, top-k, permutation, NVFP4 quantisation, the
two grouped NVFP4 GEMMs, finalize) over one synthetic batch of the chosen workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode8] [--impl ours|reference]
                  [--experts-format nvfp4|mxfp8] [--tp-shared-gpu W]

--experts-format mxfp8 measures the block-scaled FP8 variant of the experts (E4M3 values,
one power-of-two scale per 32).  --tp-shared-gpu W measures the tensor-parallel layer with
W ranks sharing this GPU, run in turn (per-rank phase timings; see run_tp_shared).

N > 1 runs under torchrun, one rank per GPU: token data parallel replicas (each rank a
full copy of the layer and its own batch, no collective on the data path; the process
group only carries the barrier and the max-over-ranks of the timing), so scaling is weak.
Rank 0 prints one JSON line.  --impl reference times the CPU oracle (FP64) instead, on
bounded samples of the same workload, on rank 0 only.
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

import moe_inputs as mi  # noqa: E402

METRIC = "moe_layer_tokens_per_s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 512 << 20  # written between timed steps (L2 is 126 MB)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ algorithmic work
# bytes per quantised value: NVFP4 0.5 B + one scale byte per 16 values; MXFP8 1 B + one
# scale byte per 32 values
BYTES_PER_VALUE = {"nvfp4": 0.5625, "mxfp8": 1.03125}


def kernel_work(shape: mi.LayerShape, T: int, counts: np.ndarray, fmt: str = "nvfp4") -> dict:
    """Algorithmic bytes and FLOPs of each kernel for one forward (T tokens).

    Quantised operands cost BYTES_PER_VALUE[fmt] per value.  Only the experts that received
    tokens have their weights read."""
    H, I, E, k = shape.hidden, shape.inter, shape.experts, shape.top_k
    R = T * k
    used = int((counts > 0).sum())
    q = BYTES_PER_VALUE[fmt]
    return {
        "router": dict(bytes=E * H * 4 + T * H * 2 + T * E * 4, flops=2 * T * H * E),
        "topk": dict(bytes=T * E * 4 + R * 8, flops=0),
        "chunk_hist": dict(bytes=R * 4, flops=0),
        "scan": dict(bytes=E * 16, flops=0),
        "scatter": dict(bytes=R * 12, flops=0),
        "quant_a1": dict(bytes=T * H * 2 + R * H * q, flops=0),
        # gate/up + down in one launch: both weight sets of the used experts, A1 read, the
        # NVFP4 intermediate A2 written and read back, y written (BF16)
        "gemm_experts": dict(bytes=used * 3 * I * H * q + R * H * q + 2 * R * I * q + R * H * 2,
                             flops=2 * R * 3 * I * H),
        "finalize": dict(bytes=R * H * 2 + 2 * T * H * 2 + H * 2, flops=0),
        "_used_experts": used,
    }


def read_traffic(kernel: str, used_experts: int, tokens: int):
    """DRAM bytes per launch from the committed ncu capture (profiles/traffic.json), scaled
    by the experts that received tokens; None when the kernel's source changed since or the
    batch is outside the regime the capture scales to."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        ent = json.load(f).get(kernel)
    if not ent:
        return None
    import hashlib
    src = os.path.join(ROOT, "sparse_moe_layer_fp32_b200", "csrc", ent["source"])
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if digest != ent["source_sha256_16"] or tokens > ent.get("applies_up_to_tokens", tokens):
        return None
    return ent["bytes_per_used_expert"] * used_experts


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [c.strip() for c in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ------------------------------------------------------------------ CPU oracle leg
def oracle_sample(shape: mi.LayerShape, tokens, seed=0, fmt="nvfp4"):
    """Inputs and quantised experts the oracle needs for a token sample (prepared untimed)."""
    from oracle import moe
    xs, rs = [], []
    for t in tokens:
        xb, rb = mi.tokens(shape, seed, t, t + 1)
        xs.append(xb[0])
        rs.append(rb[0])
    x = mi.bf16_bits_to_f32(np.stack(xs)).astype(np.float64)
    res = mi.bf16_bits_to_f32(np.stack(rs)).astype(np.float64)
    wr = mi.router_weight(shape, seed)
    g = mi.bf16_bits_to_f32(mi.gamma(shape, seed)).astype(np.float64)
    ids, _, _ = moe.route_topk(moe.router_logits(x, wr), shape.top_k)
    quantised = {int(e): moe.quantize_expert(*mi.expert_weights(shape, seed, int(e)), fmt) for e in np.unique(ids)}
    return x, res, wr, g, quantised, fmt


def oracle_step(shape, sample):
    """One oracle forward of the sample: routing, experts (dequantised from the stored
    quantised weights, FP64 matmuls), finalize.  Returns tokens processed."""
    from oracle import moe
    x, res, wr, g, quantised, fmt = sample
    a1, a2 = mi.activation_scales(shape) if fmt == "nvfp4" else (None, None)
    cache = moe.ExpertCache(lambda e: None, keep=2, fmt=fmt)
    cache._q = dict(quantised)
    moe.moe_forward_tokens(x, res, wr, g, cache, shape.top_k, a1, a2, shape.rms_eps)
    return x.shape[0]


def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_sample_tokens(shape):
    return [0] if shape.tokens <= 64 else [0, shape.tokens // 2]


def cpu_baseline(shape, budget_s=25.0, fmt="nvfp4"):
    toks = cpu_sample_tokens(shape)
    sample = oracle_sample(shape, toks, fmt=fmt)
    t0 = time.perf_counter()
    n = 0
    reps = 0
    while True:
        n += oracle_step(shape, sample)
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 3:
            break
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{len(toks)} token(s) of the {shape.name} batch x {reps} repeats: FP64 router, "
                      f"{fmt.upper()} experts dequantised from stored codes, finalize; weights pre-quantised untimed"}


def run_reference(args, shape, rank, world):
    if rank != 0:
        return
    sample = oracle_sample(shape, cpu_sample_tokens(shape), fmt=args.experts_format)
    for _ in range(args.warmup):
        oracle_step(shape, sample)
    t0 = time.perf_counter()
    n = sum(oracle_step(shape, sample) for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = n / dt
    cores = cpu_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, fmt=args.experts_format),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{len(cpu_sample_tokens(shape))} token(s) of the {shape.name} batch per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(line, rank)


def workload_config(shape, l2_flush="write", fmt="nvfp4"):
    l2 = f"flushed: {L2_FLUSH_BYTES >> 20} MiB write between timed steps"
    if l2_flush == "write+read":
        l2 = f"flushed: {L2_FLUSH_BYTES >> 20} MiB write + {L2_FLUSH_BYTES >> 21} MiB read between timed steps"
    return {"workload": shape.name, "tokens": shape.tokens, "hidden": shape.hidden, "experts": shape.experts,
            "top_k": shape.top_k, "inter": shape.inter, "routing": "zipf-skewed" if shape.skew else "uniform",
            "experts_format": fmt, "l2": l2}


# ------------------------------------------------------------------ multi-rank plumbing
def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank number over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Tokens per second of the whole job: every rank processes its own batch (weak scaling)."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def emit(line: dict, rank: int, stream=None) -> bool:
    """Rank 0 alone prints the JSON line."""
    if rank != 0:
        return False
    print(json.dumps(line), file=stream or sys.stdout, flush=True)
    return True


# ------------------------------------------------------------------ GPU leg
def run_ours(args, shape, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sparse_moe_layer_fp32_b200 as bm
    from sparse_moe_layer_fp32_b200 import synthetic

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    fmt = args.experts_format
    weights = synthetic.make_weights(shape, 0, device=dev, fmt=fmt)
    layer = synthetic.make_layer(shape, weights, fmt=fmt)
    del weights  # the handle holds its own repacked copy
    torch.cuda.empty_cache()
    x, res = synthetic.make_batch(shape, seed=rank)  # each replica its own batch
    x, res = x.to(dev), res.to(dev)
    out = torch.empty_like(res)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(L2_FLUSH_BYTES // 2 // 4, dtype=torch.float32, device=dev) if args.l2_flush == "write+read" \
        else None
    T = shape.tokens

    def flush_l2():
        """Between steps, outside the timed region: write a buffer 4x the L2; with
        write+read, then read another 2x the L2 so the step starts with L2 clean as well
        as cold (the write-back of the flush's dirty lines is not charged to the step)."""
        flush.zero_()
        if clean is not None:
            clean.sum()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        layer.forward(x, res, out)
        flush_l2()
    layer.check()
    torch.cuda.synchronize()
    barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        barrier()
        for i in range(args.steps):
            starts[i].record(stream)
            layer.forward(x, res, out)
            ends[i].record(stream)
            flush_l2()
        torch.cuda.synchronize()
        barrier()
    launches = layer.launches() * args.steps
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = reduce_max(sum(step_ms) / args.steps, world, dev)
    value = whole_job_rate(T, world, ms)
    layer.check()

    # ---- per-kernel durations (CUDA events inside the library, same stream), separate pass
    layer.profile(True)
    acc = {}
    reps = max(args.steps, 5)
    for _ in range(reps):
        layer.forward(x, res, out)
        for name, kms in layer.kernel_times():
            acc.setdefault(name, []).append(kms)
        flush_l2()
    layer.profile(False)
    kern = {n: sum(v) / len(v) for n, v in acc.items()}
    offsets = np.frombuffer(layer.debug(bm.BUF_OFFSETS).cpu().numpy().tobytes(), np.int32)
    counts = np.diff(offsets)
    work = kernel_work(shape, T, counts, fmt)
    top = max(kern, key=kern.get)
    pk = peaks()
    wk = work[top]
    # the contraction's own dtype: NVFP4 = 4 x BF16 (nominal 9 / 2.25 PF), FP8 = 2 x (4.5 / 2.25)
    ratio = 4 if fmt == "nvfp4" else 2
    if wk["flops"] > 0 and wk["flops"] / max(wk["bytes"], 1) > (ratio * pk["bf16_sus"] * 1e12) / (pk["hbm"] * 1e9):
        bound, achieved, peak, unit = ("tensor", wk["flops"] / (kern[top] / 1e3) / 1e12, ratio * pk["bf16_sus"],
                                       "TFLOP/s")
        peak_note = (f"{'NVFP4' if fmt == 'nvfp4' else 'FP8'} dense = {ratio} x {pk['src']} sustained BF16 cuBLAS "
                     f"peak (nominal {'9' if fmt == 'nvfp4' else '4.5'} / 2.25 PF ratio)")
    else:
        bound, achieved, peak, unit = "hbm", wk["bytes"] / (kern[top] / 1e3) / 1e9, pk["hbm"], "GB/s"
        peak_note = f"{pk['src']} copy bandwidth"
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": read_traffic(top if fmt == "nvfp4" else f"{top}_{fmt}", work["_used_experts"], T),
                "kernel": top, "kernel_ms": kern[top],
                "peak_source": peak_note}

    # ---- end to end through the host-buffer entry point (copies inside the timed region)
    xh = x.cpu().pin_memory()
    rh = res.cpu().pin_memory()
    oh = torch.empty_like(rh).pin_memory()
    for _ in range(3):
        layer.forward_host(xh, rh, oh)
    torch.cuda.synchronize()
    barrier()
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        e_s[i].record(stream)
        layer.forward_host(xh, rh, oh)
        e_e[i].record(stream)
        flush_l2()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in zip(e_s, e_e)) / args.steps, world, dev)
    assert torch.equal(oh.to(dev), layer.forward(x, res)), "host-buffer path differs from device path"

    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("nvfp4 (e2m1 x e4m3/16) experts" if fmt == "nvfp4" else "mxfp8 (e4m3 x ue8m0/32) experts")
                     + ", fp32 router and accumulation",
            "data": "synthetic (seeded; random-init weights of the layer's shapes)",
            "config": dict(workload_config(shape, args.l2_flush, fmt), parallelism=f"token-dp replicas x{world}"),
            "roofline": roofline,
            "kernels_ms": kern,
            "used_experts": work["_used_experts"],
            "e2e": {"value": whole_job_rate(T, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": 2 * T * shape.hidden * 2,
                    "d2h_bytes_per_step": T * shape.hidden * 2},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
    layer.close()
    return line


# ------------------------------------------------------------------ tensor parallel, one GPU
def run_tp_shared(args, shape):
    """Tensor-parallel layer (experts split over W ranks along I, finalize fused with its
    all-reduce) with all W ranks on one GPU, run in turn: every rank's phase 0 (routing,
    its slice of the expert GEMMs, its partial m and their publication), then every rank's
    phase 1 (the exchange, sum, norm, residual).  Each phase is timed with CUDA events on
    the launching stream; a rank's step = the sum of its phases.  `value` estimates the
    group's tokens/s if each rank had its own GPU: tokens / the slowest rank's step.  The
    data that rank r reads from its peers sit in this GPU's memory here, so the NVLink
    transfer of the exchange (W x T x H x 4 B per rank) is not in the estimate.

    With --ep-shared-gpu W instead: the expert-parallel layer (rank r holds experts
    [r E/W, (r+1) E/W) and its own batch of the workload's T tokens; three phases:
    dispatch, the rank's experts on the gathered W T tokens, combine + finalize); `value` =
    W T / the slowest rank's step (weak scaling of the batch)."""
    import dataclasses
    import torch
    import sparse_moe_layer_fp32_b200 as bm
    from sparse_moe_layer_fp32_b200 import synthetic, tp

    ep = bool(args.ep_shared_gpu)
    W, fmt = (args.ep_shared_gpu if ep else args.tp_shared_gpu), args.experts_format
    torch.cuda.set_device(0)
    full = synthetic.make_weights(shape, 0, fmt=fmt)
    a1, a2 = mi.activation_scales(shape) if fmt == "nvfp4" else (1.0, 1.0)
    layers = []
    for r in range(W):
        if ep:
            sh = tp.shard_experts(full, r, W, shape.experts)
            e_loc = shape.experts // W
            layers.append(bm.MoELayer(max_tokens=W * shape.tokens, hidden=shape.hidden, num_experts=shape.experts,
                                      top_k=shape.top_k, inter=shape.inter, alpha_a1=float(a1), alpha_a2=float(a2),
                                      rms_eps=shape.rms_eps, fmt=fmt, expert_begin=r * e_loc, expert_count=e_loc,
                                      **sh))
        else:
            sh = tp.shard_weights(full, r, W, shape.inter)
            layers.append(bm.MoELayer(max_tokens=shape.tokens, hidden=shape.hidden, num_experts=shape.experts,
                                      top_k=shape.top_k, inter=shape.inter // W, alpha_a1=float(a1),
                                      alpha_a2=float(a2), rms_eps=shape.rms_eps, fmt=fmt, **sh))
        del sh
    del full
    torch.cuda.empty_cache()
    grp = tp.SharedGpuGroup(layers)
    if ep:  # each rank its own batch (seeds 0..W-1)
        batches = [synthetic.make_batch(shape, r) for r in range(W)]
        xs, rs = [b[0] for b in batches], [b[1] for b in batches]
    else:
        x, res = synthetic.make_batch(shape, 0)
        xs, rs = [x] * W, [res] * W
    outs = [torch.empty_like(rs[r]) for r in range(W)]
    nphase = 3 if ep else 2
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clean = torch.ones(L2_FLUSH_BYTES // 2 // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def flush_l2():
        flush.zero_()
        clean.sum()

    def run_phase(lay, r, phase):
        if ep:
            lay.forward_ep_phase(xs[r], rs[r], outs[r], phase)
        else:
            lay.forward_tp_phase(xs[r], rs[r], outs[r], phase)

    for _ in range(max(args.warmup, 3)):
        for phase in range(nphase):
            for r, lay in enumerate(layers):
                run_phase(lay, r, phase)
        flush_l2()
    for lay in layers:
        lay.check()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ph = [[[] for _ in range(nphase)] for _ in range(W)]
    kern = {}
    with ClockSampler(0) as clk:
        for step in range(args.steps + 1):
            prof = step == args.steps  # one extra pass with the library's per-kernel events
            for lay in layers:
                lay.profile(prof)
            for phase in range(nphase):
                for r, lay in enumerate(layers):
                    flush_l2()  # each rank starts cold, as on its own GPU
                    a, b = ev(), ev()
                    a.record(stream)
                    run_phase(lay, r, phase)
                    b.record(stream)
                    if prof:
                        for name, kms in lay.kernel_times():
                            kern.setdefault(name, []).append(kms)
                    else:
                        ph[r][phase].append((a, b))
        torch.cuda.synchronize()
    for lay in layers:
        lay.check()
    if not ep:
        assert all(torch.equal(o, outs[0]) for o in outs[1:]), "ranks disagree"
    pms = [[sum(a.elapsed_time(b) for a, b in ph[r][p]) / args.steps for r in range(W)] for p in range(nphase)]
    rank_ms = [sum(pms[p][r] for p in range(nphase)) for r in range(W)]
    kms = {n: sum(v) / len(v) for n, v in kern.items()}
    T, H = shape.tokens, shape.hidden
    pk = peaks()
    red_bytes = W * T * H * 4 + 2 * T * H * 2 + H * 2  # per rank: W partials of its T tokens, residual, out
    part_bytes = T * shape.top_k * H * 2 + (W * T if ep else T) * H * 4  # y rows it holds, its partial m
    roof = {"bound": "hbm", "kernel": "tp_reduce", "kernel_ms": kms.get("tp_reduce"),
            "achieved": red_bytes / (kms["tp_reduce"] / 1e3) / 1e9, "peak": pk["hbm"], "unit": "GB/s",
            "traffic": None, "peak_source": f"{pk['src']} copy bandwidth"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    line = {
        "metric": METRIC, "value": (W * T if ep else T) / (max(rank_ms) / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": max(rank_ms), "higher_is_better": True,
        "scaling": "weak" if ep else "strong",
        "vs_baseline": None,
        "dtype": ("nvfp4" if fmt == "nvfp4" else "mxfp8") + " experts, fp32 router, accumulation and all-reduce",
        "data": "synthetic (seeded; random-init weights of the layer's shapes)",
        "config": dict(workload_config(shape, "write+read", fmt),
                       parallelism=f"{'ep' if ep else 'tp'}{W}, ranks sharing one GPU in turn"
                                   + (f", {T} tokens per rank" if ep else "")),
        "estimate": "value = tokens / slowest rank's sum of phases; peers' data read from this GPU's memory, "
                    "so the NVLink transfer of the exchange is not included",
        "tp": {"world": W, "mode": "ep" if ep else "tp", "rank_ms": rank_ms, "phase_ms": pms,
               "phase0_ms": pms[0], "phase1_ms": pms[1],
               "exchange_bytes_per_rank": W * T * H * 4, "tp_partial_bytes": part_bytes},
        "kernels_ms": kms, "roofline": roof, "gpu_launches": sum(lay.launches() for lay in layers),
        "clocks": clk.summary(),
    }
    grp.close()
    return line


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode8", choices=sorted(mi.SHAPES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tp-shared-gpu", type=int, default=0, metavar="W",
                    help="tensor-parallel layer with W ranks sharing this one GPU, run in turn (per-rank timing)")
    ap.add_argument("--ep-shared-gpu", type=int, default=0, metavar="W",
                    help="expert-parallel layer with W ranks (each its own batch) sharing this one GPU, run in turn")
    ap.add_argument("--experts-format", default="nvfp4", choices=["nvfp4", "mxfp8"],
                    help="routed experts in NVFP4 (default) or the block-scaled FP8 variant (MXFP8)")
    ap.add_argument("--l2-flush", default="write+read", choices=["write", "write+read"],
                    help="between timed steps: write 512 MiB, then (default) read 256 MiB so the step starts "
                         "with L2 cold and clean")
    args = ap.parse_args()
    shape = mi.SHAPES[args.workload]
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, shape, rank, world)
        return
    if args.tp_shared_gpu or args.ep_shared_gpu:
        emit(run_tp_shared(args, shape), 0)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, shape, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape, fmt=args.experts_format)
    emit(line, rank)


if __name__ == "__main__":
    main()
