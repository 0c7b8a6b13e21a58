#!/usr/bin/env python
"""Benchmark of the Beam-style sparse MoE layer forward (libbeam_moe) on B200 GPUs.

One step = one whole layer forward (router, top-k, permutation, NVFP4 quantisation, the
two grouped NVFP4 GEMMs, finalize) over one synthetic batch of the chosen workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload default|<name>]
                  [--impl ours|reference] [--experts-format nvfp4|mxfp8] [--tp-shared-gpu W]

The default run measures the metric's three batch sizes on one layer: the 8 x 2K prefill
(T = 16384, the headline of the JSON line), the decode verify step (T = 8) and the batched
verify (T = 1024) under "workloads", each with its own roofline, e2e, clocks, CPU baseline
and parity against the oracle.  --workload <name> measures one workload alone.
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


def read_traffic(kernel: str, used_experts: int, tokens: int, top_k: int = 8):
    """DRAM bytes per launch from the committed ncu captures (profiles/traffic.json): for the
    expert GEMM, weights per used expert (decode capture) plus, above 32 tokens, bytes per
    routed row (prefill capture); for the per-token kernels, bytes per token (batches of 256
    tokens or more).  None when the kernel's source changed since the capture or no capture
    covers the batch."""
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
    if digest != ent["source_sha256_16"]:
        return None
    if "bytes_per_token" in ent:
        return ent["bytes_per_token"] * tokens if tokens >= 256 else None
    if tokens <= ent.get("applies_up_to_tokens", tokens):
        return ent["bytes_per_used_expert"] * used_experts
    if "prefill" in ent:
        return ent["bytes_per_used_expert"] * used_experts + ent["prefill"]["bytes_per_row"] * tokens * top_k
    return None


# ------------------------------------------------------------------ clocks
REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of one GPU, sampled while a region
    runs: NVML polled every 2 ms from a thread (the timed regions last tens of ms), else
    nvidia-smi at its 200 ms period."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, pci_bus_id: str | None = None, period_s: float = 0.002):
        self.gpu = gpu_index
        self.pci = pci_bus_id
        self.period = period_s
        self.rows = []  # (sm_mhz, max_mhz, power_w, reasons bitmask)
        self.proc = None
        self.path = None
        self.thread = None
        self.stop = False
        self.source = None

    def _nvml_loop(self, nvml, handle):
        mx = float(nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM))
        while not self.stop:
            try:
                sm = float(nvml.nvmlDeviceGetClockInfo(handle, nvml.NVML_CLOCK_SM))
                pw = nvml.nvmlDeviceGetPowerUsage(handle) / 1000.0
                rs = int(nvml.nvmlDeviceGetCurrentClocksEventReasons(handle))
                self.rows.append((sm, mx, pw, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        try:
            import threading

            import pynvml as nvml
            nvml.nvmlInit()
            handle = (nvml.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci
                      else nvml.nvmlDeviceGetHandleByIndex(self.gpu))
            self.source = "nvml 2 ms"
            self.thread = threading.Thread(target=self._nvml_loop, args=(nvml, handle), daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
                self.source = "nvidia-smi 200 ms"
            except (OSError, FileNotFoundError):
                self.proc = None
        time.sleep(0.05)
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=5)
        if self.proc:
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        rows = list(self.rows)
        if self.path:
            try:
                names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
                for line in open(self.path):
                    f = [c.strip() for c in line.split(",")]
                    if len(f) >= 9 and f[1].replace(".", "").isdigit():
                        bits = sum(REASON_BITS[n] for n, v in zip(names, f[5:9]) if v.lower() == "active")
                        pw = float(f[3]) if f[3].replace(".", "").isdigit() else 0.0
                        rows.append((float(f[1]), float(f[2]), pw, bits))
            finally:
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = sorted({n for r in rows for n, b in REASON_BITS.items() if r[3] & b})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1], "reasons": reasons,
                "samples": len(rows), "power_w_max": max(r[2] for r in rows), "source": self.source}


# ------------------------------------------------------------------ CPU oracle leg
def oracle_sample(shape: mi.LayerShape, tokens, seed=0, fmt="nvfp4"):
    """Inputs of the oracle for a token sample, drawn untimed: the tokens' BF16 rows, the
    router, gamma and the FP32 weights of the experts they route to."""
    from oracle import moe
    xs, rs = [], []
    for t in tokens:
        xb, rb = mi.tokens(shape, seed, t, t + 1)
        xs.append(xb[0])
        rs.append(rb[0])
    xb, rb = np.stack(xs), np.stack(rs)
    wr = mi.router_weight(shape, seed)
    ids, _, _ = moe.route_topk(moe.router_logits(mi.bf16_bits_to_f32(xb), wr), shape.top_k)
    experts = {int(e): mi.expert_weights(shape, seed, int(e)) for e in np.unique(ids)}
    return xb, rb, wr, mi.gamma(shape, seed), experts, fmt


def oracle_step(shape, sample):
    """One forward of the sample by the C++ FP64 oracle (OpenMP over the host cores): routing,
    each expert quantised by the oracle's own quantiser and dequantised to FP64, the FP64
    expert GEMMs, finalize.  Returns (tokens processed, its result)."""
    from oracle import cpp
    xb, rb, wr, gb, experts, fmt = sample
    a1, a2 = mi.activation_scales(shape) if fmt == "nvfp4" else (1.0, 1.0)
    r = cpp.moe_forward(xb, rb, wr, gb, experts.__getitem__, shape.top_k, shape.inter, alpha_a1=a1, alpha_a2=a2,
                        eps=shape.rms_eps, fmt=fmt)
    return xb.shape[0], r


def cpu_cores() -> int:
    """Threads the C++ oracle runs on (OpenMP uses every core the process may run on)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_sample_tokens(shape):
    return [0] if shape.tokens <= 64 else [0, shape.tokens // 2]


def cpu_baseline(shape, budget_s=8.0, fmt="nvfp4", gpu=None):
    """The oracle timed on the host cores over a bounded sample of the workload.  With gpu =
    (ids [T, k], out [T, H] as FP64) of the same batch on the GPU, also the parity of that
    batch: the oracle's routing of every token (FP64 logits) against the GPU's ids, with the
    near-tie count, and the GPU's output rows of the sampled tokens against the oracle's."""
    toks = cpu_sample_tokens(shape)
    sample = oracle_sample(shape, toks, fmt=fmt)
    t0 = time.perf_counter()
    n = 0
    reps = 0
    r = None
    while True:
        dn, r = oracle_step(shape, sample)
        n += dn
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 2:
            break
    dt = time.perf_counter() - t0
    base = {"value": n / dt, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{len(toks)} token(s) of the {shape.name} batch x {reps} repeats through the C++ FP64 oracle: "
                      f"router, top-k, {fmt.upper()} quantisation of x and of each routed expert's FP32 weights, "
                      f"FP64 expert GEMMs, finalize; FP32 weights drawn untimed"}
    if gpu is None:
        return base, None
    return base, oracle_parity(shape, toks, r, *gpu)


def oracle_parity(shape, toks, ref, gpu_ids, gpu_out, seed=0):
    """Parity of the GPU's forward of a batch (routing of every token, outputs of the sampled
    tokens) against the oracle; see cpu_baseline."""
    from oracle import moe
    k = shape.top_k
    wr = mi.router_weight(shape, seed)
    near = np.zeros(shape.tokens, bool)
    differ = 0
    for t0 in range(0, shape.tokens, 4096):
        t1 = min(shape.tokens, t0 + 4096)
        xb, _ = mi.tokens(shape, seed, t0, t1)
        logits = moe.router_logits(mi.bf16_bits_to_f32(xb), wr)
        ids = moe.route_topk(logits, k)[0]
        near[t0:t1] = moe.near_tie_mask(logits, k)
        same = np.sort(ids, 1) == np.sort(gpu_ids[t0:t1], 1)
        differ += int((~same.all(1) & ~near[t0:t1]).sum())
    keep = ~near[toks]
    g, o = gpu_out[toks][keep], ref["out_pre"][keep]
    rel = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30)) if g.size else 0.0
    mx = float(np.abs(g - o).max()) if g.size else 0.0
    return {"near_ties": int(near.sum()), "tokens": shape.tokens, "ids_differ_outside_near_ties": differ,
            "sampled_tokens": len(toks), "rel_l2": rel, "max_abs": mx, "tol": {"rel_l2": 1e-2, "max_abs": 5e-2}}


def run_reference(args, shape, rank, world):
    if rank != 0:
        return
    fmt = getattr(args, "experts_format", "nvfp4")
    sample = oracle_sample(shape, cpu_sample_tokens(shape), fmt=fmt)
    for _ in range(args.warmup):
        oracle_step(shape, sample)
    t0 = time.perf_counter()
    n = sum(oracle_step(shape, sample)[0] for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = n / dt
    cores = cpu_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, fmt=fmt, world=world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{len(cpu_sample_tokens(shape))} token(s) of the {shape.name} batch per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(line, rank)


def workload_config(shape, fmt="nvfp4", world=1):
    """The workload's config keys; the same for both arms of the measurement."""
    return {"workload": shape.name, "tokens": shape.tokens, "hidden": shape.hidden, "experts": shape.experts,
            "top_k": shape.top_k, "inter": shape.inter, "routing": "zipf-skewed" if shape.skew else "uniform",
            "experts_format": fmt,
            "l2": f"flushed: {L2_FLUSH_BYTES >> 20} MiB write + {L2_FLUSH_BYTES >> 21} MiB read between timed steps",
            "parallelism": f"token-dp replicas x{world}"}


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
# The workloads of the metric (T = 16384 / 8 / 1024); the first is the headline of the line.
DEFAULT_WORKLOADS = ("prefill16k", "decode8", "spec1024")


def roofline_of(kern: dict, work: dict, fmt: str, T: int) -> dict:
    """Roofline of the dominant kernel: algorithmic bytes or FLOPs per launch over its live
    CUDA-event duration, against the measured (or fallback) peaks."""
    # the longest kernel whose algorithmic work is known (the expert GEMM in every workload;
    # a profiler's serialised, cold launches can reorder the short ones)
    top = max((n for n in kern if n in work), key=kern.get)
    pk = peaks()
    wk = work[top]
    # the contraction's own dtype: NVFP4 = 4 x BF16 (nominal 9 / 2.25 PF), FP8 = 2 x (4.5 / 2.25)
    ratio = 4 if fmt == "nvfp4" else 2
    name = "NVFP4" if fmt == "nvfp4" else "FP8"
    if wk["flops"] > 0 and wk["flops"] / max(wk["bytes"], 1) > (ratio * pk["bf16_sus"] * 1e12) / (pk["hbm"] * 1e9):
        achieved = wk["flops"] / (kern[top] / 1e3) / 1e12
        burst, sus = ratio * pk["bf16"], ratio * pk["bf16_sus"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s", "frac": achieved / burst,
                "peak_sustained": sus, "frac_sustained": achieved / sus,
                "peak_source": f"{name} dense = {ratio} x the {pk['src']} BF16 cuBLAS peak (nominal "
                               f"{'9' if fmt == 'nvfp4' else '4.5'} / 2.25 PF ratio); burst applies: the kernel runs "
                               f"ms-long stretches between L2 flushes, not a seconds-long loop at the power cap"}
    else:
        achieved = wk["bytes"] / (kern[top] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s", "frac": achieved / pk["hbm"],
                "peak_source": f"{pk['src']} copy bandwidth"}
    roof.update(traffic=read_traffic(top if fmt == "nvfp4" else f"{top}_{fmt}", work["_used_experts"], T),
                traffic_source="ncu dram__bytes_read.sum + dram__bytes_write.sum, profiles/traffic.json "
                               "(captured on a smaller case and scaled by experts used and routed rows)",
                kernel=top, kernel_ms=kern[top], algorithmic_bytes=wk["bytes"], algorithmic_flops=wk["flops"])
    return roof


def measure_workload(args, layer, shape, rank, world, dev, flush_l2, want_parity):
    """Times one workload on an existing layer: K steps with CUDA events on the launching
    stream (L2 flushed between steps, outside the events), the max over ranks; then the
    library's per-kernel events in a separate pass, and the host-buffer (e2e) path."""
    import torch
    import sparse_moe_layer_fp32_b200 as bm
    from sparse_moe_layer_fp32_b200 import synthetic
    stream = torch.cuda.current_stream()
    fmt = args.experts_format
    T = shape.tokens
    x, res = synthetic.make_batch(shape, seed=rank)  # each replica its own batch
    x, res = x.to(dev), res.to(dev)
    out = torch.empty_like(res)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        layer.forward(x, res, out)
        flush_l2()
    layer.check()
    torch.cuda.synchronize()
    barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    pci = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
    with ClockSampler(dev.index or 0, pci) as clk:
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
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms = reduce_max(sum(step_ms) / args.steps, world, dev)
    layer.check()

    # ---- per-kernel durations (CUDA events inside the library, same stream), separate pass
    layer.profile(True)
    acc = {}
    for _ in range(max(args.steps, 5)):
        layer.forward(x, res, out)
        for name, kms in layer.kernel_times():
            acc.setdefault(name, []).append(kms)
        flush_l2()
    layer.profile(False)
    kern = {n: sum(v) / len(v) for n, v in acc.items()}
    offsets = np.frombuffer(layer.debug(bm.BUF_OFFSETS).cpu().numpy().tobytes(), np.int32)
    work = kernel_work(shape, T, np.diff(offsets), fmt)

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
    ref_out = layer.forward(x, res)
    assert torch.equal(oh.to(dev), ref_out), "host-buffer path differs from device path"
    graph = graph_replay(args, layer, x, res, ref_out, flush_l2, world, dev)
    gpu = None
    if want_parity:
        ids = layer.debug(bm.BUF_IDS).cpu().numpy().view(np.int32).reshape(T, shape.top_k).astype(np.int64)
        gpu = (ids, ref_out.float().cpu().numpy().astype(np.float64))
    return {
        "value": whole_job_rate(T, world, ms), "unit": UNIT, "ms_per_step": ms, "us_per_layer": ms * 1e3,
        "steps": args.steps, "config": workload_config(shape, fmt, world),
        "roofline": roofline_of(kern, work, fmt, T), "kernels_ms": kern, "used_experts": work["_used_experts"],
        "e2e": {"value": whole_job_rate(T, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": 2 * T * shape.hidden * 2,
                "d2h_bytes_per_step": T * shape.hidden * 2},
        "gpu_launches": launches, "clocks": clk.summary(), "cuda_graph": graph,
    }, gpu


def graph_replay(args, layer, x, res, ref_out, flush_l2, world, dev):
    """The same step captured once in a CUDA graph and replayed (the plain stream above is the
    headline): per-step time with the same flush protocol, and the replay's output against
    the plain forward's bits."""
    import torch
    out = torch.empty_like(res)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.forward(x, res, out)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(x, res, out)
    for _ in range(max(args.warmup, 3)):
        g.replay()
        flush_l2()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    s_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        s_ev[i].record(stream)
        g.replay()
        e_ev[i].record(stream)
        flush_l2()
    torch.cuda.synchronize()
    layer.check()
    ms = reduce_max(sum(a.elapsed_time(b) for a, b in zip(s_ev, e_ev)) / args.steps, world, dev)
    same = bool(torch.equal(out, ref_out))
    assert same, "graph replay differs from the plain forward"
    del g
    return {"ms_per_step": ms, "same_bits_as_plain": same}


def library_peaks(steps: int = 20):
    """Dense GEMM rates of library kernels at 8192^3 on this GPU, as context for the
    rooflines: cuBLAS BF16 (torch.mm) and the block-scaled NVFP4 GEMM behind
    torch._scaled_mm (E2M1 operands, one E4M3 scale per 16 values).  L2 flushed before each
    launch; median of `steps`."""
    import statistics
    import torch
    M = N = K = 8192
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def rate(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = statistics.median(ts)
        return {"ms": ms, "tflops": 2.0 * M * N * K / ms / 1e9}

    g = torch.Generator(device="cuda").manual_seed(0)
    xa = torch.randn(M, K, dtype=torch.bfloat16, device="cuda", generator=g)
    xb = torch.randn(K, N, dtype=torch.bfloat16, device="cuda", generator=g)
    out = {"shape": [M, N, K], "bf16_torch_mm": rate(lambda: torch.mm(xa, xb))}
    del xa, xb
    a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device="cuda", generator=g)
    b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device="cuda", generator=g)
    sa = torch.full((M, K // 16), 0x38, dtype=torch.uint8, device="cuda")  # E4M3 1.0
    sb = torch.full((N, K // 16), 0x38, dtype=torch.uint8, device="cuda")
    fa, fb = a.view(torch.float4_e2m1fn_x2), b.view(torch.float4_e2m1fn_x2)
    ea, eb = sa.view(torch.float8_e4m3fn), sb.view(torch.float8_e4m3fn)
    try:
        out["nvfp4_torch_scaled_mm"] = rate(lambda: torch._scaled_mm(fa, fb.t(), ea, eb, out_dtype=torch.bfloat16))
    except Exception as ex:  # a torch build without the FP4 GEMM
        out["nvfp4_torch_scaled_mm"] = {"unavailable": f"{type(ex).__name__}: {str(ex)[:200]}"}
    return out


def run_ours(args, shapes, rank, world, local_rank):
    """Every workload of `shapes` on one layer (one set of weights, workspace for the
    largest batch); returns {name: measurement}, each with its parity inputs."""
    import torch
    from sparse_moe_layer_fp32_b200 import synthetic

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    fmt = args.experts_format
    base = shapes[0]
    key = lambda s: (s.hidden, s.experts, s.top_k, s.inter, s.skew)  # noqa: E731
    assert all(key(s) == key(base) for s in shapes), "workloads of one run share the layer's shape"
    weights = synthetic.make_weights(base, 0, device=dev, fmt=fmt)
    layer = synthetic.make_layer(base, weights, max_tokens=max(s.tokens for s in shapes), fmt=fmt)
    del weights  # the handle holds its own repacked copy
    torch.cuda.empty_cache()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(L2_FLUSH_BYTES // 2 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        """Between steps, outside the timed region: write a buffer 4x the L2, then read
        another 2x the L2 so the step starts with L2 cold and clean (the write-back of the
        flush's dirty lines is not charged to the step)."""
        flush.zero_()
        clean.sum()

    want_parity = rank == 0 and world == 1 and not args.no_cpu_baseline
    results = {}
    for shape in shapes:
        results[shape.name] = measure_workload(args, layer, shape, rank, world, dev, flush_l2, want_parity)
    layer.close()
    return results


def compose_line(args, shapes, results, world):
    """The one JSON line: the headline workload's numbers at the top level, the others under
    "workloads" with the same keys."""
    fmt = args.experts_format
    head = shapes[0].name
    line = {
        "metric": METRIC, "n_gpus": world, "warmup": max(args.warmup, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("nvfp4 (e2m1 x e4m3/16) experts" if fmt == "nvfp4" else "mxfp8 (e4m3 x ue8m0/32) experts")
                 + ", fp32 router and accumulation",
        "data": "synthetic (seeded; random-init weights of the layer's shapes)",
    }
    line.update(results[head])
    if len(shapes) > 1:
        line["workloads"] = {s.name: results[s.name] for s in shapes[1:]}
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
    [r E/W, (r+1) E/W) and its own batch of the workload's T tokens; four phases: routing of
    its tokens + count publication, layout + dispatch of the routed rows, its experts on the
    rows it received + return of the outputs, finalize of its tokens); `value` = W T / the
    slowest rank's step (weak scaling of the batch)."""
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
    nphase = tp.EP_PHASES if ep else tp.TP_PHASES
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
    T, H, k = shape.tokens, shape.hidden, shape.top_k
    pk = peaks()
    q = BYTES_PER_VALUE[fmt]
    if ep:  # dispatch: x read once, each slot's quantised row stored at its expert's rank
        top, nbytes = "ep_dispatch", T * H * 2 + T * k * H * q
        exchange = T * k * H * q + T * k * H * 2  # per rank: its rows out, their outputs back
    elif T >= bm.TP_TWO_SHOT_MIN_TOKENS:  # two-shot: the W partials of the rank's slice, residual, out and row buffer
        S = -(-T // W)
        top, nbytes = "tp_reduce", T * H * 4 + 3 * S * H * 2 + H * 2
        exchange = (W - 1) * S * H * 4 + (T - S) * H * 2  # peers' partials of the slice, peers' rows
    else:  # one-shot: the W partials of every token, residual, out
        top, nbytes = "tp_reduce", W * T * H * 4 + 2 * T * H * 2 + H * 2
        exchange = (W - 1) * T * H * 4
    roof = {"bound": "hbm", "kernel": top, "kernel_ms": kms.get(top),
            "achieved": nbytes / (kms[top] / 1e3) / 1e9, "peak": pk["hbm"], "unit": "GB/s",
            "traffic": None, "peak_source": f"{pk['src']} copy bandwidth"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    line = {
        "metric": METRIC, "value": (W * T if ep else T) / (max(rank_ms) / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": max(rank_ms), "higher_is_better": True,
        "scaling": "weak" if ep else "strong",
        "vs_baseline": None,
        "dtype": ("nvfp4" if fmt == "nvfp4" else "mxfp8") + " experts, fp32 router, accumulation and all-reduce",
        "data": "synthetic (seeded; random-init weights of the layer's shapes)",
        "config": dict(workload_config(shape, fmt),
                       parallelism=f"{'ep' if ep else 'tp'}{W}, ranks sharing one GPU in turn"
                                   + (f", {T} tokens per rank" if ep else "")),
        "estimate": "value = tokens / slowest rank's sum of phases; peers' data read from this GPU's memory, "
                    "so the NVLink transfer of the exchange is not included",
        "tp": {"world": W, "mode": "ep" if ep else "tp", "rank_ms": rank_ms, "phase_ms": pms,
               "exchange_bytes_per_rank": exchange},
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
    ap.add_argument("--workload", default="default", choices=["default"] + sorted(mi.SHAPES),
                    help="default: prefill16k (the headline), decode8 and spec1024 in one line")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tp-shared-gpu", type=int, default=0, metavar="W",
                    help="tensor-parallel layer with W ranks sharing this one GPU, run in turn (per-rank timing)")
    ap.add_argument("--ep-shared-gpu", type=int, default=0, metavar="W",
                    help="expert-parallel layer with W ranks (each its own batch) sharing this one GPU, run in turn")
    ap.add_argument("--experts-format", default="nvfp4", choices=["nvfp4", "mxfp8"],
                    help="routed experts in NVFP4 (default) or the block-scaled FP8 variant (MXFP8)")
    ap.add_argument("--library-peaks", action="store_true",
                    help="print library GEMM rates at 8192^3 (cuBLAS BF16, NVFP4 scaled_mm) and exit")
    args = ap.parse_args()
    if args.library_peaks:
        print(json.dumps({"library_peaks": library_peaks()}))
        return
    names = DEFAULT_WORKLOADS if args.workload == "default" else (args.workload,)
    shapes = [mi.SHAPES[n] for n in names]
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, shapes[0], rank, world)
        return
    if args.tp_shared_gpu or args.ep_shared_gpu:
        emit(run_tp_shared(args, shapes[0]), 0)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    try:
        results = run_ours(args, shapes, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for shape in shapes:
            meas, gpu = results[shape.name]
            meas["cpu_baseline"], meas["parity"] = cpu_baseline(shape, fmt=args.experts_format, gpu=gpu)
    results = {n: m for n, (m, _) in results.items()}
    emit(compose_line(args, shapes, results, world), rank)


if __name__ == "__main__":
    main()
