"""Host logic of the multi-rank bench path on CPU ranks (gloo, world size 2).

bench.py runs token data-parallel replicas: each rank holds the whole layer and its own
batch, the process group only carries the barrier and the max over ranks of the timing,
and rank 0 alone prints the JSON line.  These tests run that plumbing in two CPU processes.
"""

import io
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import bench
        ms = bench.reduce_max(1.0 + 2.5 * rank, world)  # the slower rank sets the job time
        rate = bench.whole_job_rate(8, world, ms)
        buf = io.StringIO()
        printed = bench.emit({"rank": rank, "ms": ms}, rank, stream=buf)
        dist.barrier()
        # the reference arm: ranks other than 0 exit without work
        class A:
            steps, warmup, gpus = 1, 0, world
        ran = False
        if rank != 0:
            bench.run_reference(A, None, rank, world)  # returns before touching the shape
            ran = True
        q.put((rank, ms, rate, printed, buf.getvalue(), ran))
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_max_timing_and_rank0_output(repo_root):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, rate0, pr0, out0, _), (r1, ms1, rate1, pr1, out1, ran1) = res
    assert ms0 == ms1 == 3.5
    assert rate0 == rate1 == pytest.approx(2 * 8 / 3.5e-3)
    assert pr0 and not pr1 and '"rank": 0' in out0 and out1 == ""
    assert ran1


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.reduce_max(4.25, 1) == 4.25
    assert bench.whole_job_rate(8, 1, 0.25) == pytest.approx(32000.0)


# ---------------------------------------------------------------- tensor-parallel host logic
# The TP layer (experts split over ranks along the intermediate size, finalize fused to its
# all-reduce) exchanges the ranks' exchange-region addresses as IPC handles over the process
# group.  Two CPU ranks run sparse_moe_layer_fp32_b200.tp.connect with a stand-in layer and
# stand-in IPC calls (no GPU): every rank must attach with all regions in rank order, its
# own address in its own slot and each peer's address opened from that peer's handle.
class _FakeLayer:
    def __init__(self, rank):
        self.rank = rank
        self.attached = None

    def tp_region(self):
        return 0x10000 * (self.rank + 1)

    def tp_attach(self, rank, world, regions):
        self.attached = (rank, world, list(regions))


def _tp_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        from sparse_moe_layer_fp32_b200 import tp
        layer = _FakeLayer(rank)
        export = lambda p: p.to_bytes(8, "little") + bytes(56)  # noqa: E731
        import_ = lambda hd: int.from_bytes(hd[:8], "little") + 0x1  # noqa: E731  (a mapping differs from the owner's address)
        opened = tp.connect(layer, rank, world, export=export, import_=import_)
        q.put((rank, layer.attached, opened))
    finally:
        dist.destroy_process_group()


def test_tp_connect_exchanges_regions_in_rank_order(repo_root):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, a0, o0), (r1, a1, o1) = res
    assert a0 == (0, 2, [0x10000, 0x20001]) and o0 == [0x20001]
    assert a1 == (1, 2, [0x10001, 0x20000]) and o1 == [0x10001]


def test_tp_shard_weights_partition_the_experts():
    from sparse_moe_layer_fp32_b200 import tp
    E, H, inter, world = 3, 64, 256, 4
    g = torch.Generator().manual_seed(0)
    full = dict(router_w=torch.randn(E, H, generator=g), gamma=torch.ones(H),
                w_gu=torch.randint(0, 255, (E, 2 * inter, H // 2), dtype=torch.uint8, generator=g),
                w_gu_sf=torch.randint(0, 255, (E, 2 * inter, H // 16), dtype=torch.uint8, generator=g),
                w_gu_alpha=torch.rand(E, generator=g),
                w_d=torch.randint(0, 255, (E, H, inter // 2), dtype=torch.uint8, generator=g),
                w_d_sf=torch.randint(0, 255, (E, H, inter // 16), dtype=torch.uint8, generator=g),
                w_d_alpha=torch.rand(E, generator=g))
    shards = [tp.shard_weights(full, r, world, inter) for r in range(world)]
    s = inter // world
    for key in ("w_gu", "w_gu_sf"):
        gate = torch.cat([sh[key][:, :s] for sh in shards], dim=1)
        up = torch.cat([sh[key][:, s:] for sh in shards], dim=1)
        assert torch.equal(torch.cat([gate, up], dim=1), full[key])
        assert all(sh[key].is_contiguous() and sh[key].shape[1] == 2 * s for sh in shards)
    for key in ("w_d", "w_d_sf"):
        assert torch.equal(torch.cat([sh[key] for sh in shards], dim=-1), full[key])
        assert all(sh[key].is_contiguous() for sh in shards)
    for key in ("router_w", "gamma", "w_gu_alpha", "w_d_alpha"):
        assert all(sh[key] is full[key] for sh in shards)
    with pytest.raises(ValueError):
        tp.shard_weights(full, 0, 3, inter)
    with pytest.raises(ValueError):
        tp.shard_weights(full, 4, 4, inter)


def test_ep_shard_experts_partition_the_expert_arrays():
    from sparse_moe_layer_fp32_b200 import tp
    E, H, inter, world = 8, 64, 128, 4
    g = torch.Generator().manual_seed(1)
    full = dict(router_w=torch.randn(E, H, generator=g), gamma=torch.ones(H),
                w_gu=torch.randint(0, 255, (E, 2 * inter, H), dtype=torch.uint8, generator=g),
                w_gu_sf=torch.randint(0, 255, (E, 2 * inter, H // 32), dtype=torch.uint8, generator=g),
                w_d=torch.randint(0, 255, (E, H, inter), dtype=torch.uint8, generator=g),
                w_d_sf=torch.randint(0, 255, (E, H, inter // 32), dtype=torch.uint8, generator=g))
    shards = [tp.shard_experts(full, r, world, E) for r in range(world)]
    for key in ("w_gu", "w_gu_sf", "w_d", "w_d_sf"):
        assert torch.equal(torch.cat([sh[key] for sh in shards]), full[key])
        assert all(sh[key].shape[0] == E // world and sh[key].is_contiguous() for sh in shards)
    assert all(sh["router_w"] is full["router_w"] and sh["gamma"] is full["gamma"] for sh in shards)
    with pytest.raises(ValueError):
        tp.shard_experts(full, 0, 3, E)


def test_bench_host_logic_for_the_expert_formats(repo_root, capsys):
    # algorithmic bytes per quantised value (NVFP4 0.5 + 1/16, MXFP8 1 + 1/32), the expert
    # GEMM's bytes and FLOPs, and the reference arm's JSON line for the MXFP8 variant on the
    # tiny workload (the CPU oracle, bounded sample)
    import json

    import numpy as np

    import bench
    import moe_inputs as mi
    shape = mi.SHAPES["decode8"]
    counts = np.zeros(shape.experts, np.int64)
    counts[:58] = 1
    w4 = bench.kernel_work(shape, 8, counts, "nvfp4")["gemm_experts"]
    w8 = bench.kernel_work(shape, 8, counts, "mxfp8")["gemm_experts"]
    assert w4["flops"] == w8["flops"] == 2 * 64 * 3 * 1536 * 5120
    weights4 = 58 * 3 * 1536 * 5120 * 0.5625
    weights8 = 58 * 3 * 1536 * 5120 * 1.03125
    assert weights4 < w4["bytes"] < weights4 * 1.01
    assert weights8 < w8["bytes"] < weights8 * 1.01

    class A:
        steps, warmup, gpus, experts_format = 1, 0, 1, "mxfp8"
    bench.run_reference(A, mi.SHAPES["tiny"], 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["experts_format"] == "mxfp8"
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0


class _PhaseLayer:
    def __init__(self, log, rank, ep):
        self.log, self.rank, self.expert_parallel = log, rank, ep
        self.attached = None

    def tp_region(self):
        return 0x1000 * (self.rank + 1)

    def tp_attach(self, rank, world, regions):
        self.attached = (rank, world, list(regions))

    def forward_tp_phase(self, x, residual, out, phase):
        self.log.append(("tp", self.rank, phase))

    def forward_ep_phase(self, x, residual, out, phase):
        self.log.append(("ep", self.rank, phase))


@pytest.mark.parametrize("ep", [False, True])
def test_shared_gpu_group_runs_every_rank_phase_by_phase(ep):
    # Ranks sharing one GPU must never have a kernel wait on a kernel that has not run: every
    # rank's phase p is enqueued before any rank's phase p + 1 (TP: 2 phases, EP: 4).
    from sparse_moe_layer_fp32_b200 import tp
    log = []
    layers = [_PhaseLayer(log, r, ep) for r in range(3)]
    grp = tp.SharedGpuGroup(layers)
    assert [lay.attached for lay in layers] == [(r, 3, [0x1000, 0x2000, 0x3000]) for r in range(3)]
    xs = [torch.zeros(2, 8) for _ in range(3)]
    if ep:
        grp.forward(xs, xs, outs=[torch.zeros(2, 8) for _ in range(3)])
    else:
        grp.forward(xs[0], xs[0], outs=[torch.zeros(2, 8) for _ in range(3)])
    phases = tp.EP_PHASES if ep else tp.TP_PHASES
    assert log == [("ep" if ep else "tp", r, p) for p in range(phases) for r in range(3)]
