"""Host side of the tensor- and expert-parallel layers: weight shards, the exchange of the
ranks' regions, and ranks that share one GPU.

Tensor parallelism over the experts' intermediate size with the finalize fused to its
all-reduce (vLLM PR "Day-0 support for Reflection's Beam-1.0", section "Status"; recipe
"reflection/Beam-1.0-501B-A23B": NVFP4 with TP4 on Blackwell).  Rank r holds features
[r I/W, (r+1) I/W) of every expert: those gate rows, the matching up rows and the same
columns of down.  Expert parallelism with attention data parallelism (the PR's Attention DP
+ MegaMoE): rank r holds experts [r E/W, (r+1) E/W) and its own batch.  The device work is
beam_moe_forward_tp / beam_moe_forward_ep (C ABI); this module only slices tensors and moves
region addresses between processes.
"""

from __future__ import annotations

from . import MoELayer, beam_moe_ipc_export, beam_moe_ipc_import

WEIGHT_KEYS = ("w_gu", "w_gu_sf", "w_d", "w_d_sf")
TP_PHASES = 3  # phases of beam_moe_forward_tp_phase
EP_PHASES = 4  # phases of beam_moe_forward_ep_phase


def shard_weights(weights: dict, rank: int, world: int, inter: int) -> dict:
    """This rank's slice of layer weights in the C-ABI layout (either expert format).

    w_gu / w_gu_sf [E][2I][..]: gate rows [r s, (r+1) s) then up rows [I + r s, I + (r+1) s),
    s = I / world; w_d / w_d_sf [E][H][cols]: the r-th of `world` equal column ranges (the
    same features, packed codes and scales alike).  Tensor scales, router weights and gamma
    are shared unchanged."""
    if world < 1 or not 0 <= rank < world or inter % world:
        raise ValueError(f"cannot take shard {rank} of {world} of an intermediate size {inter}")
    s = inter // world
    out = {k: v for k, v in weights.items() if k not in WEIGHT_KEYS}
    for key in ("w_gu", "w_gu_sf"):
        t = weights[key]
        if t.shape[1] != 2 * inter:
            raise ValueError(f"{key} must have 2 * inter rows")
        gate = t[:, rank * s:(rank + 1) * s]
        up = t[:, inter + rank * s:inter + (rank + 1) * s]
        out[key] = _cat_rows(gate, up)
    for key in ("w_d", "w_d_sf"):
        t = weights[key]
        cols = t.shape[-1]
        if cols % world:
            raise ValueError(f"{key} columns do not split over {world} ranks")
        c = cols // world
        out[key] = t[..., rank * c:(rank + 1) * c].contiguous()
    return out


def shard_experts(weights: dict, rank: int, world: int, num_experts: int) -> dict:
    """Expert parallelism: this rank's experts [r E/W, (r+1) E/W) of layer weights in the C-ABI
    layout (either format): the expert-major arrays sliced along their first dimension,
    router weights and gamma unchanged."""
    if world < 1 or not 0 <= rank < world or num_experts % world:
        raise ValueError(f"cannot take expert shard {rank} of {world} of {num_experts} experts")
    e = num_experts // world
    out = dict(weights)
    for key in WEIGHT_KEYS + ("w_gu_alpha", "w_d_alpha"):
        if key in weights:
            t = weights[key]
            if t.shape[0] != num_experts:
                raise ValueError(f"{key} must have num_experts rows")
            out[key] = t[rank * e:(rank + 1) * e].contiguous()
    return out


def _cat_rows(a, b):
    import torch
    return torch.cat([a, b], dim=1).contiguous()


def connect(layer: MoELayer, rank: int, world: int, group=None, export=None, import_=None):
    """Exchanges exchange-region addresses across processes (one per GPU) and attaches the
    layer.  Every rank exports its region as an IPC handle, all handles are gathered over
    torch.distributed (any backend), and each peer's handle is opened in this process.
    Returns the addresses this process opened (close them with beam_moe_ipc_close after
    the layer is destroyed)."""
    import torch.distributed as dist
    export = export or beam_moe_ipc_export
    import_ = import_ or beam_moe_ipc_import
    own = layer.tp_region()
    handles = [None] * world
    dist.all_gather_object(handles, bytes(export(own)), group=group)
    regions, opened = [], []
    for q, hd in enumerate(handles):
        if q == rank:
            regions.append(own)
        else:
            p = import_(hd)
            regions.append(p)
            opened.append(p)
    layer.tp_attach(rank, world, regions)
    return opened


class SharedGpuGroup:
    """W ranks of one tensor- or expert-parallel group in one process on one GPU (tests and
    measurement when fewer GPUs than ranks are available).  The ranks run one after the
    other, phase by phase: every rank's phase p before any rank's phase p + 1, so no kernel
    waits on a kernel that has not run.  Tensor parallel: phase 0 (GEMMs, partial m,
    publication), phase 1 (all-reduce + finalize, of the rank's slice from 256 tokens on),
    phase 2 (the other slices' rows, from 256 tokens on); every rank gets the same x.  Expert
    parallel (layers created with an expert range): phase 0 (routing of the rank's own
    tokens, count publication), 1 (layout, dispatch of the routed rows), 2 (the rank's
    experts on the rows it received, return of the outputs), 3 (finalize of the rank's own
    tokens); each rank its own x and residual."""

    def __init__(self, layers):
        self.layers = list(layers)
        self.expert_parallel = bool(getattr(self.layers[0], "expert_parallel", False))
        regions = [lay.tp_region() for lay in self.layers]
        for r, lay in enumerate(self.layers):
            lay.tp_attach(r, len(self.layers), regions)

    def forward(self, x, residual, outs=None):
        """Tensor parallel: x, residual tensors (the same on every rank).  Expert parallel:
        lists of each rank's x and residual."""
        import torch
        if self.expert_parallel:
            outs = outs or [torch.empty_like(r) for r in residual]
            for phase in range(EP_PHASES):
                for lay, xr, rr, o in zip(self.layers, x, residual, outs):
                    lay.forward_ep_phase(xr, rr, o, phase)
            return outs
        outs = outs or [torch.empty_like(residual) for _ in self.layers]
        for phase in range(TP_PHASES):
            for lay, o in zip(self.layers, outs):
                lay.forward_tp_phase(x, residual, o, phase)
        return outs

    def close(self):
        for lay in self.layers:
            lay.close()
