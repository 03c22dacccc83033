"""Tensor-parallel expert layer: the deployment of "Optimizing GLM4-MoE for
production" (Novita AI), section 1, where TP8 leaves each GPU an intermediate
slice of 192 of every expert.

Rank r of N holds columns [j0, j1) of every expert's intermediate dimension
(w13 gate and up rows, w2 columns, with their E4M3 scales; router weights are
replicated). The SwiGLU is per intermediate column, so the rank's layer output
over its slice (moe_forward with out_f32, unrounded) is its exact share of the
layer; the shares are summed across ranks (one all-reduce of [T, H] fp32 through
torch.distributed, NCCL on GPUs) and rounded once to bf16 by the library.
Routing is computed on every rank from the replicated inputs: the kernels are
deterministic, so all ranks pick the same experts and no exchange is needed.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib, synth
from ._lib import MOE_FFN_AUTO


def slice_bounds(I: int, rank: int, world: int) -> tuple[int, int]:
    """Columns [j0, j1) of the intermediate dimension held by `rank`."""
    if I % world:
        raise ValueError(f"intermediate size {I} does not split into {world} equal slices")
    w = I // world
    return rank * w, (rank + 1) * w


def shard_weights(weights: dict, I: int, rank: int, world: int) -> dict:
    """Rank `rank`'s slice of full-layer weights (tensors of any device)."""
    j0, j1 = slice_bounds(I, rank, world)
    w13 = weights["w13"]
    out = {
        "router_w": weights["router_w"],
        "router_bias": weights.get("router_bias"),
        "w13": torch.cat([w13[:, j0:j1], w13[:, I + j0:I + j1]], 1).contiguous(),
        "w2": weights["w2"][:, :, j0:j1].contiguous(),
        "s13": None, "s2": weights.get("s2"),
    }
    if weights.get("s13") is not None:
        s13 = weights["s13"]
        out["s13"] = torch.cat([s13[:, j0:j1], s13[:, I + j0:I + j1]], 1).contiguous()
    if "x" in weights:
        out["x"] = weights["x"]
    return out


def local_config(cfg, world: int):
    """The per-rank layer: intermediate I / world, unrounded fp32 output."""
    return synth.variant(cfg, I=cfg.I // world, out_f32=True)


class TPMoELayer:
    """One rank of a tensor-parallel expert layer.

    cfg: the full layer's LayerConfig; shard: this rank's weights (shard_weights);
    group: the torch.distributed process group of the N ranks (None: default).
    partial_fn(x) -> fp32 [T, H] and cast_fn(fp32) -> out replace the library
    calls (the CPU tests run the host logic with the oracle in their place).
    """

    def __init__(self, cfg, shard: dict, world: int, group=None, fuse_shared: bool = True,
                 impl: int = MOE_FFN_AUTO, partial_fn=None, cast_fn=None):
        self.cfg = cfg
        self.world = world
        self.group = group
        self.local = local_config(cfg, world)
        self.partial_fn = partial_fn
        self.cast_fn = cast_fn
        if partial_fn is None:
            from . import MoELayer
            self.layer = MoELayer(self.local, shard, fuse_shared=fuse_shared, impl=impl)

    def partial(self, x: torch.Tensor) -> torch.Tensor:
        """This rank's unrounded share of the layer output, fp32 [T, H]."""
        if self.partial_fn is not None:
            return self.partial_fn(x)
        part = torch.empty(x.shape[0], self.cfg.H, dtype=torch.float32, device=x.device)
        self.layer.forward(x, part)
        return part

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        part = self.partial(x)
        if self.world > 1:
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)
        if self.cast_fn is not None:
            return self.cast_fn(part)
        out = torch.empty(part.shape, dtype=torch.bfloat16, device=part.device)
        _lib.moe_cast_f32_bf16(part, out)
        return out
