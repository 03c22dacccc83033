"""Shared-experts-fused GLM4-MoE expert layer for B200 (sm_100a).

The layer: every token goes through one shared expert and through the top-k
routed experts its router picks; the outputs are aggregated with weights. The
fusion appends the shared expert to the routed ones (index n_routed) and gives
every token top_k + 1 slots, the shared expert fixed in the last one, so one
routed-MoE pass computes everything ("Optimizing GLM4-MoE for production",
Novita AI, section 1 "Shared Experts Fusion").

All compute runs in the CUDA library libsre_moe.so (C ABI in include/moe.h);
this package only marshals arguments. PyTorch supplies device memory and streams.
"""
from __future__ import annotations

import torch

from ._lib import (MOE_BF16, MOE_E4M3, MOE_F32, MOE_FFN_AUTO, MOE_FFN_SIMT, MOE_FFN_TCGEN05,
                   MoeError, alloc_workspace, make_shape, moe_clear_status, moe_combine,
                   moe_forward, moe_get_status, moe_grouped_ffn, moe_launch_count, moe_permute,
                   moe_profile_enable, moe_profile_read, moe_profile_reset, moe_qk_norm_rope,
                   moe_quant_rows_e4m3, moe_route_topk, moe_shape, moe_workspace_size)

__all__ = ["MoELayer", "moe_shape", "make_shape", "alloc_workspace", "moe_workspace_size",
           "moe_route_topk", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_forward",
           "moe_quant_rows_e4m3", "moe_qk_norm_rope", "moe_get_status", "moe_clear_status", "moe_launch_count",
           "moe_profile_enable", "moe_profile_reset", "moe_profile_read", "MoeError",
           "MOE_F32", "MOE_BF16", "MOE_E4M3", "MOE_FFN_AUTO", "MOE_FFN_SIMT", "MOE_FFN_TCGEN05"]


class MoELayer:
    """One expert layer with its weights resident on a CUDA device.

    weights: dict with router_w [E_r, H] fp32, router_bias [E_r] or None,
    w13 [E, 2I, H], s13 [E, 2I] or None, w2 [E, H, I], s2 [E, H] or None, all
    on the device. cfg: a LayerConfig-like object (T is the largest batch).
    """

    def __init__(self, cfg, weights: dict, fuse_shared: bool = True, impl: int = MOE_FFN_AUTO):
        self.cfg = cfg
        self.w = weights
        self.fuse_shared = fuse_shared
        self.impl = impl
        self.device = weights["w13"].device
        self.max_T = cfg.T
        self.ws = alloc_workspace(make_shape(cfg), fuse_shared, device=self.device)
        act = torch.bfloat16 if cfg.act_dtype == "bf16" else torch.float32
        self.act_dtype = act

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """x [T, H] on the device -> out [T, H] on the device (asynchronous)."""
        T = x.shape[0]
        if T > self.max_T:
            raise ValueError(f"batch {T} exceeds the layer's maximum {self.max_T}")
        if out is None:
            out = torch.empty_like(x)
        w = self.w
        moe_forward(make_shape(self.cfg, T), x, w["router_w"], w.get("router_bias"), w["w13"],
                    w.get("s13"), w["w2"], w.get("s2"), self.fuse_shared, out, self.ws,
                    impl=self.impl, stream=stream)
        return out

    def capture(self, x: torch.Tensor, out: torch.Tensor) -> torch.cuda.CUDAGraph:
        """Record one forward from the device buffer x into out as a CUDA graph:
        replay() reruns every kernel of the layer with one launch from the host
        (new inputs go into x in place). The kernels take no host decisions and
        allocate nothing, so the recorded launches are the eager ones."""
        was = self.profiling_off()
        try:
            self.forward(x, out)                 # one eager pass sets up every kernel
            torch.cuda.synchronize(self.device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.forward(x, out)
        finally:
            moe_profile_enable(was)
        return g

    @staticmethod
    def profiling_off() -> bool:
        """Turns per-kernel event timing off (it does not belong inside a graph)
        and returns whether it was on."""
        from ._lib import profile_enabled
        was = profile_enabled()
        moe_profile_enable(False)
        return was

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor, x_dev: torch.Tensor,
                     out_dev: torch.Tensor, stream=None) -> torch.Tensor:
        """Host buffers in and out: copy x to the device, run the layer, copy
        the result back, all enqueued on `stream` (pinned host memory makes the
        copies asynchronous)."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            x_dev.copy_(x_host, non_blocking=True)
            self.forward(x_dev, out_dev, stream=s)
            out_host.copy_(out_dev, non_blocking=True)
        return out_host

    # ---- pipelined host-buffer submission -------------------------------------
    # Batches that arrive in pinned host memory: each submit enqueues the upload
    # on one copy stream, the layer on the compute stream and the download on a
    # second copy stream, with `depth` device slots so that the copies of one
    # batch overlap the layer of its neighbours. Every batch still makes its own
    # host->device and device->host trip.

    def _pipeline(self, depth: int, T: int):
        key = (depth, T)
        if getattr(self, "_pipe_key", None) != key:
            dev = self.device
            self._pipe = {
                "h2d": torch.cuda.Stream(dev), "d2h": torch.cuda.Stream(dev),
                "comp": torch.cuda.Stream(dev),
                "x": [torch.empty(T, self.cfg.H, dtype=self.act_dtype, device=dev) for _ in range(depth)],
                "out": [torch.empty(T, self.cfg.H, dtype=self.act_dtype, device=dev) for _ in range(depth)],
                "up": [torch.cuda.Event() for _ in range(depth)],      # upload done
                "done": [torch.cuda.Event() for _ in range(depth)],    # layer done (x slot free)
                "down": [torch.cuda.Event() for _ in range(depth)],    # download done (out slot free)
                "used": [False] * depth, "next": 0, "depth": depth,
            }
            self._pipe_key = key
        return self._pipe

    def submit_host(self, x_host: torch.Tensor, out_host: torch.Tensor, depth: int = 2) -> None:
        """Enqueue one batch: pinned x_host [T, H] in, pinned out_host [T, H] out.
        Returns at once; call sync_host() before reading out_host."""
        P = self._pipeline(depth, x_host.shape[0])
        i = P["next"]
        P["next"] = (i + 1) % P["depth"]
        if P["used"][i]:
            P["h2d"].wait_event(P["done"][i])       # the layer finished reading slot i's x
            P["comp"].wait_event(P["down"][i])      # the download finished reading slot i's out
        P["used"][i] = True
        with torch.cuda.stream(P["h2d"]):
            P["x"][i].copy_(x_host, non_blocking=True)
            P["up"][i].record(P["h2d"])
        P["comp"].wait_event(P["up"][i])
        self.forward(P["x"][i], P["out"][i], stream=P["comp"])
        P["done"][i].record(P["comp"])
        P["d2h"].wait_event(P["done"][i])
        with torch.cuda.stream(P["d2h"]):
            out_host.copy_(P["out"][i], non_blocking=True)
            P["down"][i].record(P["d2h"])

    def host_streams(self):
        """(upload, compute, download) streams of the pipelined path."""
        P = self._pipe
        return P["h2d"], P["comp"], P["d2h"]

    def sync_host(self) -> None:
        for s in self.host_streams():
            s.synchronize()

    def status(self) -> int:
        return moe_get_status(self.ws)
