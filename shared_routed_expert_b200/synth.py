"""Seeded synthetic inputs for the shared-experts-fused MoE layer.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic (no routing, no GEMM, no activation quantisation). Both the
CUDA path and the CPU oracle are fed from the tensors it returns.

Workloads follow the GLM4-MoE expert layer described in "Optimizing GLM4-MoE
for production" (Novita AI blog, section 1 "Shared Experts Fusion"): 160 routed
experts plus one shared expert, top-8 routing, the shared expert appended as
expert index 160. Hidden 5120 and per-expert intermediate 1536 are the model
shapes; 192 is the per-shard intermediate the same section quotes for TP8/FP8.

Recipe (per workload, fixed draw order, one generator seeded with the
workload's seed):
  1. x      [T, H]      ~ N(0, 1)                  -> bf16 (RNE) or fp32
  2. Wr     [E_r, H]    ~ N(0, router_std)          fp32 (router weights stay fp32)
  3. for e in 0..E-1: gate [I, H], up [I, H], down [H, I] ~ N(0, weight_std)
     -> w13[e] = concat(gate, up) [2I, H], w2[e] = down [H, I]
     bf16 workloads cast with RNE; E4M3 workloads store codes with one fp32
     scale per output channel, scale = amax/448 (amax = 0 -> scale 1).
  4. skewed workloads add a router bias b[e] = -s * ln(e + 1), a Zipf(s) prior
     over expert ids (deterministic, no draw).
Small workloads draw on the CPU; full-size workloads may draw on the GPU with
torch's CUDA generator (same order, same seeds, a different random stream).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int              # tokens
    H: int              # hidden size
    I: int              # per-expert intermediate size
    n_routed: int       # routed experts E_r; the shared expert is index E_r
    top_k: int          # routed experts chosen per token (K)
    act_dtype: str      # 'f32' | 'bf16'  (x and out)
    w_dtype: str        # 'f32' | 'bf16' | 'e4m3'
    seed: int
    router_std: float | None = 0.02   # None -> 1/sqrt(H), router logits ~ N(0, 1)
    weight_std: float = 0.02
    zipf_s: float | None = None
    shared: bool = True
    shared_weight: float = 1.0
    renormalize: bool = True
    routed_scale: float = 1.0        # routed slots weigh routed_scale * softmax
    bias_select_only: bool = False   # router bias ranks the experts but does not weigh them
    out_f32: bool = False            # the layer writes its unrounded fp32 sum (tensor-parallel partials)

    @property
    def n_experts(self) -> int:
        return self.n_routed + (1 if self.shared else 0)

    @property
    def shared_id(self) -> int:
        return self.n_routed if self.shared else -1

    @property
    def slots(self) -> int:
        return self.top_k + (1 if self.shared else 0)

    @property
    def rows(self) -> int:
        return self.T * self.slots

    def gemm_flops(self) -> float:
        """2 * rows * (2I*H + H*I): the expert GEMM work of one layer pass."""
        return 2.0 * self.rows * 3 * self.H * self.I

    def router_flops(self) -> float:
        return 2.0 * self.T * self.n_routed * self.H


CONFIGS = {
    # tiny correctness workload: 8 routed + shared (index 8), top-2 + shared
    "tiny_fp32": LayerConfig("tiny_fp32", T=16, H=256, I=64, n_routed=8, top_k=2,
                             act_dtype="f32", w_dtype="f32", seed=0),
    # GLM4-MoE-shaped prefill, bf16 with fp32 accumulation
    "prefill_bf16": LayerConfig("prefill_bf16", T=4096, H=5120, I=1536, n_routed=160,
                                top_k=8, act_dtype="bf16", w_dtype="bf16", seed=1),
    # decode-sized, weight-bandwidth-bound; router logits ~ N(0, 1)
    "decode_bf16": LayerConfig("decode_bf16", T=64, H=5120, I=1536, n_routed=160, top_k=8,
                               act_dtype="bf16", w_dtype="bf16", seed=2, router_std=None),
    # FP8 E4M3 chunked prefill (16384-token chunk)
    "prefill_fp8": LayerConfig("prefill_fp8", T=16384, H=5120, I=1536, n_routed=160,
                               top_k=8, act_dtype="bf16", w_dtype="e4m3", seed=3),
    # FP8, per-shard intermediate 192, Zipf(1.2)-skewed routing
    "skewed_fp8": LayerConfig("skewed_fp8", T=4096, H=5120, I=192, n_routed=160, top_k=8,
                              act_dtype="bf16", w_dtype="e4m3", seed=4, zipf_s=1.2),
}


def variant(cfg: LayerConfig, **kw) -> LayerConfig:
    """A reduced-size copy of a workload (same dtypes and distributions)."""
    name = kw.pop("name", cfg.name + "_" + "_".join(f"{k}{v}" for k, v in kw.items()))
    return replace(cfg, name=name, **kw)


def _quantize_rows_e4m3(w: torch.Tensor):
    """Weight storage format of the E4M3 workloads: codes + per-row fp32 scale."""
    amax = w.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (w / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes.view(torch.uint8), scale.float()


def _cast_act(t: torch.Tensor, dtype: str) -> torch.Tensor:
    return t.to(torch.bfloat16) if dtype == "bf16" else t.float()


def _cast_w(t: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    return t.float()


def make_inputs(cfg: LayerConfig, device: str | torch.device = "cpu") -> dict:
    """Draw one workload. Tensors live on `device`; the draw order is fixed."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    T, H, I, Er, E = cfg.T, cfg.H, cfg.I, cfg.n_routed, cfg.n_experts

    x = torch.empty(T, H, device=device).normal_(0.0, 1.0, generator=g)
    rstd = cfg.router_std if cfg.router_std is not None else 1.0 / math.sqrt(H)
    wr = torch.empty(Er, H, device=device).normal_(0.0, rstd, generator=g)
    bias = None
    if cfg.zipf_s is not None:
        ids = torch.arange(Er, device=device, dtype=torch.float64)
        bias = (-cfg.zipf_s * torch.log(ids + 1.0)).float()

    if cfg.w_dtype == "e4m3":
        w13 = torch.empty(E, 2 * I, H, dtype=torch.uint8, device=device)
        w2 = torch.empty(E, H, I, dtype=torch.uint8, device=device)
        s13 = torch.empty(E, 2 * I, dtype=torch.float32, device=device)
        s2 = torch.empty(E, H, dtype=torch.float32, device=device)
    else:
        wdt = torch.bfloat16 if cfg.w_dtype == "bf16" else torch.float32
        w13 = torch.empty(E, 2 * I, H, dtype=wdt, device=device)
        w2 = torch.empty(E, H, I, dtype=wdt, device=device)
        s13 = s2 = None

    for e in range(E):
        gate = torch.empty(I, H, device=device).normal_(0.0, cfg.weight_std, generator=g)
        up = torch.empty(I, H, device=device).normal_(0.0, cfg.weight_std, generator=g)
        down = torch.empty(H, I, device=device).normal_(0.0, cfg.weight_std, generator=g)
        if cfg.w_dtype == "e4m3":
            c, s = _quantize_rows_e4m3(torch.cat([gate, up], 0))
            w13[e].copy_(c)
            s13[e].copy_(s)
            c, s = _quantize_rows_e4m3(down)
            w2[e].copy_(c)
            s2[e].copy_(s)
        else:
            w13[e, :I].copy_(_cast_w(gate, cfg.w_dtype))
            w13[e, I:].copy_(_cast_w(up, cfg.w_dtype))
            w2[e].copy_(_cast_w(down, cfg.w_dtype))
        del gate, up, down

    return {
        "x": _cast_act(x, cfg.act_dtype).contiguous(),
        "router_w": wr.float().contiguous(),
        "router_bias": bias,
        "w13": w13, "s13": s13, "w2": w2, "s2": s2,
    }


def to_host(inputs: dict) -> dict:
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


def to_device(inputs: dict, device) -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


# ------------------------------------------------------------------ attention pre-processing
# Inputs of the fused QK-norm + partial RoPE step (the attention's q and k heads
# normalised per head, then the first rot dimensions of each head rotated).

@dataclass(frozen=True)
class AttnConfig:
    name: str
    T: int              # tokens
    n_q: int            # query heads
    n_kv: int           # key / value heads
    d: int              # head dimension
    rot: int            # rotated dimensions per head (half of d in GLM4-MoE)
    max_pos: int        # rows of the cos/sin table
    seed: int
    theta: float = 1.0e6
    eps: float = 1.0e-5
    sequential: bool = True   # positions 0..T-1 (prefill); else random (decode)

    @property
    def row(self) -> int:
        return (self.n_q + 2 * self.n_kv) * self.d

    def moved_bytes(self) -> int:
        """q and k heads read and written once, bf16, plus positions."""
        return 2 * self.T * (self.n_q + self.n_kv) * self.d * 2 + self.T * 4


ATTN_CONFIGS = {
    "qknorm_tiny": AttnConfig("qknorm_tiny", T=5, n_q=4, n_kv=2, d=64, rot=32, max_pos=64, seed=10),
    # GLM4-MoE attention heads: 96 query and 8 key/value heads of 128, half rotated
    "qknorm_prefill": AttnConfig("qknorm_prefill", T=4096, n_q=96, n_kv=8, d=128, rot=64, max_pos=4096,
                                 seed=11),
    "qknorm_decode": AttnConfig("qknorm_decode", T=64, n_q=96, n_kv=8, d=128, rot=64, max_pos=32768,
                                seed=12, sequential=False),
}


def make_attn_inputs(cfg: AttnConfig, device: str | torch.device = "cpu") -> dict:
    """qkv [T, (n_q + 2 n_kv) d] bf16 with per-head scales spread over 10^-1..10^1,
    positions [T] int32, q/k norm weights [d] bf16 around 1, and the cos/sin
    table [max_pos, rot] fp32 (angle pos * theta^(-2j/rot), cos then sin)."""
    device = torch.device(device)
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed)
    heads = cfg.n_q + 2 * cfg.n_kv
    qkv = torch.empty(cfg.T, heads, cfg.d).normal_(0.0, 1.0, generator=g)
    scale = torch.pow(10.0, torch.empty(cfg.T, heads, 1).uniform_(-1.0, 1.0, generator=g))
    qkv = (qkv * scale).reshape(cfg.T, cfg.row).to(torch.bfloat16)
    if cfg.sequential:
        pos = torch.arange(cfg.T, dtype=torch.int32) % cfg.max_pos
    else:
        pos = torch.randint(0, cfg.max_pos, (cfg.T,), generator=g, dtype=torch.int64).to(torch.int32)
    qw = (1.0 + 0.1 * torch.empty(cfg.d).normal_(0.0, 1.0, generator=g)).to(torch.bfloat16)
    kw = (1.0 + 0.1 * torch.empty(cfg.d).normal_(0.0, 1.0, generator=g)).to(torch.bfloat16)
    half = cfg.rot // 2
    inv = torch.pow(torch.tensor(cfg.theta, dtype=torch.float64),
                    -2.0 * torch.arange(half, dtype=torch.float64) / cfg.rot)
    ang = torch.arange(cfg.max_pos, dtype=torch.float64)[:, None] * inv[None, :]
    cos_sin = torch.cat([torch.cos(ang), torch.sin(ang)], 1).float()
    out = {"qkv": qkv, "pos": pos, "q_w": qw, "k_w": kw, "cos_sin": cos_sin.contiguous()}
    return {k: v.to(device) for k, v in out.items()}
