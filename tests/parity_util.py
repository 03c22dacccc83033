"""Helpers shared by the GPU parity tests: the error metric, tolerances, and
the oracle router run over token chunks on several host threads."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle

# Tolerances on outputs (max relative error, fp32 accumulation). bf16/fp32
# layers: 1e-2; E4M3 layers: 3e-2 against an oracle that decodes the same codes.
# The reference is the oracle's exact (fp64, unrounded) layer output, so the
# GPU's own final rounding counts against the budget once, not twice.
TOL = {"f32": 1e-2, "bf16": 1e-2, "e4m3": 3e-2}


def tol_of(cfg) -> float:
    return TOL[cfg.w_dtype]


def rel_err(got, ref) -> float:
    """max_i |g_i - r_i| / max(|r_i|, rms(r)): relative error, with the RMS of
    the reference as the floor of the denominator so that outputs near zero do
    not dominate."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    den = np.maximum(np.abs(ref), rms if rms > 0 else 1e-30)
    return float(np.max(np.abs(got - ref) / den))


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def oracle_logits(x: torch.Tensor, wr: torch.Tensor, bias, rows=None) -> np.ndarray:
    """Oracle fixed-order fp32 logits for the listed token rows (all if None),
    chunked over host threads (the C call releases the GIL)."""
    xs = x if rows is None else x[torch.as_tensor(rows, dtype=torch.long, device=x.device)]
    xh = xs.detach().float().cpu().numpy()
    wh = wr.detach().float().cpu().numpy()
    bh = None if bias is None else bias.detach().float().cpu().numpy()
    n = xh.shape[0]
    chunks = [(i, min(n, i + 256)) for i in range(0, n, 256)]
    with ThreadPoolExecutor(threads()) as ex:
        parts = list(ex.map(lambda c: oracle.router_logits(xh[c[0]:c[1]], wh, bh), chunks))
    return np.concatenate(parts, 0) if parts else np.zeros((0, wh.shape[0]), np.float32)


def sample_tokens(T: int, n: int, seed: int = 123) -> np.ndarray:
    rng = np.random.default_rng(seed)
    pick = {0, T - 1}
    while len(pick) < min(n, T):
        pick.add(int(rng.integers(0, T)))
    return np.array(sorted(pick), dtype=np.int32)
