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


def full_size_sample(T: int, ids: np.ndarray, n_routed: int, n: int, unit: int = 208,
                     seed: int = 321) -> np.ndarray:
    """Tokens whose outputs a full-size parity test checks, chosen to cover the
    work units of the grouped GEMMs: every `unit`-token block of the shared
    expert's group (its rows are the tokens in order) gets at least one token
    when n allows, and for each of the 10 largest routed groups the token of its
    first row (first work unit), of its last row (last unit) and of the row
    `unit` positions before its end; the rest are random tokens. All tokens
    when n >= T."""
    if n >= T:
        return np.arange(T, dtype=np.int32)
    pick = set()
    counts = np.bincount(ids[:, :-1].ravel() if ids.shape[1] > 1 else ids.ravel(),
                         minlength=n_routed)[:n_routed]
    flat = ids.ravel()
    S = ids.shape[1]
    for e in np.argsort(-counts, kind="stable")[:10]:
        rows = np.nonzero(flat == e)[0]             # the group's rows, in slot order
        if rows.size:
            for r in (rows[0], rows[-1], rows[max(0, rows.size - unit)]):
                pick.add(int(r // S))
    n_even = max(0, n - len(pick) - 8)
    if n_even:
        pick.update(int(t) for t in np.linspace(0, T - 1, n_even).round().astype(np.int64))
    rng = np.random.default_rng(seed)
    while len(pick) < min(n, T):
        pick.add(int(rng.integers(0, T)))
    return np.array(sorted(pick), dtype=np.int32)
