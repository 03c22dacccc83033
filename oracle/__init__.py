"""ctypes wrapper of the CPU oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``. The product path (the CUDA library
and its binding) never imports this package.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
F32, BF16, E4M3 = 0, 1, 2
_DT = {"f32": F32, "bf16": BF16, "e4m3": E4M3}


def build(force: bool = False) -> str:
    """Compile the oracle with plain gcc: no fast-math, no fp contraction."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-pthread", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(build())
        p, i, f, d = C.c_void_p, C.c_int, C.c_float, C.c_double
        L.orc_bf16_to_double.restype = d
        L.orc_bf16_to_double.argtypes = [C.c_uint16]
        L.orc_round_bf16.restype = C.c_uint16
        L.orc_round_bf16.argtypes = [d]
        L.orc_e4m3_decode.restype = d
        L.orc_e4m3_decode.argtypes = [C.c_uint8]
        L.orc_e4m3_encode.restype = C.c_uint8
        L.orc_e4m3_encode.argtypes = [f]
        L.orc_quant_row_e4m3.restype = f
        L.orc_quant_row_e4m3.argtypes = [i, p, p]
        L.orc_router_logits.restype = None
        L.orc_router_logits.argtypes = [i, i, i, p, p, p, p]
        L.orc_router_logits_f64.restype = None
        L.orc_router_logits_f64.argtypes = [i, i, i, p, p, p, p]
        L.orc_topk.restype = None
        L.orc_topk.argtypes = [i, i, i, p, p, i, f, i, f, p, p]
        L.orc_permute.restype = i
        L.orc_permute.argtypes = [i, i, p, p, p, p, p]
        L.orc_expert_ffn.restype = None
        L.orc_expert_ffn.argtypes = [p, i, p, p]
        L.orc_forward.restype = i
        L.orc_forward.argtypes = [p, i, p, i, p, p, p, p, i]
        L.orc_qk_norm_rope.restype = None
        L.orc_qk_norm_rope.argtypes = [i, i, i, i, i, f, p, p, p, p, p, p]
        L.orc_combine.restype = None
        L.orc_combine.argtypes = [i, i, i, p, p, p, i, p]
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _np(t: torch.Tensor | None):
    """Host numpy view of a tensor; bf16 as uint16 bits, E4M3 codes as uint8."""
    if t is None:
        return None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def act_as_f32(x: torch.Tensor) -> np.ndarray:
    return np.ascontiguousarray(x.detach().cpu().float().numpy(), dtype=np.float32)


# ------------------------------------------------------------------ codecs

def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib().orc_e4m3_decode(int(c)) for c in codes], dtype=np.float64)


def e4m3_encode(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float32).ravel()
    return np.array([lib().orc_e4m3_encode(float(a)) for a in v], dtype=np.uint8)


def round_bf16(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64).ravel()
    return np.array([lib().orc_round_bf16(float(a)) for a in v], dtype=np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def quant_rows_e4m3(v: np.ndarray):
    """Per-row E4M3 quantisation: returns (codes [n, m] uint8, scales [n] fp32)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    n, m = v.shape
    codes = np.empty((n, m), dtype=np.uint8)
    scales = np.empty(n, dtype=np.float32)
    for r in range(n):
        scales[r] = lib().orc_quant_row_e4m3(m, _ptr(v[r]), _ptr(codes[r]))
    return codes, scales


# ------------------------------------------------------------------ router

def router_logits(x: np.ndarray, wr: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    wr = np.ascontiguousarray(wr, dtype=np.float32)
    T, H = x.shape
    E = wr.shape[0]
    assert H % 256 == 0
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    L = np.empty((T, E), dtype=np.float32)
    lib().orc_router_logits(T, H, E, _ptr(x), _ptr(wr), _ptr(b), _ptr(L))
    return L


def router_logits_f64(x, wr, bias=None) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    wr = np.ascontiguousarray(wr, dtype=np.float32)
    T, H = x.shape
    E = wr.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    L = np.empty((T, E), dtype=np.float64)
    lib().orc_router_logits_f64(T, H, E, _ptr(x), _ptr(wr), _ptr(b), _ptr(L))
    return L


def topk(L: np.ndarray, K: int, renormalize: bool = True, shared_id: int = -1,
         shared_weight: float = 1.0, weight_logits: np.ndarray | None = None, routed_scale: float = 1.0):
    """Top-K by the ranking keys L; weights from weight_logits (default: L),
    routed slots scaled by routed_scale."""
    L = np.ascontiguousarray(L, dtype=np.float32)
    T, E = L.shape
    Lw = None if weight_logits is None else np.ascontiguousarray(weight_logits, dtype=np.float32)
    S = K + (1 if shared_id >= 0 else 0)
    ids = np.empty((T, S), dtype=np.int32)
    w = np.empty((T, S), dtype=np.float64)
    lib().orc_topk(T, E, K, _ptr(L), _ptr(Lw), int(renormalize), routed_scale, shared_id, shared_weight,
                   _ptr(ids), _ptr(w))
    return ids, w


def permute(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, dtype=np.int32).ravel()
    R = ids.size
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(R, dtype=np.int32)
    inv = np.empty(R, dtype=np.int32)
    rc = lib().orc_permute(R, E, _ptr(ids), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv))
    if rc != 0:
        raise ValueError("expert id out of range")
    return counts, offsets, perm, inv


def combine(Y: np.ndarray, inv: np.ndarray, w: np.ndarray, act_dtype: str) -> np.ndarray:
    Y = np.ascontiguousarray(Y, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    T, S = w.shape
    H = Y.shape[1]
    inv = np.ascontiguousarray(inv, dtype=np.int32)
    out = np.empty((T, H), dtype=np.float64)
    lib().orc_combine(T, S, H, _ptr(Y), _ptr(inv), _ptr(w), _DT[act_dtype], _ptr(out))
    return out


# ------------------------------------------------------------------ QK-norm + partial RoPE

def qk_norm_rope(qkv_bits: np.ndarray, pos: np.ndarray, qw_bits: np.ndarray, kw_bits: np.ndarray,
                 cos_sin: np.ndarray, n_q: int, n_kv: int, d: int, rot: int, eps: float) -> np.ndarray:
    """qkv_bits [T, (n_q + 2 n_kv) d] bf16 bits, pos [T], norm weights [d] bf16
    bits, cos_sin [max_pos, rot] fp32 -> normalised and rotated q and k heads,
    [T, n_q + n_kv, d] fp64 (unrounded)."""
    qkv_bits = np.ascontiguousarray(qkv_bits, dtype=np.uint16)
    T = qkv_bits.shape[0]
    assert qkv_bits.shape[1] == (n_q + 2 * n_kv) * d and rot % 2 == 0 and rot <= d
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    assert pos.shape == (T,) and (T == 0 or (pos.min() >= 0 and pos.max() < cos_sin.shape[0]))
    cos_sin = np.ascontiguousarray(cos_sin, dtype=np.float32)
    qw_bits = np.ascontiguousarray(qw_bits, dtype=np.uint16)
    kw_bits = np.ascontiguousarray(kw_bits, dtype=np.uint16)
    out = np.empty((T, n_q + n_kv, d), dtype=np.float64)
    lib().orc_qk_norm_rope(T, n_q, n_kv, d, rot, eps, _ptr(qkv_bits), _ptr(pos), _ptr(qw_bits),
                           _ptr(kw_bits), _ptr(cos_sin), _ptr(out))
    return out


# ------------------------------------------------------------------ layer

class _Layer(C.Structure):
    _fields_ = [("T", C.c_int), ("H", C.c_int), ("I", C.c_int), ("E_r", C.c_int),
                ("K", C.c_int), ("shared_id", C.c_int), ("shared_weight", C.c_float),
                ("renormalize", C.c_int), ("act_dtype", C.c_int), ("w_dtype", C.c_int),
                ("routed_scale", C.c_float), ("bias_select_only", C.c_int), ("x", C.c_void_p), ("router_w", C.c_void_p), ("router_bias", C.c_void_p),
                ("w13", C.c_void_p), ("s13", C.c_void_p), ("w2", C.c_void_p),
                ("s2", C.c_void_p)]


class Layer:
    """The oracle's view of one layer: host copies of the inputs plus shape."""

    def __init__(self, cfg, inputs: dict):
        self.cfg = cfg
        self._keep = {k: _np(v) for k, v in inputs.items()}
        k = self._keep
        self.s = _Layer(cfg.T, cfg.H, cfg.I, cfg.n_routed, cfg.top_k, cfg.shared_id,
                        cfg.shared_weight, int(cfg.renormalize), _DT[cfg.act_dtype],
                        _DT[cfg.w_dtype], float(getattr(cfg, "routed_scale", 1.0)),
                        int(getattr(cfg, "bias_select_only", False)), _ptr(k["x"]), _ptr(k["router_w"]),
                        _ptr(k["router_bias"]), _ptr(k["w13"]), _ptr(k["s13"]),
                        _ptr(k["w2"]), _ptr(k["s2"]))

    def expert_ffn(self, e: int, v: np.ndarray) -> np.ndarray:
        v = np.ascontiguousarray(v, dtype=np.float32)
        y = np.empty(self.cfg.H, dtype=np.float64)
        lib().orc_expert_ffn(C.byref(self.s), e, _ptr(v), _ptr(y))
        return y

    def forward(self, tokens=None, fuse_shared: bool = True, n_threads: int | None = None):
        """Returns dict(out fp64, out_rnd, ids, w, threads) for the listed tokens."""
        cfg = self.cfg
        tok = np.arange(cfg.T, dtype=np.int32) if tokens is None else \
            np.ascontiguousarray(tokens, dtype=np.int32)
        n = tok.size
        S = cfg.top_k + (1 if (fuse_shared and cfg.shared) else 0)
        out = np.empty((n, cfg.H), dtype=np.float64)
        out_rnd = np.empty((n, cfg.H), dtype=np.float64)
        ids = np.empty((n, S), dtype=np.int32)
        w = np.empty((n, S), dtype=np.float64)
        if n_threads is None:
            n_threads = len(os.sched_getaffinity(0))
        used = lib().orc_forward(C.byref(self.s), n, _ptr(tok), int(fuse_shared), _ptr(out),
                                 _ptr(out_rnd), _ptr(ids), _ptr(w), n_threads)
        return {"out": out, "out_rnd": out_rnd, "ids": ids, "w": w, "threads": used,
                "tokens": tok}
