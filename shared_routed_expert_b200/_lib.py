"""ctypes binding of libsre_moe.so (include/moe.h). Argument marshalling only:
every step of the layer runs in the library's CUDA kernels. There is no CPU
path; if the library is missing, loading fails loudly."""
from __future__ import annotations

import ctypes as C
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsre_moe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE = 4, 5, 6
MOE_F32, MOE_BF16, MOE_E4M3 = 0, 1, 2
(MOE_FFN_AUTO, MOE_FFN_SIMT, MOE_FFN_TCGEN05, MOE_FFN_TCGEN05_M128, MOE_FFN_TCGEN05_M256,
 MOE_FFN_TCGEN05_PAIR, MOE_FFN_TCGEN05_WIDE, MOE_FFN_TCGEN05_SWAP) = 0, 1, 2, 3, 4, 5, 6, 7
MOE_FFN_COMBINE_FOLD = 512         # flag: the fused layer's aggregation inside its down-projection
DTYPES = {"f32": MOE_F32, "bf16": MOE_BF16, "e4m3": MOE_E4M3}

EXPORTS = ("moe_workspace_size", "moe_route_topk", "moe_permute", "moe_grouped_ffn",
           "moe_combine", "moe_forward", "moe_quant_rows_e4m3", "moe_get_status",
           "moe_clear_status", "moe_status_string", "moe_launch_count", "moe_profile_enable",
           "moe_profile_reset", "moe_profile_read", "moe_inject_wait_timeout",
           "moe_permute_noalloc", "moe_qk_norm_rope", "moe_cast_f32_bf16", "moe_inject_fold_timeout",
           "moe_inject_route_timeout")


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {status_string(code)} (status {code})")


class moe_shape(C.Structure):
    _fields_ = [("T", C.c_int32), ("H", C.c_int32), ("I", C.c_int32), ("n_routed", C.c_int32),
                ("top_k", C.c_int32), ("shared_id", C.c_int32), ("shared_weight", C.c_float),
                ("renormalize", C.c_int32), ("act_dtype", C.c_int32), ("w_dtype", C.c_int32),
                ("routed_scale", C.c_float), ("bias_select_only", C.c_int32), ("out_f32", C.c_int32)]


_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run python -m shared_routed_expert_b200.build")
        L = C.CDLL(LIB_PATH)
        p, i, u64, sz, f = C.c_void_p, C.c_int, C.c_uint64, C.c_size_t, C.c_float
        S = C.POINTER(moe_shape)
        L.moe_workspace_size.restype = sz
        L.moe_workspace_size.argtypes = [S, i]
        L.moe_route_topk.restype = i
        L.moe_route_topk.argtypes = [S, p, p, p, p, p, p, p, sz, p]
        L.moe_permute.restype = i
        L.moe_permute.argtypes = [S, p, p, p, p, p, p, sz, p]
        L.moe_grouped_ffn.restype = i
        L.moe_grouped_ffn.argtypes = [S, p, p, p, p, p, p, p, p, p, sz, i, p]
        L.moe_combine.restype = i
        L.moe_combine.argtypes = [S, p, p, p, p, p]
        L.moe_forward.restype = i
        L.moe_forward.argtypes = [S, p, p, p, p, p, p, p, i, p, p, sz, i, p]
        L.moe_quant_rows_e4m3.restype = i
        L.moe_quant_rows_e4m3.argtypes = [C.c_int32, C.c_int32, p, p, p, p]
        L.moe_get_status.restype = i
        L.moe_get_status.argtypes = [p, p]
        L.moe_clear_status.restype = i
        L.moe_clear_status.argtypes = [p, p]
        L.moe_status_string.restype = C.c_char_p
        L.moe_status_string.argtypes = [i]
        L.moe_launch_count.restype = u64
        L.moe_launch_count.argtypes = []
        L.moe_profile_enable.restype = None
        L.moe_profile_enable.argtypes = [i]
        L.moe_profile_reset.restype = None
        L.moe_profile_reset.argtypes = []
        L.moe_profile_read.restype = i
        L.moe_profile_read.argtypes = [C.c_char_p, C.POINTER(C.c_int64), C.POINTER(C.c_double)]
        L.moe_permute_noalloc.restype = i
        L.moe_permute_noalloc.argtypes = [S, p, p, p, p, p, p]
        L.moe_inject_wait_timeout.restype = None
        L.moe_inject_wait_timeout.argtypes = [i]
        L.moe_inject_fold_timeout.restype = None
        L.moe_inject_fold_timeout.argtypes = [i]
        L.moe_inject_route_timeout.restype = None
        L.moe_inject_route_timeout.argtypes = [i]
        L.moe_cast_f32_bf16.restype = i
        L.moe_cast_f32_bf16.argtypes = [sz, p, p, p]
        L.moe_qk_norm_rope.restype = i
        L.moe_qk_norm_rope.argtypes = [i, i, i, i, i, f, p, p, i, p, p, p, p, p]
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def make_shape(cfg, T: int | None = None) -> moe_shape:
    """moe_shape of a LayerConfig-like object (T overrides cfg.T)."""
    return moe_shape(cfg.T if T is None else T, cfg.H, cfg.I, cfg.n_routed, cfg.top_k,
                     cfg.shared_id, cfg.shared_weight, int(cfg.renormalize),
                     DTYPES[cfg.act_dtype], DTYPES[cfg.w_dtype],
                     float(getattr(cfg, "routed_scale", 1.0)), int(getattr(cfg, "bias_select_only", False)),
                     int(getattr(cfg, "out_f32", False)))


def moe_workspace_size(shape: moe_shape, fuse_shared: bool = True) -> int:
    n = lib().moe_workspace_size(C.byref(shape), int(fuse_shared))
    if n == 0:
        raise MoeError("moe_workspace_size", MOE_ERR_INVALID_ARG)
    return n


def alloc_workspace(shape: moe_shape, fuse_shared: bool = True, device="cuda") -> torch.Tensor:
    n = moe_workspace_size(shape, fuse_shared)
    ws = torch.zeros(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def moe_route_topk(shape, x, router_w, router_bias, ids, weights, logits, ws, stream=None):
    _check("moe_route_topk", lib().moe_route_topk(
        C.byref(shape), _p(x), _p(router_w), _p(router_bias), _p(ids), _p(weights), _p(logits),
        _p(ws), ws.numel(), _stream(stream)))


def moe_permute(shape, ids, counts, offsets, perm, inv, ws, stream=None):
    _check("moe_permute", lib().moe_permute(
        C.byref(shape), _p(ids), _p(counts), _p(offsets), _p(perm), _p(inv), _p(ws), ws.numel(),
        _stream(stream)))


def moe_grouped_ffn(shape, x, perm, offsets, w13, s13, w2, s2, y, ws, impl=MOE_FFN_AUTO,
                    stream=None):
    _check("moe_grouped_ffn", lib().moe_grouped_ffn(
        C.byref(shape), _p(x), _p(perm), _p(offsets), _p(w13), _p(s13), _p(w2), _p(s2), _p(y),
        _p(ws), ws.numel(), impl, _stream(stream)))


def moe_combine(shape, y, inv, weights, out, stream=None):
    _check("moe_combine", lib().moe_combine(
        C.byref(shape), _p(y), _p(inv), _p(weights), _p(out), _stream(stream)))


def moe_forward(shape, x, router_w, router_bias, w13, s13, w2, s2, fuse_shared, out, ws,
                impl=MOE_FFN_AUTO, stream=None):
    _check("moe_forward", lib().moe_forward(
        C.byref(shape), _p(x), _p(router_w), _p(router_bias), _p(w13), _p(s13), _p(w2), _p(s2),
        int(fuse_shared), _p(out), _p(ws), ws.numel(), impl, _stream(stream)))


def moe_permute_noalloc(shape, ids, counts, offsets, perm, inv, stream=None):
    """moe_permute for callers that cannot allocate: the library's own fixed
    device scratch replaces the workspace (see include/moe.h)."""
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(
        C.byref(shape), _p(ids), _p(counts), _p(offsets), _p(perm), _p(inv), _stream(stream)))


def moe_qk_norm_rope(cfg, qkv, positions, q_norm_w, k_norm_w, cos_sin, bad_positions=None, stream=None):
    """In place on the q and k heads of qkv [T, (n_q + 2 n_kv) d] bf16; cfg
    carries T, n_q, n_kv, d, rot, eps and max_pos = cos_sin rows."""
    _check("moe_qk_norm_rope", lib().moe_qk_norm_rope(
        qkv.shape[0], cfg.n_q, cfg.n_kv, cfg.d, cfg.rot, cfg.eps, _p(qkv), _p(positions), cos_sin.shape[0],
        _p(q_norm_w), _p(k_norm_w), _p(cos_sin if cfg.rot > 0 else None), _p(bad_positions), _stream(stream)))


def moe_cast_f32_bf16(inp, out, stream=None):
    """out (bf16) = inp (fp32) rounded to nearest even, same element count."""
    _check("moe_cast_f32_bf16", lib().moe_cast_f32_bf16(inp.numel(), _p(inp), _p(out), _stream(stream)))


def moe_quant_rows_e4m3(rows, cols, inp, codes, scales, stream=None):
    _check("moe_quant_rows_e4m3", lib().moe_quant_rows_e4m3(
        rows, cols, _p(inp), _p(codes), _p(scales), _stream(stream)))


def moe_get_status(ws, stream=None) -> int:
    return lib().moe_get_status(_p(ws), _stream(stream))


def moe_clear_status(ws, stream=None):
    _check("moe_clear_status", lib().moe_clear_status(_p(ws), _stream(stream)))


def moe_launch_count() -> int:
    return int(lib().moe_launch_count())


_prof_on = False


def moe_profile_enable(on: bool):
    global _prof_on
    lib().moe_profile_enable(int(on))
    _prof_on = bool(on)


def profile_enabled() -> bool:
    """Whether per-kernel event timing was last switched on through this module."""
    return _prof_on


def moe_profile_reset():
    lib().moe_profile_reset()


def moe_inject_wait_timeout(n_calls: int):
    lib().moe_inject_wait_timeout(int(n_calls))


def moe_inject_fold_timeout(n_calls: int):
    lib().moe_inject_fold_timeout(int(n_calls))


def moe_inject_route_timeout(n_calls: int):
    lib().moe_inject_route_timeout(int(n_calls))


def moe_profile_read(name: str):
    n = C.c_int64()
    ms = C.c_double()
    _check("moe_profile_read", lib().moe_profile_read(name.encode(), C.byref(n), C.byref(ms)))
    return n.value, ms.value
