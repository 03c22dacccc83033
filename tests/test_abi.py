"""The C ABI without a GPU: the library loads, exports every entry point that
include/moe.h declares, and rejects bad arguments on the host before any CUDA
call is made."""
import ctypes as C
import os
import re

import pytest

from shared_routed_expert_b200 import _lib, build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_layer_entry_points():
    names = declared_functions()
    for must in ("moe_route_topk", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_forward"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) <= set(_lib.EXPORTS)


def test_status_strings(L):
    for code in range(7):
        assert _lib.status_string(code)
    assert _lib.status_string(_lib.MOE_ERR_WORKSPACE) == "workspace too small"


def _shape(**kw):
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=64, H=512, I=128, n_routed=16, top_k=4)
    s = _lib.make_shape(cfg)
    for k, v in kw.items():
        setattr(s, k, v)
    return s


def test_workspace_size_and_invalid_shapes(L):
    s = _shape()
    n_f = _lib.moe_workspace_size(s, True)
    n_u = _lib.moe_workspace_size(s, False)
    assert n_f > 0 and n_u > 0 and n_f % 256 == 0
    for bad in (dict(H=500), dict(I=100), dict(top_k=17), dict(shared_id=3),
                dict(act_dtype=_lib.MOE_F32), dict(w_dtype=_lib.MOE_F32), dict(T=-1),
                dict(renormalize=2), dict(n_routed=300, top_k=8, shared_id=300),
                dict(n_routed=257, top_k=8, shared_id=257)):
        assert L.moe_workspace_size(C.byref(_shape(**bad)), 1) == 0, bad
    # 256 routed experts (+ the shared one) is the largest layer accepted
    assert L.moe_workspace_size(C.byref(_shape(n_routed=256, top_k=8, shared_id=256)), 1) > 0


FAKE = 1 << 20        # aligned non-null addresses; the host checks never dereference them


def test_forward_rejects_bad_arguments_on_the_host(L):
    s = _shape()
    n = _lib.moe_workspace_size(s, True)
    f = L.moe_forward
    ok = [C.byref(s), FAKE, FAKE, None, FAKE, None, FAKE, None, 1, FAKE, FAKE, n, 0, None]

    def call(**over):
        args = list(ok)
        pos = {"x": 1, "w13": 4, "out": 9, "ws": 10, "ws_bytes": 11, "impl": 12, "fuse": 8,
               "router_w": 2}
        for k, v in over.items():
            args[pos[k]] = v
        return f(*args)

    assert call(x=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(w13=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(x=FAKE + 8) == _lib.MOE_ERR_INVALID_ARG           # not 16-byte aligned
    assert call(ws=FAKE + 16) == _lib.MOE_ERR_INVALID_ARG         # workspace not 256-aligned
    assert call(ws_bytes=n - 1) == _lib.MOE_ERR_WORKSPACE
    assert call(impl=8) == _lib.MOE_ERR_INVALID_ARG
    s0 = _shape(shared_id=-1)
    assert f(C.byref(s0), FAKE, FAKE, None, FAKE, None, FAKE, None, 0, FAKE, FAKE, 1 << 30, 0,
             None) == _lib.MOE_ERR_INVALID_ARG                   # unfused needs a shared expert
    s8 = _shape(w_dtype=_lib.MOE_E4M3)
    n8 = _lib.moe_workspace_size(s8, True)
    assert f(C.byref(s8), FAKE, FAKE, None, FAKE, None, FAKE, None, 1, FAKE, FAKE, n8, 0,
             None) == _lib.MOE_ERR_INVALID_ARG                   # E4M3 needs weight scales
    s32 = _shape(act_dtype=_lib.MOE_F32, w_dtype=_lib.MOE_F32)
    assert f(C.byref(s32), FAKE, FAKE, None, FAKE, None, FAKE, None, 1, FAKE, FAKE, 1 << 30,
             _lib.MOE_FFN_TCGEN05, None) == _lib.MOE_ERR_UNSUPPORTED


def test_other_entry_points_reject_bad_arguments(L):
    s = _shape()
    n = _lib.moe_workspace_size(s, True)
    assert L.moe_route_topk(C.byref(s), None, FAKE, None, FAKE, FAKE, None, FAKE, n, None) == 1
    assert L.moe_route_topk(C.byref(s), FAKE, FAKE, None, FAKE, FAKE, None, FAKE, n - 256,
                            None) == _lib.MOE_ERR_WORKSPACE
    assert L.moe_permute(C.byref(s), FAKE, None, FAKE, FAKE, FAKE, FAKE, n, None) == 1
    assert L.moe_grouped_ffn(C.byref(s), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE,
                             n - 1, 0, None) == _lib.MOE_ERR_WORKSPACE
    assert L.moe_combine(C.byref(s), FAKE, None, FAKE, FAKE, None) == 1
    assert L.moe_quant_rows_e4m3(4, 12, FAKE, FAKE, FAKE, None) == 1      # cols % 8
    assert L.moe_get_status(None, None) == 1
    assert L.moe_launch_count() == 0


def test_zero_tokens_is_a_no_op(L):
    s = _shape(T=0)
    n = _lib.moe_workspace_size(s, True)
    assert L.moe_forward(C.byref(s), FAKE, FAKE, None, FAKE, None, FAKE, None, 1, FAKE, FAKE, n,
                         0, None) == _lib.MOE_OK
    assert L.moe_launch_count() == 0


def test_a_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU path: without the built CUDA library every entry point raises
    instead of computing anything."""
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libsre_moe.so"))
    with pytest.raises(ImportError):
        _lib.lib()
    with pytest.raises(ImportError):
        _lib.moe_workspace_size(_shape(), True)


def _noalloc_bound(E: int) -> int:
    """Largest ceil(T*S/512) * E the fixed scratch of moe_permute_noalloc holds:
    1 MiB less the 256-byte status word and the (E+1)-int tile prefix rounded
    up to 256 bytes, in ints."""
    return (1048576 - 256 - (4 * (E + 1) + 255) // 256 * 256) // 4


@pytest.mark.parametrize("E_r,K", [(40, 6), (160, 8), (191, 4), (256, 8)])
def test_permute_noalloc_size_limit_is_exact(L, E_r, K):
    """The host check of moe_permute_noalloc rejects exactly the batches whose
    histograms do not fit its fixed array: at the bound the call gets past the
    check (and, with no GPU here, fails in the CUDA runtime); one 512-slot chunk
    more is MOE_ERR_UNSUPPORTED before any CUDA call."""
    E, S = E_r + 1, K + 1
    chunks = _noalloc_bound(E) // E
    T_ok = chunks * 512 // S                  # ceil(T_ok * S / 512) == chunks
    T_bad = T_ok + 1
    assert -(-T_ok * S // 512) == chunks and -(-T_bad * S // 512) == chunks + 1
    for T, want in ((T_ok, None), (T_bad, _lib.MOE_ERR_UNSUPPORTED)):
        cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=T, H=256, I=64, n_routed=E_r, top_k=K)
        rc = L.moe_permute_noalloc(C.byref(_lib.make_shape(cfg)), FAKE, FAKE, FAKE, FAKE, FAKE, None)
        if want is None:
            assert rc != _lib.MOE_ERR_UNSUPPORTED
        else:
            assert rc == want
