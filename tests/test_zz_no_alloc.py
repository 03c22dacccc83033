"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (their buffers all come from a host framework, or they may not call
cudaMalloc where they enqueue work). It must give exactly what moe_permute gives
with a caller-provided workspace, on consecutive calls that reuse the library's
fixed scratch array. This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from shared_routed_expert_b200 import _lib, build, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ids(T, E_r, K, seed):
    rng = np.random.default_rng(seed)
    routed = np.stack([rng.permutation(E_r)[:K] for _ in range(T)]).astype(np.int32)
    return np.concatenate([routed, np.full((T, 1), E_r, np.int32)], 1)


def _outputs(E, R):
    return [torch.full((n,), -1, dtype=torch.int32, device=DEV) for n in (E, E + 1, R, R)]


def _both(T, E_r, K, ids_np):
    """(noalloc outputs, workspace-entry outputs, the latter's status)."""
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=T, H=256, I=64, n_routed=E_r, top_k=K)
    s = _lib.make_shape(cfg)
    ids = torch.from_numpy(ids_np).to(DEV)
    E, R = cfg.n_experts, cfg.rows
    ref = _outputs(E, R)
    ws = _lib.alloc_workspace(s, True)
    _lib.moe_permute(s, ids, *ref, ws)
    got = _outputs(E, R)
    _lib.moe_permute_noalloc(s, ids, *got)
    torch.cuda.synchronize()
    return got, ref, _lib.moe_get_status(ws)


def test_permute_noalloc_matches_the_workspace_entry_point_on_consecutive_calls():
    build.build()
    # two calls in a row, both on the multi-kernel path (more than 8192 slots),
    # with different expert counts and numbers of 512-slot chunks, sharing the
    # fixed scratch: a GLM-shaped batch (72 chunks x 161 experts), then a
    # ragged one (21 chunks x 41 experts)
    for T, E_r, K, seed in [(4096, 160, 8, 1), (1500, 40, 6, 2)]:
        assert T * (K + 1) > 8192
        got, ref, st = _both(T, E_r, K, _ids(T, E_r, K, seed))
        assert st == _lib.MOE_OK
        for a, b in zip(got, ref):        # integer outputs: bit for bit
            assert torch.equal(a, b)


@pytest.mark.parametrize("T,E_r,K", [(333, 40, 6), (1500, 40, 6)])
def test_permute_noalloc_drops_an_out_of_range_id(T, E_r, K):
    """An out-of-range id is dropped without a report (this call has no status
    word the caller can read): MOE_OK, the counts sum to R - 1, and every output
    equals moe_permute's, which reports the id. One-block path (333 tokens) and
    multi-kernel path (1500 tokens)."""
    build.build()
    ids = _ids(T, E_r, K, 7)
    ids[T // 2, 1] = E_r + 5                      # past the shared expert's id
    got, ref, st = _both(T, E_r, K, ids)          # raises unless noalloc returned MOE_OK
    assert st == _lib.MOE_ERR_DEVICE              # the workspace entry point saw it
    R = ids.size
    assert int(got[0].sum()) == R - 1 and int(got[1][-1]) == R - 1
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_permute_noalloc_rejects_sizes_beyond_its_fixed_scratch():
    build.build()
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=100000, H=256, I=64)
    s = _lib.make_shape(cfg)
    with pytest.raises(_lib.MoeError) as ei:
        _lib.moe_permute_noalloc(s, 16, 16, 16, 16, 16)      # host check fires before any use
    assert ei.value.code == _lib.MOE_ERR_UNSUPPORTED
