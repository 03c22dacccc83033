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


def test_permute_noalloc_matches_the_workspace_entry_point_on_consecutive_calls():
    build.build()
    # two calls in a row: a GLM-shaped batch, then a ragged one, sharing the scratch
    for T, E_r, K, seed in [(4096, 160, 8, 1), (333, 40, 6, 2)]:
        cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=T, H=256, I=64, n_routed=E_r, top_k=K)
        s = _lib.make_shape(cfg)
        ids = torch.from_numpy(_ids(T, E_r, K, seed)).to(DEV)
        E, R = cfg.n_experts, cfg.rows
        ref = _outputs(E, R)
        ws = _lib.alloc_workspace(s, True)
        _lib.moe_permute(s, ids, *ref, ws)
        got = _outputs(E, R)
        _lib.moe_permute_noalloc(s, ids, *got)
        torch.cuda.synchronize()
        assert _lib.moe_get_status(ws) == _lib.MOE_OK
        for a, b in zip(got, ref):        # integer outputs: bit for bit
            assert torch.equal(a, b)


def test_permute_noalloc_rejects_sizes_beyond_its_fixed_scratch():
    build.build()
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=100000, H=256, I=64)
    s = _lib.make_shape(cfg)
    with pytest.raises(_lib.MoeError) as ei:
        _lib.moe_permute_noalloc(s, 16, 16, 16, 16, 16)      # host check fires before any use
    assert ei.value.code == _lib.MOE_ERR_UNSUPPORTED
