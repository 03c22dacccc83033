"""The tensor-parallel layer's kernel side on one GPU: every rank's share
(moe_forward over its slice of each expert's intermediate dimension, unrounded
fp32) is computed by the CUDA library, the shares are summed as the all-reduce
would sum them, and moe_cast_f32_bf16 rounds once. Compared with the oracle's
slices and, for bf16 layers, with the full layer."""
import numpy as np
import pytest
import torch

import oracle
from shared_routed_expert_b200 import _lib, build, synth, tp
from tests.parity_util import rel_err, to_f64, tol_of

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = {
    "bf16_tp2": (synth.variant(synth.CONFIGS["prefill_bf16"], T=100, H=512, I=512, n_routed=16, top_k=4), 2),
    "bf16_tp8": (synth.variant(synth.CONFIGS["prefill_bf16"], T=100, H=512, I=512, n_routed=16, top_k=4), 8),
    "fp8_tp2": (synth.variant(synth.CONFIGS["prefill_fp8"], T=90, H=512, I=384, n_routed=12, top_k=3), 2),
    "fp8_zipf_tp3": (synth.variant(synth.CONFIGS["skewed_fp8"], T=90, H=512, I=384, n_routed=12, top_k=3), 3),
}


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("fuse", [True, False], ids=["fused", "unfused"])
def test_tensor_parallel_shares_sum_to_the_layer(name, fuse):
    cfg, world = CASES[name]
    inp = synth.make_inputs(cfg)
    d = synth.to_device(inp, DEV)
    parts, oracle_parts = [], []
    for r in range(world):
        layer = tp.TPMoELayer(cfg, tp.shard_weights(d, cfg.I, r, world), world, fuse_shared=fuse)
        part = layer.partial(d["x"])
        assert layer.layer.status() == _lib.MOE_OK
        ref = oracle.Layer(tp.local_config(cfg, world), tp.shard_weights(inp, cfg.I, r, world)) \
            .forward(fuse_shared=fuse)["out"]
        assert rel_err(part.double().cpu().numpy(), ref) <= tol_of(cfg), r      # each share
        parts.append(part)
        oracle_parts.append(ref)
    total = torch.stack(parts).sum(0)
    out = torch.empty(total.shape, dtype=torch.bfloat16, device=DEV)
    _lib.moe_cast_f32_bf16(total, out)
    torch.cuda.synchronize()
    assert torch.equal(out, total.to(torch.bfloat16))            # the cast rounds to nearest even
    assert rel_err(to_f64(out), sum(oracle_parts)) <= tol_of(cfg)
    if cfg.w_dtype == "bf16":
        # bf16: the shares of the slices are the full layer's output
        assert rel_err(to_f64(out), oracle.Layer(cfg, inp).forward()["out"]) <= tol_of(cfg)
