"""A seeded random sweep of layer shapes through moe_forward against the CPU
oracle: token counts with ragged tails, hidden and intermediate sizes the
tensor-core tiles divide differently, expert counts from 1 to 48, top-k from 1
to 8, bf16 and E4M3 weights, routed scaling factors and selection-only bias,
fused and unfused, and every GEMM variant (the CUDA-core one, single-CTA 128-
and 256-row units, CTA pairs with 256 x 256 and 256 x 512 tiles, and CTA pairs
with the tokens as the MMA's N dimension). Each case
compares every output and the routing of every token."""
import numpy as np
import pytest
import torch

import oracle
from shared_routed_expert_b200 import MoELayer, _lib, build, synth
from tests.parity_util import oracle_logits, rel_err, to_f64, tol_of

pytestmark = pytest.mark.gpu
DEV = "cuda"

IMPLS = [_lib.MOE_FFN_AUTO, _lib.MOE_FFN_SIMT, _lib.MOE_FFN_TCGEN05_M128, _lib.MOE_FFN_TCGEN05_M256,
         _lib.MOE_FFN_TCGEN05_PAIR, _lib.MOE_FFN_TCGEN05_WIDE, _lib.MOE_FFN_TCGEN05_SWAP]


def _case(seed: int):
    rng = np.random.default_rng(1000 + seed)
    w_dtype = ["bf16", "e4m3"][seed % 2]
    base = synth.CONFIGS["prefill_bf16" if w_dtype == "bf16" else "prefill_fp8"]
    E_r = int(rng.choice([1, 3, 8, 17, 32, 48]))
    K = int(rng.integers(1, min(8, E_r) + 1))
    cfg = synth.variant(base, T=int(rng.integers(1, 301)), H=int(rng.choice([256, 512, 768, 1024])),
                        I=int(rng.choice([64, 128, 192, 256, 384])), n_routed=E_r, top_k=K,
                        seed=seed, renormalize=bool(rng.integers(0, 4) > 0),
                        shared_weight=float(rng.choice([1.0, 1.0, 0.5])),
                        zipf_s=(1.1 if rng.integers(0, 3) == 0 else None))
    cfg = synth.variant(cfg, routed_scale=float(rng.choice([1.0, 1.0, 2.5])),
                        bias_select_only=bool(cfg.zipf_s is not None and rng.integers(0, 2)))
    impl = IMPLS[int(rng.integers(0, len(IMPLS)))]
    fuse = bool(rng.integers(0, 4) > 0)
    return cfg, impl, fuse


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


@pytest.mark.parametrize("seed", range(24))
def test_random_layer_matches_oracle(seed):
    cfg, impl, fuse = _case(seed)
    inp = synth.make_inputs(cfg)
    d = synth.to_device(inp, DEV)
    layer = MoELayer(cfg, d, fuse_shared=fuse, impl=impl)
    out = layer.forward(d["x"])
    assert layer.status() == _lib.MOE_OK, (cfg, impl, fuse)
    # routing of every token, bit for bit
    s = _lib.make_shape(cfg)
    ids = torch.empty(cfg.T, cfg.slots, dtype=torch.int32, device=DEV)
    w = torch.empty(cfg.T, cfg.slots, dtype=torch.float32, device=DEV)
    ws = _lib.alloc_workspace(s, True)      # the routing entry point takes the fused layout
    _lib.moe_route_topk(s, d["x"], d["router_w"], d["router_bias"], ids, w, None, ws)
    torch.cuda.synchronize()
    rid, _ = oracle.topk(oracle_logits(d["x"], d["router_w"], d["router_bias"]), cfg.top_k, cfg.renormalize,
                         cfg.shared_id, cfg.shared_weight)
    assert np.array_equal(ids.cpu().numpy(), rid), (cfg, impl)
    # every output
    ref = oracle.Layer(cfg, inp).forward()
    assert rel_err(to_f64(out), ref["out"]) <= tol_of(cfg), (cfg, impl, fuse)
