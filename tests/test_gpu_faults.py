"""Failure detection on the GPU without a GPU fault: a tensor-core GEMM whose
producer never issues its loads runs its bounded waits out, returns, frees its
tensor memory and leaves MOE_ERR_TIMEOUT in the status word; the context stays
usable and the next call is correct."""
import numpy as np
import pytest
import torch

import oracle
from shared_routed_expert_b200 import MoELayer, _lib, build, synth
from tests.parity_util import rel_err, to_f64, tol_of

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("impl,I", [(_lib.MOE_FFN_AUTO, 128), (_lib.MOE_FFN_TCGEN05_PAIR, 128),
                                    (_lib.MOE_FFN_TCGEN05_WIDE, 128), (_lib.MOE_FFN_TCGEN05_SWAP, 256)],
                         ids=["auto", "cta_pair", "cta_pair_wide", "cta_pair_swap"])
def test_wait_timeout_is_reported_and_the_context_survives(impl, I):
    build.build()
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=64, H=512, I=I, n_routed=8, top_k=2)
    inp = synth.make_inputs(cfg)
    d = synth.to_device(inp, "cuda")
    layer = MoELayer(cfg, d, impl=impl)
    _lib.moe_inject_wait_timeout(1)
    layer.forward(d["x"])
    assert layer.status() == _lib.MOE_ERR_TIMEOUT
    # the status word was cleared by the read; the next pass is clean and right
    out = layer.forward(d["x"])
    assert layer.status() == _lib.MOE_OK
    ref = oracle.Layer(cfg, inp).forward()["out"]
    assert rel_err(to_f64(out), ref) <= tol_of(cfg)
    torch.cuda.synchronize()


@pytest.mark.parametrize("impl,T", [(_lib.MOE_FFN_AUTO, 64), (_lib.MOE_FFN_AUTO, 1100),
                                    (_lib.MOE_FFN_TCGEN05_PAIR, 64)],
                         ids=["single_cta", "cta_pair_wide", "cta_pair"])
def test_folded_combine_wait_timeout_is_reported(impl, T):
    """The shared expert's down-projection units wait for the routed units of
    their columns before aggregating; with one arrival too many expected the
    wait runs out (~10 ms), the kernel drains and returns MOE_ERR_TIMEOUT, and
    the next pass is clean and right."""
    build.build()
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=T, H=1024, I=256, n_routed=8, top_k=4)
    inp = synth.make_inputs(cfg)
    d = synth.to_device(inp, "cuda")
    layer = MoELayer(cfg, d, impl=impl | _lib.MOE_FFN_COMBINE_FOLD)
    _lib.moe_inject_fold_timeout(1)
    layer.forward(d["x"])
    assert layer.status() == _lib.MOE_ERR_TIMEOUT
    out = layer.forward(d["x"])
    assert layer.status() == _lib.MOE_OK
    ref = oracle.Layer(cfg, inp).forward()["out"]
    assert rel_err(to_f64(out), ref) <= tol_of(cfg)
    torch.cuda.synchronize()


def test_routing_wait_timeout_is_reported():
    """Routing through approximate tensor-core logits (batches over 256 tokens):
    when its GEMM's producer issues no loads, the waits run out (~10 ms), the
    kernel drains and returns MOE_ERR_TIMEOUT, every id stays in range (the
    layer still runs), and the next pass is clean and right."""
    build.build()
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=300, H=512, I=128, n_routed=40, top_k=6)
    inp = synth.make_inputs(cfg)
    d = synth.to_device(inp, "cuda")
    layer = MoELayer(cfg, d)
    _lib.moe_inject_route_timeout(1)
    layer.forward(d["x"])
    assert layer.status() == _lib.MOE_ERR_TIMEOUT
    out = layer.forward(d["x"])
    assert layer.status() == _lib.MOE_OK
    ref = oracle.Layer(cfg, inp).forward()["out"]
    assert rel_err(to_f64(out), ref) <= tol_of(cfg)
    torch.cuda.synchronize()
