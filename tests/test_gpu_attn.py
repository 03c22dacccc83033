"""The fused QK-norm + partial RoPE kernel against the CPU oracle: every
output of the q and k heads within one bf16 rounding of the oracle's fp64
value, v heads untouched bit for bit, for several head shapes, rotation
widths, the full prefill and decode shapes, and out-of-range positions."""
import numpy as np
import pytest
import torch

import oracle
from shared_routed_expert_b200 import _lib, build, synth
from tests.parity_util import rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2.0 ** -8       # one bf16 rounding of an fp32 result (2^-9) with room for fp32 error

CASES = {
    "tiny": synth.ATTN_CONFIGS["qknorm_tiny"],
    "mid_d128": synth.AttnConfig("mid_d128", T=300, n_q=12, n_kv=4, d=128, rot=64, max_pos=1024, seed=21,
                                 sequential=False),
    "d64_rot32": synth.AttnConfig("d64_rot32", T=77, n_q=6, n_kv=2, d=64, rot=32, max_pos=100, seed=22),
    "d256_rot128": synth.AttnConfig("d256_rot128", T=33, n_q=4, n_kv=1, d=256, rot=128, max_pos=64, seed=23),
    "norm_only": synth.AttnConfig("norm_only", T=20, n_q=3, n_kv=3, d=128, rot=0, max_pos=32, seed=24),
    "full_rotation": synth.AttnConfig("full_rotation", T=20, n_q=2, n_kv=2, d=128, rot=128, max_pos=32,
                                      seed=25),
    "prefill": synth.ATTN_CONFIGS["qknorm_prefill"],
    "decode": synth.ATTN_CONFIGS["qknorm_decode"],
}


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _run(cfg, inp, bad=None):
    qkv = inp["qkv"].clone()
    _lib.moe_qk_norm_rope(cfg, qkv, inp["pos"], inp["q_w"], inp["k_w"], inp["cos_sin"], bad)
    torch.cuda.synchronize()
    return qkv


@pytest.mark.parametrize("name", list(CASES))
def test_qk_norm_rope_matches_oracle(name):
    cfg = CASES[name]
    inp = synth.make_attn_inputs(cfg, DEV)
    out = _run(cfg, inp)
    ref = oracle.qk_norm_rope(_bits(inp["qkv"]), inp["pos"].cpu().numpy(), _bits(inp["q_w"]), _bits(inp["k_w"]),
                              inp["cos_sin"].cpu().numpy(), cfg.n_q, cfg.n_kv, cfg.d, cfg.rot, cfg.eps)
    heads = out.reshape(cfg.T, cfg.n_q + 2 * cfg.n_kv, cfg.d)
    got = heads[:, :cfg.n_q + cfg.n_kv].double().cpu().numpy()
    # per head: the error relative to that head's scale (heads span 10^-1..10^1)
    for t in range(0, cfg.T, max(1, cfg.T // 64)):
        for h in range(cfg.n_q + cfg.n_kv):
            assert rel_err(got[t, h], ref[t, h]) <= TOL, (t, h)
    # v heads untouched
    v_in = inp["qkv"].reshape(cfg.T, -1, cfg.d)[:, cfg.n_q + cfg.n_kv:]
    assert torch.equal(heads[:, cfg.n_q + cfg.n_kv:].view(torch.int16), v_in.view(torch.int16))


def test_out_of_range_positions_leave_heads_unchanged_and_are_counted():
    cfg = CASES["mid_d128"]
    inp = synth.make_attn_inputs(cfg, DEV)
    inp["pos"][5] = cfg.max_pos          # one past the table
    inp["pos"][9] = -1
    bad = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = _run(cfg, inp, bad)
    assert int(bad.item()) == 2 * (cfg.n_q + cfg.n_kv)
    for t in (5, 9):
        assert torch.equal(out[t].view(torch.int16), inp["qkv"][t].view(torch.int16))
    assert not torch.equal(out[6].view(torch.int16), inp["qkv"][6].view(torch.int16))


def test_rejects_unsupported_head_shapes():
    cfg = synth.AttnConfig("bad", T=4, n_q=2, n_kv=1, d=96, rot=48, max_pos=8, seed=0)
    inp = synth.make_attn_inputs(synth.AttnConfig("ok", T=4, n_q=2, n_kv=1, d=96 + 32, rot=64, max_pos=8,
                                                  seed=0), DEV)
    with pytest.raises(_lib.MoeError):
        _lib.moe_qk_norm_rope(cfg, inp["qkv"], inp["pos"], inp["q_w"], inp["k_w"], inp["cos_sin"])
