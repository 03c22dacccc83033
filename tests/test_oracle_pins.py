"""Pins of the CPU oracle to things other than itself.

Each test fixes a value from the pages, a closed form, a library routine or a
brute-force enumeration, chosen so that a plausible slip in the oracle (a
dropped term, a swapped operand, a wrong index or sign, a missing rounding)
fails at least one of them. No GPU is used.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from shared_routed_expert_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ E4M3 codec

def test_e4m3_decode_matches_torch_for_all_256_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert nan.sum() == 2                          # 0x7F and 0xFF only
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9    # largest, smallest subnormal


def test_e4m3_encode_matches_torch_on_every_bf16_value_in_range():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals)]
    for scale in (1.0, 1.0 / 3.0, 97.25):
        v = (vals * np.float32(scale)).astype(np.float32)
        ok = np.isfinite(v) & (np.abs(v) <= 448.0)
        v = v[ok]
        ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = oracle.e4m3_encode(v)
        assert np.array_equal(got, ref), scale


def test_e4m3_encode_ties_and_saturation():
    # midway between 1.0 (0x38) and 1.125 (0x39): ties go to the even code
    assert oracle.e4m3_encode([1.0625])[0] == 0x38
    # midway between 1.125 and 1.25 (0x3A): even code is 0x3A
    assert oracle.e4m3_encode([1.1875])[0] == 0x3A
    # above the largest finite value: saturate (not NaN)
    assert list(oracle.e4m3_encode([449.0, 1e6, -1e30])) == [0x7E, 0x7E, 0xFE]
    # half of the smallest subnormal rounds to (signed) zero; just above rounds up
    assert list(oracle.e4m3_encode([2.0 ** -10, -2.0 ** -10, 2.0 ** -10 * 1.01])) == [0x00, 0x80, 0x01]
    assert oracle.e4m3_encode([float("nan")])[0] == 0x7F


def test_e4m3_quant_row_closed_form():
    v = np.array([[1.0, -2.0, 0.5, 4.0], [0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    codes, scales = oracle.quant_rows_e4m3(v)
    assert scales[0] == np.float32(4.0) / np.float32(448.0)
    assert scales[1] == 1.0
    dec = oracle.e4m3_decode(codes[0])
    assert list(dec) == [112.0, -224.0, 56.0, 448.0]
    assert list(codes[1]) == [0, 0, 0, 0]


# ------------------------------------------------------------------ bf16 rounding

def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 32, size=20000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_bf16(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_round_bf16_rounds_doubles_once():
    # 1 + 2^-8 + 2^-30 lies just above the midpoint of 1 and 1 + 2^-7. Rounding
    # through fp32 first would land on the midpoint and tie down to 1.0.
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle.bf16_bits_to_f64(oracle.round_bf16([v]))[0] == 1.0 + 2.0 ** -7
    assert oracle.bf16_bits_to_f64(oracle.round_bf16([1.0 + 2.0 ** -8]))[0] == 1.0


# ------------------------------------------------------------------ router logits

def test_router_logits_exact_on_integer_inputs():
    rng = np.random.default_rng(1)
    x = rng.integers(-8, 9, size=(5, 512)).astype(np.float32)
    w = rng.integers(-8, 9, size=(7, 512)).astype(np.float32)
    b = rng.integers(-3, 4, size=7).astype(np.float32)
    L = oracle.router_logits(x, w, b)
    ref = x.astype(np.int64) @ w.astype(np.int64).T + b.astype(np.int64)
    assert np.array_equal(L.astype(np.int64), ref)


def test_router_logits_follow_the_segmented_fma_order():
    # Two 256-wide segments. Segment sums are formed first, then added, so the
    # +1 survives: seg0 = 2^24, seg1 = 1 - 2^24 (exact), total = 1. A single
    # running chain over all of H would absorb the +1 into 2^24 and give 0.
    x = np.zeros((1, 512), dtype=np.float32)
    w = np.zeros((1, 512), dtype=np.float32)
    x[0, 0], w[0, 0] = 1.0, 2.0 ** 24
    x[0, 256], w[0, 256] = 1.0, 1.0
    x[0, 257], w[0, 257] = 1.0, -(2.0 ** 24)
    assert oracle.router_logits(x, w)[0, 0] == 1.0
    # The same three terms inside one segment (h = 0, 128, 129) share one chain:
    # 2^24 + 1 ties back to 2^24 and the -2^24 cancels it, giving 0. A segment
    # shorter than 256 would split them and give 1.
    x[:] = 0.0
    w[:] = 0.0
    x[0, 0], w[0, 0] = 1.0, 2.0 ** 24
    x[0, 128], w[0, 128] = 1.0, 1.0
    x[0, 129], w[0, 129] = 1.0, -(2.0 ** 24)
    assert oracle.router_logits(x, w)[0, 0] == 0.0


def test_router_logits_use_fused_multiply_add():
    # (1 + 2^-7)(1 + 2^-17) = 1 + 2^-7 + 2^-17 + 2^-24: the last term is half an
    # fp32 ulp, so a separately rounded product would lose it and cancel to 0.
    x = np.zeros((1, 256), dtype=np.float32)
    w = np.zeros((1, 256), dtype=np.float32)
    x[0, 0], w[0, 0] = 1.0, -(1.0 + 2.0 ** -7 + 2.0 ** -17)
    x[0, 1], w[0, 1] = 1.0 + 2.0 ** -7, 1.0 + 2.0 ** -17
    assert oracle.router_logits(x, w)[0, 0] == np.float32(2.0 ** -24)


def test_router_logits_close_to_fp64_within_bound():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 1024)).astype(np.float32)
    w = (0.02 * rng.standard_normal((9, 1024))).astype(np.float32)
    L = oracle.router_logits(x, w).astype(np.float64)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    bound = (np.abs(x).astype(np.float64) @ np.abs(w).astype(np.float64).T) * (256 + 4) * 2.0 ** -24
    assert np.all(np.abs(L - exact) <= bound)


# ------------------------------------------------------------------ top-K

def _brute_topk(l, K):
    """Max-sum K-subset, lexicographically smallest ids among ties; slots then
    ordered by (logit desc, id asc)."""
    best, best_sum = None, None
    for sub in itertools.combinations(range(len(l)), K):
        s = sum(float(l[e]) for e in sub)
        if best_sum is None or s > best_sum:
            best, best_sum = sub, s
    return sorted(best, key=lambda e: (-float(l[e]), e))


@pytest.mark.parametrize("E,K", [(8, 2), (8, 3), (6, 6), (9, 1)])
def test_topk_matches_subset_enumeration_with_ties(E, K):
    rng = np.random.default_rng(E * 10 + K)
    L = rng.integers(-3, 4, size=(40, E)).astype(np.float32)   # many exact ties
    ids, _ = oracle.topk(L, K)
    for t in range(L.shape[0]):
        assert list(ids[t]) == _brute_topk(L[t], K)


def test_topk_zero_router_gives_lowest_ids_and_uniform_weights():
    ids, w = oracle.topk(np.zeros((3, 160), np.float32), 8, shared_id=160)
    assert np.array_equal(ids, np.tile(np.r_[np.arange(8), 160], (3, 1)))
    assert np.allclose(w[:, :8], 1.0 / 8, rtol=0, atol=1e-15)
    assert np.all(w[:, 8] == 1.0)


def test_topk_softmax_closed_forms():
    L = np.array([[0.0, math.log(3.0), -5.0, -7.0]], np.float32)
    ids, w = oracle.topk(L, 2)
    assert list(ids[0]) == [1, 0]
    assert abs(w[0, 0] - 0.75) < 1e-7 and abs(w[0, 1] - 0.25) < 1e-7
    # without renormalisation: the full softmax evaluated at the selected ids
    ids, w = oracle.topk(np.zeros((1, 4), np.float32), 2, renormalize=False)
    assert np.allclose(w, 0.25, rtol=0, atol=1e-15)


def test_topk_nan_ranks_last():
    L = np.array([[np.nan, 1.0, np.nan, 0.5]], np.float32)
    ids, _ = oracle.topk(L, 3)
    assert list(ids[0]) == [1, 3, 0]


# ------------------------------------------------------------------ permute

def test_permute_equals_stable_argsort_and_inverts():
    rng = np.random.default_rng(3)
    T, K, E = 37, 3, 6
    ids = np.concatenate([rng.integers(0, E - 1, size=(T, K)), np.full((T, 1), E - 1)], 1).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    flat = ids.ravel()
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert np.array_equal(offsets, np.r_[0, np.cumsum(counts)])
    assert np.array_equal(inv[perm], np.arange(flat.size))
    # the shared block (last expert) is every token, in token order
    assert np.array_equal(perm[offsets[E - 1]:] // (K + 1), np.arange(T))


def test_permute_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 5]], np.int32), 5)


# ------------------------------------------------------------------ expert FFN

def _layer(cfg, inputs):
    return oracle.Layer(cfg, inputs)


def _np_swiglu(w13, w2, v):
    I = w13.shape[0] // 2
    g = w13[:I] @ v
    u = w13[I:] @ v
    return w2 @ ((g / (1.0 + np.exp(-g))) * u)


def test_expert_ffn_matches_numpy_matmul_fp32_layer():
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg)
    L = _layer(cfg, inp)
    x = inp["x"].double().numpy()
    for e in (0, 5, cfg.shared_id):
        y = L.expert_ffn(e, inp["x"][3].numpy())
        ref = _np_swiglu(inp["w13"][e].double().numpy(), inp["w2"][e].double().numpy(), x[3])
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_expert_ffn_gate_up_order_closed_form():
    # x = e_0; gate row 0 sees 2, up row 0 sees 3; w2 = identity on row 0.
    # silu(2) = 2 * sigmoid(2) = 1 + tanh(1); swapping gate and up would give
    # silu(3) * 2 instead.
    cfg = synth.variant(synth.CONFIGS["tiny_fp32"], T=1, H=256, I=8, n_routed=1, top_k=1)
    inp = synth.make_inputs(cfg)
    inp["w13"].zero_()
    inp["w2"].zero_()
    inp["w13"][0, 0, 0] = 2.0
    inp["w13"][0, cfg.I + 0, 0] = 3.0
    inp["w2"][0, 0, 0] = 1.0
    L = _layer(cfg, inp)
    v = np.zeros(cfg.H, np.float32)
    v[0] = 1.0
    y = L.expert_ffn(0, v)
    assert abs(y[0] - 3.0 * (1.0 + math.tanh(1.0))) < 1e-14
    assert np.all(y[1:] == 0.0)


def test_expert_ffn_bf16_rounds_h_before_the_down_projection():
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=1, H=256, I=8, n_routed=1, top_k=1)
    inp = synth.make_inputs(cfg)
    inp["w13"].zero_()
    inp["w2"].zero_()
    # g = 64.5 and u = 1 + 2^-7 are bf16 values; silu(64.5) == 64.5 in fp64.
    # h = g * u = 65.00390625 needs 14 mantissa bits; bf16 spacing at 64 is 0.5,
    # so the stored h is 65.0.
    inp["w13"][0, 0, 0] = 64.5
    inp["w13"][0, cfg.I, 0] = 1.0 + 2.0 ** -7
    inp["w2"][0, 0, 0] = 1.0
    L = _layer(cfg, inp)
    v = np.zeros(cfg.H, np.float32)
    v[0] = 1.0
    h_exact = 64.5 * (1.0 + 2.0 ** -7)
    h_bf16 = 65.0
    assert h_exact == 65.00390625
    y = L.expert_ffn(0, v)
    assert y[0] == h_bf16


def test_expert_ffn_e4m3_closed_form():
    # x = 448 e_0 -> scale 1, codes exact. Gate/up codes 1.0 and 0.5 with
    # channel scales 1: g = 448, u = 224, silu(448) = 448 in fp64, h = 100352
    # (a bf16 value). h's row scale 100352/448 = 224 makes its code 448 -> the
    # down projection sees 100352 exactly; w2 code 0.25 with scale 2 -> y = 50176.
    cfg = synth.variant(synth.CONFIGS["prefill_fp8"], T=1, H=256, I=8, n_routed=1, top_k=1)
    inp = synth.make_inputs(cfg)
    enc = lambda v: int(torch.tensor([v]).to(torch.float8_e4m3fn).view(torch.uint8)[0])
    inp["w13"].zero_()
    inp["w2"].zero_()
    inp["s13"].fill_(1.0)
    inp["s2"].fill_(2.0)
    inp["w13"][0, 0, 0] = enc(1.0)
    inp["w13"][0, cfg.I, 0] = enc(0.5)
    inp["w2"][0, 5, 0] = enc(0.25)
    L = _layer(cfg, inp)
    v = np.zeros(cfg.H, np.float32)
    v[0] = 448.0
    y = L.expert_ffn(0, v)
    assert y[5] == 50176.0
    assert np.count_nonzero(y) == 1


# ------------------------------------------------------------------ layer

def _dense_bruteforce(cfg, inp):
    """Every expert on every token (numpy fp64 matmuls), top-K by subset
    enumeration, softmax over the chosen logits, plus the shared expert."""
    x = inp["x"].double().numpy()
    L = oracle.router_logits(inp["x"].float().numpy(), inp["router_w"].numpy(),
                             None if inp["router_bias"] is None else inp["router_bias"].numpy())
    Y = np.stack([np.stack([_np_swiglu(inp["w13"][e].double().numpy(), inp["w2"][e].double().numpy(), x[t])
                            for t in range(cfg.T)]) for e in range(cfg.n_experts)])   # [E, T, H]
    out = np.zeros((cfg.T, cfg.H))
    for t in range(cfg.T):
        sel = _brute_topk(L[t], cfg.top_k)
        z = np.array([float(L[t, e]) for e in sel])
        p = np.exp(z - z.max())
        p /= p.sum()
        out[t] = sum(p[k] * Y[sel[k], t] for k in range(cfg.top_k)) + cfg.shared_weight * Y[cfg.shared_id, t]
    return out


def test_forward_matches_dense_bruteforce_tiny():
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg)
    res = oracle.Layer(cfg, inp).forward(fuse_shared=True, n_threads=2)
    ref = _dense_bruteforce(cfg, inp)
    assert np.allclose(res["out"], ref, rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("cfg", [synth.CONFIGS["tiny_fp32"],
                                 synth.variant(synth.CONFIGS["prefill_bf16"], T=6, H=256, I=64,
                                               n_routed=12, top_k=3),
                                 synth.variant(synth.CONFIGS["skewed_fp8"], T=6, H=256, I=64,
                                               n_routed=12, top_k=3)],
                         ids=["f32", "bf16", "e4m3"])
def test_fused_equals_unfused_exactly(cfg):
    """The fusion only re-partitions the work: shared(x) + sum of the routed
    top-K (the unfused pseudocode) equals the top-(K+1) pass bit for bit."""
    inp = synth.make_inputs(cfg)
    Ly = oracle.Layer(cfg, inp)
    a = Ly.forward(fuse_shared=True, n_threads=3)
    b = Ly.forward(fuse_shared=False, n_threads=1)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["ids"][:, :cfg.top_k], b["ids"])
    # the zh page's own acceptance check (allclose with atol 1e-5) holds a fortiori
    assert np.allclose(a["out"], b["out"], atol=1e-5)


def test_identical_experts_give_twice_one_expert():
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg)
    inp["w13"][:] = inp["w13"][0].clone()
    inp["w2"][:] = inp["w2"][0].clone()
    Ly = oracle.Layer(cfg, inp)
    res = Ly.forward(n_threads=2)
    for t in range(cfg.T):
        y = Ly.expert_ffn(0, inp["x"][t].numpy())
        assert np.allclose(res["out"][t], 2.0 * y, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("s", [2.5, 0.25])
def test_identical_experts_with_routed_scale(s):
    """Identical experts and a routed scaling factor s: the routed weights sum
    to s and the shared slot keeps weight 1, so out = (s + 1) * FFN(x)."""
    cfg = synth.variant(synth.CONFIGS["tiny_fp32"], routed_scale=s)
    inp = synth.make_inputs(cfg)
    inp["w13"][:] = inp["w13"][0].clone()
    inp["w2"][:] = inp["w2"][0].clone()
    Ly = oracle.Layer(cfg, inp)
    res = Ly.forward(n_threads=2)
    for t in range(cfg.T):
        y = Ly.expert_ffn(0, inp["x"][t].numpy())
        assert np.allclose(res["out"][t], (s + 1.0) * y, rtol=1e-12, atol=1e-15)


def test_routed_scale_equals_scaling_the_fused_sum_with_shared_weight_one_over_s():
    """An engine that scales the whole fused sum by s must give the shared slot
    1/s; scaling the routed slots by s instead yields the same output (s = 4:
    1/s is exact in fp32, so the two differ only by fp64 rounding)."""
    s = 4.0
    base = synth.variant(synth.CONFIGS["prefill_bf16"], T=12, H=256, I=64, n_routed=8, top_k=3)
    inp = synth.make_inputs(base)
    a = oracle.Layer(synth.variant(base, routed_scale=s), inp).forward(n_threads=2)
    b = oracle.Layer(synth.variant(base, shared_weight=1.0 / s), inp).forward(n_threads=2)
    assert np.array_equal(a["ids"], b["ids"])
    assert np.allclose(a["out"], s * b["out"], rtol=1e-12, atol=1e-12)


def test_bias_for_selection_only_weighs_with_the_unbiased_logits():
    """A bias that forces experts 3 and 5 into a top-2: they are selected in
    either mode, but with bias_select_only the weights are the softmax of their
    unbiased logits (numpy, fp64), otherwise of the biased ones."""
    base = synth.variant(synth.CONFIGS["prefill_bf16"], T=10, H=256, I=64, n_routed=8, top_k=2)
    inp = synth.make_inputs(base)
    bias = torch.zeros(8)
    bias[3], bias[5] = 40.0, 39.0
    inp["router_bias"] = bias
    x = inp["x"].float().numpy()
    raw = oracle.router_logits_f64(x, inp["router_w"].numpy())[:, [3, 5]]
    for sel_only in (True, False):
        cfg = synth.variant(base, bias_select_only=sel_only)
        r = oracle.Layer(cfg, inp).forward(n_threads=2)
        assert np.array_equal(r["ids"][:, :2], np.tile([3, 5], (10, 1)))
        z = raw if sel_only else raw + np.array([40.0, 39.0])
        ref = np.exp(z - z.max(1, keepdims=True))
        ref /= ref.sum(1, keepdims=True)
        assert np.allclose(r["w"][:, :2], ref, rtol=0, atol=1e-6)
        assert np.all(r["w"][:, 2] == 1.0)


def test_bias_for_selection_only_without_bias_changes_nothing():
    base = synth.variant(synth.CONFIGS["skewed_fp8"], T=16, H=256, I=64, n_routed=12, top_k=3)
    inp = synth.make_inputs(base)
    inp["router_bias"] = torch.zeros(12)
    a = oracle.Layer(base, inp).forward(n_threads=2)
    b = oracle.Layer(synth.variant(base, bias_select_only=True), inp).forward(n_threads=2)
    assert np.array_equal(a["ids"], b["ids"]) and np.array_equal(a["out"], b["out"])


def test_single_routed_expert_is_two_dense_mlps():
    cfg = synth.variant(synth.CONFIGS["tiny_fp32"], n_routed=1, top_k=1)
    inp = synth.make_inputs(cfg)
    res = oracle.Layer(cfg, inp).forward(n_threads=1)
    x = inp["x"].double().numpy()
    for t in range(cfg.T):
        ref = sum(_np_swiglu(inp["w13"][e].double().numpy(), inp["w2"][e].double().numpy(), x[t])
                  for e in (0, 1))
        assert np.allclose(res["out"][t], ref, rtol=1e-12, atol=1e-15)
    assert np.all(res["w"][:, 0] == 1.0)


def test_glm47_structure_from_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "glm47_shared_fusion.json")))
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=24, H=256, I=32,
                        n_routed=g["n_routed"], top_k=g["top_k_routed"])
    assert cfg.n_experts == g["n_experts_fused"] and cfg.slots == g["top_k_fused"]
    assert cfg.shared_id == g["shared_expert_index"] == g["shared_expert_number_one_based"] - 1
    inp = synth.make_inputs(cfg)
    res = oracle.Layer(cfg, inp).forward(n_threads=4)
    ids = res["ids"]
    assert ids.shape[1] == g["top_k_fused"]
    assert np.all(ids[:, g["shared_slot_index"]] == g["shared_expert_index"])
    assert np.all(ids[:, :g["top_k_routed"]] < g["n_routed"])
    assert all(len(set(r)) == g["top_k_fused"] for r in ids.tolist())
    counts, offsets, perm, _ = oracle.permute(ids, cfg.n_experts)
    assert counts[g["shared_expert_index"]] == cfg.T
    assert synth.CONFIGS["skewed_fp8"].I == g["tp8_fp8_intermediate"]


def test_combine_hand_example():
    # two tokens, two slots, three rows per expert output
    Y = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0], [0.5, -0.5]], np.float32)
    inv = np.array([2, 0, 1, 3], np.int32)          # t0 -> rows 2, 0 ; t1 -> rows 1, 3
    w = np.array([[0.25, 0.75], [1.0, 2.0]])
    out = oracle.combine(Y, inv, w, "f32")
    assert np.array_equal(out, [[25.75, 51.5], [11.0, 19.0]])


def test_weights_sum_to_one_and_ids_distinct_on_a_glm_shape():
    cfg = synth.variant(synth.CONFIGS["skewed_fp8"], T=64, H=512, I=64)
    inp = synth.make_inputs(cfg)
    L = oracle.router_logits(inp["x"].float().numpy(), inp["router_w"].numpy(),
                             inp["router_bias"].numpy())
    ids, w = oracle.topk(L, cfg.top_k, shared_id=cfg.shared_id)
    assert np.allclose(w[:, :cfg.top_k].sum(1), 1.0, atol=1e-12)
    assert all(len(set(r)) == cfg.slots for r in ids.tolist())
    # the Zipf prior pulls routing toward low expert ids
    counts = np.bincount(ids[:, :cfg.top_k].ravel(), minlength=cfg.n_routed)
    assert counts[:16].sum() > counts[-16:].sum()


# ------------------------------------------------------------------ QK-norm + partial RoPE

def _attn(cfg):
    inp = synth.make_attn_inputs(cfg)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)     # noqa: E731
    out = oracle.qk_norm_rope(bits(inp["qkv"]), inp["pos"].numpy(), bits(inp["q_w"]), bits(inp["k_w"]),
                              inp["cos_sin"].numpy(), cfg.n_q, cfg.n_kv, cfg.d, cfg.rot, cfg.eps)
    return inp, out


def test_qk_norm_matches_torch_rms_norm_and_rope_matches_complex_rotation():
    """Norm: torch's rms_norm (fp64, eps as the fp32 value the call takes).
    Rotation: the pair (u_i, u_{i+rot/2}) as the complex number u_i + i u_{i+rot/2}
    times exp(i angle), angle read back from the table with atan2; dimensions
    past rot unchanged."""
    cfg = synth.ATTN_CONFIGS["qknorm_tiny"]
    inp, out = _attn(cfg)
    half = cfg.rot // 2
    heads = inp["qkv"].double().reshape(cfg.T, cfg.n_q + 2 * cfg.n_kv, cfg.d)
    for t in range(cfg.T):
        cs = inp["cos_sin"][inp["pos"][t]].double().numpy()
        ang = np.arctan2(cs[half:], cs[:half])
        rad = np.hypot(cs[half:], cs[:half])          # 1 up to fp32 rounding of the table
        for h in range(cfg.n_q + cfg.n_kv):
            w = (inp["q_w"] if h < cfg.n_q else inp["k_w"]).double()
            u = torch.nn.functional.rms_norm(heads[t, h], (cfg.d,), w, float(np.float32(cfg.eps))).numpy()
            z = (u[:half] + 1j * u[half:cfg.rot]) * rad * np.exp(1j * ang)
            ref = np.concatenate([z.real, z.imag, u[cfg.rot:]])
            assert np.allclose(out[t, h], ref, rtol=1e-12, atol=1e-12)


def test_rope_dot_products_depend_only_on_the_position_difference():
    """The defining property of rotary embeddings: over the rotated dimensions
    <q at m, k at n> = <q at m + s, k at n + s> (unit norm weights, fp32 table)."""
    base = synth.ATTN_CONFIGS["qknorm_tiny"]
    cfg = synth.replace(base, T=2, max_pos=64)
    inp = synth.make_attn_inputs(cfg)
    inp["q_w"][:] = 1.0
    inp["k_w"][:] = 1.0
    qkv = inp["qkv"].clone()
    qkv[1] = qkv[0]                     # the same token content at two positions
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)     # noqa: E731
    dots = []
    for m, n in [(3, 10), (20, 27), (50, 57)]:
        pos = np.array([m, n], np.int32)
        o = oracle.qk_norm_rope(bits(qkv), pos, bits(inp["q_w"]), bits(inp["k_w"]),
                                inp["cos_sin"].numpy(), cfg.n_q, cfg.n_kv, cfg.d, cfg.rot, cfg.eps)
        q, k = o[0, 0, :cfg.rot], o[1, cfg.n_q, :cfg.rot]
        dots.append(float(q @ k))
    assert np.allclose(dots, dots[0], rtol=1e-5, atol=1e-6)


def test_qk_norm_is_scale_invariant_and_position_zero_is_the_identity_rotation():
    cfg = synth.ATTN_CONFIGS["qknorm_tiny"]
    inp = synth.make_attn_inputs(cfg)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)     # noqa: E731
    args = (bits(inp["q_w"]), bits(inp["k_w"]), inp["cos_sin"].numpy(), cfg.n_q, cfg.n_kv, cfg.d, cfg.rot, 0.0)
    pos0 = np.zeros(cfg.T, np.int32)
    a = oracle.qk_norm_rope(bits(inp["qkv"]), pos0, *args)
    b = oracle.qk_norm_rope(bits((inp["qkv"].float() * 4.0).to(torch.bfloat16)), pos0, *args)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-13)       # x4 is exact in bf16; eps = 0
    # position 0: cos 1, sin 0, so every output is the normalised value
    heads = inp["qkv"].double().reshape(cfg.T, -1, cfg.d)[:, :cfg.n_q + cfg.n_kv]
    rms = torch.sqrt((heads ** 2).mean(-1, keepdim=True))
    w = torch.cat([inp["q_w"].double().expand(cfg.n_q, -1), inp["k_w"].double().expand(cfg.n_kv, -1)])
    assert np.allclose(a, (heads / rms * w).numpy(), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ tensor-parallel slices

@pytest.mark.parametrize("world", [2, 4])
def test_intermediate_slices_sum_to_the_layer(world):
    """The SwiGLU is per intermediate column, so the layers of the N slices of
    every expert's intermediate dimension (router replicated) sum to the full
    layer (bf16: h is rounded per element either way; fp64 sums)."""
    from shared_routed_expert_b200 import tp
    cfg = synth.variant(synth.CONFIGS["prefill_bf16"], T=10, H=256, I=256, n_routed=8, top_k=3)
    inp = synth.make_inputs(cfg)
    full = oracle.Layer(cfg, inp).forward(n_threads=2)["out"]
    parts = [oracle.Layer(tp.local_config(cfg, world), tp.shard_weights(inp, cfg.I, r, world))
             .forward(n_threads=2)["out"] for r in range(world)]
    assert np.allclose(sum(parts), full, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ E4M3 exactness case

def _e4m3_codes(values: torch.Tensor) -> torch.Tensor:
    """Codes of values that lie on the E4M3 grid (checked by the round trip)."""
    c = values.float().to(torch.float8_e4m3fn)
    assert torch.equal(c.float(), values.float()), "value off the E4M3 grid"
    return c.view(torch.uint8)


def test_e4m3_layer_equals_bf16_layer_when_every_quantisation_is_lossless():
    """Weights on the E4M3 grid with power-of-two channel scales, tokens whose
    amax / 448 is a power of two, and an FFN whose h rows are +-amax * 2^-p: then
    every quantisation the E4M3 layer performs (x per token, h per row) is exact,
    and the layer must equal the bf16-weight layer on the dequantised weights bit
    for bit. Gate rows read x_0 = 56 only (silu(56) = 56 in fp64), up rows read
    x_1 only, so h_j = 56 * x_1 * d_j."""
    T, H, I, E_r = 4, 256, 64, 2
    f8 = synth.variant(synth.CONFIGS["prefill_fp8"], T=T, H=H, I=I, n_routed=E_r, top_k=1)
    b16 = synth.variant(synth.CONFIGS["prefill_bf16"], T=T, H=H, I=I, n_routed=E_r, top_k=1)
    E = f8.n_experts
    g = torch.Generator().manual_seed(11)
    grid = torch.tensor([0.0, 0.25, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])     # E4M3 values
    # x: x_0 = 56 = 448 * 2^-3 is each token's amax, so its scale is 2^-3
    x = grid[torch.randint(0, len(grid), (T, H), generator=g)] * 0.125
    x = x * torch.where(torch.rand(T, H, generator=g) < 0.5, -1.0, 1.0)
    x[:, 0] = 56.0
    x[:, 1] = torch.tensor([0.5, 1.0, 2.0, 0.25])
    x[:, 2] = torch.tensor([0.125, 0.125, -0.125, -0.125])   # routes tokens 0, 1 -> 0 and 2, 3 -> 1
    router_w = torch.zeros(E_r, H)
    router_w[0, 2], router_w[1, 2] = 1.0, -1.0
    # weights as E4M3 values times power-of-two channel scales
    w13 = torch.zeros(E, 2 * I, H)
    s13 = torch.zeros(E, 2 * I)
    w2 = grid[torch.randint(0, len(grid), (E, H, I), generator=g)] * 0.5
    w2 = w2 * torch.where(torch.rand(E, H, I, generator=g) < 0.5, -1.0, 1.0)
    s2 = torch.pow(2.0, torch.randint(-9, -5, (E, H), generator=g).float())
    for e in range(E):
        w13[e, :I, 0] = 256.0                          # gate_j = 256 * 2^-8 * x_0 = 56
        s13[e, :I] = 2.0 ** -8
        p = torch.randint(0, 6, (I,), generator=g)     # d_j = +-2^-p, max |d| = 1
        p[0] = 0
        sign = torch.where(torch.rand(I, generator=g) < 0.5, -1.0, 1.0)
        w13[e, I:, 1] = sign * torch.pow(2.0, -p.float()) * 64.0
        s13[e, I:] = 2.0 ** -6
    inp8 = synth.make_inputs(f8)
    inp8.update(x=x.to(torch.bfloat16), router_w=router_w, w13=_e4m3_codes(w13), s13=s13,
                w2=_e4m3_codes(w2), s2=s2)
    inp16 = synth.make_inputs(b16)
    deq13 = w13 * s13[:, :, None]
    deq2 = w2 * s2[:, :, None]
    assert torch.equal(deq13.to(torch.bfloat16).float(), deq13) and torch.equal(deq2.to(torch.bfloat16).float(), deq2)
    inp16.update(x=x.to(torch.bfloat16), router_w=inp8["router_w"], router_bias=inp8["router_bias"],
                 w13=deq13.to(torch.bfloat16), w2=deq2.to(torch.bfloat16))
    r8 = oracle.Layer(f8, inp8).forward(n_threads=2)
    r16 = oracle.Layer(b16, inp16).forward(n_threads=2)
    assert np.array_equal(r8["ids"], r16["ids"])
    assert np.any(r8["out"] != 0.0)
    assert np.array_equal(r8["out"], r16["out"])
    assert r8["ids"][:, 0].tolist() == [0, 0, 1, 1]          # both routed experts in use
    # one up-row scale of the shared expert (used by every token) off by 2: not equal
    inp8["s13"] = s13.clone()
    inp8["s13"][E_r, I + 3] *= 2.0
    r8b = oracle.Layer(f8, inp8).forward(n_threads=2)
    assert not np.array_equal(r8b["out"], r16["out"])
