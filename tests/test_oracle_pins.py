"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against something fixed independently: the OCP MX
FP4 table (golden fixture), torch's own bf16 / E8M0 decoders, a brute-force
search over expert subsets, a dense re-derivation with numpy float64 matmul and
scipy's sigmoid/softmax, closed forms (zero input, single-expert routing) and
a case worked out by hand.  A dropped term, a wrong sign, a swapped nibble, a
transposed operand or a wrong tie rule in the oracle fails at least one.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from mxfp4_latent_moe_router_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fp4_table():
    tab = {}
    with open(os.path.join(GOLDEN, "ocp_mx_fp4_e2m1.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, val = line.split()
            tab[int(bits, 2)] = float(val)
    assert len(tab) == 16
    return tab


FP4 = _fp4_table()


def _e8m0_torch(s: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(s, dtype=np.uint8).copy()).view(torch.float8_e8m0fnu)
    return t.to(torch.float64).numpy()


def _bf16_torch(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16).copy()).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def _dequant_independent(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP4 dequantisation from the golden table and torch's E8M0 decoder."""
    lut = np.array([FP4[c] for c in range(16)])
    lo = lut[codes & 0xF]
    hi = lut[codes >> 4]
    rows = codes.shape[:-1]
    K = codes.shape[-1] * 2
    vals = np.empty(rows + (K,))
    vals[..., 0::2] = lo
    vals[..., 1::2] = hi
    sc = np.repeat(_e8m0_torch(scales), 32, axis=-1)
    return vals * sc


# --------------------------------------------------------------------------
# element decoders


def test_e2m1_matches_ocp_table():
    for code, val in FP4.items():
        got = oracle.e2m1_value(code)
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), code


def test_e8m0_matches_torch_decoder():
    s = np.arange(256, dtype=np.uint8)
    ref = _e8m0_torch(s)
    got = np.array([oracle.e8m0_value(int(v)) for v in s])
    assert np.isnan(got[255]) and np.isnan(ref[255])
    np.testing.assert_array_equal(got[:255], ref[:255])


def test_bf16_decoder_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = _bf16_torch(bits)
    # every one of the 65536 patterns
    got = np.array([oracle.bf16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert math.copysign(1.0, oracle.bf16_value(0x8000)) == -1.0


def test_dequant_exhaustive_codes_and_scales():
    # every (code, scale) pair: 16 codes x 256 scale bytes, both nibble positions
    codes = np.zeros((256, 16), dtype=np.uint8)
    for c in range(16):
        codes[:, c] = c | (((c + 5) & 15) << 4)
    codes = np.tile(codes, (1, 2))  # K = 64 -> 2 scale blocks
    scales = np.stack([np.arange(256, dtype=np.uint8), np.arange(256, dtype=np.uint8)[::-1]], axis=1)
    got = oracle.dequant_mx(codes, scales)
    ref = _dequant_independent(codes, scales)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_nibble_order_single_element():
    # one nonzero code at (row 3, k 37): low/high nibble and scale block must land there
    rows, K = 8, 64
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.full((rows, K // 32), 127, np.uint8)
    codes[3, 37 // 2] = 0x7 << 4          # k=37 is odd -> high nibble, code 0111 = 6.0
    scales[3, 1] = 127 - 3                # block 1 scale 2^-3
    d = oracle.dequant_mx(codes, scales)
    expect = np.zeros((rows, K))
    expect[3, 37] = 6.0 / 8.0
    np.testing.assert_array_equal(d, expect)


# --------------------------------------------------------------------------
# selection


def _bias_shape(E, k):
    return synth.custom_shape("sel", 1, 32, 32, E, k, 32, 0, synth.SCORE_SIGMOID)


def _route_with_bias(bias, k):
    E = len(bias)
    shape = _bias_shape(E, k)
    w = synth.make_weights(shape)
    w["router_bias"] = np.asarray(bias, np.float32)
    x = np.zeros((1, 32), np.uint16)  # zero logits: keys = sigmoid(0) + bias = 0.5 + bias
    return oracle.route(shape, w, x)


def _brute_force_topk(keys, k):
    best = None
    for sub in itertools.combinations(range(len(keys)), k):
        s = sum(keys[i] for i in sub)
        cand = (-s, sub)  # max sum, then lexicographically smallest index set
        if best is None or cand < best:
            best = cand
    return sorted(best[1])


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_subset_brute_force(seed):
    rng = np.random.default_rng(seed)
    E, k = 9, 3
    # small integer-valued biases -> many exact ties in float32 and float64
    bias = rng.integers(-3, 3, size=E).astype(np.float32) / 8.0
    r = _route_with_bias(bias, k)
    keys = [0.5 + float(b) for b in bias]
    assert sorted(r["ids"][0].tolist()) == _brute_force_topk(keys, k)
    # key-descending order inside the selection, ties by index
    ids = r["ids"][0].tolist()
    assert ids == sorted(ids, key=lambda e: (-keys[e], e))


def test_zero_input_sigmoid_selects_by_bias_with_equal_weights():
    bias = np.array([0.1, -0.2, 0.3, 0.3, 0.0, -0.1], np.float32)
    r = _route_with_bias(bias, 3)
    assert r["ids"][0].tolist() == [2, 3, 0]
    np.testing.assert_allclose(r["weights"][0], [1 / 3] * 3, rtol=0, atol=1e-15)


def test_zero_input_softmax_full_block_is_zero():
    shape = synth.SHAPES["tiny"]
    w = synth.make_weights(shape)
    x = np.zeros((2, shape.hidden), np.uint16)
    r = oracle.forward(shape, w, x)
    assert r["ids"].tolist() == [[0, 1], [0, 1]]     # all logits tie -> lowest indices
    np.testing.assert_array_equal(r["weights"], 0.5)
    assert np.all(r["out"] == 0.0) and np.all(r["z"] == 0.0) and np.all(r["y"] == 0.0)


def test_renormalised_weights_sum_to_one():
    for name in ("tiny",):
        shape = synth.SHAPES[name]
        w = synth.make_weights(shape)
        x = synth.make_x(shape, tokens=16)
        r = oracle.forward(shape, w, x, intermediates=False)
        np.testing.assert_allclose(r["weights"].sum(1), 1.0, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# the whole block, re-derived densely with library routines


def _dense_reference(shape, w, x):
    """Every expert evaluated densely, then masked by a brute-force selection."""
    B = x.shape[0]
    H, L, E, k, I, Is = (shape.hidden, shape.latent, shape.num_experts, shape.top_k,
                         shape.expert_inter, shape.shared_inter)
    xf = _bf16_torch(x).reshape(B, H)
    Wr = _bf16_torch(w["router_w"]).reshape(H, E)
    Win = _bf16_torch(w["w_in"]).reshape(H, L)
    Wout = _bf16_torch(w["w_out"]).reshape(L, H)
    logits = xf @ Wr
    if shape.score_fn == synth.SCORE_SOFTMAX:
        src = scipy.special.softmax(logits, axis=1)
        keys = src
    else:
        src = scipy.special.expit(logits)
        keys = src + (0 if w["router_bias"] is None else w["router_bias"].astype(np.float64))
    z = xf @ Win
    gu = _dequant_independent(w["gu_codes"], w["gu_scales"])   # [E][2I][L]
    dn = _dequant_independent(w["dn_codes"], w["dn_scales"])   # [E][L][I]
    out = np.zeros((B, H))
    sel_all = []
    for b in range(B):
        sel = _brute_force_topk(list(keys[b]), k)
        sel_all.append(sel)
        tot = sum(src[b, e] for e in sel) if shape.renormalize else 1.0
        mask = np.zeros(E)
        for e in sel:
            mask[e] = src[b, e] / tot * shape.routed_scale
        c = np.zeros(L)
        for e in range(E):
            g = gu[e, :I] @ z[b]
            u = gu[e, I:] @ z[b]
            hh = g * scipy.special.expit(g) * u
            c += mask[e] * (dn[e] @ hh)
        out[b] = c @ Wout
        if Is:
            Wg = _bf16_torch(w["sh_gate"]).reshape(H, Is)
            Wu = _bf16_torch(w["sh_up"]).reshape(H, Is)
            Wd = _bf16_torch(w["sh_down"]).reshape(Is, H)
            g = xf[b] @ Wg
            hs = g * scipy.special.expit(g) * (xf[b] @ Wu)
            out[b] += hs @ Wd
    return out, logits, sel_all


@pytest.mark.parametrize("score_fn,k,renorm,scale", [(synth.SCORE_SOFTMAX, 2, 1, 1.0),
                                                     (synth.SCORE_SIGMOID, 3, 1, 1.0),
                                                     (synth.SCORE_SIGMOID, 1, 1, 1.0),
                                                     (synth.SCORE_SIGMOID, 3, 0, 2.5),
                                                     (synth.SCORE_SOFTMAX, 2, 0, 0.5)])
def test_block_matches_dense_enumeration(score_fn, k, renorm, scale):
    # also without renormalisation and with a routed scale: the combine weight
    # is then the raw score times the scale
    shape = synth.custom_shape("enum", 3, 96, 64, 6, k, 64, 32, score_fn, seed=11 + k,
                               scale_exp_lo=-5, scale_exp_hi=-2, renormalize=renorm,
                               routed_scale=scale)
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    r = oracle.forward(shape, w, x)
    ref, logits, sel = _dense_reference(shape, w, x)
    np.testing.assert_allclose(r["logits"], logits, rtol=1e-12, atol=1e-14)
    for b in range(shape.tokens):
        assert sorted(r["ids"][b].tolist()) == sel[b]
    scale = np.abs(ref).max()
    np.testing.assert_allclose(r["out"], ref, rtol=1e-11, atol=1e-12 * scale)


def test_single_expert_routing_is_dense_swiglu_mlp():
    # k = 1 with renormalisation: the weight is exactly 1 and the block is a
    # dense SwiGLU MLP through the chosen expert (plus the shared expert).
    shape = synth.custom_shape("k1", 2, 64, 64, 3, 1, 32, 0, synth.SCORE_SIGMOID, seed=5)
    w = synth.make_weights(shape)
    x = synth.make_x(shape)
    r = oracle.forward(shape, w, x)
    np.testing.assert_array_equal(r["weights"], 1.0)
    xf = _bf16_torch(x).reshape(2, 64)
    z = xf @ _bf16_torch(w["w_in"]).reshape(64, 64)
    gu = _dequant_independent(w["gu_codes"], w["gu_scales"])
    dn = _dequant_independent(w["dn_codes"], w["dn_scales"])
    Wout = _bf16_torch(w["w_out"]).reshape(64, 64)
    for b in range(2):
        e = int(r["ids"][b, 0])
        g = np.matmul(gu[e, :32], z[b])
        u = np.matmul(gu[e, 32:], z[b])
        hh = g / (1 + np.exp(-g)) * u
        ref = np.matmul(np.matmul(dn[e], hh), Wout)
        np.testing.assert_allclose(r["out"][b], ref, rtol=1e-12, atol=1e-13 * np.abs(ref).max())


# --------------------------------------------------------------------------
# a case worked out by hand


def _bf(v):
    return synth.to_bf16_bits(np.asarray(v, np.float32))


def test_hand_computed_tiny_case():
    """H=64, L=64, E=4, k=2 softmax, I=64, I_s=32; values derived on paper.

    x = e0 + 2 e1 + 0.5 e2.  Router columns give logits (0.5, 0.75, 1.0, -1):
    experts 2 and 1 win; renormalised softmax over the pair is a logistic of
    the logit gap: w = (sig(0.25), sig(-0.25)).
    W_in is one-hot: z[0] = 1, z[1] = 2, z[33] = 0.5.
    Expert 2: gate row 0 = {k0: 1.0, k1: 0.5, k33: 1.5 * 2^2} -> g = 1 + 1 + 3 = 5;
              up row 0 = {k0: 2.0} -> u = 2;  h0 = silu(5) * 2 = 10 sig(5);
              down row 3 = {k0: 4.0 * 2^-1} -> y[3] = 20 sig(5).
    Expert 1: gate row 5 = {k1: -1.0} -> g = -2;  up row 5 = {k0: 6.0 * 2^-2} -> u = 1.5;
              h5 = silu(-2) * 1.5 = -3 sig(-2);  down row 3 = {k5: 3.0} -> y[3] = -9 sig(-2).
    c[3] = sig(0.25) 20 sig(5) - sig(-0.25) 9 sig(-2);  W_out[3][7] = 0.5.
    Shared: g_s[4] = x0 = 1, u_s[4] = 0.25 x1 = 0.5 -> h_s[4] = 0.5 sig(1);
            W_sd[4][7] = 2, W_sd[4][0] = -1.
    out[7] = 0.5 c[3] + sig(1);  out[0] = -0.5 sig(1);  all other outputs 0.
    """
    H, L, E, k, I, Is = 64, 64, 4, 2, 64, 32
    shape = synth.custom_shape("hand", 1, H, L, E, k, I, Is, synth.SCORE_SOFTMAX)
    sig = lambda t: 1.0 / (1.0 + math.exp(-t))
    x = np.zeros((1, H), np.float32)
    x[0, 0], x[0, 1], x[0, 2] = 1.0, 2.0, 0.5
    Wr = np.zeros((H, E), np.float32)
    Wr[0] = [0.5, 0.25, 0.0, -1.0]
    Wr[1] = [0.0, 0.25, 0.5, 0.0]
    Win = np.zeros((H, L), np.float32)
    Win[0, 0] = 1.0
    Win[1, 1] = 1.0
    Win[2, 33] = 1.0
    Wout = np.zeros((L, H), np.float32)
    Wout[3, 7] = 0.5
    gu_codes = np.zeros((E, 2 * I, L // 2), np.uint8)
    gu_scales = np.full((E, 2 * I, L // 32), 127, np.uint8)
    dn_codes = np.zeros((E, L, I // 2), np.uint8)
    dn_scales = np.full((E, L, I // 32), 127, np.uint8)
    # expert 2
    gu_codes[2, 0, 0] = 0b0010 | (0b0001 << 4)      # k0 = 1.0 (low), k1 = 0.5 (high)
    gu_codes[2, 0, 16] = 0b0011 << 4                # k33 = 1.5 (high nibble of byte 16)
    gu_scales[2, 0, 1] = 129                        # block 1 scale 2^2
    gu_codes[2, I + 0, 0] = 0b0100                  # up row 0, k0 = 2.0
    dn_codes[2, 3, 0] = 0b0110                      # down row 3, k0 = 4.0
    dn_scales[2, 3, 0] = 126                        # 2^-1
    # expert 1
    gu_codes[1, 5, 0] = 0b1010 << 4                 # gate row 5, k1 = -1.0
    gu_codes[1, I + 5, 0] = 0b0111                  # up row 5, k0 = 6.0
    gu_scales[1, I + 5, 0] = 125                    # 2^-2
    dn_codes[1, 3, 2] = 0b0101 << 4                 # down row 3, k5 = 3.0 (high nibble of byte 2)
    # experts 0 and 3 carry large weights that must not leak into the output
    gu_codes[0] = 0x77
    gu_codes[3] = 0x77
    dn_codes[0] = 0x77
    dn_codes[3] = 0x77
    Wsg = np.zeros((H, Is), np.float32)
    Wsu = np.zeros((H, Is), np.float32)
    Wsd = np.zeros((Is, H), np.float32)
    Wsg[0, 4] = 1.0
    Wsu[1, 4] = 0.25
    Wsd[4, 7] = 2.0
    Wsd[4, 0] = -1.0
    w = {"router_w": _bf(Wr), "router_bias": None, "w_in": _bf(Win), "w_out": _bf(Wout),
         "gu_codes": gu_codes, "gu_scales": gu_scales, "dn_codes": dn_codes, "dn_scales": dn_scales,
         "sh_gate": _bf(Wsg), "sh_up": _bf(Wsu), "sh_down": _bf(Wsd)}
    r = oracle.forward(shape, w, _bf(x))
    assert r["ids"][0].tolist() == [2, 1]
    w0, w1 = sig(0.25), sig(-0.25)
    np.testing.assert_allclose(r["weights"][0], [w0, w1], rtol=1e-15)
    c3 = w0 * 20 * sig(5) - w1 * 9 * sig(-2)
    expect = np.zeros(H)
    expect[7] = 0.5 * c3 + sig(1)
    expect[0] = -0.5 * sig(1)
    np.testing.assert_allclose(r["out"][0], expect, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(r["h_s"][0][4], 0.5 * sig(1), rtol=1e-15)


# --------------------------------------------------------------------------
# the selection margin and the router-only entry point
#
# The margin (k-th minus (k+1)-th selection key) decides which tokens the GPU
# parity tests hold to exact ids, so it is pinned on its own: hand cases whose
# keys are closed forms, and the dense numpy/scipy route at non-zero input.


def _one_hot_router(logit_row, k, score_fn, bias=None, renorm=1, scale=1.0):
    """x = e0, W_r row 0 = logit_row: the logits are exactly logit_row."""
    E = len(logit_row)
    shape = synth.custom_shape("margin", 1, 32, 32, E, k, 32, 0, score_fn, renormalize=renorm,
                               routed_scale=scale)
    w = synth.make_weights(shape)
    Wr = np.zeros((32, E), np.float32)
    Wr[0] = logit_row
    w["router_w"] = _bf(Wr)
    w["router_bias"] = None if bias is None else np.asarray(bias, np.float32)
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 1.0
    return shape, w, _bf(x)


def test_margin_softmax_hand_case():
    # logits (1, 0.5, 2, -1, 0.25), top-2: experts 2 then 0; the next is 1.
    # margin = p_0 - p_1 = (e^1 - e^0.5) / sum_e e^{l_e}
    lg = [1.0, 0.5, 2.0, -1.0, 0.25]
    shape, w, x = _one_hot_router(lg, 2, synth.SCORE_SOFTMAX)
    den = sum(math.exp(v) for v in lg)
    for r in (oracle.route(shape, w, x), oracle.forward(shape, w, x, intermediates=False)):
        assert r["ids"][0].tolist() == [2, 0]
        assert r["margin"][0] == pytest.approx((math.exp(1.0) - math.exp(0.5)) / den, rel=1e-14)
        e2, e0 = math.exp(2.0) / den, math.exp(1.0) / den
        np.testing.assert_allclose(r["weights"][0], [e2 / (e2 + e0), e0 / (e2 + e0)], rtol=1e-14)


def test_margin_sigmoid_with_bias_hand_case():
    # keys s_e + b_e with s = sigmoid(logit).  Logits (0, 2, -1, 1), biases
    # (0.25, -0.5, 0.5, 0): keys 0.75, sig(2)-0.5 = 0.3808, sig(-1)+0.5 = 0.7689,
    # sig(1) = 0.7311.  Top-2: experts 2 and 0; the next is 3.
    sig = lambda t: 1.0 / (1.0 + math.exp(-t))
    lg, bias = [0.0, 2.0, -1.0, 1.0], [0.25, -0.5, 0.5, 0.0]
    shape, w, x = _one_hot_router(lg, 2, synth.SCORE_SIGMOID, bias=bias)
    for r in (oracle.route(shape, w, x), oracle.forward(shape, w, x, intermediates=False)):
        assert r["ids"][0].tolist() == [2, 0]
        assert r["margin"][0] == pytest.approx((sig(0.0) + 0.25) - sig(1.0), rel=1e-14)
        # weights come from the unbiased scores
        np.testing.assert_allclose(r["weights"][0],
                                   [sig(-1.0) / (sig(-1.0) + 0.5), 0.5 / (sig(-1.0) + 0.5)], rtol=1e-14)


def test_margin_is_infinite_when_every_expert_is_chosen():
    shape, w, x = _one_hot_router([0.5, -0.25, 1.0], 3, synth.SCORE_SIGMOID, bias=[0.0, 0.1, -0.1])
    for r in (oracle.route(shape, w, x), oracle.forward(shape, w, x, intermediates=False)):
        assert math.isinf(r["margin"][0]) and r["margin"][0] > 0
        assert sorted(r["ids"][0].tolist()) == [0, 1, 2]


def test_margin_of_exact_tie_is_zero():
    # two experts tie at the k-th place: the lower index is taken, margin 0
    shape, w, x = _one_hot_router([1.0, 0.5, 0.5, -2.0], 2, synth.SCORE_SOFTMAX)
    r = oracle.route(shape, w, x)
    assert r["ids"][0].tolist() == [0, 1]
    assert r["margin"][0] == 0.0


@pytest.mark.parametrize("score_fn,k,renorm,scale", [(synth.SCORE_SOFTMAX, 2, 1, 1.0),
                                                     (synth.SCORE_SIGMOID, 3, 1, 1.0),
                                                     (synth.SCORE_SIGMOID, 4, 0, 2.5),
                                                     (synth.SCORE_SOFTMAX, 3, 0, 0.5)])
def test_route_matches_dense_route_at_nonzero_input(score_fn, k, renorm, scale):
    """The router-only entry point at random (non-zero) input: logits, ids,
    weights and margins against numpy/scipy, with the selection from a sort
    of the dense keys; and the same values as the full forward."""
    shape = synth.custom_shape("route", 7, 96, 64, 12, k, 64, 0, score_fn, seed=31 + k,
                               renormalize=renorm, routed_scale=scale)
    w = synth.make_weights(shape)
    if score_fn == synth.SCORE_SIGMOID:
        w["router_bias"] = (np.random.default_rng(5).standard_normal(12) * 0.05).astype(np.float32)
    x = synth.make_x(shape)
    r = oracle.route(shape, w, x)
    f = oracle.forward(shape, w, x, intermediates=False)
    xf = _bf16_torch(x).reshape(7, 96)
    logits = xf @ _bf16_torch(w["router_w"]).reshape(96, 12)
    if score_fn == synth.SCORE_SOFTMAX:
        src = scipy.special.softmax(logits, axis=1)
        keys = src
    else:
        src = scipy.special.expit(logits)
        keys = src + w["router_bias"].astype(np.float64)
    np.testing.assert_allclose(r["logits"], logits, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["keys"], keys, rtol=1e-12, atol=1e-14)
    for b in range(7):
        order = np.lexsort((np.arange(12), -keys[b]))     # key descending, index ascending
        sel = order[:k]
        assert r["ids"][b].tolist() == sel.tolist()
        assert r["margin"][b] == pytest.approx(keys[b][order[k - 1]] - keys[b][order[k]], rel=1e-9,
                                               abs=1e-14)
        tot = src[b][sel].sum() if renorm else 1.0
        np.testing.assert_allclose(r["weights"][b], src[b][sel] / tot * scale, rtol=1e-12)
    for key in ("logits", "ids", "weights", "margin"):
        np.testing.assert_array_equal(r[key], f[key])
