"""Edge cases of the CUDA path against the CPU oracle: the largest expert count
and top-k the library takes, the largest batch, sigmoid scoring without a
selection bias, the fused single launch with a tail activation too large to
keep in shared memory, the tail on formed records (tensor-core and warp-level
MMA), 32-token virtual experts, raw (unrenormalised)
scores with a routed scale, and the host-side geometry query against a real
plan."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mxfp4_latent_moe_router_b200 as moe  # noqa: E402
from mxfp4_latent_moe_router_b200 import synth  # noqa: E402
from helpers import assert_close, bf16_to_f32, check_routing  # noqa: E402

pytestmark = pytest.mark.gpu


def _run(shape, w, x, max_tokens):
    plan = moe.MoePlan(moe.config_from_shape(shape, max_tokens=max_tokens))
    try:
        plan.load(moe.weights_to_device(w))
        xd = torch.from_numpy(x.view(np.int16)).cuda()
        out = torch.empty_like(xd)
        plan.forward(xd, out)
        torch.cuda.synchronize()
        assert plan.sync_status() == 0
        B = x.shape[0]
        ids, wts = plan.routing(B)
        logits = plan.fetch(moe.MOE_DBG_LOGITS, B)
        return out.cpu().numpy().view(np.uint16), ids, wts, logits
    finally:
        plan.close()


def _check(shape, w, x, max_tokens):
    out, ids, wts, logits = _run(shape, w, x, max_tokens)
    orc = oracle.forward(shape, w, x, intermediates=False)
    near = check_routing(shape, w, x, ids, wts, logits, orc)
    ok = [b for b in range(x.shape[0]) if b not in near]
    assert_close(bf16_to_f32(out[ok]), orc["out"][ok], shape.name + " out")
    return ids, near


@pytest.mark.parametrize("B", [3, 9])
def test_largest_expert_count_and_top_k(B):
    # E = 1024 and k = 16 are the library's limits; B = 3 splits each token's
    # experts over two warps, B = 9 selects from two 512-expert slices on one
    shape = synth.custom_shape("e1024", B, 256, 128, 1024, 16, 64, 64, synth.SCORE_SIGMOID,
                               seed=61 + B, scale_exp_lo=-5, scale_exp_hi=-2)
    w = synth.make_weights(shape)
    ids, near = _check(shape, w, synth.make_x(shape), max_tokens=16)
    assert all(len(set(r.tolist())) == 16 for r in ids)


def test_largest_batch():
    # B = 128 (the library's limit) in one forward: sixteen 8-token tiles in
    # the front kernel, token groups in the expert kernels, several tail passes
    shape = synth.custom_shape("b128-small", 128, 512, 256, 32, 4, 128, 128,
                               synth.SCORE_SOFTMAX, seed=71)
    w = synth.make_weights(shape)
    _check(shape, w, synth.make_x(shape), max_tokens=128)


def test_sigmoid_without_selection_bias():
    shape = synth.custom_shape("nobias", 6, 256, 128, 24, 3, 64, 64, synth.SCORE_SIGMOID, seed=81)
    w = dict(synth.make_weights(shape))
    w["router_bias"] = None
    _check(shape, w, synth.make_x(shape), max_tokens=8)


def test_fused_launch_with_staged_tail(monkeypatch):
    # L + I_s = 3072: eight tokens' tail activation (about 98 KB as bf16 hi/lo)
    # does not fit the shared-memory budget, so the fused launch stages y and
    # h_s per chunk instead
    shape = synth.custom_shape("staged", 8, 256, 1024, 16, 2, 128, 2048, synth.SCORE_SOFTMAX,
                               seed=91, scale_exp_lo=-5, scale_exp_hi=-2)
    w = synth.make_weights(shape)
    monkeypatch.setenv("MOE_FUSED", "1")
    monkeypatch.setenv("MOE_UMMA", "0")  # (the fused launch keeps the warp-level MMA)
    _check(shape, w, synth.make_x(shape), max_tokens=8)


@pytest.mark.parametrize("umma_tail", ["1", "0"])
@pytest.mark.parametrize("B", [5, 8, 37, 64, 77])
def test_tail_from_formed_records(B, umma_tail, monkeypatch):
    # L + I_s = 3072: the tail's activation is formed once per token group as
    # bf16 hi/lo records (too large to keep resident from 6 tokens on); on the
    # tensor cores the tail multiplies them with a bf16 MMA, the records' two
    # parts as two rows a token.  1 to 8 token tiles, two passes at 77 tokens.
    monkeypatch.setenv("MOE_UMMA_TAIL", umma_tail)
    shape = synth.custom_shape("formed", B, 256, 1024, 16, 2, 128, 2048, synth.SCORE_SOFTMAX,
                               seed=61 + B, scale_exp_lo=-5, scale_exp_hi=-2)
    w = synth.make_weights(shape)
    _check(shape, w, synth.make_x(shape), max_tokens=max(B, 8))


@pytest.mark.parametrize("umma", ["1", "0"])
@pytest.mark.parametrize("B,E,k", [(24, 8, 4), (48, 4, 3)])
def test_thirty_two_token_expert_groups(B, E, k, umma, monkeypatch):
    # with 8-token groups switched off, an expert's slots form groups of up to
    # 32 tokens: ~12 per expert in one group, or 36 per expert in groups of
    # 32 and 4.  The expert kernels run four token tiles at one CTA per SM
    # and gather more than 8 activation rows per stage with 16-byte copies.
    monkeypatch.setenv("MOE_EXPERT_SMALL_MAX_B", "0")
    monkeypatch.setenv("MOE_UMMA", umma)
    shape = synth.custom_shape("tg32", B, 256, 256, E, k, 256, 64, synth.SCORE_SOFTMAX,
                               seed=101 + B, scale_exp_lo=-5, scale_exp_hi=-2)
    w = synth.make_weights(shape)
    _check(shape, w, synth.make_x(shape), max_tokens=B)


@pytest.mark.parametrize("score_fn", [synth.SCORE_SOFTMAX, synth.SCORE_SIGMOID])
def test_raw_scores_with_routed_scale(score_fn):
    # renormalisation off and a routed scale: each combine weight is the
    # chosen expert's raw score times 2.5
    shape = synth.custom_shape("raw", 5, 256, 128, 24, 3, 64, 64, score_fn, seed=111 + score_fn,
                               renormalize=0, routed_scale=2.5)
    w = synth.make_weights(shape)
    _check(shape, w, synth.make_x(shape), max_tokens=8)


def test_geometry_query_matches_the_plan():
    # the host-only geometry query and a plan on this device choose alike
    shape = synth.SHAPES["tiny"]
    for B in (1, 16):
        cfg = moe.config_from_shape(shape, max_tokens=B)
        plan = moe.MoePlan(cfg)
        try:
            info = plan.info()
            front, egu, edn, tail = moe.moe_debug_geometry(cfg, info.num_sms, B)[:4]
            # + the routing CTAs: one per 8 tokens
            assert front["grid"] == info.front_ctas + max(1, min(16, (B + 7) // 8))
            assert egu["grid"] == edn["grid"] == info.expert_ctas
        finally:
            plan.close()
