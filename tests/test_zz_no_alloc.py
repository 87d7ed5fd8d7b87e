"""The allocation-free routing entry point against the regular one.

moe_route_noalloc serves callers that cannot allocate device memory (a fixed
memory budget, an allocator that must see every byte, a thread that may not
call cudaMalloc) and so cannot create a plan.  Its ids and combine weights
are checked against the oracle directly (exact ids unless the selection
margin is within the fp32 logit bound's effect on the keys, weights to 1e-5)
and against the routing that moe_forward produces for the same tokens, on two
calls in a row, up to the largest batch and expert count its scratch holds.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mxfp4_latent_moe_router_b200 as moe  # noqa: E402
from mxfp4_latent_moe_router_b200 import synth  # noqa: E402
from helpers import check_routing, logit_tolerance  # noqa: E402

pytestmark = pytest.mark.gpu


def _regular_routing(plan, x):
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    out = torch.empty_like(xt)
    plan.forward(xt, out)
    torch.cuda.synchronize()
    return plan.routing(x.shape[0]) + (plan.fetch(moe.MOE_DBG_LOGITS, x.shape[0]),)


def _noalloc_routing(shape, dw, x):
    B = x.shape[0]
    xt = torch.from_numpy(x.view(np.int16)).cuda()
    ids = torch.full((B, shape.top_k), -1, dtype=torch.int32, device="cuda")
    wts = torch.zeros((B, shape.top_k), dtype=torch.float32, device="cuda")
    st = moe.moe_route_noalloc(xt, dw["router_w"], dw.get("router_bias"), B, shape.hidden,
                               shape.num_experts, shape.top_k, shape.score_fn, shape.renormalize,
                               shape.routed_scale, ids, wts)
    assert st == 0, moe.moe_status_str(st)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), wts.cpu().numpy()


def _key_bound(shape, w, x):
    """Bound on how far a GPU selection key may sit from the oracle's: the
    fp32 logit bound, through the sigmoid's slope (at most 1/4); softmax is
    ranked by logit."""
    kb = logit_tolerance(shape, w, x)
    return kb / 4.0 if shape.score_fn == synth.SCORE_SIGMOID else kb


def _rank_keys(shape, w, logits):
    lg = np.asarray(logits, np.float64)
    if shape.score_fn == synth.SCORE_SIGMOID:
        b = 0.0 if w["router_bias"] is None else w["router_bias"].astype(np.float64)
        return 1.0 / (1.0 + np.exp(-lg)) + b
    return lg


def _check_vs_oracle(shape, w, x, ids, wts, orc):
    """The no-alloc ids and weights against the oracle directly.  Where the
    oracle's k-th and (k+1)-th keys are further apart than twice the key
    bound, the ids must be exactly the oracle's and the weights within 1e-5;
    closer calls must still be a valid top-k: every expert clearly above the
    k-th key chosen, none clearly below it.  Returns the near-tie tokens."""
    kb = _key_bound(shape, w, x)
    ko = _rank_keys(shape, w, orc["logits"])
    k = shape.top_k
    near = []
    for b in range(x.shape[0]):
        srt = np.sort(ko[b])[::-1]
        gap = srt[k - 1] - srt[k] if k < ko.shape[1] else np.inf
        d = kb[b].max()
        got = sorted(ids[b].tolist())
        assert len(set(got)) == k and min(got) >= 0 and max(got) < ko.shape[1], (b, got)
        if gap > 2 * d:
            assert got == sorted(orc["ids"][b].tolist()), (b, got, orc["ids"][b])
            order = {e: j for j, e in enumerate(orc["ids"][b].tolist())}
            np.testing.assert_allclose(wts[b], [orc["weights"][b][order[e]] for e in ids[b].tolist()],
                                       rtol=1e-5, atol=1e-7)
        else:
            near.append(b)
            must = set(np.nonzero(ko[b] > srt[k - 1] + 2 * d)[0].tolist())
            may = set(np.nonzero(ko[b] >= srt[k - 1] - 2 * d)[0].tolist())
            assert must <= set(got) <= may, (b, got)
    return near


# (E, k, score function, batch of the first call, batch of the second call)
CASES = [(384, 8, synth.SCORE_SIGMOID, 16, 5),
         (16, 2, synth.SCORE_SOFTMAX, 16, 3),
         # the whole static array (B = 128, E = 1024) with the largest top-k
         (1024, 16, synth.SCORE_SIGMOID, 128, 128),
         # an expert count that splits unevenly over the selection slices
         (600, 8, synth.SCORE_SOFTMAX, 40, 7)]


@pytest.mark.parametrize("E,k,score_fn,B0,B1", CASES)
def test_noalloc_matches_oracle_and_forward_routing_twice(E, k, score_fn, B0, B1):
    shape = synth.custom_shape("route", B0, 1024, 256, E, k, 128, 64, score_fn, seed=31 + k + E)
    w = synth.make_weights(shape)
    dw = moe.weights_to_device(w)
    plan = moe.MoePlan(moe.config_from_shape(shape, max_tokens=max(B0, B1)))
    plan.load(dw)
    for step, B in ((0, B0), (1, B1)):  # two calls in a row, different inputs
        x = synth.make_x(shape, tokens=B, step=40 + step)
        ids_f, w_f, logits_f = _regular_routing(plan, x)
        ids_n, w_n = _noalloc_routing(shape, dw, x)
        orc = oracle.route(shape, w, x)
        # the no-alloc call against the oracle directly
        near_n = _check_vs_oracle(shape, w, x, ids_n, w_n, orc)
        # the regular forward under the parity rule
        near_f = check_routing(shape, w, x, ids_f, w_f, logits_f, orc)
        # and the two entry points against each other where neither is near a tie
        for b in range(B):
            if b in near_f or b in near_n:
                continue
            assert sorted(ids_n[b].tolist()) == sorted(ids_f[b].tolist()), b
            order = {e: j for j, e in enumerate(ids_f[b].tolist())}
            np.testing.assert_allclose(w_n[b], [w_f[b][order[e]] for e in ids_n[b].tolist()],
                                       rtol=1e-5, atol=1e-7)
    plan.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    x = torch.zeros((129, 64), dtype=torch.int16, device="cuda")
    wr = torch.zeros((64, 16), dtype=torch.int16, device="cuda")
    ids = torch.zeros((129, 2), dtype=torch.int32, device="cuda")
    wts = torch.zeros((129, 2), dtype=torch.float32, device="cuda")
    assert moe.moe_route_noalloc(x, wr, None, 129, 64, 16, 2, 0, 1, 1.0, ids, wts) == 2
    wr2 = torch.zeros((64, 2048), dtype=torch.int16, device="cuda")
    assert moe.moe_route_noalloc(x, wr2, None, 4, 64, 2048, 2, 0, 1, 1.0, ids, wts) == 2
    assert moe.moe_route_noalloc(x, wr, None, 0, 64, 16, 2, 0, 1, 1.0, ids, wts) == 1
    # top-k beyond 16 (with enough experts to choose from)
    wr3 = torch.zeros((64, 32), dtype=torch.int16, device="cuda")
    ids3 = torch.zeros((4, 17), dtype=torch.int32, device="cuda")
    wts3 = torch.zeros((4, 17), dtype=torch.float32, device="cuda")
    assert moe.moe_route_noalloc(x, wr3, None, 4, 64, 32, 17, 0, 1, 1.0, ids3, wts3) == 2
    # outputs that are not 4-byte aligned
    raw = torch.zeros(64, dtype=torch.uint8, device="cuda")
    assert moe.moe_route_noalloc(x, wr, None, 4, 64, 16, 2, 0, 1, 1.0, raw[2:], wts) == 1
    assert moe.moe_route_noalloc(x, wr, None, 4, 64, 16, 2, 0, 1, 1.0, ids, raw[1:]) == 1
