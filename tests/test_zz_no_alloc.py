"""The allocation-free routing entry point against the regular one.

moe_route_noalloc serves callers that cannot allocate device memory (a fixed
memory budget, an allocator that must see every byte, a thread that may not
call cudaMalloc) and so cannot create a plan.  Its ids and combine weights
must equal the routing that moe_forward produces for the same tokens, under
the same rule the parity tests use (exact ids unless the selection margin is
within the measured key deviation, weights to 1e-5), on two calls in a row.

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


@pytest.mark.parametrize("score_fn,k", [(synth.SCORE_SIGMOID, 8), (synth.SCORE_SOFTMAX, 2)])
def test_noalloc_matches_forward_routing_twice(score_fn, k):
    shape = synth.custom_shape("route", 16, 1024, 256, 384 if k == 8 else 16, k, 128, 64, score_fn,
                               seed=31 + k)
    w = synth.make_weights(shape)
    dw = moe.weights_to_device(w)
    plan = moe.MoePlan(moe.config_from_shape(shape, max_tokens=16))
    plan.load(dw)
    for step, B in ((0, 16), (1, 5)):  # two calls in a row, different inputs
        x = synth.make_x(shape, tokens=B, step=40 + step)
        ids_f, w_f, logits_f = _regular_routing(plan, x)
        ids_n, w_n = _noalloc_routing(shape, dw, x)
        # both against the oracle under the parity rule ...
        orc = oracle.route(shape, w, x)
        near_f = check_routing(shape, w, x, ids_f, w_f, logits_f, orc)
        # ... and directly against each other where the choice is unambiguous:
        # the no-alloc logits obey the same fp32 bound, so a margin above twice
        # the bound's effect on the keys cannot flip
        kb = logit_tolerance(shape, w, x).max(1)
        if shape.score_fn == synth.SCORE_SIGMOID:
            kb = kb / 4.0
        for b in range(B):
            if b in near_f or orc["margin"][b] <= 2 * kb[b]:
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
