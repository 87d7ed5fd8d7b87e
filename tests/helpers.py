"""Shared helpers of the parity tests: error metrics and GPU/oracle runners."""
import numpy as np

from mxfp4_latent_moe_router_b200 import synth


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def rel_errors(got, ref):
    """max |g-o| / max(|o|, rms(o)) and sum|g-o| / sum|o| (the block's tolerance metrics)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    denom = np.maximum(np.abs(ref), rms)
    denom[denom == 0] = 1.0
    max_rel = float(np.max(np.abs(got - ref) / denom)) if ref.size else 0.0
    s = np.sum(np.abs(ref))
    mean_rel = float(np.sum(np.abs(got - ref)) / s) if s > 0 else float(np.sum(np.abs(got - ref)))
    return max_rel, mean_rel


MAX_REL = 2e-2
MEAN_REL = 2e-3


def assert_close(got, ref, what, max_rel=MAX_REL, mean_rel=MEAN_REL):
    mx, mn = rel_errors(got, ref)
    assert mx <= max_rel and mn <= mean_rel, "%s: max_rel %.3g (<= %.3g), mean_rel %.3g (<= %.3g)" % (
        what, mx, max_rel, mn, mean_rel)
    return mx, mn


def logit_tolerance(shape, w, x):
    """Bound on the fp32 router logits: 2^-14 of the sum of |x_h W_he|, about the
    worst-case rounding of the few hundred fp32 additions behind each logit."""
    xf = np.abs(bf16_to_f32(x).astype(np.float64))
    Wr = np.abs(bf16_to_f32(w["router_w"]).astype(np.float64).reshape(shape.hidden, shape.num_experts))
    return (xf @ Wr) * 2.0 ** -14 + 1e-30


def _keys(shape, w, logits):
    lg = np.asarray(logits, np.float64)
    if shape.score_fn == synth.SCORE_SIGMOID:
        return 1 / (1 + np.exp(-lg)) + (0 if w["router_bias"] is None else w["router_bias"].astype(np.float64))
    return lg  # softmax ranks by logit (monotone in the probability)


def check_routing(shape, w, x, gpu_ids, gpu_w, gpu_logits, orc, max_near=None):
    """Top-k parity.

    The GPU's logits must sit within the fp32 rounding bound of the oracle's.
    If every selection key moved by at most d, any gap wider than 2d keeps its
    order, so for tokens whose oracle margin (k-th minus (k+1)-th key) exceeds
    twice the measured key deviation (plus the fp32 rounding of the key
    itself) the ids must match exactly.  Closer calls are reported as near
    ties and checked for validity: the GPU's ids must be the top-k of its own
    logits under the same rule.  At most max_near tokens (default: one per 32
    tokens, at least one) may be near ties, so that logits drifting away from
    the oracle's cannot quietly turn the exact check into the validity one."""
    B, k, E = x.shape[0], shape.top_k, shape.num_experts
    tol = logit_tolerance(shape, w, x)
    dl = np.abs(gpu_logits.astype(np.float64) - orc["logits"])
    assert np.all(dl <= tol), "router logits off by %.3g (tolerance %.3g)" % (
        float(np.max(dl - tol)), float(tol.max()))
    kg = _keys(shape, w, gpu_logits)
    ko = _keys(shape, w, orc["logits"])
    dev = np.max(np.abs(kg - ko), axis=1) + 2.0 ** -22 * (np.max(np.abs(ko), axis=1) + 1.0)
    near = []
    for b in range(B):
        if orc["margin"][b] > 2 * dev[b]:
            assert sorted(gpu_ids[b].tolist()) == sorted(orc["ids"][b].tolist()), (
                "token %d: ids %s vs oracle %s (margin %.3g, key deviation %.3g)" % (
                    b, gpu_ids[b], orc["ids"][b], orc["margin"][b], dev[b]))
            order = {e: j for j, e in enumerate(orc["ids"][b].tolist())}
            wo = np.array([orc["weights"][b][order[e]] for e in gpu_ids[b].tolist()])
            np.testing.assert_allclose(gpu_w[b], wo, rtol=1e-5, atol=1e-7)
        else:
            near.append(b)
            order = sorted(range(E), key=lambda e: (-kg[b][e], e))[:k]
            assert sorted(order) == sorted(gpu_ids[b].tolist()), "near-tie token %d invalid" % b
    if max_near is None:
        max_near = max(1, B // 32)
    assert len(near) <= max_near, "%d near-tie tokens (at most %d): %s" % (len(near), max_near, near)
    return near
