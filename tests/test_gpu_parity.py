"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Each step of the block is checked on its own (router logits and top-k, latent
z, expert SwiGLU h, expert outputs y, shared-expert h_s) and the block output
against the oracle's fp64 result: top-k ids exact (up to reported near ties),
combine weights to 1e-5, floating outputs within max-rel 2e-2 / mean-rel 2e-3.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mxfp4_latent_moe_router_b200 as moe  # noqa: E402
from mxfp4_latent_moe_router_b200 import synth  # noqa: E402
from helpers import assert_close, bf16_to_f32, check_routing  # noqa: E402

pytestmark = pytest.mark.gpu


class GpuBlock:
    def __init__(self, shape, w, max_tokens, shared_sms=0):
        self.shape = shape
        self.w = w
        self.plan = moe.MoePlan(moe.config_from_shape(shape, max_tokens=max_tokens,
                                                      shared_sms=shared_sms))
        self.dev_w = moe.weights_to_device(w)
        self.plan.load(self.dev_w)
        torch.cuda.synchronize()

    def run(self, x_bits: np.ndarray):
        x = torch.from_numpy(x_bits.view(np.int16)).cuda()
        out = torch.empty_like(x)
        self.plan.forward(x, out)
        torch.cuda.synchronize()
        assert self.plan.sync_status() == 0
        return out.cpu().numpy().view(np.uint16)

    def fetch_all(self, B):
        r = {"logits": self.plan.fetch(moe.MOE_DBG_LOGITS, B),
             "z": self.plan.fetch(moe.MOE_DBG_Z, B),
             "h": self.plan.fetch(moe.MOE_DBG_H, B),
             "y": self.plan.fetch(moe.MOE_DBG_Y, B)}
        if self.shape.shared_inter:
            r["h_s"] = self.plan.fetch(moe.MOE_DBG_HS, B)
        r["ids"], r["w"] = self.plan.routing(B)
        return r


def _slot_order(gpu_ids, orc_ids):
    """Map GPU slot j of token b to the oracle's slot of the same expert."""
    perm = np.zeros_like(gpu_ids)
    for b in range(gpu_ids.shape[0]):
        pos = {e: j for j, e in enumerate(orc_ids[b].tolist())}
        perm[b] = [pos.get(e, -1) for e in gpu_ids[b].tolist()]
    return perm


def full_check(blk: GpuBlock, x, tokens=None, intermediates=True):
    shape, w = blk.shape, blk.w
    out = blk.run(x)
    B = x.shape[0]
    sel = np.arange(B) if tokens is None else np.asarray(tokens)
    orc = oracle.forward(shape, w, x[sel], intermediates=intermediates)
    g = blk.fetch_all(B)
    near = check_routing(shape, w, x[sel], g["ids"][sel], g["w"][sel], g["logits"][sel], orc)
    if intermediates:
        assert_close(g["z"][sel], orc["z"], "z (latent)")
        if shape.shared_inter:
            assert_close(g["h_s"][sel], orc["h_s"], "h_s (shared SwiGLU)")
        ok = [i for i, b in enumerate(sel) if b not in near]
        perm = _slot_order(g["ids"][sel], orc["ids"])
        for i in ok:
            hg = g["h"][sel[i]]
            yg = g["y"][sel[i]]
            ho = orc["h"][i][perm[i]]
            yo = orc["y"][i][perm[i]]
            assert_close(hg, ho, "h (expert SwiGLU) token %d" % sel[i])
            assert_close(yg, yo, "y (expert out) token %d" % sel[i])
    ok_rows = [i for i, b in enumerate(sel) if b not in near]
    res = assert_close(bf16_to_f32(out[sel][ok_rows]), orc["out"][ok_rows], "out")
    return out, res, near


# Launch modes chosen when a plan is made: the expert kernels on the
# tensor cores (the default), on the warp-level MMA, and the single fused
# launch (which keeps the warp-level MMA)
MODES = {"umma": {"MOE_UMMA": "1", "MOE_FUSED": "0"},
         "warp": {"MOE_UMMA": "0", "MOE_FUSED": "0"},
         "fused": {"MOE_UMMA": "0", "MOE_FUSED": "1"}}


def set_mode(monkeypatch, mode):
    for k, v in MODES[mode].items():
        monkeypatch.setenv(k, v)


# ---------------------------------------------------------------------------
# small shapes: several tiles, ragged tails, every branch


@pytest.fixture(scope="module")
def tiny():
    shape = synth.SHAPES["tiny"]
    return shape, synth.make_weights(shape)


def test_tiny_single_token(tiny):
    shape, w = tiny
    blk = GpuBlock(shape, w, max_tokens=1)
    full_check(blk, synth.make_x(shape))


@pytest.mark.parametrize("B", [1, 13])
def test_next_layer_prefetch(tiny, B):
    """Two plans as consecutive layers, each pulling the other's front
    weights into L2 during its forward: outputs bit-identical to the same
    forwards without the prefetch, and within the oracle's bounds; bad
    arguments are rejected and destroying the next plan turns it off."""
    shape, w = tiny
    w2 = synth.make_weights(shape, instance=1)
    a = GpuBlock(shape, w, max_tokens=16)
    b = GpuBlock(shape, w2, max_tokens=16)
    xs = [synth.make_x(shape, tokens=B, step=40 + i) for i in range(4)]

    def run_pair():
        return [blk.run(x) for blk, x in zip([a, b, a, b], xs)]

    plain = run_pair()
    a.plan.set_next_layer(b.plan, 1 << 30)  # (clamped to b's front weights)
    b.plan.set_next_layer(a.plan, 4096)
    pref = run_pair()
    for u, v in zip(plain, pref):
        np.testing.assert_array_equal(u, v)
    full_check(a, xs[0])
    full_check(b, xs[1])
    with pytest.raises(RuntimeError):
        a.plan.set_next_layer(b.plan, -1)
    b.plan.close()
    np.testing.assert_array_equal(a.run(xs[2]), plain[2])
    st = moe.moe_set_next_layer(a.plan.handle, 12345, 1 << 20)  # not a live plan
    assert st == 1
    a.plan.set_next_layer(None, 0)
    a.plan.set_next_layer(a.plan, 1 << 20)  # its own weights: allowed
    np.testing.assert_array_equal(a.run(xs[0]), plain[0])


@pytest.mark.parametrize("B", [2, 13, 16])
def test_tiny_ragged_batches(tiny, B):
    shape, w = tiny
    blk = GpuBlock(shape, w, max_tokens=16)
    full_check(blk, synth.make_x(shape, tokens=B, step=B))


@pytest.mark.parametrize("score_fn,k,Is", [(synth.SCORE_SIGMOID, 3, 32), (synth.SCORE_SOFTMAX, 1, 64),
                                           (synth.SCORE_SIGMOID, 4, 0)])
def test_ragged_shapes(score_fn, k, Is):
    # H=96 (dense chunks 64+32), L=96 and I=96 (MXFP4 chunks of 3 blocks), E=10
    # (router rows padded), I_s=32 or none
    shape = synth.custom_shape("ragged", 5, 96, 96, 10, k, 96, Is, score_fn, seed=21 + k,
                               scale_exp_lo=-5, scale_exp_hi=-2)
    w = synth.make_weights(shape)
    blk = GpuBlock(shape, w, max_tokens=40)
    full_check(blk, synth.make_x(shape))
    full_check(blk, synth.make_x(shape, tokens=37, step=3))


def test_zero_input_gives_exact_zero(tiny):
    shape, w = tiny
    blk = GpuBlock(shape, w, max_tokens=4)
    x = np.zeros((3, shape.hidden), np.uint16)
    out = blk.run(x)
    assert np.all(out == 0)
    ids, wts = blk.plan.routing(3)
    assert ids.tolist() == [[0, 1]] * 3
    np.testing.assert_allclose(wts, 0.5, rtol=0, atol=1e-7)


@pytest.mark.parametrize("mode", list(MODES))
def test_back_to_back_forwards_read_their_own_inputs(tiny, mode, monkeypatch):
    """Two forwards on one stream with different x: a read hoisted above a
    dependency wait would pick up the other step's activations."""
    shape, w = tiny
    set_mode(monkeypatch, mode)
    blk = GpuBlock(shape, w, max_tokens=8)
    xa = synth.make_x(shape, tokens=8, step=100)
    xb = synth.make_x(shape, tokens=8, step=101)
    ta = torch.from_numpy(xa.view(np.int16)).cuda()
    tb = torch.from_numpy(xb.view(np.int16)).cuda()
    oa, ob = torch.empty_like(ta), torch.empty_like(tb)
    for _ in range(3):
        blk.plan.forward(ta, oa)
        blk.plan.forward(tb, ob)
    torch.cuda.synchronize()
    for x, o in ((xa, oa), (xb, ob)):
        ref = oracle.forward(shape, w, x, intermediates=False)
        assert_close(bf16_to_f32(o.cpu().numpy().view(np.uint16)), ref["out"], "out")


@pytest.mark.parametrize("mode", list(MODES))
def test_deterministic_and_graph_replay(tiny, mode, monkeypatch):
    shape, w = tiny
    set_mode(monkeypatch, mode)
    blk = GpuBlock(shape, w, max_tokens=8)
    x = torch.from_numpy(synth.make_x(shape, tokens=8, step=7).view(np.int16)).cuda()
    o1, o2, o3 = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    blk.plan.forward(x, o1)
    blk.plan.forward(x, o2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        blk.plan.forward(x, o3, stream=s)  # warm-up outside capture
        s.synchronize()
        o3.zero_()
        with torch.cuda.graph(g, stream=s):
            blk.plan.forward(x, o3, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o1, o3)


def test_host_buffer_entry_point(tiny):
    shape, w = tiny
    blk = GpuBlock(shape, w, max_tokens=4)
    x = synth.make_x(shape, tokens=4, step=9)
    dev = blk.run(x)
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    blk.plan.forward_host(xh, oh)
    torch.cuda.synchronize()
    assert np.array_equal(oh.numpy().view(np.uint16), dev)


def test_argument_errors(tiny):
    shape, w = tiny
    blk = GpuBlock(shape, w, max_tokens=4)
    x = torch.zeros((4, shape.hidden), dtype=torch.int16, device="cuda")
    out = torch.empty_like(x)
    h = blk.plan.handle
    assert moe.moe_forward(h, x, 0, out) == 1
    assert moe.moe_forward(h, x, 5, out) == 1
    assert moe.moe_forward(h, x, 4, x) == 1                      # aliasing
    xb = torch.zeros(4 * shape.hidden + 8, dtype=torch.int16, device="cuda")
    assert moe.moe_forward(h, xb[1:], 4, out) == 1               # misaligned
    fresh = moe.MoePlan(moe.config_from_shape(shape, max_tokens=4))
    assert moe.moe_forward(fresh.handle, x, 4, out) == 3         # not loaded
    bad = dict(w)
    bad["gu_scales"] = w["gu_scales"].copy()
    bad["gu_scales"][3, 5, 1] = 0xFF
    with pytest.raises(moe.MoeError) as ei:
        fresh.load(moe.weights_to_device(bad))
    assert ei.value.status == 7
    assert moe.moe_forward(fresh.handle, x, 4, out) == 3


@pytest.mark.parametrize("B", [1, 4, 8])
def test_fused_launch_matches_multi_kernel_path(tiny, B, monkeypatch):
    """With MOE_FUSED=1 at plan creation, up to 8 tokens run as one fused
    launch; it must agree with the four-kernel path and with the oracle.
    The split-K piece boundaries differ, so agreement is to rounding."""
    shape, w = tiny
    x = synth.make_x(shape, tokens=B, step=40 + B)
    set_mode(monkeypatch, "fused")
    fused = GpuBlock(shape, w, max_tokens=8)
    monkeypatch.delenv("MOE_FUSED")
    monkeypatch.delenv("MOE_UMMA")
    assert fused.plan.info().kernels_per_forward == 1
    multi = GpuBlock(shape, w, max_tokens=8)
    assert multi.plan.info().kernels_per_forward == 4
    of = bf16_to_f32(fused.run(x))
    om = bf16_to_f32(multi.run(x))
    ref = oracle.forward(shape, w, x, intermediates=False)
    assert_close(of, ref["out"], "fused out")
    assert_close(om, ref["out"], "multi-kernel out")
    assert_close(of, om, "fused vs multi-kernel", max_rel=1e-2, mean_rel=1e-3)
    ids_f, w_f = fused.plan.routing(B)
    ids_m, w_m = multi.plan.routing(B)
    assert np.array_equal(np.sort(ids_f, axis=1), np.sort(ids_m, axis=1))


@pytest.mark.parametrize("case", ["tiny1", "tiny13", "tiny16", "ragged3", "ragged1"])
def test_expert_mma_paths_agree(tiny, case, monkeypatch):
    """The expert kernels on the tensor cores (e2m1 x three e4m3 terms of the
    activations, block-scaled) and on the warp-level MMA (e2m1 decoded to
    f16 x f16 activations): each within tolerance of the oracle, step by
    step, and of each other."""
    if case.startswith("tiny"):
        shape, w = tiny
        B = int(case[4:])
        x = synth.make_x(shape, tokens=B, step=60 + B)
    else:
        k = int(case[6:])
        shape = synth.custom_shape("ragged", 5, 96, 96, 10, k, 96, 32, synth.SCORE_SIGMOID,
                                   seed=31 + k, scale_exp_lo=-5, scale_exp_hi=-2)
        w = synth.make_weights(shape)
        x = synth.make_x(shape, tokens=37, step=5)
    outs = {}
    for mode in ("umma", "warp"):
        set_mode(monkeypatch, mode)
        blk = GpuBlock(shape, w, max_tokens=max(16, x.shape[0]))
        outs[mode], _, _ = full_check(blk, x)
        blk.plan.close()
    assert_close(bf16_to_f32(outs["umma"]), bf16_to_f32(outs["warp"]), "tensor-core vs warp MMA",
                 max_rel=1e-2, mean_rel=1e-3)


# ---------------------------------------------------------------------------
# full-size decode shapes (H=7168, L=2048, E=384, k=8, I=2048, I_s=2048), each
# with the seeded weights the benchmark loads for it (instance 0 of that
# workload), in a plan of 128 tokens as the benchmark creates


@pytest.fixture(scope="module")
def full_weights():
    return synth.make_weights(synth.SHAPES["b1"], 0)


@pytest.fixture(scope="module")
def full_block(full_weights):
    shape = synth.SHAPES["b1"]
    blk = GpuBlock(shape, full_weights, max_tokens=128)
    yield blk
    blk.plan.close()


def test_b1_full_size(full_block):
    shape = synth.SHAPES["b1"]
    _, (mx, mn), near = full_check(full_block, synth.make_x(shape))
    print("b1: max_rel %.3g mean_rel %.3g near-ties %s" % (mx, mn, near))


def test_b1_full_size_warp_mma(full_weights, monkeypatch):
    shape = synth.SHAPES["b1"]
    set_mode(monkeypatch, "warp")
    blk = GpuBlock(shape, full_weights, max_tokens=128)
    try:
        _, (mx, mn), near = full_check(blk, synth.make_x(shape))
        print("b1 (warp MMA): max_rel %.3g mean_rel %.3g near-ties %s" % (mx, mn, near))
    finally:
        blk.plan.close()


@pytest.mark.parametrize("ppr", ["0", "4"])
def test_b1_full_size_split_expert_pieces(full_weights, monkeypatch, ppr):
    """The expert kernels' split-K path on the tensor cores (partial sums out
    of tensor memory, tickets, the finalising sum): the makespan model's
    factor (0) and 4 pieces a row block, against the oracle."""
    shape = synth.SHAPES["b1"]
    monkeypatch.setenv("MOE_EXPERT_PPR", ppr)
    blk = GpuBlock(shape, full_weights, max_tokens=128)
    try:
        _, (mx, mn), near = full_check(blk, synth.make_x(shape, step=3))
        print("b1 (expert pieces %s): max_rel %.3g mean_rel %.3g near-ties %s" % (ppr, mx, mn, near))
    finally:
        blk.plan.close()


# sampled tokens for the whole-block check at B = 64 and 128 (every token's
# routing is checked): spread over the batch, both ends included
SAMPLES = {"b8": None,
           "b64": [0, 5, 9, 17, 22, 31, 38, 44, 50, 57, 61, 63],
           "b128": [0, 5, 13, 22, 31, 40, 47, 64, 71, 80, 95, 101, 110, 119, 127]}


@pytest.mark.parametrize("name", ["b8", "b64", "b128"])
def test_batched_full_size_as_benchmarked(name):
    shape = synth.SHAPES[name]
    w = synth.make_weights(shape, 0)
    blk = GpuBlock(shape, w, max_tokens=128)
    try:
        x = synth.make_x(shape)
        out = blk.run(x)
        # routing of every token, with the cheap router-only oracle
        r = oracle.route(shape, w, x)
        ids, wts = blk.plan.routing(x.shape[0])
        logits = blk.plan.fetch(moe.MOE_DBG_LOGITS, x.shape[0])
        near = check_routing(shape, w, x, ids, wts, logits, r)
        # whole block on sampled tokens
        sample = SAMPLES[name]
        sel = np.arange(x.shape[0]) if sample is None else np.array(sample)
        sel = np.array([b for b in sel if b not in near])
        orc = oracle.forward(shape, w, x[sel], intermediates=False)
        mx, mn = assert_close(bf16_to_f32(out[sel]), orc["out"], name + " out")
        distinct = len(np.unique(ids))
        print("%s: distinct experts %d, near ties %s, max_rel %.3g mean_rel %.3g"
              % (name, distinct, near, mx, mn))
        if shape.routing == "zipf":
            # the Zipf bias concentrates the tokens: far fewer experts than
            # uniform routing would touch (about 358 of 384 at B = 128)
            assert distinct < 200, distinct
    finally:
        blk.plan.close()
        del blk
        torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# the shared expert as a side lane (B <= 4): on, off, bounded


@pytest.mark.parametrize("shared_sms", [0, -1, 24, 148])
@pytest.mark.parametrize("B", [1, 3, 4])
def test_side_lane_settings_agree_with_the_oracle(tiny, shared_sms, B):
    shape, w = tiny
    plan = moe.MoePlan(moe.config_from_shape(shape, max_tokens=4, shared_sms=shared_sms))
    try:
        plan.load(moe.weights_to_device(w))
        x = synth.make_x(shape, tokens=B, step=60 + B)
        xt = torch.from_numpy(x.view(np.int16)).cuda()
        out = torch.empty_like(xt)
        plan.forward(xt, out)
        torch.cuda.synchronize()
        assert plan.sync_status() == 0
        ref = oracle.forward(shape, w, x)
        ids, wts = plan.routing(B)
        check_routing(shape, w, x, ids, wts, plan.fetch(moe.MOE_DBG_LOGITS, B), ref)
        assert_close(plan.fetch(moe.MOE_DBG_HS, B), ref["h_s"], "h_s")
        assert_close(bf16_to_f32(out.cpu().numpy().view(np.uint16)), ref["out"], "out")
        side = shared_sms > 0
        assert plan.info().kernels_per_forward == (6 if side else 4)
    finally:
        plan.close()


def test_side_lane_graph_replay_and_back_to_back(tiny):
    """The side stream's fork and join captured into a CUDA graph; forwards
    back to back on one stream keep their own inputs."""
    shape, w = tiny
    blk = GpuBlock(shape, w, max_tokens=4, shared_sms=148)
    xa = synth.make_x(shape, tokens=3, step=70)
    xb = synth.make_x(shape, tokens=3, step=71)
    ta = torch.from_numpy(xa.view(np.int16)).cuda()
    tb = torch.from_numpy(xb.view(np.int16)).cuda()
    oa, ob, og = torch.empty_like(ta), torch.empty_like(tb), torch.empty_like(ta)
    for _ in range(3):
        blk.plan.forward(ta, oa)
        blk.plan.forward(tb, ob)
    torch.cuda.synchronize()
    for x, o in ((xa, oa), (xb, ob)):
        ref = oracle.forward(shape, w, x, intermediates=False)
        assert_close(bf16_to_f32(o.cpu().numpy().view(np.uint16)), ref["out"], "out")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        blk.plan.forward(ta, og, stream=s)
        s.synchronize()
        og.zero_()
        with torch.cuda.graph(g, stream=s):
            blk.plan.forward(tb, ob, stream=s)
            blk.plan.forward(ta, og, stream=s)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(og, oa)
    assert blk.plan.sync_status() == 0
