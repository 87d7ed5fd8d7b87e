"""The launch planner, checked on the host for every batch size.

``moe_debug_geometry`` reports the geometry ``moe_forward`` would launch with
(the same functions choose it), without a device.  These tests hold it to the
limits the kernels rely on: shared memory per CTA and per SM, the token
columns a ring stage holds, the kernel instantiations that exist, the split-K
scratch a plan allocates, the routing CTA's logit staging and the tail's
resident activation."""
import ctypes

import pytest

import mxfp4_latent_moe_router_b200 as moe
from mxfp4_latent_moe_router_b200 import synth

KB = 1024
SMEM_PER_CTA = 227 * KB      # opt-in maximum of one CTA
HALF_SM = 113 * KB           # two CTAs on one SM (228 KB, 1 KB reserved each)
ONE_PER_SM = 116 * KB        # more than half: never two CTAs of these kernels on one SM
RESIDENT_MAX = 72 * KB
SIDE_MAX_TOKENS = 4           # largest batch with the shared expert as a side lane
INVALID_ARG, UNSUPPORTED = 1, 2  # moe_status codes
# token-tile instantiations the library compiles, per kind
TILES = {0: {1, 2, 4, 8, 16}, 1: {1, 2, 4}, 2: {1, 2, 4}, 3: {1, 2, 4, 8}, 4: {1}, 5: {1}}


def _cfg(shape, max_tokens=128):
    return moe.config_from_shape(shape, max_tokens=max_tokens)


def _side(cfg, n=148):
    c = moe.moe_config.from_buffer_copy(cfg)
    c.shared_sms = n
    return c


SHAPES = [
    ("b1 dims", _cfg(synth.SHAPES["b1"])),
    ("b1 dims, side lane", _side(_cfg(synth.SHAPES["b1"]))),
    ("tiny dims, side lane of 40", _side(_cfg(synth.SHAPES["tiny"]), 40)),
    ("tiny dims", _cfg(synth.SHAPES["tiny"])),
    ("E1024 k16", _cfg(synth.custom_shape("e1024", 1, 256, 128, 1024, 16, 64, 64, synth.SCORE_SIGMOID))),
    ("no shared expert", _cfg(synth.custom_shape("nos", 1, 512, 256, 64, 6, 256, 0, synth.SCORE_SOFTMAX))),
    ("k1", _cfg(synth.custom_shape("k1", 1, 1024, 512, 32, 1, 512, 256, synth.SCORE_SIGMOID))),
]


def _geometry(cfg, sms, B):
    return moe.moe_debug_geometry(cfg, sms, B)


@pytest.mark.parametrize("name,cfg", SHAPES, ids=[s[0] for s in SHAPES])
@pytest.mark.parametrize("sms", [148, 132])
def test_every_batch_size_fits_the_kernels(name, cfg, sms):
    E = cfg.num_experts
    res_k = {}
    for B in range(1, cfg.max_tokens + 1):
        geo = _geometry(cfg, sms, B)
        assert [g["kind"] for g in geo] == [0, 1, 2, 3, 4, 5]
        # with shared_sms > 0 the shared expert runs as a side lane (kinds 4,
        # 5) for at most 4 tokens when there is one; every front and tail
        # kernel then fits in half an SM, so one CTA of each lane shares an SM
        side = cfg.shared_inter > 0 and cfg.shared_sms > 0 and B <= SIDE_MAX_TOKENS
        assert (geo[4]["grid"] > 0) == side and (geo[5]["grid"] > 0) == side
        for g in geo:
            if g["grid"] == 0:
                continue
            where = "%s B=%d kind %d" % (name, B, g["kind"])
            assert g["stages"] >= 2, where
            assert g["stage_bytes"] % 128 == 0, where
            assert g["smem_bytes"] <= SMEM_PER_CTA, where
            assert g["token_tiles"] in TILES[g["kind"]], where
            # a ring stage holds 8 token columns per tile
            assert 8 * g["token_tiles"] >= g["max_piece_tokens"] >= 1, where
            assert g["partial_floats_needed"] <= g["partial_floats_capacity"], where
            assert g["pieces_per_row_block"] >= 1, where
            if g["kind"] >= 4:
                assert g["grid"] == min(cfg.shared_sms, sms), where  # the side lane's own size
            else:
                assert g["grid"] == sms * g["ctas_per_sm"], where
            if g["ctas_per_sm"] == 2:
                # only the expert kernels are compiled for two CTAs an SM: at one
                # token tile, and (tensor-core instantiation) at two
                assert g["kind"] in (1, 2) and g["token_tiles"] in (1, 2), where
                assert g["smem_bytes"] <= HALF_SM and g["stages"] >= 3, where
            elif side and g["kind"] in (0, 3, 4, 5):
                assert g["smem_bytes"] <= HALF_SM and g["stages"] >= 2, where
            else:
                assert g["ctas_per_sm"] == 1 and g["smem_bytes"] >= ONE_PER_SM, where
        front, egu, edn, tail = geo[:4]
        if side:
            # the two lanes' tails fill the same row blocks' partial-sum slots
            # and count the same tickets: one split for both
            assert geo[5]["pieces_per_row_block"] == tail["pieces_per_row_block"]
        # the front streams every token of the batch in one piece
        assert front["max_piece_tokens"] == B
        # the routing CTA stages at least one token's logits in its idle ring
        assert front["route_logit_floats"] >= E
        # expert pieces gather at most one row per producer lane
        assert egu["max_piece_tokens"] <= 32 and edn["max_piece_tokens"] <= 32
        assert egu["token_tiles"] == edn["token_tiles"] and egu["grid"] == edn["grid"]
        # the tail keeps the combined activation resident only when it fits
        assert tail["resident_tail_bytes"] <= RESIDENT_MAX
        for g in (tail, geo[5]):
            if g["grid"] and g["resident_tail_bytes"]:
                assert g["resident_tail_bytes"] <= RESIDENT_MAX
                per_token = g["resident_tail_bytes"] // B
                assert per_token * B == g["resident_tail_bytes"]
                key = (g["kind"], side)
                res_k.setdefault(key, per_token)
                assert per_token == res_k[key]  # the same record size for every B


@pytest.mark.parametrize("umma", ["1", "0"])
def test_expert_kernel_choices(umma, monkeypatch):
    # 8-token virtual experts up to 64 tokens; above, 16-token ones on the
    # tensor-core path (two token tiles).  Either MMA path runs two expert
    # CTAs an SM there (the tensor-core one holding half the SM's tensor
    # memory each).
    monkeypatch.setenv("MOE_UMMA", umma)
    cfg = _cfg(synth.SHAPES["b1"])
    for B in (1, 8, 64, 65, 128):
        front, egu, edn, tail = _geometry(cfg, 148, B)[:4]
        tg = 16 if (umma == "1" and B > 64) else 8
        assert egu["ctas_per_sm"] == 2 and egu["grid"] == 296
        assert egu["max_piece_tokens"] == min(B, tg)
        assert egu["token_tiles"] == tg // 8
        assert egu["stages"] >= 3 and edn["stages"] >= 3


def test_full_size_choices():
    # the measured configuration at full size: one token per stage at B = 1
    cfg = _cfg(synth.SHAPES["b1"])
    for B, front_tiles in ((1, 1), (8, 1), (64, 8), (128, 16)):
        front, egu, edn, tail = _geometry(cfg, 148, B)[:4]
        assert front["token_tiles"] == front_tiles
    front, egu, edn, tail, side_front, side_tail = _geometry(cfg, 148, 1)
    assert tail["resident_tail_bytes"] > 0  # B = 1 keeps c and h_s in shared memory
    assert front["pieces_per_row_block"] > 1  # the dense front splits K
    assert side_front["grid"] == side_tail["grid"] == 0  # no side lane by default
    front, egu, edn, tail, side_front, side_tail = _geometry(_side(cfg), 148, 1)
    assert side_tail["resident_tail_bytes"] > 0  # the side lane keeps h_s resident
    assert side_front["grid"] == side_tail["grid"] == 148
    # shared_sms bounds the side lane's CTAs; -1 turns it off
    bounded = moe.moe_config.from_buffer_copy(cfg)
    bounded.shared_sms = 40
    geo = _geometry(bounded, 148, 1)
    assert geo[4]["grid"] == geo[5]["grid"] == 40
    assert geo[5]["pieces_per_row_block"] == geo[3]["pieces_per_row_block"]
    off = moe.moe_config.from_buffer_copy(cfg)
    off.shared_sms = -1
    geo = _geometry(off, 148, 1)
    assert geo[4]["grid"] == geo[5]["grid"] == 0
    assert geo[0]["smem_bytes"] >= ONE_PER_SM


def test_bad_arguments_rejected():
    cfg = _cfg(synth.SHAPES["tiny"], max_tokens=16)
    lib = moe.load_library()
    out = (moe.moe_geometry * 6)()
    for sms, B in ((148, 0), (148, 17), (1, 1)):
        assert lib.moe_debug_geometry(ctypes.byref(cfg), sms, B, out) == INVALID_ARG
    assert lib.moe_debug_geometry(None, 148, 1, out) == INVALID_ARG
    assert lib.moe_debug_geometry(ctypes.byref(cfg), 148, 1, None) == INVALID_ARG
    bad = moe.moe_config.from_buffer_copy(cfg)
    bad.hidden = 100  # not a multiple of 32
    assert lib.moe_debug_geometry(ctypes.byref(bad), 148, 1, out) == INVALID_ARG
    big = moe.moe_config.from_buffer_copy(cfg)
    big.num_experts = 2048
    assert lib.moe_debug_geometry(ctypes.byref(big), 148, 1, out) == UNSUPPORTED
    neg = moe.moe_config.from_buffer_copy(cfg)
    neg.shared_sms = -2
    assert lib.moe_debug_geometry(ctypes.byref(neg), 148, 1, out) == INVALID_ARG
