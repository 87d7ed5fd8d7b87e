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
INVALID_ARG, UNSUPPORTED = 1, 2  # moe_status codes
# token-tile instantiations the library compiles, per kind
TILES = {0: {1, 2, 4, 8, 16}, 1: {1, 2, 4}, 2: {1, 2, 4}, 3: {1, 2}}


def _cfg(shape, max_tokens=128):
    return moe.config_from_shape(shape, max_tokens=max_tokens)


SHAPES = [
    ("b1 dims", _cfg(synth.SHAPES["b1"])),
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
    res_k = None
    for B in range(1, cfg.max_tokens + 1):
        geo = _geometry(cfg, sms, B)
        assert [g["kind"] for g in geo] == [0, 1, 2, 3]
        for g in geo:
            where = "%s B=%d kind %d" % (name, B, g["kind"])
            assert g["stages"] >= 2, where
            assert g["stage_bytes"] % 128 == 0, where
            assert g["smem_bytes"] <= SMEM_PER_CTA, where
            assert g["token_tiles"] in TILES[g["kind"]], where
            # a ring stage holds 8 token columns per tile
            assert 8 * g["token_tiles"] >= g["max_piece_tokens"] >= 1, where
            assert g["partial_floats_needed"] <= g["partial_floats_capacity"], where
            assert g["pieces_per_row_block"] >= 1, where
            assert g["grid"] == sms * g["ctas_per_sm"], where
            if g["ctas_per_sm"] == 2:
                # only the expert kernels at one tile are compiled for two CTAs an SM
                assert g["kind"] in (1, 2) and g["token_tiles"] == 1, where
                assert g["smem_bytes"] <= HALF_SM and g["stages"] >= 3, where
            else:
                assert g["ctas_per_sm"] == 1 and g["smem_bytes"] >= ONE_PER_SM, where
        front, egu, edn, tail = geo
        # the front streams every token of the batch in one piece
        assert front["max_piece_tokens"] == B
        # the routing CTA stages at least one token's logits in its idle ring
        assert front["route_logit_floats"] >= E
        # expert pieces gather at most one row per producer lane
        assert egu["max_piece_tokens"] <= 32 and edn["max_piece_tokens"] <= 32
        assert egu["token_tiles"] == edn["token_tiles"] and egu["grid"] == edn["grid"]
        # the tail keeps the combined activation resident only when it fits
        assert tail["resident_tail_bytes"] <= RESIDENT_MAX
        if tail["resident_tail_bytes"]:
            per_token = tail["resident_tail_bytes"] // B
            assert per_token * B == tail["resident_tail_bytes"]
            res_k = per_token if res_k is None else res_k
            assert per_token == res_k  # the same record size for every B


def test_full_size_choices():
    # the measured configuration at full size: one token per stage at B = 1,
    # the expert kernels two CTAs an SM with 8-token virtual experts
    cfg = _cfg(synth.SHAPES["b1"])
    for B, front_tiles in ((1, 1), (8, 1), (64, 8), (128, 16)):
        front, egu, edn, tail = _geometry(cfg, 148, B)
        assert front["token_tiles"] == front_tiles
        assert egu["ctas_per_sm"] == 2 and egu["grid"] == 296
        assert egu["max_piece_tokens"] == min(B, 8)
    front, egu, edn, tail = _geometry(cfg, 148, 1)
    assert tail["resident_tail_bytes"] > 0  # B = 1 keeps c and h_s in shared memory
    assert front["pieces_per_row_block"] > 1  # the dense front splits K


def test_bad_arguments_rejected():
    cfg = _cfg(synth.SHAPES["tiny"], max_tokens=16)
    lib = moe.load_library()
    out = (moe.moe_geometry * 4)()
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
