"""Pins of the oracle's Tier-1 encoding (per-channel INT8 keys, per-group INT4
values, eta_b annotations, nibble packing) against hand-worked fixtures and
the rounding bounds the encoding must satisfy."""

import numpy as np
import pytest

from oracle import (BLOCK, VGROUP, build_unit, pack_int4, quantize_keys_block,
                    quantize_values_block, unpack_int4)
from tests.golden import load


def test_keys_hand_fixture():
    g = load("key_quant_hand.txt")
    codes, scale = quantize_keys_block(g["k"].astype(np.float16))
    assert codes.dtype == np.int8
    np.testing.assert_array_equal(codes, g["codes"].astype(np.int8))
    np.testing.assert_array_equal(scale, g["scale"].astype(np.float32))


def test_values_hand_fixture():
    g = load("value_quant_hand.txt")
    v = np.stack([
        g["v0"],
        1.0 + 2.0 * (np.arange(32) % 16),
        np.full(32, 3.0),
    ]).astype(np.float16)
    codes, scale, offset, v_hat, eta = quantize_values_block(v)
    np.testing.assert_array_equal(codes[0], g["codes0"].astype(np.uint8))
    np.testing.assert_array_equal(codes[1], (np.arange(32) % 16).astype(np.uint8))
    np.testing.assert_array_equal(codes[2], np.zeros(32, np.uint8))
    np.testing.assert_array_equal(scale[:, 0], g["scale"].astype(np.float32))
    np.testing.assert_array_equal(offset[:, 0], g["offset"].astype(np.float32))
    np.testing.assert_array_equal(v_hat[1:], v[1:].astype(np.float32))
    assert eta == np.float32(g["eta"][0])
    np.testing.assert_array_equal(pack_int4(codes[1]), g["packed1"].astype(np.uint8))


def _blocks(rng, n, d, heavy=False):
    x = rng.standard_normal((n, BLOCK, d))
    if heavy:
        x = rng.standard_t(3, size=(n, BLOCK, d))
    x[:, :, : d // 16] *= 10.0
    return x.astype(np.float16)


@pytest.mark.parametrize("d", [64, 128])
def test_key_roundtrip_half_step(rng, d):
    for blk in _blocks(rng, 20, d):
        codes, s = quantize_keys_block(blk)
        assert np.all(np.abs(codes.astype(np.int32)) <= 127)
        # each channel's largest |k| lands on +-127
        am = np.argmax(np.abs(blk.astype(np.float32)), axis=0)
        assert np.all(np.abs(codes[am, np.arange(d)]) == 127)
        err = np.abs(blk.astype(np.float64) - codes.astype(np.float64) * s.astype(np.float64))
        # half a step, plus the float32 rounding of k/s (|k/s| <= 127)
        assert np.all(err <= s.astype(np.float64) * (0.5 + 127 * 2.0 ** -23))


def test_key_zero_channel():
    blk = np.zeros((BLOCK, 64), np.float16)
    blk[:, 1] = 2.0
    codes, s = quantize_keys_block(blk)
    assert s[0] == 0 and np.all(codes[:, 0] == 0)
    assert np.all(codes[:, 1] == 127)


@pytest.mark.parametrize("heavy", [False, True])
def test_value_roundtrip_and_eta(rng, heavy):
    d = 128
    for blk in _blocks(rng, 10, d, heavy):
        codes, s, z, v_hat, eta = quantize_values_block(blk)
        assert codes.max() <= 15
        v = blk.astype(np.float64).reshape(BLOCK, d // VGROUP, VGROUP)
        np.testing.assert_array_equal(z, v.min(axis=2).astype(np.float32))
        err = np.abs(v - v_hat.astype(np.float64).reshape(v.shape))
        zz = np.abs(z.astype(np.float64))[:, :, None]
        bound = (s.astype(np.float64)[:, :, None] * (0.5 + 16 * 2.0 ** -23)
                 + (np.abs(v) + zz) * 2.0 ** -22)
        assert np.all(err <= bound)
        # eta is the largest reconstruction error in the block (brute force)
        brute = 0.0
        for t in range(BLOCK):
            for c in range(d):
                brute = max(brute, abs(float(blk[t, c]) - float(v_hat[t, c])))
        assert abs(float(eta) - brute) <= 1e-6 * max(1.0, brute)


def test_pack_unpack_roundtrip(rng):
    codes = rng.integers(0, 16, size=(BLOCK, 128)).astype(np.uint8)
    p = pack_int4(codes)
    assert p.shape == (BLOCK, 64)
    assert p[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))
    np.testing.assert_array_equal(unpack_int4(p), codes)


def test_build_unit_blocks_and_residual(rng):
    T, d = 3 * BLOCK + 17, 64
    K = rng.standard_normal((T, d)).astype(np.float16)
    V = rng.standard_normal((T, d)).astype(np.float16)
    u = build_unit(K, V)
    assert u["nb"] == 3 and u["r"] == 17
    c1, s1 = quantize_keys_block(K[BLOCK:2 * BLOCK])
    np.testing.assert_array_equal(u["kcodes"][1], c1)
    np.testing.assert_array_equal(u["kscale"][1], s1)
    np.testing.assert_array_equal(u["vmin"], V.astype(np.float32).min(0))
    np.testing.assert_array_equal(u["vmax"], V.astype(np.float32).max(0))


# ---- binary16 metadata with directed rounding ----

def _all_finite_fp16_ascending():
    h = np.arange(1 << 16, dtype=np.uint16).view(np.float16)
    h = h[np.isfinite(h)].astype(np.float32)
    return np.unique(h)


def test_fp16_round_up_brute_force(rng):
    """The smallest binary16 >= x, against a search over every finite binary16."""
    from oracle import fp16_round_up
    table = _all_finite_fp16_ascending()
    x = np.concatenate([
        rng.uniform(0, 1, 2000), rng.uniform(0, 1e-3, 2000) ** 2, rng.uniform(0, 600, 2000),
        table[(table >= 0) & (table < 600)][::97],  # exact binary16 values map to themselves
        [0.0, 1.0 / 127, 1.0 / 15, 65504.0],
    ]).astype(np.float32)
    got = fp16_round_up(x)
    want = table[np.searchsorted(table, x, side="left")]
    np.testing.assert_array_equal(got, want)


def test_fp16_meta_hand_fixture():
    g = load("fp16_meta_hand.txt")
    d = 32
    K = np.zeros((BLOCK, d), np.float16)
    K[:5, 0] = g["k"]
    codes, scale = quantize_keys_block(K, fp16_meta=True)
    assert float(scale[0]) == float(g["key_scale"][0])
    np.testing.assert_array_equal(codes[:5, 0], g["key_codes"].astype(np.int8))
    V = np.zeros((BLOCK, d), np.float16)
    V[0, :4] = g["v"]
    vcodes, vscale, voff, v_hat, eta = quantize_values_block(V, fp16_meta=True)
    assert float(vscale[0, 0]) == float(g["value_scale"][0])
    assert float(voff[0, 0]) == 0.0
    np.testing.assert_array_equal(vcodes[0, :4], g["value_codes"].astype(np.uint8))
    assert float(eta) == float(g["eta"][0])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("heavy", [False, True])
def test_fp16_meta_bounds_hold(rng, d, heavy):
    """With binary16 metadata: the scales are binary16 values rounded up from the
    float32 ones, no code is clamped, and the errors stay within half a stored
    step (keys) and within the measured eta_b (values)."""
    for blk in _blocks(rng, 12, d, heavy):
        codes32, s32 = quantize_keys_block(blk)
        codes, s = quantize_keys_block(blk, fp16_meta=True)
        assert np.all(s.astype(np.float16).astype(np.float32) == s)
        assert np.all(s >= s32)
        ratio = np.abs(blk.astype(np.float64)) / np.where(s > 0, s, 1.0)
        assert np.all(ratio <= 127.0 * (1 + 2.0 ** -22))
        err = np.abs(blk.astype(np.float64) - codes.astype(np.float64) * s.astype(np.float64))
        assert np.all(err <= s.astype(np.float64) * (0.5 + 127 * 2.0 ** -23))
        vc, vs, vz, vh, eta = quantize_values_block(blk, fp16_meta=True)
        vc32, vs32, vz32, vh32, eta32 = quantize_values_block(blk)
        assert np.all(vs.astype(np.float16).astype(np.float32) == vs)
        assert np.all(vz.astype(np.float16).astype(np.float32) == vz)
        np.testing.assert_array_equal(vz, vz32)  # the offset is the group min, exact
        assert np.all(vs >= vs32)
        v = blk.astype(np.float32).reshape(BLOCK, d // VGROUP, VGROUP)
        r = (v - vz[:, :, None]) / np.where(vs > 0, vs, 1.0)[:, :, None]
        assert np.all(r <= 15.0 * (1 + 2.0 ** -22))
        verr = np.abs(blk.astype(np.float32) - vh)
        assert float(verr.max()) == float(eta)
        assert float(eta) <= float(vs.max()) * (0.5 + 2.0 ** -20)
