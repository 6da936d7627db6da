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
