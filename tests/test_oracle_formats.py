"""Pins of the oracle's codecs against brute force and library casts (CPU only).

Each pin uses a method other than the oracle's own: nearest-value search over
every code, torch's float8_e4m3fn cast, or an explicit exponent loop.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_e2m1(y):
    """Nearest of the 15 signed e2m1 values; at a tie the even code wins."""
    vals = [(c, F.E2M1_MAGNITUDES[c & 7] * (-1 if c & 8 else 1)) for c in range(16) if c != 8]
    out = []
    for v in np.asarray(y, np.float32).ravel().tolist():
        v = max(-6.0, min(6.0, v))
        best = min(vals, key=lambda cv: (abs(v - cv[1]), cv[0] & 1, cv[0]))
        c = best[0]
        out.append(0 if best[1] == 0 else c)
    return np.array(out, np.uint8)


def brute_e4m3(x):
    table = [(c, F.e4m3_decode(np.uint8(c)).item()) for c in range(256)]
    table = [(c, v) for c, v in table if not math.isnan(v)]
    out = []
    for v in np.asarray(x, np.float32).ravel().tolist():
        v = max(-448.0, min(448.0, v))
        best = min(table, key=lambda cv: (abs(v - cv[1]), cv[0] & 1, cv[0] & 0x80))
        out.append(0 if best[1] == 0 else best[0])
    return np.array(out, np.uint8)


def test_e2m1_grid_and_ties_brute_force():
    mags = list(F.E2M1_MAGNITUDES)
    mids = [(a + b) / 2 for a, b in zip(mags, mags[1:])]
    pts = set(mags + mids + [6.5, 7.0, 100.0, 1e30, 0.1, 0.2499, 0.2501, 5.01, 4.99])
    for m in list(pts):
        pts.add(float(np.nextafter(np.float32(m), np.float32(10))))
        pts.add(float(np.nextafter(np.float32(m), np.float32(-10))))
    ys = np.array(sorted(pts | {-p for p in pts}), np.float32)
    rng = np.random.default_rng(1)
    ys = np.concatenate([ys, rng.normal(0, 3, 4000).astype(np.float32), np.float32([-0.0])])
    np.testing.assert_array_equal(F.e2m1_encode(ys), brute_e2m1(ys))


def test_e2m1_documented_ties():
    # round half to even on the e2m1 grid
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for y, want in ties.items():
        assert F.e2m1_decode(F.e2m1_encode(np.float32(y))) == want
        assert F.e2m1_decode(F.e2m1_encode(np.float32(-y))) == -want


def test_e2m1_negative_zero_is_code_zero():
    assert F.e2m1_encode(np.float32(-0.0)) == 0
    assert F.e2m1_encode(np.float32(-0.1)) == 0


def test_e4m3_against_brute_force_every_midpoint():
    vals = sorted(set(F.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).tolist()))
    pts = set(vals)
    for a, b in zip(vals, vals[1:]):
        m = (a + b) / 2
        pts |= {m, float(np.nextafter(np.float32(m), np.float32(1e9))),
                float(np.nextafter(np.float32(m), np.float32(-1e9)))}
    pts |= {448.0, 460.0, 464.0, 465.0, 1e6, 1e-12, 2.0 ** -10, 3 * 2.0 ** -11}
    xs = np.array(sorted(pts | {-p for p in pts}), np.float32)
    np.testing.assert_array_equal(F.e4m3_encode(xs), brute_e4m3(xs))


def test_e4m3_against_torch_cast():
    rng = np.random.default_rng(2)
    xs = np.concatenate([rng.normal(0, s, 20000) for s in (1e-3, 0.1, 1, 30, 300)]).astype(np.float32)
    xs = np.clip(xs, -448, 448)
    ours = F.e4m3_decode(F.e4m3_encode(xs))
    theirs = torch.from_numpy(xs).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, theirs)


def test_e4m3_saturates():
    assert F.e4m3_encode(np.float32(1e9)) == 0x7E
    assert F.e4m3_encode(np.float32(-1e9)) == 0xFE


def test_e8m0_ceil_exponent_brute_force():
    rng = np.random.default_rng(3)
    qs = np.concatenate([np.exp2(rng.uniform(-140, 127.9, 3000)),
                         np.exp2(np.arange(-130, 127, dtype=np.float64)),
                         [1.0, 1.5, 2.0, 3.0, 1e-45, 3e38]]).astype(np.float32)
    qs = qs[np.isfinite(qs) & (qs > 0)]
    got = F.e8m0_ceil_exponent(qs)
    for q, e in zip(qs.tolist(), got.tolist()):
        want = next((x for x in range(-127, 128) if 2.0 ** x >= q), 127)
        assert e == want, (q, e, want)


def test_nibble_order_low_first():
    codes = np.array([1, 2, 3, 4], np.uint8)
    np.testing.assert_array_equal(F.pack_nibbles(codes), [0x21, 0x43])
    np.testing.assert_array_equal(F.unpack_nibbles(F.pack_nibbles(codes)), codes)


def _nearest_scaled(x, s):
    """Nearest e2m1 multiple of s (brute force), for one block."""
    if s == 0:
        return np.zeros_like(x, dtype=np.float64)
    y = np.array([np.float32(v) / np.float32(s) for v in x], np.float32)
    return F.e2m1_decode(brute_e2m1(y)) * s


def test_pack_main_layout_and_nearest_values():
    rng = np.random.default_rng(4)
    x = rng.normal(0, 1, (7, 512)).astype(np.float32)
    x[3, 16:32] = 0.0                     # an all-zero block
    x[5, :16] *= 1e-4                     # a block with a subnormal E4M3 scale
    codes, scales = F.pack_main(x)
    assert codes.shape == (7, 256) and scales.shape == (7, 32)
    assert codes.shape[1] + scales.shape[1] == 288
    v = F.unpack_main(codes, scales)
    for r in range(7):
        for b in range(32):
            blk = x[r, 16 * b:16 * b + 16]
            s = F.e4m3_decode(brute_e4m3(np.float32([np.max(np.abs(blk)) / np.float32(6)])))[0]
            np.testing.assert_array_equal(v[r, 16 * b:16 * b + 16], _nearest_scaled(blk, s))
    assert scales[3, 1] == 0 and not codes[3, 8:16].any()


def test_pack_indexer_layout_and_minimal_power_of_two():
    rng = np.random.default_rng(5)
    x = rng.normal(0, 1, (9, 128)).astype(np.float32)
    x[2, 32:64] = 0.0
    x[4] *= 1e-30
    codes, scales = F.pack_indexer(x)
    assert codes.shape == (9, 64) and scales.shape == (9, 4)
    assert codes.shape[1] + scales.shape[1] == 68
    v = F.unpack_indexer(codes, scales)
    for r in range(9):
        for b in range(4):
            blk = x[r, 32 * b:32 * b + 32]
            amax = np.max(np.abs(blk))
            if amax == 0:
                assert scales[r, b] == 0 and not v[r, 32 * b:32 * b + 32].any()
                continue
            q = float(np.float32(amax) / np.float32(6))
            e = int(scales[r, b]) - 127
            assert 2.0 ** e >= q and (e == -127 or 2.0 ** (e - 1) < q)
            np.testing.assert_array_equal(v[r, 32 * b:32 * b + 32], _nearest_scaled(blk, 2.0 ** e))


def test_pack_swa_nearest_and_amax_maps_to_448():
    rng = np.random.default_rng(6)
    x = rng.normal(0, 1, (5, 512)).astype(np.float32)
    x[1] = 0.0
    codes, scale = F.pack_swa(x)
    assert codes.shape == (5, 512) and scale.dtype == np.float32
    for r in range(5):
        if scale[r] == 0:
            assert not codes[r].any()
            continue
        y = x[r] / scale[r]
        np.testing.assert_array_equal(codes[r], brute_e4m3(y))
        assert np.max(np.abs(F.e4m3_decode(codes[r]))) == 448.0


def test_roundtrip_on_grid_is_identity():
    # values already on the grid at the scale the packer will pick come back exactly
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    row = np.tile(np.concatenate([mags, -mags]), 32)[:512] * np.float32(0.5)
    codes, scales = F.pack_main(row[None])
    np.testing.assert_array_equal(F.unpack_main(codes, scales)[0], row)
    irow = np.tile(np.concatenate([mags, -mags]), 8)[:128] * np.float32(2.0 ** -3)
    c, s = F.pack_indexer(irow[None])
    np.testing.assert_array_equal(F.unpack_indexer(c, s)[0], irow)


def test_entry_sizes_match_pages():
    g = json.load(open(os.path.join(GOLDEN, "byte_accounting.json")))
    assert F.MAIN_ENTRY_BYTES == g["main_entry"]["bytes"]
    assert F.MAIN_DIM * g["main_entry"]["bits_per_value"] // 8 + g["main_entry"]["scale_bytes"] == 288
    assert F.IX_ENTRY_BYTES == g["indexer_entry"]["bytes"]
    assert F.MAIN_SCALE_BYTES == g["main_entry"]["scale_bytes"]
    assert F.IX_SCALE_BYTES == g["indexer_entry"]["scale_bytes"]
    assert F.MAIN_ENTRY_BYTES + F.IX_ENTRY_BYTES == g["bytes_per_entry_pair"]["value"]
