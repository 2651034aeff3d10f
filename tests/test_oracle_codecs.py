"""Pins for the oracle's number formats against independent library codecs
(PyTorch float8_e4m3fn / bfloat16 casts and ml_dtypes), plus the saturation rule."""

import json
import os

import numpy as np
import pytest
import torch

from oracle import bf16_round, e4m3_decode, e4m3_encode

ml_dtypes = pytest.importorskip("ml_dtypes")


def _all_e4m3_values():
    return e4m3_decode(np.arange(256, dtype=np.uint8))


def test_e4m3_decode_all_codes_match_libraries():
    ours = e4m3_decode(np.arange(256, dtype=np.uint8))
    lib_t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    lib_m = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib_t))
    fin = ~np.isnan(ours)
    np.testing.assert_array_equal(ours[fin], lib_t[fin])
    np.testing.assert_array_equal(ours[fin], lib_m[fin])
    assert np.nanmax(ours) == 448.0 and np.nanmin(ours) == -448.0
    assert ours[1] == 2.0 ** -9  # smallest subnormal


def _probe_values(rng, n=200_000):
    vals = _all_e4m3_values()
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (fin[:-1] + fin[1:]) / 2.0  # exact halfway points (ties)
    near = np.concatenate([np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                           np.nextafter(mids.astype(np.float32), np.float32(-np.inf))])
    mags = np.exp2(rng.uniform(-14, np.log2(463.0), n)).astype(np.float32)
    signs = np.where(rng.random(n) < 0.5, -1.0, 1.0).astype(np.float32)
    x = np.concatenate([fin, mids, near, mags * signs, [0.0, -0.0, 2.0 ** -10, 2.0 ** -11]])
    x = x.astype(np.float32)
    return x[np.abs(x) < 464.0]  # libraries give NaN at/above 464; saturation is tested apart


def test_e4m3_encode_matches_libraries_in_range():
    x = _probe_values(np.random.default_rng(0))
    ours = e4m3_encode(x)
    lib_t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    lib_m = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    # both libraries encode -0.0 as 0x80 like we do
    np.testing.assert_array_equal(ours, lib_t)
    np.testing.assert_array_equal(ours, lib_m)


def test_e4m3_encode_saturates():
    x = np.array([448.0, 463.99, 464.0, 480.0, 1e6, np.inf], dtype=np.float32)
    np.testing.assert_array_equal(e4m3_decode(e4m3_encode(x)), np.full(6, 448.0))
    np.testing.assert_array_equal(e4m3_decode(e4m3_encode(-x)), np.full(6, -448.0))
    assert e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_e4m3_roundtrip_is_identity_on_codes():
    codes = np.arange(256, dtype=np.uint8)
    fin = ~np.isnan(e4m3_decode(codes))
    back = e4m3_encode(e4m3_decode(codes[fin]).astype(np.float32))
    np.testing.assert_array_equal(back, codes[fin])


def test_bf16_round_matches_library():
    rng = np.random.default_rng(1)
    u = rng.integers(0, 2 ** 32, 500_000, dtype=np.uint64).astype(np.uint32)
    # force many exact ties: low 16 bits = 0x8000
    u[:50_000] = (u[:50_000] & 0xFFFF0000) | 0x8000
    x = u.view(np.float32)
    x = x[np.isfinite(x)]
    x = x[np.abs(x) < 3.3e38]  # keep away from overflow to inf
    ours = bf16_round(x)
    lib = torch.from_numpy(x.copy()).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(ours.view(np.uint32), lib.view(np.uint32))
