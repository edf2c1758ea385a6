"""Pins for the oracle's number formats against independent implementations.

e2m1 / e4m3fn / bf16 are checked against ml_dtypes and torch (separate code
bases), plus hand-worked anchor values of the formats' definitions."""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3fn_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decode_matches_ml_dtypes_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ours = O.e4m3fn_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_anchor_values():
    # bias 7: 0x38 = 2^(7-7) = 1.0; 0x7E = 1.75 * 2^8 = 448; 0x01 = 2^-9 (smallest subnormal)
    assert O.e4m3fn_decode(np.uint8(0x38)) == 1.0
    assert O.e4m3fn_decode(np.uint8(0x7E)) == 448.0
    assert O.e4m3fn_decode(np.uint8(0x01)) == 2.0 ** -9
    assert O.e4m3fn_decode(np.uint8(0x08)) == 2.0 ** -6
    assert math.isnan(O.e4m3fn_decode(np.uint8(0x7F)))
    assert math.isnan(O.e4m3fn_decode(np.uint8(0xFF)))
    assert O.e4m3fn_decode(np.uint8(0xB8)) == -1.0


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(O.e2m1_decode(codes), ref)


def test_e2m1_normals_match_rebiased_e4m3():
    # An e2m1 normal (s, e>0, m) equals the e4m3fn value with exponent e+6 and
    # mantissa m<<2 (biases 1 and 7): a second, format-level cross-check.
    for s in (0, 1):
        for e in (1, 2, 3):
            for m in (0, 1):
                c = (s << 3) | (e << 1) | m
                b = (s << 7) | ((e + 6) << 3) | (m << 2)
                assert O.e2m1_decode(np.uint8(c)) == O.e4m3fn_decode(np.uint8(b))


def test_unpack_low_nibble_first():
    q = np.array([[0x21, 0x7F]], dtype=np.uint8)
    assert O.unpack_e2m1(q).tolist() == [[1, 2, 0xF, 0x7]]


def test_dequant_hand_computed():
    # row 0: codes (2, 0xD) = (1.0, -3.0) ..., scale 0x40 = 2.0, gs 0.5
    q = np.zeros((2, 8), np.uint8)
    q[0, 0] = 0xD2            # element0 = 2 (1.0), element1 = 0xD (-3.0)
    q[1, 7] = 0x70            # element14 = 0, element15 = 7 (6.0)
    sf = np.array([[0x40], [0x30]], np.uint8)   # 2.0 and 0.5
    W = O.dequant_nvfp4(q, sf, np.float32(0.5))
    assert W[0, 0] == 1.0 * 2.0 * 0.5
    assert W[0, 1] == -3.0 * 2.0 * 0.5
    assert np.count_nonzero(W[0]) == 2
    assert W[1, 15] == 6.0 * 0.5 * 0.5
    assert np.count_nonzero(W[1]) == 1


def test_dequant_blocks_follow_k():
    # scale block i covers elements 16i..16i+15 along K
    q = np.full((1, 16), 0x22, np.uint8)       # 32 elements, all 1.0
    sf = np.array([[0x38, 0x40]], np.uint8)    # 1.0 then 2.0
    W = O.dequant_nvfp4(q, sf, np.float32(1.0))
    assert np.all(W[0, :16] == 1.0) and np.all(W[0, 16:] == 2.0)


def test_e2m1_rne_ties_and_saturation():
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 1e9, -0.25, -5.0, -2.6, 0.26])
    got = O.e2m1_decode(O.e2m1_rne_satfinite_codes(v))
    assert got.tolist() == [0, 1, 1, 2, 2, 4, 4, 6, 6, 0, -4, -3, 0.5]


def test_e2m1_rne_matches_ml_dtypes_random():
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 3,
                        (np.arange(-28, 29) / 4).astype(np.float32)])   # every tie point
    ours = O.e2m1_decode(O.e2m1_rne_satfinite_codes(v))
    ref = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(ours, ref)


def test_e4m3_rne_matches_torch_in_range():
    rng = np.random.default_rng(6)
    v = np.concatenate([np.exp(rng.uniform(-13, 6.1, 50000)).astype(np.float32),
                        O.E4M3_POSITIVE.astype(np.float32),
                        ((O.E4M3_POSITIVE[1:] + O.E4M3_POSITIVE[:-1]) / 2).astype(np.float32)])
    v = v[v <= 448]
    ours = O.e4m3_rne_satfinite(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    assert O.e4m3_rne_satfinite(np.array([500.0, 1e6]))[0] == 448.0


def test_bf16_rne_matches_torch_on_fp32_values():
    rng = np.random.default_rng(7)
    v = rng.standard_normal(100000).astype(np.float32) * np.float32(100)
    ours = O.f64_to_bf16_bits_rne(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rne_ties_from_fp64():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0);
    # 1 + 3*2^-8 is a tie -> 1 + 2^-6 (even); 1 + 2^-8 + 2^-40 rounds up.
    v = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -40, -3.0, 0.0])
    bits = O.f64_to_bf16_bits_rne(v)
    back = O.bf16_bits_to_f64(bits)
    assert back.tolist() == [1.0, 1 + 2 ** -6, 1 + 2 ** -7, -3.0, 0.0]


def test_quantizer_idempotent_on_grid():
    # A block that holds a +-6 code has amax = 6*sf, so its scale is recovered
    # exactly and the codes come back unchanged: q(deq(q)) = q.
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 16, size=(64, 16)).astype(np.uint8)
    codes[:, 3] = 7
    sf = O.E4M3_POSITIVE[rng.integers(8, 100, size=64)]
    vals = O.e2m1_decode(codes) * sf[:, None]
    qc, qsf, deq = O.quantize_act_nvfp4(vals.astype(np.float32))
    canon = np.where((codes & 7) == 0, 0, codes)        # -0 has no code of its own
    assert np.array_equal(qc, canon)
    assert np.array_equal(qsf[:, 0], sf)
    assert np.array_equal(deq, vals)


def test_quantizer_hand_block():
    # amax 12 -> scale 2.0; v/2 = [6, 1.5, 0.625, -1.1, 0...] -> codes 6, 1.5, 0.5, -1
    v = np.zeros(16, np.float32)
    v[:4] = [12.0, 3.0, 1.25, -2.2]
    _, sf, deq = O.quantize_act_nvfp4(v)
    assert sf.tolist() == [2.0]
    assert deq[:4].tolist() == [12.0, 3.0, 1.0, -2.0]
    zero = O.quantize_act_nvfp4(np.zeros(16, np.float32))
    assert zero[1].tolist() == [0.0] and not np.any(zero[2])
