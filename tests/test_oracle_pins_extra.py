"""More pins of the oracle, each against something other than the oracle itself.

- The activation quantiser's decisions (reading R4: sf = e4m3_rn(fp32(amax/6)),
  q = e2m1_rn(fp32(v/sf))) against an exact-rational quantiser written here
  with Python Fractions, on blocks built to sit on and next to every rounding
  midpoint.  For bf16/fp32 inputs the IEEE fp32 quotient never crosses an
  e4m3 or e2m1 midpoint that the exact quotient does not cross (the midpoints
  have few significant bits), so R4's fp32 decisions equal the exact ones;
  these blocks show it, and a quantiser that divided in bf16/fp16, truncated,
  or broke ties away from zero fails them.
- The fp32 router-logit error bound against an input whose sequential fp32
  sum provably loses about half of it, so the bound cannot be inflated by a
  large factor unnoticed.
- The per-expert output normalisation (reading R12; "Optimizing Muse Spark Open
  on TPU v7 with SGLang-TorchTPU", section 8) against closed forms on the
  hand-worked example and against its invariances."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from nvfp4_expert_layer_b200 import workloads as W
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# ----------------------------------------------------------------- exact quantiser

_E2M1 = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
         Fraction(6)]


def _e4m3_values():
    out = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        out.append(Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7))
    return out


_E4M3 = _e4m3_values()


def _rne_index(v: Fraction, grid):
    """Index of the grid value nearest to v >= 0; ties to the even index; clamps."""
    if v >= grid[-1]:
        return len(grid) - 1
    hi = next(i for i, g in enumerate(grid) if g >= v)
    if hi == 0:
        return 0
    lo = hi - 1
    dlo, dhi = v - grid[lo], grid[hi] - v
    if dlo < dhi:
        return lo
    if dhi < dlo:
        return hi
    return lo if lo % 2 == 0 else hi


def _exact_quantize_block(vals32):
    """16 fp32 values -> (scale value, 16 e2m1 codes) with exact division."""
    vs = [Fraction(float(v)) for v in vals32]
    amax = max(abs(v) for v in vs)
    sf = _E4M3[_rne_index(amax / 6, _E4M3)]
    codes = []
    for v in vs:
        if sf == 0:
            codes.append(0)
            continue
        mag = _rne_index(abs(v) / sf, _E2M1)
        codes.append(mag | 8 if (v < 0 and mag) else mag)
    return sf, codes


def _adversarial_blocks():
    """Blocks whose amax sits on, and within a few ulps of, 6 x an e4m3
    midpoint, with elements on and next to e2m1 midpoint x scale."""
    rng = np.random.default_rng(5)
    e4 = [float(v) for v in _E4M3]
    mids4 = [(a + b) / 2 for a, b in zip(e4[:-1], e4[1:])]
    mids2 = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    blocks = []
    for m in mids4[8::3]:
        a0 = np.float32(6.0 * m)
        for steps in (-2, -1, 0, 1, 2):
            a = a0
            for _ in range(abs(steps)):
                a = np.nextafter(a, np.float32(np.inf if steps > 0 else -np.inf), dtype=np.float32)
            # the scale this amax gets decides the grid of the other elements
            sf = float(_E4M3[_rne_index(Fraction(float(a)) / 6, _E4M3)])
            blk = [a]
            for mid in rng.choice(mids2, size=15):
                v = np.float32(mid * sf)
                st = int(rng.integers(-1, 2))
                for _ in range(abs(st)):
                    v = np.nextafter(v, np.float32(np.inf if st > 0 else -np.inf), dtype=np.float32)
                blk.append(np.float32(v if rng.random() < 0.5 else -v))
            blk = np.array(blk, np.float32)
            rng.shuffle(blk)
            blocks.append(blk)
    return np.stack(blocks)


def test_quantizer_decisions_equal_exact_rational_rounding():
    blocks = _adversarial_blocks()
    codes, sf, _ = O.quantize_act_nvfp4(blocks)
    ties = 0
    for i, blk in enumerate(blocks):
        esf, ecodes = _exact_quantize_block(blk)
        assert Fraction(float(sf[i, 0])) == esf, (blk, sf[i, 0], esf)
        assert codes[i].tolist() == ecodes, (blk, codes[i], ecodes)
        ties += sum(1 for v in blk if esf and (abs(Fraction(float(v))) / esf) in
                    (Fraction(1, 4), Fraction(3, 4), Fraction(5, 4), Fraction(7, 4), Fraction(5, 2),
                     Fraction(7, 2), Fraction(5)))
    assert ties > 50                                   # the blocks do exercise exact ties


def test_quantizer_hand_ties():
    # amax = 6.375 = 6 x 1.0625, the midpoint of e4m3 1.0 (0x38) and 1.125
    # (0x39): ties to the even code, 1.0.  With sf = 1: 0.25 -> 0 (0.0),
    # 0.75 -> code 2 (1.0), 1.25 -> 2 (1.0), 1.75 -> 4 (2.0), 2.5 -> 4 (2.0),
    # 3.5 -> 6 (4.0), 5.0 -> 6 (4.0), -0.75 -> 0xA (-1.0); 6.375 saturates to 6.0 (7).
    blk = np.array([6.375, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.75, 0, 0, 0, 0, 0, 0, 0], np.float32)
    codes, sf, deq = O.quantize_act_nvfp4(blk)
    assert sf[0] == 1.0
    assert codes[:9].tolist() == [7, 0, 2, 2, 4, 4, 6, 6, 0xA]
    assert deq[:9].tolist() == [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -1.0]


# ----------------------------------------------------------------- fp32 logit bound

def test_fp32_logit_bound_is_tight_on_a_worst_case_sum():
    # x = 1, w = [1, 1.5 * 2^-24, 1.5 * 2^-24, ...]: a sequential fp32 sum adds
    # 1.5u to a value in [1, 2) each step, which rounds up by u/2 every time
    # (u = 2^-24; ulp in [1, 2) is 2u), so the error grows by about u/2 per
    # term, about half of the bound gamma_{d+1} * sum|x w|.
    d = 4096
    x_bits = np.full((1, d), 0x3F80, np.uint16)
    w = np.full((1, d), np.float32(1.5 * 2.0 ** -24), np.float32)
    w[0, 0] = 1.0
    s = np.float32(0.0)
    for v in w[0]:
        s = np.float32(s + v)
    exact = 1.0 + (d - 1) * 1.5 * 2.0 ** -24
    err = abs(float(s) - exact)
    bound = O.fp32_logit_error_bound(x_bits, w)[0, 0]
    assert err <= bound
    assert err >= 0.4 * bound, (err, bound)


# ----------------------------------------------------------------- per-expert norm

class _ArrayExperts:
    def __init__(self, mats):
        self.mats = mats

    def expert(self, e):
        return self.mats[e]


def _hand_layer():
    d = f = 16
    q = np.full((f, d // 2), 0x22, np.uint8)
    sf = np.full((f, d // 16), 0x38, np.uint8)
    one = np.float32(1)
    mats = {0: {0: (q, sf, one), 1: (q, sf, one), 2: (q, sf, one)}}
    x = np.full((1, d), 0x3F80, np.uint16)
    rw = np.zeros((1, d), np.float32)
    return mats, x, rw


def test_expert_norm_hand_example():
    # hand example (tests/golden/hand_example_d16.txt): y[r] = 16 h for every
    # r, so mean(y^2) = (16 h)^2 and the normalised output is 1 with eps = 0,
    # and exactly 1/2 with eps = 3 (16 h)^2
    mats, x, rw = _hand_layer()
    res = O.forward(x, rw, _ArrayExperts(mats), 1, 1, thr=1 << 30, expert_norm_eps=0.0)
    np.testing.assert_allclose(res["out64"], 1.0, rtol=1e-15)
    y = res["y"][0, 0]
    res = O.forward(x, rw, _ArrayExperts(mats), 1, 1, thr=1 << 30, expert_norm_eps=3 * y * y)
    np.testing.assert_allclose(res["out64"], 0.5, rtol=1e-14)
    assert np.array_equal(res["partial"][0], res["out64"][0])


def test_expert_norm_removes_each_experts_scale():
    # the norm makes every expert's contribution independent of its down
    # tensor scale: scaling gs_d of one expert by 2^5 leaves the output alone
    cfg = W.custom_config(T=6, d=64, E=4, k=2, f=32, seed=19, router="unit")
    x, rw, ex = W.gen_all(cfg)
    a = O.forward(x, rw, ex, cfg.E, cfg.k, expert_norm_eps=0.0)
    ex.down_gs = ex.down_gs.copy()
    ex.down_gs[a["ids"][0, 0]] *= np.float32(32.0)
    b = O.forward(x, rw, ex, cfg.E, cfg.k, expert_norm_eps=0.0)
    np.testing.assert_allclose(b["out64"], a["out64"], rtol=1e-12, atol=1e-14)
    plain = O.forward(x, rw, ex, cfg.E, cfg.k)
    assert not np.allclose(plain["out64"], b["out64"])


def test_expert_norm_keeps_the_routing_weights():
    # a token whose top expert has almost all of the weight: the output is
    # that expert's normalised output (rms 1), not a sum of k unit vectors
    cfg = W.custom_config(T=3, d=64, E=8, k=4, f=32, seed=23, router="unit")
    x, rw, ex = W.gen_all(cfg)
    rw = rw.copy()
    rw[5] = 0
    rw[5, :] = np.float32(40.0 / 64)
    x = x.copy()
    x[:, :] = 0x3F80                                  # x = 1: logit of expert 5 is 40
    res = O.forward(x, rw, ex, cfg.E, cfg.k, expert_norm_eps=0.0)
    assert np.all(res["ids"][:, 0] == 5) and np.all(res["w"][:, 0] > 1 - 1e-12)
    rms = np.sqrt(np.mean(res["out64"] ** 2, axis=1))
    np.testing.assert_allclose(rms, 1.0, rtol=1e-9)
    yn = O.expert_rms_norm(res["y"][res["inv"][0]][None], 0.0)[0]
    np.testing.assert_allclose(res["out64"][0], yn, rtol=1e-9, atol=1e-12)


# ----------------------------------------------------------------- dynamic activation scale (R13)

def test_pow2_tensor_scale_is_the_smallest_power_of_two():
    rng = np.random.default_rng(9)
    for a in list(np.exp(rng.uniform(-60, 60, size=200))) + [2688.0, 1344.0, 2688 * 2.0 ** -20, 1.0]:
        g = O.pow2_tensor_scale(a)
        e = int(round(math.log2(g)))
        assert g == 2.0 ** e and a <= 2688.0 * g and not a <= 2688.0 * g / 2
    assert O.pow2_tensor_scale(0.0) == 1.0


def test_dynamic_scale_makes_the_dense_class_homogeneous_in_the_up_scale():
    # h = SiLU(g) u is linear in u: scaling the up tensor scale by 2^-12
    # scales h, the dynamic h scale, and so the output, by exactly 2^-12.  With
    # the fixed scale 1 the small h underflows the e4m3 block scales instead.
    cfg = W.custom_config(T=6, d=64, E=4, k=2, f=32, seed=29, router="unit")
    x, rw, ex = W.gen_all(cfg)
    a = O.forward(x, rw, ex, cfg.E, cfg.k, thr=1, act_scale="dynamic")
    ex.up_gs = (ex.up_gs * np.float32(2.0 ** -12)).astype(np.float32)
    b = O.forward(x, rw, ex, cfg.E, cfg.k, thr=1, act_scale="dynamic")
    np.testing.assert_array_equal(b["out64"], a["out64"] * 2.0 ** -12)
    assert b["gs_h"] == a["gs_h"] * 2.0 ** -12
    fixed = O.forward(x, rw, ex, cfg.E, cfg.k, thr=1)
    assert not np.allclose(fixed["out64"], b["out64"], rtol=1e-3, atol=0)


def test_dynamic_scale_quantises_x_independently_of_its_magnitude():
    # x * 2^-12 quantises to the same codes and block scales as x under the
    # dynamic scale: the gate and up values scale by exactly 2^-12
    cfg = W.custom_config(T=5, d=64, E=4, k=2, f=32, seed=31, router="unit")
    x, rw, ex = W.gen_all(cfg)
    xs = W.f32_to_bf16_bits_trunc(W.bf16_bits_to_f32(x) * np.float32(2.0 ** -12))
    a = O.forward(x, rw, ex, cfg.E, cfg.k, thr=1, act_scale="dynamic", magnitudes=True)
    b = O.forward(xs, rw, ex, cfg.E, cfg.k, thr=1, act_scale="dynamic", magnitudes=True)
    rows = np.arange(cfg.T * cfg.k)
    np.testing.assert_array_equal(b["mags"]["g"][rows], a["mags"]["g"][rows] * 2.0 ** -12)
    np.testing.assert_array_equal(b["mags"]["u"][rows], a["mags"]["u"][rows] * 2.0 ** -12)
    assert b["gs_x"] == a["gs_x"] * 2.0 ** -12


# ----------------------------------------------------------------- residual add (R14)

def test_residual_of_a_zero_expert_is_the_identity():
    # down weights all zero: the block adds nothing, out = x exactly
    cfg = W.custom_config(T=4, d=64, E=2, k=1, f=32, seed=37, router="unit")
    x, rw, ex = W.gen_all(cfg)
    ex.down_q[:] = 0
    res = O.forward(x, rw, ex, cfg.E, cfg.k, residual=True)
    assert np.array_equal(res["out_bits"], x)
    plain = O.forward(x, rw, ex, cfg.E, cfg.k)
    assert not np.any(plain["out64"])
