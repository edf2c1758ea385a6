"""CPU checks of the parity helpers themselves (no GPU).

quant_deviation must bound the quantiser's output change for every input
inside the stated interval; it is checked here by brute force: random points
of each element's interval, re-quantised by the oracle's quantiser, never
move further from the oracle's quantised value than the bound says."""
import numpy as np

from oracle import moe_oracle as O
from tests.parity import quant_deviation


def test_quant_deviation_bounds_random_perturbations():
    rng = np.random.default_rng(7)
    n, K = 6, 64
    h = rng.standard_normal((n, K)) * np.exp(rng.uniform(-3, 3, (n, 1)))
    # place some values right at e2m1 / e4m3 rounding boundaries
    _, sf, _ = O.quantize_act_nvfp4(h.astype(np.float32))
    h[0, :16] = np.repeat(sf[0, :1], 16) * 2.5            # code midpoint 2 | 3
    h[1, 16] = 6 * O.E4M3_POSITIVE[40] * (1 + 1 / 32)     # amax/6 near an e4m3 midpoint
    hb = np.abs(h) * 1e-3 + 1e-6
    dev, hq = quant_deviation(h, hb)
    assert np.all(dev >= 0)
    assert dev.max() > 0, "boundary cases must allow a flip"
    for _ in range(200):
        v = h + hb * rng.uniform(-1, 1, h.shape)
        q = O.quantize_act_nvfp4(v.astype(np.float32))[2]
        assert np.all(np.abs(q - hq) <= dev + 1e-30)


def test_quant_deviation_is_zero_for_exact_h():
    rng = np.random.default_rng(8)
    h = rng.standard_normal((3, 32))
    dev, hq = quant_deviation(h, np.zeros_like(h))
    # a zero-width interval can still straddle a tie only through the widening
    assert np.mean(dev == 0) > 0.95
    assert np.array_equal(hq, O.quantize_act_nvfp4(h.astype(np.float32))[2])
