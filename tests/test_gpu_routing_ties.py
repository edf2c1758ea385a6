"""GPU routing on exactly tied router logits: ties go to the lower expert index.

Identical router rows give bit-identical logits on both sides (the layer's
fp32 dot products and the oracle's fp64 ones), so the selection is fully
determined by the tie rule ("top-k ... ties to the lower expert index" of the
problem statement) and the ids must match the oracle on every token, with no
near-tie exclusion.  T = 1 and 3 run the fused small-batch routing kernel
(warp top-k, one-warp permutation); T = 300 runs the tensor-core router, the
top-k kernel and the three-launch permutation."""
import numpy as np
import pytest

from nvfp4_expert_layer_b200 import workloads as W
from tests.parity import U32, W_RTOL, Case

pytestmark = pytest.mark.gpu


def _bf16_bits(v: float) -> np.uint16:
    return np.uint16(np.float32(v).view(np.uint32) >> 16)


def _tied_inputs(T, k, seed, case):
    cfg = W.custom_config(T=T, d=256, E=16, k=k, f=128, seed=seed, router="unit")
    x, rw = W.gen_x_router(cfg)
    x, rw = x.copy(), rw.copy()
    x[:, 0] = _bf16_bits(8.0)
    x[:, 1] = _bf16_bits(8.0)
    if case == "top":
        # experts 2, 5, 9 share the largest logit (about 24), 1 and 7 the next (about 16)
        rw[2, 0] = 3.0
        rw[5] = rw[2]
        rw[9] = rw[2]
        rw[1, 1] = 2.0
        rw[7] = rw[1]
        expect = [2, 5, 9, 1, 7][:k]
    else:
        # experts 0..7 sit near -8; 8..15 are zero rows: eight exact zero logits
        rw[:8, 0] = -1.0
        rw[8:] = 0.0
        expect = list(range(8, 16))[:k]
    return cfg, x, rw, expect


@pytest.mark.parametrize("T", [1, 3, 300])
@pytest.mark.parametrize("case,k", [("top", 4), ("zeros", 8)])
def test_exact_logit_ties(T, case, k):
    cfg, x, rw, expect = _tied_inputs(T, k, 80 + T, case)
    c = Case(cfg, x=x, rw=rw).run_gpu().run_oracle()
    assert np.array_equal(c.o["ids"], np.tile(np.array(expect, np.int32), (T, 1)))
    assert np.array_equal(c.g["topk_ids"], c.o["ids"])
    # weights within the tolerance the parity contract derives from the logit deviation
    dl = np.abs(c.g["logits"].astype(np.float64) - c.o["logits"])
    delta = np.take_along_axis(dl, c.o["ids"], axis=1).max(axis=1)
    w_rtol = np.maximum(W_RTOL, 2 * delta + 4 * delta ** 2 + (k + 8) * U32)[:, None]
    assert np.all(np.abs(c.g["topk_w"].astype(np.float64) - c.o["w"]) <= w_rtol * c.o["w"])
    # counts, offsets and the permutation of the tied selection are the oracle's, bit for bit
    assert np.array_equal(c.g["counts"], c.o["counts"])
    assert np.array_equal(c.g["offsets"], c.o["offsets"])
    assert np.array_equal(c.g["perm"], c.o["perm"])
    if case == "zeros":
        c.check_all()     # "top" puts an exact tie at the k-th place: every token is a near tie
