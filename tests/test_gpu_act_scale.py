"""GPU parity of the dense class with dynamic activation tensor scales
(moe_fp4_set_act_scale, reading R13): x and h are quantised as a / gs with
gs the smallest power of two bringing the call's max|a| to at most 6 * 448.
Small-magnitude activations, which the fixed scale 1 rounds to zero, then
keep their values; parity holds at the same tolerances as the fixed scale."""
import numpy as np
import pytest

from nvfp4_expert_layer_b200 import workloads as W
from tests.parity import Case
from tests.test_gpu_edge_cases import _scaled

pytestmark = pytest.mark.gpu


def test_dynamic_scale_tiny_every_expert_dense():
    c = Case(W.CONFIGS["tiny"], thr=1, act_dynamic=True).run_gpu().run_oracle()
    c.check_all()
    assert c.n_dense_rows == c.cfg.T * c.cfg.k


@pytest.mark.parametrize("x_pow,gs_pow", [(-12, 0), (8, 0), (0, -10), (-12, -10)],
                         ids=["x*2^-12", "x*2^8", "gs*2^-10", "both"])
def test_dynamic_scale_magnitude_sweep(x_pow, gs_pow):
    cfg = W.custom_config(T=40, d=512, E=8, k=2, f=256, seed=74, router="unit")
    x, rw, ex = _scaled(cfg, x_pow, gs_pow)
    c = Case(cfg, thr=1, experts=ex, x=x, rw=rw, act_dynamic=True).run_gpu().run_oracle()
    c.check_all()
    # the output keeps its values: not the zeros the fixed scale gives at small magnitudes
    assert np.sqrt(np.mean(c.o["out64"] ** 2)) > 0


def test_dynamic_scale_mixed_classes_and_ragged_tiles():
    cfg = W.custom_config(T=600, d=1024, E=16, k=4, f=768, seed=52, router="unit")
    c = Case(cfg, thr=150, act_dynamic=True).run_gpu().run_oracle()
    c.check_all()
    assert 0 < c.n_dense_rows < cfg.T * cfg.k


def test_dynamic_scale_back_to_fixed():
    cfg = W.custom_config(T=300, d=512, E=8, k=2, f=256, seed=53, router="unit")
    c = Case(cfg, thr=32, act_dynamic=True).run_gpu().run_oracle()
    c.check_all()
    c2 = Case(cfg, thr=32, layer=c.layer, experts=c.experts).run_gpu().run_oracle()
    c2.check_all()
