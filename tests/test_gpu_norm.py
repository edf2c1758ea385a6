"""GPU parity of the per-expert output normalisation ("Optimizing Muse Spark
Open on TPU v7 with SGLang-TorchTPU", section 8: each expert's output is
normalised before the weighted sum, in the one combine pass; reading R12: an
RMS norm over d with no learned gain).  The down epilogues then store the
unweighted expert outputs, and the combine normalises and weights them."""
import numpy as np
import pytest

from nvfp4_expert_layer_b200 import workloads as W
from tests.parity import Case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("thr", [128, 1], ids=["light", "dense"])
def test_norm_tiny(thr):
    Case(W.CONFIGS["tiny"], thr=thr, norm_eps=1e-6).run_gpu().run_oracle().check_all()


@pytest.mark.parametrize("T", [3, 40, 300])
def test_norm_ragged_batches(T):
    cfg = W.custom_config(T=T, d=512, E=16, k=4, f=256, seed=80 + T, router="unit")
    Case(cfg, thr=64, norm_eps=1e-6).run_gpu().run_oracle().check_all()


def test_norm_large_eps_dominates():
    # eps far above mean(y^2): the output shrinks towards sum_j w_j y_j / sqrt(eps)
    cfg = W.custom_config(T=9, d=512, E=8, k=2, f=256, seed=88, router="unit")
    c = Case(cfg, norm_eps=1e4).run_gpu().run_oracle()
    c.check_all()
    assert np.max(np.abs(c.o["out64"])) < 0.1


def test_norm_decode1_full_size():
    Case(W.CONFIGS["decode1"], norm_eps=1e-6).run_gpu().run_oracle().check_all()


def test_norm_switches_back_to_plain_sum():
    cfg = W.custom_config(T=12, d=512, E=8, k=2, f=256, seed=89, router="unit")
    c = Case(cfg, norm_eps=1e-6).run_gpu().run_oracle()
    c.check_all()
    c2 = Case(cfg, layer=c.layer, experts=c.experts).run_gpu().run_oracle()
    c2.check_all()
    assert not np.array_equal(c.g["out_bits"], c2.g["out_bits"])
