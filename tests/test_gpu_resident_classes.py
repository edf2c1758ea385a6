"""Resident weight copies chosen by the caller (moe_fp4_set_resident_classes).

A handle keeps the register-dequant copy of the experts, the tensor-core
copy, or both.  Each copy holds exactly the canonical NVFP4 bytes, so a
handle that keeps one class costs 1.0x the expert weights; with one copy
every expert runs in that class whatever its row count, and the result
matches the oracle for that class."""
import numpy as np
import pytest
import torch

from nvfp4_expert_layer_b200 import _lib
from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from tests.parity import Case, to_dev_x

pytestmark = pytest.mark.gpu


def canonical_bytes(cfg):
    return cfg.E * 3 * cfg.f * cfg.d * 9 // 16       # 1/2 byte per value + 1 scale byte per 16


def _layer(cfg, ex, light, dense):
    layer = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
    layer.set_resident_classes(light, dense)
    layer.load_experts(experts_to_device(ex))
    return layer


@pytest.mark.parametrize("T,thr", [(40, 1), (300, 32)])
def test_light_copy_only(T, thr):
    # even with a threshold every expert reaches, each expert runs light
    cfg = W.custom_config(T=T, d=512, E=8, k=2, f=256, seed=110 + T, router="unit")
    ex = W.gen_experts(cfg)
    layer = _layer(cfg, ex, True, False)
    assert layer.device_bytes()[0] == canonical_bytes(cfg)
    c = Case(cfg, thr=thr, layer=layer, experts=ex, oracle_thr=1 << 40).run_gpu().run_oracle()
    c.check_all()
    assert c.n_dense_rows == 0


@pytest.mark.parametrize("T", [1, 5, 200])
def test_dense_copy_only(T):
    # with the default threshold 128 every expert still runs dense (NVFP4 activations)
    cfg = W.custom_config(T=T, d=512, E=8, k=2, f=256, seed=120 + T, router="unit")
    ex = W.gen_experts(cfg)
    layer = _layer(cfg, ex, False, True)
    assert layer.device_bytes()[0] == canonical_bytes(cfg)
    c = Case(cfg, thr=128, layer=layer, experts=ex, oracle_thr=1).run_gpu().run_oracle()
    c.check_all()
    assert c.n_dense_rows == c.n_rows_compared > 0


def test_both_copies_and_reload_rules():
    cfg = W.custom_config(T=8, d=512, E=8, k=2, f=256, seed=131, router="unit")
    ex = W.gen_experts(cfg)
    layer = _layer(cfg, ex, True, True)
    assert layer.device_bytes()[0] == 2 * canonical_bytes(cfg)
    x, rw = W.gen_x_router(cfg)
    xd, rwd = to_dev_x(x), torch.from_numpy(rw).cuda()
    layer(xd, rwd)
    layer.set_resident_classes(False, True)             # takes effect at the next load
    with pytest.raises(_lib.MoeFp4Error) as ei:
        layer(xd, rwd)
    assert ei.value.status == _lib.STATUS_CODE["MOE_FP4_ERR_NOT_LOADED"]
    layer.load_experts(experts_to_device(ex))
    assert layer.device_bytes()[0] == canonical_bytes(cfg)
    layer(xd, rwd)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    with pytest.raises(_lib.MoeFp4Error):
        layer.set_resident_classes(False, False)


def test_dense_only_needs_a_dense_shape():
    cfg = W.custom_config(T=4, d=384, E=4, k=2, f=256, seed=132)
    layer = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
    with pytest.raises(_lib.MoeFp4Error) as ei:
        layer.set_resident_classes(False, True)
    assert ei.value.status == _lib.STATUS_CODE["MOE_FP4_ERR_UNSUPPORTED"]
