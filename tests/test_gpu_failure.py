"""Failure detection on the GPU without a fault: a bounded device wait that
runs out, and a non-finite input.  Both are recorded in the handle's device
error word, and the handle keeps working afterwards.

The wait is made to run out by a test hook (moe_fp4_set_unreachable_wait):
the light-class down tiles then wait for a completion count that is never
reached; the wait gives up after the handle's bound (set to a few
milliseconds here), records MOE_FP4_ERR_DEVICE_TIMEOUT, drains the copies the
kernel issued and returns.  Nothing traps, faults or spins without a bound."""
import numpy as np
import pytest
import torch

from nvfp4_expert_layer_b200 import _lib
from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from tests.parity import bf16_to_bits, to_dev_x

pytestmark = pytest.mark.gpu

TIMEOUT = _lib.STATUS_CODE["MOE_FP4_ERR_DEVICE_TIMEOUT"]
NUMERIC = _lib.STATUS_CODE["MOE_FP4_ERR_NUMERIC"]


def _layer(cfg, ex):
    layer = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
    layer.load_experts(experts_to_device(ex))
    return layer


@pytest.mark.parametrize("T", [4, 40])
def test_wait_timeout_is_reported_and_the_handle_recovers(T):
    cfg = W.custom_config(T=T, d=512, E=8, k=2, f=256, seed=90 + T, router="unit")
    x, rw = W.gen_x_router(cfg)
    ex = W.gen_experts(cfg)
    xd, rwd = to_dev_x(x), torch.from_numpy(rw).cuda()
    fresh = _layer(cfg, ex)
    ref = bf16_to_bits(fresh(xd, rwd))
    assert fresh.device_error() == 0
    layer = _layer(cfg, ex)
    layer.set_wait_timeout_ms(5)
    layer.set_unreachable_wait(True)
    layer(xd, rwd)
    torch.cuda.synchronize()
    assert layer.device_error() == TIMEOUT
    assert layer.device_error() == 0                       # read and cleared
    layer.set_unreachable_wait(False)
    out = bf16_to_bits(layer(xd, rwd))
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert np.array_equal(out, ref)


def test_non_finite_input_is_reported():
    cfg = W.custom_config(T=5, d=512, E=8, k=2, f=256, seed=95, router="unit")
    x, rw = W.gen_x_router(cfg)
    ex = W.gen_experts(cfg)
    layer = _layer(cfg, ex)
    rwd = torch.from_numpy(rw).cuda()
    ref = bf16_to_bits(layer(to_dev_x(x), rwd))
    bad = x.copy()
    bad[2, 7] = 0x7F80                                    # +inf
    layer(to_dev_x(bad), rwd)
    torch.cuda.synchronize()
    assert layer.device_error() == NUMERIC
    assert np.array_equal(bf16_to_bits(layer(to_dev_x(x), rwd)), ref)
    assert layer.device_error() == 0
