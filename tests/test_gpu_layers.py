"""A stack of layers on one stream (moe_fp4_forward_layers): the chained
result equals the layers run one by one (bit for bit: the same kernels on the
same inputs; the L2 prefetch of the next router only moves data earlier),
every layer matches the oracle on its own input, and the whole stack is
captured into one CUDA graph.  Source: "Optimizing Muse Spark Open on TPU v7
with SGLang-TorchTPU", sections 1-2 (one program over all layers, the next
layer's weights fetched while the current one computes)."""
import numpy as np
import pytest
import torch

from nvfp4_expert_layer_b200 import _lib
from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device, forward_layers
from tests.parity import Case, bf16_to_bits, to_dev_x

pytestmark = pytest.mark.gpu


def _stack(L, T, residual, E=8, k=2, thr=128):
    cfgs = [W.custom_config(T=T, d=512, E=E + 8 * (l % 2), k=k, f=256, seed=180 + l, router="unit")
            for l in range(L)]
    exs = [W.gen_experts(c) for c in cfgs]
    rws = [W.gen_x_router(c)[1] for c in cfgs]
    layers = []
    for c, ex in zip(cfgs, exs):
        layer = MoeFp4Layer(c.E, c.k, c.d, c.f)
        layer.load_experts(experts_to_device(ex))
        layer.set_residual(residual)
        layer.set_dense_threshold(thr)
        layers.append(layer)
    x, _ = W.gen_x_router(cfgs[0])
    return cfgs, exs, rws, layers, x


@pytest.mark.parametrize("T,residual,thr", [(1, True, 128), (40, True, 128), (300, False, 64)])
def test_stack_equals_layers_one_by_one_and_each_matches_the_oracle(T, residual, thr):
    cfgs, exs, rws, layers, x = _stack(3, T, residual, thr=thr)
    rwd = [torch.from_numpy(r).cuda() for r in rws]
    out = bf16_to_bits(forward_layers(layers, to_dev_x(x), rwd))
    xs = [x]
    for layer, rw in zip(layers, rwd):
        xs.append(bf16_to_bits(layer(to_dev_x(xs[-1]), rw)))
    assert np.array_equal(out, xs[-1])
    for l, (c, ex, rw) in enumerate(zip(cfgs, exs, rws)):
        Case(c, thr=thr, layer=layers[l], experts=ex, x=xs[l], rw=rw,
             residual=residual).run_gpu().run_oracle().check_all()


def test_stack_captured_in_one_graph():
    cfgs, exs, rws, layers, x = _stack(4, 2, True)
    rwd = [torch.from_numpy(r).cuda() for r in rws]
    for layer in layers:
        layer.reserve(2)
    xd = to_dev_x(x)
    ref = bf16_to_bits(forward_layers(layers, xd, rwd))
    out = torch.empty_like(xd)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            forward_layers(layers, xd, rwd, out=out, stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert all(layer.device_error() == 0 for layer in layers)
    assert np.array_equal(bf16_to_bits(out), ref)


def test_stack_rejects_a_handle_twice_in_a_row():
    cfgs, exs, rws, layers, x = _stack(2, 4, False)
    rwd = [torch.from_numpy(r).cuda() for r in rws]
    with pytest.raises(_lib.MoeFp4Error) as ei:
        forward_layers([layers[0], layers[0]], to_dev_x(x), rwd)
    assert ei.value.status == _lib.STATUS_CODE["MOE_FP4_ERR_INVALID_ARG"]
