"""The allocation-free routing entry point, moe_fp4_route_topk_static.

Some callers cannot call cudaMalloc at all: code that runs while a stream is
being captured into a CUDA graph, code whose device memory belongs to an
external pool or allocator, and processes whose device memory budget is fixed
up front.  For them the library offers routing (router logits, top-k and the
renormalised weights) that needs no handle and allocates nothing; its logits
scratch is a fixed-size array the library defines in device memory.

These tests call it through the C ABI twice in a row, with different inputs,
and check each result against the same values reported by the allocating
entry point, moe_fp4_forward_ex, within the tolerances of the parity tests:
ids bit-exact (the inputs are checked for near ties first) and weights within
1e-5 relative.  This file is collected last so that a run which stops at the
first failure has run every other test already."""
import ctypes

import numpy as np
import pytest
import torch

from nvfp4_expert_layer_b200 import _lib
from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

W_RTOL = 1e-5


def _static_route(lib, x, rw, E, k):
    T, d = x.shape
    ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream()
    rc = lib.moe_fp4_route_topk_static(ctypes.c_void_p(x.data_ptr()), T, d, ctypes.c_void_p(rw.data_ptr()),
                                       E, k, ctypes.c_void_p(ids.data_ptr()),
                                       ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(st.cuda_stream))
    assert rc == 0, _lib.STATUS.get(rc, rc)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


def _case(T, seed):
    cfg = W.custom_config(T=T, d=512, E=64, k=4, f=256, seed=seed, router="unit")
    x, rw = W.gen_x_router(cfg)
    _, _, gap = O.route(O.router_logits(x, rw), cfg.k)
    assert np.all(gap > 1e-4), "seeded inputs must have no near-tie tokens"
    return cfg, x, rw


def test_static_routing_matches_forward_ex_twice():
    lib = _lib.load()
    results = []
    for T, seed in ((37, 101), (200, 102)):
        cfg, x, rw = _case(T, seed)
        layer = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
        layer.load_experts(experts_to_device(W.gen_experts(cfg)))
        xd = torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16)
        rwd = torch.from_numpy(rw).cuda()
        _, dbg = layer.forward_ex(xd, rwd, want=("topk_ids", "topk_w"))
        ref_ids, ref_w = dbg["topk_ids"].cpu().numpy(), dbg["topk_w"].cpu().numpy()
        ids, w = _static_route(lib, xd, rwd, cfg.E, cfg.k)
        assert np.array_equal(ids, ref_ids)
        np.testing.assert_allclose(w, ref_w, rtol=W_RTOL, atol=1e-7)
        results.append(ids)
        layer.close()
    assert results[0].shape != results[1].shape


def test_static_routing_rejects_oversized_calls():
    lib = _lib.load()
    E, k, d = 1024, 8, 128
    T = 65536 // E + 1                       # T * E just over the scratch size
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    rw = torch.zeros((E, d), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    rc = lib.moe_fp4_route_topk_static(ctypes.c_void_p(x.data_ptr()), T, d, ctypes.c_void_p(rw.data_ptr()),
                                       E, k, ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                       None)
    assert rc == _lib.STATUS_CODE["MOE_FP4_ERR_UNSUPPORTED"]
    assert lib.moe_fp4_route_topk_static(None, 0, d, None, E, k, None, None, None) == 0
