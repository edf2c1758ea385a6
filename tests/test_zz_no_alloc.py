"""The allocation-free routing entry point, moe_fp4_route_topk_static.

Some callers cannot call cudaMalloc at all: code that runs while a stream is
being captured into a CUDA graph, code whose device memory belongs to an
external pool or allocator, and processes whose device memory budget is fixed
up front.  For them the library offers routing (router logits, top-k and the
renormalised weights) that needs no handle and allocates nothing; its logits
scratch is a fixed-size array the library defines in device memory.

These tests call it through the C ABI, twice in a row with different inputs,
and check each result against the oracle's routing of the same inputs (ids
bit-exact, near ties excluded; weights within the tolerance the parity tests
derive from the fp32 logit bound) and against the allocating entry point
moe_fp4_forward_ex (ids bit-exact, weights within 1e-5 relative).  One case
fills the scratch array exactly (T * E = 65536).  This file is collected last
so that a run which stops at the first failure has run every other test
already."""
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
U32 = 2.0 ** -24


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


def _check_against_oracle(x, rw, k, ids, w):
    """ids bit-exact on tokens without a near tie; weights within
    max(1e-5, 2 delta + 4 delta^2 + (k + 8) 2^-24) relative, delta bounded by
    the fp32 logit bound of the token's selected experts."""
    logits = O.router_logits(x, rw)
    oids, ow, gap = O.route(logits, k)
    keep = ~O.near_tie_flags(gap)
    assert keep.sum() >= len(keep) - 2 - len(keep) // 100
    assert np.array_equal(ids[keep], oids[keep])
    bound = O.fp32_logit_error_bound(x, rw)
    delta = np.take_along_axis(bound, oids, axis=1).max(axis=1)
    tol = np.maximum(W_RTOL, 2 * delta + 4 * delta ** 2 + (k + 8) * U32)[:, None]
    assert np.all((np.abs(w.astype(np.float64) - ow) <= tol * ow + 1e-7)[keep])


def test_static_routing_matches_oracle_and_forward_ex_twice():
    lib = _lib.load()
    results = []
    for T, seed in ((37, 101), (200, 102)):
        cfg = W.custom_config(T=T, d=512, E=64, k=4, f=256, seed=seed, router="unit")
        x, rw = W.gen_x_router(cfg)
        layer = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
        layer.load_experts(experts_to_device(W.gen_experts(cfg)))
        xd = torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16)
        rwd = torch.from_numpy(rw).cuda()
        _, dbg = layer.forward_ex(xd, rwd, want=("topk_ids", "topk_w"))
        ref_ids, ref_w = dbg["topk_ids"].cpu().numpy(), dbg["topk_w"].cpu().numpy()
        ids, w = _static_route(lib, xd, rwd, cfg.E, cfg.k)
        _check_against_oracle(x, rw, cfg.k, ids, w)
        assert np.array_equal(ids, ref_ids)
        np.testing.assert_allclose(w, ref_w, rtol=W_RTOL, atol=1e-7)
        results.append(ids)
        layer.close()
    assert results[0].shape != results[1].shape


def test_static_routing_fills_the_scratch_exactly():
    # T * E = 65536 logits, the largest call the scratch array holds
    lib = _lib.load()
    cfg = W.custom_config(T=256, d=512, E=256, k=8, f=256, seed=103, router="unit")
    x, rw = W.gen_x_router(cfg)
    assert cfg.T * cfg.E == 65536
    xd = torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16)
    rwd = torch.from_numpy(rw).cuda()
    for _ in range(2):
        ids, w = _static_route(lib, xd, rwd, cfg.E, cfg.k)
        _check_against_oracle(x, rw, cfg.k, ids, w)


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
