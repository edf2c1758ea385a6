"""Expert parallelism on the GPU: the library's kernels behind the exchange
of nvfp4_expert_layer_b200.ep.  G ranks are held in one process on one GPU
(the all-to-alls become slices), each with its own handle for its E/G
experts; the sharded forward must match the single-device layer (bf16
outputs within one ulp or 1e-5 rms: the routing weight is applied in the
combine instead of the down epilogue, a different fp32 rounding) and the
oracle (1e-2 rms + half an ulp).  A one-rank NCCL process group runs the torch.distributed path
(all-to-all through NCCL) on the same GPU.  Not measured across GPUs: this
pool gives one GPU per run."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.ep import CudaEpBackend, ep_forward_local, shard_experts
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from oracle import moe_oracle as O
from tests.parity import bf16_to_bits, to_dev_x

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _close_to_single_device(got, ref):
    """Within one bf16 ulp of the single-device output, or 1e-5 rms absolutely
    (the weight enters in the combine instead of the down epilogue, an fp32
    rounding apart; near zero a sum may change sign by that much)."""
    a, b = O.bf16_bits_to_f64(got), O.bf16_bits_to_f64(ref)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126))) - 7)
    rms = np.sqrt(np.mean(b ** 2))
    assert np.all(np.abs(a - b) <= ulp + 1e-5 * rms)


def _oracle_check(x, rw, ex, cfg, thr, out_bits):
    res = O.forward(x, rw, ex, cfg.E, cfg.k, thr=thr)
    keep = ~O.near_tie_flags(res["gap"])
    ov = res["out64"][keep]
    rms = np.sqrt(np.mean(ov ** 2))
    half = np.exp2(np.floor(np.log2(np.maximum(np.abs(ov), 2.0 ** -126))) - 8)
    assert np.all(np.abs(O.bf16_bits_to_f64(out_bits[keep]) - ov) <= 1e-2 * rms + half)


@pytest.mark.parametrize("G,T,thr", [(2, 37, 128), (4, 300, 64), (8, 5, 128)])
def test_virtual_ranks_match_single_device_and_oracle(G, T, thr):
    cfg = W.custom_config(T=T, d=512, E=16, k=4, f=256, seed=160 + G, router="unit")
    x, rw = W.gen_x_router(cfg)
    ex = W.gen_experts(cfg)
    dev = experts_to_device(ex)
    rwd = torch.from_numpy(rw).cuda()
    single = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
    single.load_experts(dev)
    single.set_dense_threshold(thr)
    ref = bf16_to_bits(single(to_dev_x(x), rwd))
    Eq = cfg.E // G
    backends = [CudaEpBackend(cfg.E, cfg.k, cfg.d, cfg.f, r, G, shard_experts(dev, r * Eq, (r + 1) * Eq), rwd)
                for r in range(G)]
    for b in backends:
        b.expert_handle.set_dense_threshold(thr)
    xs = [to_dev_x(s) for s in np.array_split(x, G)]
    outs = ep_forward_local(backends, xs)
    torch.cuda.synchronize()
    assert all(b.device_error() == 0 for b in backends)
    got = np.concatenate([bf16_to_bits(o) for o in outs])
    _close_to_single_device(got, ref)
    _oracle_check(x, rw, ex, cfg, thr, got)
    for b in backends:
        b.close()


def test_routed_rows_reject_out_of_range_experts():
    from nvfp4_expert_layer_b200 import _lib
    cfg = W.custom_config(T=6, d=512, E=4, k=1, f=256, seed=171)
    h = MoeFp4Layer(cfg.E, 1, cfg.d, cfg.f)
    h.load_experts(experts_to_device(W.gen_experts(cfg)))
    x, _ = W.gen_x_router(cfg)
    b = CudaEpBackend.__new__(CudaEpBackend)
    b.lib, b.d, b.expert_handle = _lib.load(), cfg.d, h
    ids = torch.tensor([0, 1, 2, 3, 4, 1], dtype=torch.int32, device="cuda")
    b.forward_routed(to_dev_x(x), ids)
    torch.cuda.synchronize()
    assert h.device_error() == _lib.STATUS_CODE["MOE_FP4_ERR_INVALID_ARG"]


_NCCL_RANK = r'''
import os, sys, datetime
import numpy as np, torch, torch.distributed as dist
sys.path.insert(0, sys.argv[1])
from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.ep import CudaEpBackend, ep_forward
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
torch.cuda.set_device(0)
dist.init_process_group("nccl", init_method="tcp://127.0.0.1:" + sys.argv[2], rank=0, world_size=1,
                        timeout=datetime.timedelta(seconds=60))
cfg = W.custom_config(T=21, d=512, E=8, k=2, f=256, seed=172, router="unit")
x, rw = W.gen_x_router(cfg)
dev = experts_to_device(W.gen_experts(cfg))
rwd = torch.from_numpy(rw).cuda()
xd = torch.from_numpy(x.view(np.int16).copy()).cuda().view(torch.bfloat16)
single = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
single.load_experts(dev)
ref = single(xd, rwd).view(torch.int16).cpu().numpy()
b = CudaEpBackend(cfg.E, cfg.k, cfg.d, cfg.f, 0, 1, dev, rwd)
out = ep_forward(b, xd).view(torch.int16).cpu().numpy()
torch.cuda.synchronize()
f = lambda v: (v.view(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
a, r = f(out), f(ref)
ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(r), 2.0 ** -126))) - 7)
ok = bool(np.all(np.abs(a - r) <= ulp + 1e-5 * np.sqrt(np.mean(r ** 2))))
print("close", ok, "err", b.device_error(), flush=True)
b.close()
dist.destroy_process_group()
sys.exit(0 if ok else 3)
'''


def test_one_rank_nccl_all_to_all_path():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", _NCCL_RANK, ROOT, str(port)], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "err 0" in r.stdout
