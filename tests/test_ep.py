"""Expert parallelism on the host: the exchange's index math and collectives
(nvfp4_expert_layer_b200.ep) with the oracle's arithmetic in place of the
kernels.  G ranks each own E/G experts and a slice of the tokens; the
sharded forward must give every token the output the single-device oracle
gives it (fp64, up to summation order).  Two of the tests run the ranks as
gloo processes, one holds G ranks in one process."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.ep import EpPlan, ep_forward, ep_forward_local
from oracle import moe_oracle as O
from tests._ep_host_backend import HostEpBackend

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_plan_ownership_and_send_counts():
    plan = EpPlan(8, 4)
    assert [plan.owner_range(q) for q in range(4)] == [(0, 2), (2, 4), (4, 6), (6, 8)]
    assert plan.send_counts([1, 0, 3, 2, 0, 0, 5, 1]) == [1, 5, 0, 6]
    with pytest.raises(ValueError):
        EpPlan(10, 4)


def _setup(cfg, world):
    x, rw = W.gen_x_router(cfg)
    ex = W.gen_experts(cfg)
    xs = np.array_split(x, world)                 # ragged token slices
    return x, rw, ex, xs


@pytest.mark.parametrize("world,thr", [(2, 128), (4, 128), (4, 6)])
def test_sharded_forward_matches_oracle_in_one_process(world, thr):
    cfg = W.custom_config(T=13, d=128, E=8, k=3, f=128, seed=140 + world, router="unit")
    x, rw, ex, xs = _setup(cfg, world)
    backends = [HostEpBackend(cfg.E, cfg.k, cfg.d, cfg.f, r, world, ex, rw, thr) for r in range(world)]
    outs = ep_forward_local(backends, [torch.from_numpy(s.view(np.int16).copy()) for s in xs])
    ref = O.forward(x, rw, ex, cfg.E, cfg.k, thr=thr)["out64"]
    np.testing.assert_allclose(np.concatenate([o.numpy() for o in outs]), ref, rtol=1e-11, atol=1e-13)


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        cfg = W.custom_config(T=11, d=128, E=8, k=2, f=128, seed=150, router="unit")
        x, rw, ex, xs = _setup(cfg, world)
        b = HostEpBackend(cfg.E, cfg.k, cfg.d, cfg.f, rank, world, ex, rw)
        out = ep_forward(b, torch.from_numpy(xs[rank].view(np.int16).copy()))
        q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_the_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = W.custom_config(T=11, d=128, E=8, k=2, f=128, seed=150, router="unit")
    x, rw = W.gen_x_router(cfg)
    ref = O.forward(x, rw, W.gen_experts(cfg), cfg.E, cfg.k)["out64"]
    np.testing.assert_allclose(np.concatenate([res[0], res[1]]), ref, rtol=1e-11, atol=1e-13)
