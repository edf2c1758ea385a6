"""GPU parity of the dense expert class (tcgen05 block-scaled NVFP4 GEMMs).

Experts that receive at least `thr` rows quantise x and h to NVFP4 and run on
the FP4 tensor cores; the oracle applies the same activation quantiser
(reading R4) and the parity helpers bound the effect of quantiser decisions
that may round the other way when h moves inside its accumulation bound."""
import os

import numpy as np
import pytest
import torch

from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from oracle import moe_oracle as O
from tests.parity import Case, bf16_to_bits, to_dev_x

pytestmark = pytest.mark.gpu


def _run(cfg, thr, **kw):
    c = Case(cfg, thr=thr, **kw).run_gpu().run_oracle()
    c.check_all()
    return c


@pytest.fixture(params=["pairs", "single"])
def gemm_tiles(request, monkeypatch):
    """The dense GEMMs on CTA pairs (256 x 256 tiles) or on single CTAs
    (128-row tiles, the default); the choice is read when a layer is created."""
    monkeypatch.setenv("MOE_FP4_DENSE_PAIRS", "1" if request.param == "pairs" else "0")
    return request.param


def test_dense_tiny_every_expert_dense(gemm_tiles):
    # thr = 1: every active expert is dense; each holds <= 4 rows of a token tile
    c = _run(W.CONFIGS["tiny"], thr=1)
    assert c.n_dense_rows == c.cfg.T * c.cfg.k


def test_dense_and_light_classes_small_batch():
    # 32 pairs (the small-batch routing path): experts with >= 3 rows dense, the rest light
    cfg = W.custom_config(T=4, d=512, E=16, k=8, f=256, seed=56, router="unit")
    c = _run(cfg, thr=3)
    counts = c.o["counts"]
    assert np.any(counts >= 3) and np.any((counts > 0) & (counts < 3)), counts
    assert 0 < c.n_dense_rows < cfg.T * cfg.k


def test_dense_ragged_multi_tile_experts(gemm_tiles):
    # ~175 rows per expert: two 128-token tiles (one 256-token pair tile), the second ragged
    cfg = W.custom_config(T=700, d=512, E=8, k=2, f=512, seed=51, router="unit")
    c = _run(cfg, thr=64)
    counts = c.o["counts"]
    assert np.any((counts > 128) & (counts % 128 != 0))
    assert c.n_dense_rows > 0


def test_dense_and_light_classes_in_one_call(gemm_tiles):
    cfg = W.custom_config(T=600, d=1024, E=16, k=4, f=768, seed=52, router="unit")
    c = Case(cfg, thr=150).run_gpu().run_oracle()
    counts = c.o["counts"]
    assert np.any(counts >= 150) and np.any((counts > 0) & (counts < 150)), counts
    c.check_all()
    assert 0 < c.n_dense_rows < cfg.T * cfg.k


def test_dense_threshold_is_inclusive():
    cfg = W.custom_config(T=300, d=512, E=8, k=2, f=256, seed=53, router="unit")
    x, rw = W.gen_x_router(cfg)
    ex = W.gen_experts(cfg)
    probe = Case(cfg, thr=1 << 30, experts=ex, x=x, rw=rw).run_oracle()
    counts = np.sort(probe.o["counts"][probe.o["counts"] > 0])
    thr = int(counts[len(counts) // 2])          # one expert sits exactly at thr
    c = _run(cfg, thr=thr, experts=ex, x=x, rw=rw)
    assert np.any(c.o["counts"] == thr)
    # compared rows of experts at or above thr are exactly the dense rows
    ro = c._rows()[:, 1]
    e_of = np.searchsorted(c.o["offsets"], ro, side="right") - 1
    assert c.n_dense_rows == int(np.sum(c.o["counts"][e_of] >= thr)) > 0


def test_dense_unsupported_shape_runs_light():
    # d = 384 is not a multiple of 256: every expert stays in the light class
    cfg = W.custom_config(T=40, d=384, E=4, k=2, f=256, seed=54, router="unit")
    c = _run(cfg, thr=1)
    assert c.n_dense_rows == 0


def test_dense_deterministic_and_graph_replay():
    cfg = W.custom_config(T=400, d=512, E=8, k=2, f=256, seed=55, router="unit")
    x, rw = W.gen_x_router(cfg)
    layer = MoeFp4Layer(cfg.E, cfg.k, cfg.d, cfg.f)
    layer.load_experts(experts_to_device(W.gen_experts(cfg)))
    layer.set_dense_threshold(32)
    layer.reserve(cfg.T)
    xd, rwd = to_dev_x(x), torch.from_numpy(rw).cuda()
    a = bf16_to_bits(layer(xd, rwd))
    b = bf16_to_bits(layer(xd, rwd))
    assert np.array_equal(a, b)
    out = torch.empty_like(xd)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            layer(xd, rwd, out=out, stream=s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert np.array_equal(bf16_to_bits(out), a)


def _cover_every_tile(ids, E, tile=128, seed=0):
    """Tokens such that every (expert, 128-row tile of its permuted rows) holds
    at least one of their pairs: walk the tiles, and for a tile no chosen
    token covers yet, take a random token of it."""
    rng = np.random.default_rng(seed)
    T, k = ids.shape
    counts, offsets, perm, _ = O.permute(ids, E)
    tile_of = np.empty(T * k, np.int64)              # pair -> global tile id
    tid = 0
    starts = []
    for e in range(E):
        for r0 in range(offsets[e], offsets[e + 1], tile):
            r1 = min(r0 + tile, offsets[e + 1])
            tile_of[perm[r0:r1]] = tid
            starts.append((r0, r1))
            tid += 1
    covered = np.zeros(tid, bool)
    chosen = []
    for t_id, (r0, r1) in enumerate(starts):
        if covered[t_id]:
            continue
        tok = int(perm[rng.integers(r0, r1)] // k)
        chosen.append(tok)
        covered[tile_of[tok * k:(tok + 1) * k]] = True
    return sorted(chosen), tid


def test_prefill_full_size_every_expert_tile():
    # 8 x 2048 tokens, d = 7168, E = 256, k = 8, f = 2048: every expert dense.
    # One row or more of every (expert, 128-token tile) is compared element by
    # element, so every expert and every tile position of the persistent
    # schedulers is covered; the oracle's per-expert work runs in a spawned
    # process pool (started before any work in it touches the GPU).
    import multiprocessing as mp
    cfg = W.CONFIGS["prefill"]
    x, rw = W.gen_x_router(cfg)
    ids, _, _ = O.route(O.router_logits(x, rw), cfg.k)
    toks, ntiles = _cover_every_tile(ids, cfg.E)
    workers = max(1, min(16, (os.cpu_count() or 2) - 1))
    with mp.get_context("spawn").Pool(workers) as pool:
        c = Case(cfg, token_subset=toks, x=x, rw=rw, oracle_experts=W.LazyExperts(cfg),
                 map_fn=pool.map).run_gpu().run_oracle()
        assert np.all(c.o["counts"] >= 128)
        c.check_all()
    rows = c._rows()
    assert c.n_dense_rows == len(rows) > 0
    # every (expert, tile) position holds a compared row
    e_of = np.searchsorted(c.o["offsets"], rows[:, 1], side="right") - 1
    seen = set(zip(e_of.tolist(), ((rows[:, 1] - c.o["offsets"][e_of]) // 128).tolist()))
    assert len(seen) >= ntiles - c.n_excluded * cfg.k, (len(seen), ntiles)
