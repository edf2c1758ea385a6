"""The seeded generators: shapes, determinism and value distributions."""
import numpy as np

from nvfp4_expert_layer_b200 import workloads as W
from oracle import moe_oracle as O


def test_tiny_shapes_and_determinism():
    cfg = W.CONFIGS["tiny"]
    x1, r1, e1 = W.gen_all(cfg)
    x2, r2, e2 = W.gen_all(cfg)
    assert x1.shape == (4, 512) and x1.dtype == np.uint16
    assert r1.shape == (8, 512) and r1.dtype == np.float32
    assert e1.gate_q.shape == (8, 256, 256) and e1.gate_sf.shape == (8, 256, 32)
    assert e1.down_q.shape == (8, 512, 128) and e1.down_sf.shape == (8, 512, 16)
    for a, b in ((x1, x2), (r1, r2), (e1.down_q, e2.down_q), (e1.up_sf, e2.up_sf)):
        assert np.array_equal(a, b)
    assert np.all(np.isfinite(O.e4m3fn_decode(e1.gate_sf)))


def test_weight_distribution_close_to_requested():
    cfg = W.CONFIGS["tiny"]
    ex = W.gen_experts(cfg)
    Wg = O.dequant_nvfp4(ex.gate_q[1], ex.gate_sf[1], ex.gate_gs[1])
    assert 0.017 < Wg.std() < 0.023
    assert abs(Wg.mean()) < 1e-3


def test_pooled_matrix_matches_per_expert_regeneration():
    cfg = W.custom_config(T=1, d=2048, E=4, k=2, f=2560, seed=3, router="unit")  # 5.2M > 2^22
    ex = W.gen_experts(cfg)
    q, sf, gs = W.gen_expert_matrix(cfg, 2, W.DOWN)
    assert np.array_equal(q, ex.down_q[2]) and np.array_equal(sf, ex.down_sf[2]) and gs == ex.down_gs[2]
    Wd = O.dequant_nvfp4(q, sf, gs)
    assert 0.013 < Wd.std() < 0.027
    assert len(set(ex.gate_gs.tolist())) == cfg.E      # per-tensor scales differ


def test_router_recipes():
    z = W.CONFIGS["decode64"]
    x, rw = W.gen_x_router(z)
    xf = W.bf16_bits_to_f32(x)
    assert np.all(xf[:, -1] == 1.0)
    p = np.exp(rw[:, -1].astype(np.float64))
    np.testing.assert_allclose(p.sum(), 1.0, rtol=1e-5)
    v = W.CONFIGS["verify"]
    x, rw = W.gen_x_router(v)
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    L = xf @ rw.T.astype(np.float64)
    same = np.mean([np.corrcoef(L[4 * r], L[4 * r + 1])[0, 1] for r in range(32)])
    other = np.mean([np.corrcoef(L[4 * r], L[4 * r + 4])[0, 1] for r in range(31)])
    assert 0.7 < same < 0.9 and abs(other) < 0.2
