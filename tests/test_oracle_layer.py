"""Pins for the oracle's layer arithmetic: brute force, closed forms, invariants."""
import os

import numpy as np
import pytest

from nvfp4_expert_layer_b200 import workloads as W
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split()
            vals[key] = val
    return vals


class _ArrayExperts:
    def __init__(self, mats):
        self.mats = mats

    def expert(self, e):
        return self.mats[e]


def _tiny():
    cfg = W.CONFIGS["tiny"]
    x, rw, ex = W.gen_all(cfg)
    return cfg, x, rw, ex


# ---------------------------------------------------------------- routing

def test_route_matches_brute_force_sort():
    cfg, x, rw, _ = _tiny()
    logits = O.router_logits(x, rw)
    ids, w, gap = O.route(logits, cfg.k)
    for t in range(cfg.T):
        order = sorted(range(cfg.E), key=lambda e: (-logits[t, e], e))
        assert ids[t].tolist() == order[:cfg.k]
        # softmax restricted to S equals the renormalised full softmax
        sel = logits[t, order[:cfg.k]]
        ref = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
        np.testing.assert_allclose(w[t], ref, rtol=1e-14)
        assert gap[t] == logits[t, order[cfg.k - 1]] - logits[t, order[cfg.k]]


def test_route_invariants_and_ties():
    logits = np.array([[0.5, 2.0, 2.0, -1.0, 2.0, 0.1]])
    ids, w, gap = O.route(logits, 2)
    assert ids.tolist() == [[1, 2]]              # three-way tie: lowest indices win
    assert gap[0] == 0.0 and O.near_tie_flags(gap)[0]
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(w[0], [0.5, 0.5])
    rng = np.random.default_rng(3)
    L = rng.standard_normal((50, 32))
    ids, w, _ = O.route(L, 5)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)
    sel = np.take_along_axis(L, ids, axis=1)
    assert np.all(np.diff(sel, axis=1) <= 0)        # listed by descending logit
    assert np.all(np.diff(w, axis=1) <= 1e-15)


def test_router_logits_fp64_dot():
    cfg, x, rw, _ = _tiny()
    xf = W.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.array([[sum(float(a) * float(b) for a, b in zip(xf[t], rw[e]))
                     for e in range(cfg.E)] for t in range(cfg.T)])
    np.testing.assert_allclose(O.router_logits(x, rw), ref, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- permutation

def test_permute_invariants_and_brute_force():
    rng = np.random.default_rng(11)
    E, T, k = 16, 37, 4
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = O.permute(ids, E)
    assert np.array_equal(counts, np.bincount(ids.ravel(), minlength=E))
    assert offsets[0] == 0 and offsets[E] == T * k
    assert np.array_equal(perm[inv], np.arange(T * k))
    assert np.array_equal(inv[perm], np.arange(T * k))
    brute = [t * k + j for e in range(E) for t in range(T) for j in range(k) if ids[t, j] == e]
    assert perm.tolist() == brute


# ---------------------------------------------------------------- layer

def _dense_brute_force(x_bits, rw, experts, E, k, thr):
    """Every expert on every token, times a gate that is zero outside the top-k."""
    logits = O.router_logits(x_bits, rw)
    ids, w, _ = O.route(logits, k)
    T = x_bits.shape[0]
    G = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            G[t, ids[t, j]] = w[t, j]
    counts = np.bincount(ids.ravel(), minlength=E)
    x = O.bf16_bits_to_f64(x_bits)
    out = np.zeros_like(x)
    for e in range(E):
        mats = experts.expert(e)
        Wg, Wu, Wd = (O.dequant_nvfp4(*mats[m]) for m in (0, 1, 2))
        quant = counts[e] >= thr
        xin = np.stack([O.quantize_act_nvfp4(x[t])[2] for t in range(T)]) if quant else x
        g = np.einsum("fd,td->tf", Wg, xin)
        u = np.einsum("fd,td->tf", Wu, xin)
        h = g / (1 + np.exp(-g)) * u
        if quant:
            h = np.stack([O.quantize_act_nvfp4(h[t].astype(np.float32))[2] for t in range(T)])
        y = np.einsum("df,tf->td", Wd, h)
        out += G[:, e:e + 1] * y
    return out


@pytest.mark.parametrize("thr", [128, 1])
def test_layer_matches_dense_brute_force(thr):
    cfg, x, rw, ex = _tiny()
    res = O.forward(x, rw, ex, cfg.E, cfg.k, thr=thr)
    ref = _dense_brute_force(x, rw, ex, cfg.E, cfg.k, thr)
    np.testing.assert_allclose(res["out64"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.array_equal(res["out_bits"], O.f64_to_bf16_bits_rne(ref))


def test_single_expert_top1_is_dense_swiglu():
    cfg = W.custom_config(T=5, d=64, E=1, k=1, f=32, seed=9)
    x, rw, ex = W.gen_all(cfg)
    res = O.forward(x, rw, ex, 1, 1, thr=1 << 30)
    assert np.all(res["w"] == 1.0)
    Wg, Wu, Wd = (O.dequant_nvfp4(*ex.expert(0)[m]) for m in (0, 1, 2))
    xf = O.bf16_bits_to_f64(x)
    g, u = xf @ Wg.T, xf @ Wu.T
    ref = (g * (1.0 / (1.0 + np.exp(-g))) * u) @ Wd.T      # textbook SwiGLU FFN
    np.testing.assert_allclose(res["out64"], ref, rtol=1e-13, atol=1e-13)


def test_hand_worked_example():
    gold = _read_golden("hand_example_d16.txt")
    d = f = 16
    q = np.full((f, d // 2), 0x22, np.uint8)
    sf = np.full((f, d // 16), 0x38, np.uint8)
    mats = {0: {0: (q, sf, np.float32(1)), 1: (q, sf, np.float32(1)), 2: (q, sf, np.float32(1))}}
    x = np.full((1, d), 0x3F80, np.uint16)
    rw = np.zeros((1, d), np.float32)
    res = O.forward(x, rw, _ArrayExperts(mats), 1, 1, thr=1 << 30)
    assert res["h"][0, 0] == pytest.approx(float(gold["h"]), rel=1e-15)
    assert res["out64"][0, 0] == pytest.approx(float(gold["y"]), rel=1e-15)
    assert np.all(res["out_bits"] == int(gold["out_bf16_bits"], 16))


def test_weighted_combine_scales_with_routing_weight():
    # Dropping the routing weight or a pair would break linearity in w.
    cfg, x, rw, ex = _tiny()
    res = O.forward(x, rw, ex, cfg.E, cfg.k)
    for t in range(cfg.T):
        acc = np.zeros(cfg.d)
        for j in range(cfg.k):
            acc += res["partial"][res["inv"][t * cfg.k + j]]
        np.testing.assert_allclose(res["out64"][t], acc, rtol=1e-13, atol=1e-15)
        # each partial is w * y; recover y and recompute
        e = res["ids"][t, 0]
        pos = res["inv"][t * cfg.k]
        mats = ex.expert(e)
        Wg, Wu, Wd = (O.dequant_nvfp4(*mats[m]) for m in (0, 1, 2))
        xf = O.bf16_bits_to_f64(x[t])
        g, u = Wg @ xf, Wu @ xf
        y = Wd @ (g / (1 + np.exp(-g)) * u)
        np.testing.assert_allclose(res["partial"][pos], res["w"][t, 0] * y, rtol=1e-12)


def test_token_subset_matches_full():
    cfg, x, rw, ex = _tiny()
    full = O.forward(x, rw, ex, cfg.E, cfg.k)
    sub = O.forward(x, rw, ex, cfg.E, cfg.k, token_subset=[2])
    np.testing.assert_allclose(sub["out64"][2], full["out64"][2], rtol=1e-13, atol=1e-16)
    assert not np.any(sub["out64"][0])


def test_quantized_class_changes_result_but_stays_close():
    cfg, x, rw, ex = _tiny()
    a16 = O.forward(x, rw, ex, cfg.E, cfg.k, thr=128)["out64"]
    a4 = O.forward(x, rw, ex, cfg.E, cfg.k, thr=1)["out64"]
    rel = np.sqrt(np.mean((a4 - a16) ** 2)) / np.sqrt(np.mean(a16 ** 2))
    assert 1e-3 < rel < 0.5


def test_fp32_bound_is_conservative():
    cfg, x, rw, _ = _tiny()
    xf = W.bf16_bits_to_f32(x)
    l32 = (xf.astype(np.float32) @ rw.T.astype(np.float32)).astype(np.float64)
    l64 = O.router_logits(x, rw)
    assert np.all(np.abs(l32 - l64) <= O.fp32_logit_error_bound(x, rw))
