"""Run the CUDA layer and compare it with the oracle on the same seeded inputs.

Parity contract, applied per compared token (near-tie tokens excluded):
  - ids and the permutation bit-exact, except near-tie tokens (k-th vs
    (k+1)-th fp64 logit closer than 1e-6) and mismatches explained by the
    fp32 dot-product error bound of the two logits involved;
  - router logits within the fp32 dot-product bound gamma_{d+1} sum|x w|;
  - routing weights within 1e-5 relative;
  - h element-wise within the propagated fp32 accumulation bound
    (d+2) 2^-24 (|Wg||x|, |Wu||x|) through SiLU(g)*u, times 2 for second
    order terms;
  - partial element-wise within |w| 2^-10 (|Wd||h|): h enters the down
    projection as fp16 (relative rounding 2^-11), doubled for the fp32
    accumulation and the propagated error of h;
  - out: the bf16 output is exactly bf16_rn of the fp32 slot-order sum of the
    partials; that fp32 sum is within 1e-2 * rms(out_oracle) of the oracle's
    exact output; the bf16 output is within 1e-2 * rms + half a bf16 ulp (the
    layer's own final rounding) of it."""
from __future__ import annotations

import numpy as np
import torch

from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from oracle import moe_oracle as O

OUT_TOL = 1e-2
W_RTOL = 1e-5
U32 = 2.0 ** -24


def silu_prime(z):
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def to_dev_x(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_bits.view(np.int16).copy()).cuda().view(torch.bfloat16)


def bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class Case:
    """Inputs, the CUDA layer's results and the oracle's for one config."""

    def __init__(self, cfg, thr=128, layer=None, experts=None, token_subset=None, x=None, rw=None):
        self.cfg = cfg
        self.thr = thr
        if x is None:
            x, rw = W.gen_x_router(cfg)
        self.x, self.rw = x, rw
        self.experts = experts if experts is not None else W.gen_experts(cfg)
        self.layer = layer
        self.token_subset = token_subset

    def run_gpu(self):
        if self.layer is None:
            self.layer = MoeFp4Layer(self.cfg.E, self.cfg.k, self.cfg.d, self.cfg.f)
            self.layer.load_experts(experts_to_device(self.experts))
        self.layer.set_dense_threshold(self.thr)
        xd = to_dev_x(self.x)
        rwd = torch.from_numpy(self.rw).cuda()
        out, dbg = self.layer.forward_ex(xd, rwd)
        torch.cuda.synchronize()
        self.err = self.layer.device_error()
        self.g = {n: t.cpu().numpy() for n, t in dbg.items()}
        self.g["out_bits"] = bf16_to_bits(out)
        return self

    def run_oracle(self):
        self.o = O.forward(self.x, self.rw, self.experts, self.cfg.E, self.cfg.k, thr=self.thr,
                           token_subset=self.token_subset, magnitudes=True)
        return self

    # ------------------------------------------------------------- checks
    def check_routing(self):
        cfg, g, o = self.cfg, self.g, self.o
        bound = O.fp32_logit_error_bound(self.x, self.rw)
        dl = np.abs(g["logits"].astype(np.float64) - o["logits"])
        assert np.all(dl <= bound), f"logit error {dl.max()} above the fp32 bound"
        flagged = O.near_tie_flags(o["gap"])
        explained = np.zeros(cfg.T, bool)
        for t in np.nonzero(np.any(g["topk_ids"] != o["ids"], axis=1))[0]:
            if flagged[t]:
                continue
            a = set(o["ids"][t].tolist()) ^ set(g["topk_ids"][t].tolist())
            lt = o["logits"][t]
            kth = np.sort(lt)[::-1][cfg.k - 1]
            ok = all(abs(lt[e] - kth) <= 2 * bound[t].max() for e in a) or \
                sorted(o["ids"][t]) == sorted(g["topk_ids"][t])
            assert ok, f"token {t}: unexplained id mismatch {o['ids'][t]} vs {g['topk_ids'][t]}"
            explained[t] = True
        self.skip = flagged | explained
        keep = ~self.skip
        assert np.array_equal(g["topk_ids"][keep], o["ids"][keep])
        np.testing.assert_allclose(g["topk_w"][keep], o["w"][keep], rtol=W_RTOL, atol=1e-7)
        if not self.skip.any():
            assert np.array_equal(g["counts"], o["counts"])
            assert np.array_equal(g["offsets"], o["offsets"])
            assert np.array_equal(g["perm"], o["perm"])
        else:   # property check of the GPU permutation of its own ids
            ids = g["topk_ids"].reshape(-1)
            perm = g["perm"]
            assert np.array_equal(np.sort(perm), np.arange(perm.size))
            keys = ids[perm].astype(np.int64) * perm.size + perm
            assert np.all(np.diff(keys) > 0)
        return self

    def _rows(self):
        """(gpu_row, oracle_row) for pairs of compared tokens with oracle values."""
        k = self.cfg.k
        inv_o = self.o["inv"]
        rows = []
        toks = self.o["tokens"]
        want = np.zeros(self.cfg.T, bool)
        want[toks] = True
        for r, pair in enumerate(self.g["perm"]):
            t = pair // k
            if want[t] and not self.skip[t]:
                rows.append((r, inv_o[pair]))
        return np.array(rows, dtype=np.int64).reshape(-1, 2)

    def check_intermediates(self):
        rows = self._rows()
        g, o, m = self.g, self.o, self.o["mags"]
        d = self.cfg.d
        ro, rg = rows[:, 1], rows[:, 0]
        # h = SiLU(g) * u with g, u accumulated in fp32
        dg = (d + 2) * U32 * m["gabs"][ro]
        du = (d + 2) * U32 * m["uabs"][ro]
        gg, uu = m["g"][ro], m["u"][ro]
        sil = gg / (1.0 + np.exp(-gg))
        hb = 2.0 * (np.abs(silu_prime(gg) * uu) * dg + np.abs(sil) * du) + 16 * U32 * np.abs(o["h"][ro])
        hg = g["h"][rg].astype(np.float64)
        assert np.all(np.isfinite(hg)), "h: unwritten rows"
        excess = np.abs(hg - o["h"][ro]) - hb - 1e-30
        assert np.all(excess <= 0), f"h: {np.sum(excess > 0)} elements outside the bound"
        # partial = w * (Wd h16)
        wpair = np.abs(o["w"].reshape(-1)[o["perm"][ro]])
        pb = wpair[:, None] * (2.0 ** -10) * m["yabs"][ro] + 1e-30
        pg = g["partial"][rg].astype(np.float64)
        assert np.all(np.isfinite(pg)), "partial: unwritten rows"
        excess = np.abs(pg - o["partial"][ro]) - pb
        assert np.all(excess <= 0), f"partial: {np.sum(excess > 0)} elements outside the bound"
        return self

    def check_out(self):
        k = self.cfg.k
        toks = np.array([t for t in self.o["tokens"] if not self.skip[t]], dtype=np.int64)
        inv_g = np.argsort(self.g["perm"])
        # the combine: fp32 sum of the k partials in slot order, then bf16_rn
        s32 = np.zeros((len(toks), self.cfg.d), np.float32)
        for j in range(k):
            s32 = (s32 + self.g["partial"][inv_g[toks * k + j]].astype(np.float32)).astype(np.float32)
        assert np.array_equal(O.f64_to_bf16_bits_rne(s32.astype(np.float64)), self.g["out_bits"][toks]), \
            "out is not bf16_rn of the fp32 slot-order sum of the partials"
        ov = self.o["out64"][toks]
        rms = np.sqrt(np.mean(ov ** 2))
        pre = np.abs(s32.astype(np.float64) - ov).max()
        self.out_err_rel = pre / rms
        assert pre <= OUT_TOL * rms, f"out (pre-rounding): max err {pre:.3e} > {OUT_TOL} * rms {rms:.3e}"
        gv = O.bf16_bits_to_f64(self.g["out_bits"][toks])
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ov), 2.0 ** -126))) - 8)
        assert np.all(np.abs(gv - ov) <= OUT_TOL * rms + half_ulp), "out (bf16) outside tolerance"
        return self

    def check_all(self):
        assert self.err == 0, f"device error word {self.err}"
        return self.check_routing().check_intermediates().check_out()
