"""Run the CUDA layer and compare it with the oracle on the same seeded inputs.

Parity contract, applied per compared token (near-tie tokens excluded):
  - ids and the permutation bit-exact, except near-tie tokens (k-th vs
    (k+1)-th fp64 logit closer than 1e-6) and mismatches explained by the
    fp32 dot-product error bound of the two logits involved;
  - router logits within the fp32 dot-product bound gamma_{d+1} sum|x w|;
  - routing weights within max(1e-5, 2 delta + 4 delta^2 + (k + 8) 2^-24)
    relative, delta the largest |layer logit - oracle logit| among the
    token's selected experts (itself checked against the fp32 bound above):
    the renormalised top-k softmax moves by at most e^(2 delta) - 1 when its
    logits move by at most delta; the rest covers exp, the sum and the
    division in fp32;
  - h element-wise within the propagated fp32 accumulation bound
    (d+2) 2^-24 (|Wg||x|, |Wu||x|) through SiLU(g)*u, times 2 for second
    order terms;
  - partial element-wise within |w| 2^-10 (|Wd||h|): h enters the down
    projection as fp16 (relative rounding 2^-11), doubled for the fp32
    accumulation and the propagated error of h;
  - dense-class rows (experts with n_e >= thr, where x and h are NVFP4): the
    same h bound over the quantised x (the quantiser's decisions on x are the
    same fp32 operations on both sides); partial within |w| (|Wd| dev +
    gamma_f (|Wd||hq| + |Wd| dev)), where dev bounds, element by element, how
    far the layer's quantised h can sit from the oracle's when h moves inside
    its bound (a block scale or a code may round the other way), and gamma_f
    = (f + 2) 2^-24 + 2^-22 covers the fp32 accumulation and epilogue scaling;
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


def dense_supported(cfg) -> bool:
    """The layer's dense class needs d and f to be multiples of 256."""
    return cfg.d % 256 == 0 and cfg.f % 256 == 0


def _widen32(v, up):
    """fp32 value on the far side of v (v * (1 +- 2^-22) rounded to fp32)."""
    f = 1.0 + 2.0 ** -22 if up else 1.0 - 2.0 ** -22
    return (np.asarray(v, np.float64) * f).astype(np.float32)


def quant_deviation(h, hb):
    """Bound on |q(v) - q(h32)| per element for every v with |v - h| <= hb.

    q is the oracle's NVFP4 activation quantiser (block of 16, sf =
    e4m3_rn(amax/6), code = e2m1_rn(v/sf), decisions in fp32).  The block
    scale is monotone in amax and each code is monotone in v for a fixed
    scale, so the candidates are every e4m3 value between the scales of the
    smallest and the largest possible amax, each with the codes at both ends
    of the element's interval."""
    n, K = h.shape
    _, _, hq = O.quantize_act_nvfp4(h.astype(np.float32))
    lo = _widen32(h - hb, up=False).astype(np.float64)
    hi = _widen32(h + hb, up=True).astype(np.float64)
    lo, hi = np.minimum(lo, hi), np.maximum(lo, hi)
    amag_lo = np.where((lo <= 0) & (hi >= 0), 0.0, np.minimum(np.abs(lo), np.abs(hi)))
    amag_hi = np.maximum(np.abs(lo), np.abs(hi))
    a_lo = amag_lo.reshape(n, K // 16, 16).max(-1)
    a_hi = amag_hi.reshape(n, K // 16, 16).max(-1)
    s_lo = O.e4m3_rne_satfinite((a_lo.astype(np.float32) / np.float32(6.0)).astype(np.float32))
    s_hi = O.e4m3_rne_satfinite((a_hi.astype(np.float32) / np.float32(6.0)).astype(np.float32))
    grid = O.E4M3_POSITIVE
    i_lo = np.searchsorted(grid, s_lo)
    i_hi = np.searchsorted(grid, s_hi)
    assert np.all(grid[i_lo] == s_lo) and np.all(grid[i_hi] == s_hi)
    dev = np.zeros_like(h)
    for j in range(int((i_hi - i_lo).max()) + 1):
        sf = grid[np.minimum(i_lo + j, i_hi)]
        sfe = np.repeat(sf, 16, axis=-1)
        sf32 = sfe.astype(np.float32)
        safe = np.where(sf32 == 0, np.float32(1), sf32)
        for v in (lo, hi):
            r = (v.astype(np.float32) / safe).astype(np.float32)
            q = np.where(sf32 == 0, 0.0, O.e2m1_decode(O.e2m1_rne_satfinite_codes(r)) * sfe)
            dev = np.maximum(dev, np.abs(q - hq))
    return dev, hq


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
        # without dense-class support every expert runs in the light class
        thr = self.thr if dense_supported(self.cfg) else 1 << 40
        self.o = O.forward(self.x, self.rw, self.experts, self.cfg.E, self.cfg.k, thr=thr,
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
        delta = np.take_along_axis(dl, o["ids"], axis=1).max(axis=1)
        w_rtol = np.maximum(W_RTOL, 2 * delta + 4 * delta ** 2 + (cfg.k + 8) * U32)[:, None]
        dw = np.abs(g["topk_w"].astype(np.float64) - o["w"])
        bad = (dw > w_rtol * np.abs(o["w"]) + 1e-7) & keep[:, None]
        assert not bad.any(), f"routing weights: {int(bad.sum())} outside the derived tolerance"
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

    def dense_rows(self, ro):
        """Mask of oracle rows whose expert ran in the dense class."""
        o = self.o
        if not dense_supported(self.cfg):
            return np.zeros(len(ro), bool)
        e = np.searchsorted(o["offsets"], ro, side="right") - 1
        return o["counts"][e] >= self.thr

    def check_intermediates(self):
        rows = self._rows()
        g, o, m = self.g, self.o, self.o["mags"]
        d, f = self.cfg.d, self.cfg.f
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
        dense = self.dense_rows(ro)
        self.n_dense_rows = int(dense.sum())
        if dense.any():     # partial = w * (Wd q(h)): quantiser decisions may flip inside the h bound
            gam = (f + 2) * U32 + 2.0 ** -22
            e_of = np.searchsorted(o["offsets"], ro, side="right") - 1
            for e in np.unique(e_of[dense]):
                sel = np.nonzero(dense & (e_of == e))[0]
                dev, _ = quant_deviation(o["h"][ro[sel]], hb[sel])
                Wd_abs = np.abs(O.dequant_nvfp4(*self.experts.expert(int(e))[2]))
                flip = dev @ Wd_abs.T
                pb[sel] = wpair[sel, None] * (flip + gam * (m["yabs"][ro[sel]] + flip)) + 1e-30
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
