"""Run the CUDA layer and compare it with the oracle on the same seeded inputs.

Parity contract, applied per compared token:
  - ids: the GPU's selected expert set of every token equals the oracle's,
    except near-tie tokens (k-th vs (k+1)-th fp64 logit closer than 1e-6) and
    tokens whose differing experts all sit within twice the fp32 dot-product
    bound of the k-th logit ("explained").  Both kinds are excluded from the
    numeric checks, counted, and capped (exclude_cap).  A token whose set
    matches but whose listing order differs must have every misordered pair
    of experts within twice the fp32 bound of each other; such a token stays
    in every check, its rows matched by (token, expert);
  - counts, offsets bit-exact, and the permutation bit-exact as the sequence
    of (token, expert) keys it lists, when no token is excluded (the
    permutation is also checked bit-exact as pair indices when no token's
    order differs); otherwise the GPU permutation is checked to be the
    stable (expert, pair) order of its own ids;
  - router logits within the fp32 dot-product bound gamma_{d+1} sum|x w|;
  - routing weights within max(1e-5, 2 delta + 4 delta^2 + (k + 8) 2^-24)
    relative, delta the largest |layer logit - oracle logit| among the
    token's selected experts: the renormalised top-k softmax moves by at most
    e^(2 delta) - 1 when its logits move by at most delta; the rest covers
    exp, the sum and the division in fp32;
  - h element-wise within the propagated fp32 accumulation bound
    (d+2) 2^-24 (|Wg||x|, |Wu||x|) through SiLU(g)*u, times 2 for second
    order terms;
  - every partial additionally within (w_rtol |w| + 2^-149) |Wd||h|: the
    layer's fp32 routing weight carries the weight tolerance above;
  - light-class partial element-wise within |w| (2^-10 |Wd||h| + 2 L1d hfl):
    h enters the down projection as fp16 after a power-of-two scale 2^e_h
    (relative rounding 2^-11, doubled for the fp32 accumulation and the
    propagated error of h), plus the fp16 subnormal floor: an element of h
    loses at most 2^-25 2^-e_h absolutely, and the layer's choice of e_h
    implies 2^-e_h <= 2^-10 L1g L1u xmax^2 (L1 = largest row L1 norm of the
    expert's matrix, xmax = max|x| of the token), so hfl = 2^-35 L1g L1u xmax^2;
  - dense-class rows (experts with n_e >= thr, where x and h are NVFP4): the
    same h bound over the quantised x; partial within |w| (|Wd| dev +
    gamma_f (|Wd||hq| + |Wd| dev)), where dev bounds, element by element, how
    far the layer's quantised h can sit from the oracle's when h moves inside
    its bound (a block scale or a code may round the other way), and gamma_f
    = (f + 2) 2^-24 + 2^-22 covers the fp32 accumulation and epilogue scaling;
  - out: the bf16 output is exactly bf16_rn of the fp32 slot-order sum of the
    partials; that fp32 sum is within 1e-2 * rms(out_oracle) of the oracle's
    exact output; the bf16 output is within 1e-2 * rms + half a bf16 ulp (the
    layer's own final rounding) of it.  Quantiser near ties: a dense-class h
    element inside its fp32 bound of an NVFP4 rounding midpoint may round
    either way on the two sides, like a routing near tie; the propagated
    effect of such elements (|w| |Wd| dev, the flip term above) is allowed on
    top of 1e-2 * rms, and the output elements that need it are counted.  With the per-expert norm the GPU's
    partials are the unweighted expert outputs y; the fp64 value
    sum_j w_j y_j / sqrt(mean y_j^2 + eps) of the GPU's own partials must be
    within 1e-2 * rms of the oracle, and the bf16 output within half an ulp
    (plus 1e-5 relative for the fp32 combine) of that value."""
from __future__ import annotations

import math
import os

import numpy as np
import torch

from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from oracle import moe_oracle as O
from tests._oracle_tasks import abs_wd_times

OUT_TOL = 1e-2
# one summary per checked case of this session (printed by tests/conftest.py)
PARITY_REPORT = []
W_RTOL = 1e-5
U32 = 2.0 ** -24


def exclude_cap(T: int) -> int:
    """Largest number of excluded tokens a case may have: 2 plus 1 % of T."""
    return 2 + T // 100


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


def bf16_ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> int:
    """Largest distance, in bf16 ulps of the reference value b, between two
    arrays of bf16 bit patterns, over the elements with |b| >= rms(b) / 64
    (near zero an ulp is tiny and the absolute tolerance governs)."""
    a = O.bf16_bits_to_f64(np.asarray(a_bits))
    b = O.bf16_bits_to_f64(np.asarray(b_bits))
    if not b.size:
        return 0
    big = (np.abs(b) >= np.sqrt(np.mean(b * b)) / 64) & (b != 0)
    if not big.any():
        return 0
    ulp = np.exp2(np.floor(np.log2(np.abs(b[big]))) - 7)
    return int(np.round(np.abs(a[big] - b[big]) / ulp).max())


def oracle_pool(workers: int = 16):
    """A spawned process pool for the oracle's per-expert work (spawn: a
    forked child of a process that has touched the GPU can hang)."""
    import multiprocessing as mp
    return mp.get_context("spawn").Pool(max(1, min(workers, (os.cpu_count() or 2) - 1)))


class Case:
    """Inputs, the CUDA layer's results and the oracle's for one config."""

    def __init__(self, cfg, thr=128, layer=None, experts=None, token_subset=None, x=None, rw=None,
                 norm_eps=None, oracle_experts=None, map_fn=map, oracle_thr=None, act_dynamic=False,
                 residual=False):
        self.cfg = cfg
        self.thr = thr
        # the class threshold the oracle applies (by default the layer's)
        self.oracle_thr = oracle_thr
        if x is None:
            x, rw = W.gen_x_router(cfg)
        self.x, self.rw = x, rw
        self.experts = experts if experts is not None else W.gen_experts(cfg)
        # what the oracle reads the experts from (a LazyExperts for process pools)
        self.oracle_experts = oracle_experts if oracle_experts is not None else self.experts
        self.layer = layer
        self.token_subset = token_subset
        self.norm_eps = norm_eps
        self.map_fn = map_fn
        self.act_dynamic = act_dynamic
        self.residual = residual

    def run_gpu(self):
        if self.layer is None:
            self.layer = MoeFp4Layer(self.cfg.E, self.cfg.k, self.cfg.d, self.cfg.f)
            self.layer.load_experts(experts_to_device(self.experts))
        self.layer.set_dense_threshold(self.thr)
        self.layer.set_expert_norm(self.norm_eps is not None, 0.0 if self.norm_eps is None else self.norm_eps)
        self.layer.set_act_scale(self.act_dynamic)
        self.layer.set_residual(self.residual)
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
        if self.oracle_thr is not None:
            thr = self.oracle_thr
        self.o = O.forward(self.x, self.rw, self.oracle_experts, self.cfg.E, self.cfg.k, thr=thr,
                           token_subset=self.token_subset, magnitudes=True,
                           expert_norm_eps=self.norm_eps, map_fn=self.map_fn,
                           act_scale="dynamic" if self.act_dynamic else "fixed", residual=self.residual)
        if self.act_dynamic and self.o["h_amax"]:
            # the two sides pick the same power of two for h unless max|h| sits
            # within h's fp32 error of a boundary 6 * 448 * 2^e (checked here)
            r = math.log2(self.o["h_amax"] / 2688.0)
            assert abs(r - round(r)) > 1e-4, "seeded input has max|h| on a tensor-scale boundary"
        return self

    # ------------------------------------------------------------- checks
    def check_routing(self):
        cfg, g, o = self.cfg, self.g, self.o
        k = cfg.k
        bound = O.fp32_logit_error_bound(self.x, self.rw)
        dl = np.abs(g["logits"].astype(np.float64) - o["logits"])
        assert np.all(dl <= bound), f"logit error {dl.max()} above the fp32 bound"
        flagged = O.near_tie_flags(o["gap"])
        gi, oi = g["topk_ids"], o["ids"]
        same_set = np.all(np.sort(gi, axis=1) == np.sort(oi, axis=1), axis=1)
        self.near_tie = np.zeros(cfg.T, bool)
        self.explained = np.zeros(cfg.T, bool)
        for t in np.nonzero(~same_set)[0]:
            if flagged[t]:
                self.near_tie[t] = True
                continue
            lt = o["logits"][t]
            kth = lt[oi[t, k - 1]]
            diff = set(oi[t].tolist()) ^ set(gi[t].tolist())
            assert all(abs(lt[e] - kth) <= 2 * bound[t].max() for e in diff), \
                f"token {t}: unexplained id mismatch {oi[t]} vs {gi[t]}"
            self.explained[t] = True
        self.skip = self.near_tie | self.explained
        self.n_excluded = int(self.skip.sum())
        assert self.n_excluded <= exclude_cap(cfg.T), \
            f"{self.n_excluded} excluded tokens ({int(self.near_tie.sum())} near ties) > cap {exclude_cap(cfg.T)}"
        # same set, other order: every misordered pair must be an fp32 near-tie
        self.reordered = same_set & np.any(gi != oi, axis=1)
        for t in np.nonzero(self.reordered)[0]:
            lt = o["logits"][t]
            rank_o = {e: j for j, e in enumerate(oi[t].tolist())}
            seq = gi[t].tolist()
            for a in range(k):
                for b in range(a + 1, k):
                    if rank_o[seq[a]] > rank_o[seq[b]]:
                        assert abs(lt[seq[a]] - lt[seq[b]]) <= 2 * bound[t].max(), \
                            f"token {t}: listing order {gi[t]} vs {oi[t]} not explained by fp32"
        # weights, matched by expert
        keep = ~self.skip
        order_g = np.argsort(gi, axis=1)
        order_o = np.argsort(oi, axis=1)
        wg = np.take_along_axis(g["topk_w"].astype(np.float64), order_g, axis=1)
        wo = np.take_along_axis(o["w"], order_o, axis=1)
        delta = np.take_along_axis(dl, oi, axis=1).max(axis=1)
        w_rtol = np.maximum(W_RTOL, 2 * delta + 4 * delta ** 2 + (k + 8) * U32)[:, None]
        self.w_rtol_tok = w_rtol[:, 0]          # the weights' own error enters every partial
        bad = (np.abs(wg - wo) > w_rtol * np.abs(wo) + 1e-7) & keep[:, None]
        assert not bad.any(), f"routing weights: {int(bad.sum())} outside the derived tolerance"
        # permutation
        P = cfg.T * k
        key_g = (g["perm"] // k).astype(np.int64) * cfg.E + gi.reshape(-1)[g["perm"]]
        if self.n_excluded == 0:
            assert np.array_equal(g["counts"], o["counts"])
            assert np.array_equal(g["offsets"], o["offsets"])
            key_o = (o["perm"] // k).astype(np.int64) * cfg.E + oi.reshape(-1)[o["perm"]]
            assert np.array_equal(key_g, key_o), "permutation: (token, expert) sequence differs"
            if not self.reordered.any():
                assert np.array_equal(g["perm"], o["perm"])
        ids = gi.reshape(-1)
        perm = g["perm"]
        assert np.array_equal(np.sort(perm), np.arange(P))
        keys = ids[perm].astype(np.int64) * P + perm
        assert np.all(np.diff(keys) > 0), "permutation is not the stable (expert, pair) order"
        return self

    def _rows(self):
        """(gpu_row, oracle_row) for the pairs of compared tokens with oracle
        values, matched by (token, expert)."""
        k = self.cfg.k
        inv_o = self.o["inv"]
        gi, oi = self.g["topk_ids"], self.o["ids"]
        want = np.zeros(self.cfg.T, bool)
        want[self.o["tokens"]] = True
        rows = []
        for r, pair in enumerate(self.g["perm"]):
            t = pair // k
            if want[t] and not self.skip[t]:
                e = gi[t, pair % k]
                jo = int(np.nonzero(oi[t] == e)[0][0])
                rows.append((r, inv_o[t * k + jo]))
        return np.array(rows, dtype=np.int64).reshape(-1, 2)

    def dense_rows(self, ro):
        """Mask of oracle rows whose expert ran in the dense class."""
        o = self.o
        thr = self.oracle_thr if self.oracle_thr is not None else self.thr
        if not dense_supported(self.cfg) and self.oracle_thr is None:
            return np.zeros(len(ro), bool)
        e = np.searchsorted(o["offsets"], ro, side="right") - 1
        return o["counts"][e] >= thr

    def check_intermediates(self):
        rows = self._rows()
        self.n_rows_compared = len(rows)
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
        # partial = w * (Wd h16) (light); with the norm the partial is the unweighted y
        wpair = np.abs(o["w"].reshape(-1)[o["perm"][ro]])
        wscale = np.ones_like(wpair) if self.norm_eps is not None else wpair
        # the layer's fp32 routing weight is within w_rtol |w| (+ 2^-149 below
        # fp32's range) of the oracle's; that error scales the whole partial
        wrt = np.zeros_like(wpair) if self.norm_eps is not None else \
            self.w_rtol_tok[o["perm"][ro] // self.cfg.k] * wpair + 2.0 ** -149
        hfl = 2.0 ** -35 * m["l1g"][ro, 0] * m["l1u"][ro, 0] * m["xmax"][ro, 0] ** 2
        pb = wscale[:, None] * ((2.0 ** -10) * m["yabs"][ro] + (2 * hfl * m["l1d"][ro, 0])[:, None]) + \
            wrt[:, None] * m["yabs"][ro] + 1e-30
        dense = self.dense_rows(ro)
        self.n_dense_rows = int(dense.sum())
        self.flip_rows = {}      # GPU row -> |Wd| dev: effect of h codes that may round either way
        if dense.any():     # partial = w * (Wd q(h)): quantiser decisions may flip inside the h bound
            gam = (f + 2) * U32 + 2.0 ** -22
            e_of = np.searchsorted(o["offsets"], ro, side="right") - 1
            tasks, sels = [], []
            for e in np.unique(e_of[dense]):
                sel = np.nonzero(dense & (e_of == e))[0]
                gh = o["gs_h"]                  # h quantised as h / gs_h (1 unless dynamic)
                dev, _ = quant_deviation(o["h"][ro[sel]] / gh, hb[sel] / gh)
                tasks.append((self.oracle_experts, int(e), dev * gh))
                sels.append(sel)
            for sel, flip in zip(sels, self.map_fn(abs_wd_times, tasks)):
                pb[sel] = wscale[sel, None] * (flip + gam * (m["yabs"][ro[sel]] + flip)) + \
                    wrt[sel, None] * (m["yabs"][ro[sel]] + flip) + 1e-30
                for n_i, r in enumerate(rg[sel]):
                    self.flip_rows[int(r)] = flip[n_i]
        ref = o["y"][ro] if self.norm_eps is not None else o["partial"][ro]
        pg = g["partial"][rg].astype(np.float64)
        assert np.all(np.isfinite(pg)), "partial: unwritten rows"
        excess = np.abs(pg - ref) - pb
        assert np.all(excess <= 0), f"partial: {np.sum(excess > 0)} elements outside the bound"
        return self

    def check_out(self):
        k = self.cfg.k
        toks = np.array([t for t in self.o["tokens"] if not self.skip[t]], dtype=np.int64)
        self.n_tokens_compared = len(toks)
        inv_g = np.argsort(self.g["perm"])
        ov = self.o["out64"][toks]
        rms = np.sqrt(np.mean(ov ** 2))
        gv = O.bf16_bits_to_f64(self.g["out_bits"][toks])
        self.ulp_distance = bf16_ulp_distance(self.g["out_bits"][toks], self.o["out_bits"][toks])
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ov), 2.0 ** -126))) - 8)
        if self.norm_eps is not None:
            # the GPU's own partials (unweighted y), normalised and weighted in fp64
            wg = self.g["topk_w"].astype(np.float64)
            pre = O.bf16_bits_to_f64(self.x[toks]) if self.residual else np.zeros((len(toks), self.cfg.d))
            for j in range(k):
                y = self.g["partial"][inv_g[toks * k + j]].astype(np.float64)
                pre += wg[toks, j][:, None] * O.expert_rms_norm(y, self.norm_eps)
            hu = np.exp2(np.floor(np.log2(np.maximum(np.abs(pre), 2.0 ** -126))) - 8)
            # fp32 combine: the norm factors and a sum of k terms, relative to the terms' magnitudes
            mag = np.abs(O.bf16_bits_to_f64(self.x[toks])) if self.residual else np.zeros_like(pre)
            for j in range(k):
                y = self.g["partial"][inv_g[toks * k + j]].astype(np.float64)
                mag += np.abs(wg[toks, j][:, None] * O.expert_rms_norm(y, self.norm_eps))
            assert np.all(np.abs(gv - pre) <= hu + (k + 8) * 2.0 ** -23 * mag + 1e-30), \
                "out is not bf16 of its combine"
        else:
            # the combine: fp32 sum of the k partials in slot order, then bf16_rn
            s32 = (O.bf16_bits_to_f64(self.x[toks]).astype(np.float32) if self.residual
                   else np.zeros((len(toks), self.cfg.d), np.float32))
            for j in range(k):
                s32 = (s32 + self.g["partial"][inv_g[toks * k + j]].astype(np.float32)).astype(np.float32)
            assert np.array_equal(O.f64_to_bf16_bits_rne(s32.astype(np.float64)), self.g["out_bits"][toks]), \
                "out is not bf16_rn of the fp32 slot-order sum of the partials"
            pre = s32.astype(np.float64)
        # quantiser near ties: a dense-class h element within its fp32 bound of an
        # NVFP4 rounding midpoint may round either way on the two sides (the
        # analogue of a routing near tie); its propagated effect (the flip term
        # of the partial bound) is allowed on top of the tolerance and counted
        allow = np.zeros_like(pre)
        if getattr(self, "flip_rows", None):
            wo = self.g["topk_w"].astype(np.float64)
            for j in range(k):
                rows = inv_g[toks * k + j]
                for i, r in enumerate(rows):
                    fl = self.flip_rows.get(int(r))
                    if fl is None:
                        continue
                    if self.norm_eps is None:
                        allow[i] += np.abs(wo[toks[i], j]) * fl
                    else:
                        y = self.g["partial"][r].astype(np.float64)
                        rr = math.sqrt(np.mean(y * y) + self.norm_eps)
                        allow[i] += 1.1 * np.abs(wo[toks[i], j]) * (fl / rr + np.abs(y) / rr *
                                                                   math.sqrt(np.mean(fl * fl)) / rr)
        e_el = np.abs(pre - ov)
        err = e_el.max() if len(toks) else 0.0
        self.out_err_rel = err / rms if rms > 0 else (0.0 if err == 0 else math.inf)
        self.flip_elems = int(np.sum(e_el > OUT_TOL * rms))
        assert np.all(e_el <= OUT_TOL * rms + allow), \
            f"out (pre-rounding): max err {err:.3e} > {OUT_TOL} * rms {rms:.3e} (+ quantiser near-tie allowance)"
        assert np.all(np.abs(gv - ov) <= OUT_TOL * rms + allow + half_ulp), "out (bf16) outside tolerance"
        return self

    def check_all(self):
        assert self.err == 0, f"device error word {self.err}"
        self.check_routing().check_intermediates().check_out()
        name = os.environ.get("PYTEST_CURRENT_TEST", self.cfg.name).split(" ")[0]
        PARITY_REPORT.append((name, self.summary()))
        return self

    def summary(self) -> dict:
        return dict(excluded=self.n_excluded, near_tie=int(self.near_tie.sum()),
                    explained=int(self.explained.sum()), reordered=int(self.reordered.sum()),
                    rows=self.n_rows_compared, tokens=self.n_tokens_compared,
                    out_err_over_rms=self.out_err_rel, ulp=self.ulp_distance, flip_elems=self.flip_elems)
