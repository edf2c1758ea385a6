"""Run the CUDA layer and compare it with the oracle on the same seeded inputs.

Tolerances (the layer's parity contract):
  - ids and the permutation bit-exact, except near-tie tokens (k-th vs
    (k+1)-th fp64 logit closer than 1e-6) and mismatches explained by the
    fp32 dot-product error bound of the two logits involved;
  - router logits within the fp32 dot-product bound;
  - routing weights within 1e-5 relative;
  - h and partial rows within 2e-3 * rms of the oracle's (fp32 accumulation
    and fp16 operand staging; NVFP4 activation rounding for dense experts
    is identical on both sides);
  - out: max |out - out_oracle| <= 1e-2 * rms(out_oracle) over compared tokens."""
from __future__ import annotations

import numpy as np
import torch

from nvfp4_expert_layer_b200 import workloads as W
from nvfp4_expert_layer_b200.layer import MoeFp4Layer, experts_to_device
from oracle import moe_oracle as O

OUT_TOL = 1e-2
INTER_TOL = 2e-3
W_RTOL = 1e-5


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
                           token_subset=self.token_subset)
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
        for name in ("h", "partial"):
            gv = self.g[name][rows[:, 0]].astype(np.float64)
            ov = self.o[name][rows[:, 1]]
            assert np.all(np.isfinite(gv)), f"{name}: unwritten rows"
            rms = np.sqrt(np.mean(ov ** 2))
            err = np.abs(gv - ov).max()
            assert err <= INTER_TOL * rms, f"{name}: max err {err:.3e} > {INTER_TOL} * rms {rms:.3e}"
        return self

    def check_out(self):
        toks = np.array([t for t in self.o["tokens"] if not self.skip[t]], dtype=np.int64)
        gv = O.bf16_bits_to_f64(self.g["out_bits"][toks])
        ov = self.o["out64"][toks]
        rms = np.sqrt(np.mean(ov ** 2))
        err = np.abs(gv - ov).max()
        self.out_err_rel = err / rms
        assert err <= OUT_TOL * rms, f"out: max err {err:.3e} > {OUT_TOL} * rms {rms:.3e}"
        return self

    def check_all(self):
        assert self.err == 0, f"device error word {self.err}"
        return self.check_routing().check_intermediates().check_out()
