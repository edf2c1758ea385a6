"""A host backend for the expert-parallel exchange tests: the oracle's
arithmetic on CPU tensors in place of the library's kernels, so the index
math and the collectives of nvfp4_expert_layer_b200.ep run without a GPU
(test infrastructure; it calls only oracle/ and the input generators)."""
import numpy as np
import torch

from nvfp4_expert_layer_b200.ep import EpPlan
from oracle import moe_oracle as O


class HostEpBackend:
    def __init__(self, E, k, d, f, rank, world, experts, router_w, thr=128):
        self.plan = EpPlan(E, world)
        self.E, self.k, self.d, self.f, self.rank, self.thr = E, k, d, f, rank, thr
        self.experts = experts                   # .expert(e) for the global expert id
        self.router_w = router_w
        self.lo, _ = self.plan.owner_range(rank)

    def route(self, x):
        xb = x.numpy().view(np.uint16)
        ids, w, _ = O.route(O.router_logits(xb, self.router_w), self.k)
        counts, offsets, perm, inv = O.permute(ids, self.E)
        t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).astype(dt))
        return {"ids": t(ids, np.int32), "w": t(w, np.float64), "counts": t(counts, np.int32),
                "offsets": t(offsets, np.int32), "perm": t(perm, np.int32), "inv": t(inv, np.int32)}

    def gather_rows(self, x, perm):
        return x[perm.long() // self.k].contiguous()

    def pair_experts(self, R):
        return R["ids"].reshape(-1)[R["perm"].long()].contiguous()

    def forward_routed(self, rows, local_ids):
        xb = rows.numpy().view(np.uint16)
        ids = local_ids.numpy()
        y = np.zeros((len(ids), self.d))
        for le in np.unique(ids):
            sel = np.nonzero(ids == le)[0]
            mats = self.experts.expert(int(le) + self.lo)
            Wg, Wu, Wd = (O.dequant_nvfp4(*mats[m]) for m in (0, 1, 2))
            _, y[sel] = O.expert_ffn(O.bf16_bits_to_f64(xb[sel]), Wg, Wu, Wd, quantized=len(sel) >= self.thr)
        return torch.from_numpy(y)

    def combine(self, y, R):
        w, inv = R["w"].numpy(), R["inv"].numpy()
        T = w.shape[0]
        out = np.zeros((T, self.d))
        for j in range(self.k):
            out += w[:, j:j + 1] * y.numpy()[inv[np.arange(T) * self.k + j]]
        return torch.from_numpy(out)
