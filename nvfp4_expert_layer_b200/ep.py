"""Expert parallelism for the NVFP4 MoE layer: experts sharded over G ranks.

Rank r owns the contiguous experts [r E/G, (r+1) E/G) and the tokens of its
own batch.  One forward of a rank ("Optimizing Muse Spark Open on TPU v7
with SGLang-TorchTPU", section 8, "Sequence-parallel prefill": each device
keeps its own tokens, routing travels with them and the MoE output returns
through an all-to-all; "Day-0 Inference Adaptation for Ultra-Large Sparse
Models": expert-parallel deployment):

  1. route its tokens (router weights replicated): ids, weights, per-expert
     counts, the permutation by (expert, token, slot) and its inverse;
  2. gather the token row of every (token, expert) pair in permutation
     order.  The permutation sorts pairs by expert, so the rows bound for
     rank q are one contiguous run: positions [offsets[q E/G],
     offsets[(q+1) E/G]);
  3. all-to-all: row counts, then the rows (bf16) and their expert ids;
  4. the local experts on the received rows (one expert per row, weight 1:
     unweighted fp32 outputs y).  An expert's row count on its owner is its
     count over all ranks' tokens, so its class (light / dense) is the one a
     single device would choose for the whole batch;
  5. all-to-all back: y returns to the pair's rank in the order it was sent,
     i.e. permutation order;
  6. combine: out[t] = bf16( sum_j fl(w[t,j] * y[inv[t,j]]) ).

Steps 1, 2, 4 and 6 run in the library's CUDA kernels (CudaEpBackend);
this module holds only the index arithmetic of the exchange and the
collective calls.  The exchange is NCCL's all-to-all through
torch.distributed (remote rows land in local HBM before any kernel reads
them), or, for tests, a backend and an exchange on the host."""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib


class EpPlan:
    """Ownership and exchange sizes: rank q owns experts [q Eq, (q+1) Eq)."""

    def __init__(self, E: int, world: int):
        if E % world:
            raise ValueError(f"E = {E} experts do not split evenly over {world} ranks")
        self.E, self.world, self.Eq = E, world, E // world

    def owner_range(self, q: int):
        return q * self.Eq, (q + 1) * self.Eq

    def send_counts(self, counts) -> list:
        """Rows this rank sends to each rank: its pairs per owner."""
        c = np.asarray(counts, dtype=np.int64).reshape(self.world, self.Eq)
        return c.sum(axis=1).tolist()


def shard_experts(experts: dict, lo: int, hi: int) -> dict:
    """Experts [lo, hi) of canonical expert tensors (dim 0 is the expert)."""
    return {n: t[lo:hi].contiguous() for n, t in experts.items()}


# ---------------------------------------------------------------------------
# device side: the library's kernels through the C ABI
# ---------------------------------------------------------------------------

def _p(t):
    return ctypes.c_void_p(t.data_ptr())


class CudaEpBackend:
    """One rank's device work.  Holds a routing handle over all E experts (no
    expert weights) and a handle with this rank's E/G experts (top_k = 1)."""

    def __init__(self, E: int, k: int, d: int, f: int, rank: int, world: int, local_experts: dict,
                 router_w: torch.Tensor):
        from .layer import MoeFp4Layer
        self.lib = _lib.load()
        self.plan = EpPlan(E, world)
        self.E, self.k, self.d, self.f, self.rank = E, k, d, f, rank
        self.router_w = router_w
        self.route_handle = MoeFp4Layer(E, k, d, f)
        self.expert_handle = MoeFp4Layer(self.plan.Eq, 1, d, f)
        self.expert_handle.load_experts(local_experts)

    def _stream(self):
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def route(self, x: torch.Tensor) -> dict:
        T, dev = x.shape[0], x.device
        P = T * self.k
        out = {"ids": torch.empty((T, self.k), dtype=torch.int32, device=dev),
               "w": torch.empty((T, self.k), dtype=torch.float32, device=dev),
               "counts": torch.empty((self.E,), dtype=torch.int32, device=dev),
               "offsets": torch.empty((self.E + 1,), dtype=torch.int32, device=dev),
               "perm": torch.empty((P,), dtype=torch.int32, device=dev),
               "inv": torch.empty((P,), dtype=torch.int32, device=dev)}
        r = _lib.Routing()
        r.topk_ids, r.topk_w, r.counts = out["ids"].data_ptr(), out["w"].data_ptr(), out["counts"].data_ptr()
        r.offsets, r.perm, r.inv = out["offsets"].data_ptr(), out["perm"].data_ptr(), out["inv"].data_ptr()
        _lib.check(self.lib.moe_fp4_route(self.route_handle._h, _p(x), T, _p(self.router_w), ctypes.byref(r),
                                          self._stream()), "moe_fp4_route")
        return out

    def gather_rows(self, x: torch.Tensor, perm: torch.Tensor) -> torch.Tensor:
        P = perm.numel()
        rows = torch.empty((P, self.d), dtype=x.dtype, device=x.device)
        _lib.check(self.lib.moe_fp4_gather_rows(_p(x), x.shape[0], self.d, _p(perm), P, self.k, _p(rows),
                                                self._stream()), "moe_fp4_gather_rows")
        return rows

    def pair_experts(self, R: dict) -> torch.Tensor:
        """Global expert of every pair in permutation order."""
        return R["ids"].reshape(-1)[R["perm"].long()].contiguous()

    def forward_routed(self, rows: torch.Tensor, local_ids: torch.Tensor) -> torch.Tensor:
        n = rows.shape[0]
        y = torch.empty((n, self.d), dtype=torch.float32, device=rows.device)
        if n:
            _lib.check(self.lib.moe_fp4_forward_routed(self.expert_handle._h, _p(rows), n, _p(local_ids), _p(y),
                                                       self._stream()), "moe_fp4_forward_routed")
        return y

    def combine(self, y: torch.Tensor, R: dict) -> torch.Tensor:
        T = R["ids"].shape[0]
        out = torch.empty((T, self.d), dtype=torch.bfloat16, device=y.device)
        _lib.check(self.lib.moe_fp4_combine_rows(_p(y), _p(R["inv"]), _p(R["w"]), T, self.k, self.d, _p(out),
                                                 self._stream()), "moe_fp4_combine_rows")
        return out

    def device_error(self) -> int:
        return max(self.route_handle.device_error(), self.expert_handle.device_error())

    def close(self):
        self.route_handle.close()
        self.expert_handle.close()


# ---------------------------------------------------------------------------
# the forward, in three local stages around two exchanges
# ---------------------------------------------------------------------------

def dispatch_prep(backend, x):
    """Stages 1-2: routing, the gathered rows in permutation order, their
    global experts, and the rows this rank sends to every rank."""
    R = backend.route(x)
    rows = backend.gather_rows(x, R["perm"])
    gids = backend.pair_experts(R)
    send = backend.plan.send_counts(R["counts"].cpu().numpy())
    return R, rows, gids, send


def ep_forward(backend, x, group=None):
    """One rank's expert-parallel forward through torch.distributed
    (all-to-all over `group`, NCCL for device tensors)."""
    import torch.distributed as dist
    R, rows, gids, send = dispatch_prep(backend, x)
    sc = torch.tensor(send, dtype=torch.int64, device=rows.device)
    rc = torch.empty_like(sc)
    dist.all_to_all_single(rc, sc, group=group)
    recv = rc.cpu().tolist()
    # rows travel as raw bytes (bf16 is not an all-to-all type on every backend)
    rb = rows.view(torch.uint8) if rows.element_size() == 2 else rows
    rows_in = rb.new_empty((sum(recv), rb.shape[1]))
    dist.all_to_all_single(rows_in, rb, output_split_sizes=recv, input_split_sizes=send, group=group)
    rows_in = rows_in.view(rows.dtype)
    gids_in = gids.new_empty((sum(recv),))
    dist.all_to_all_single(gids_in, gids, output_split_sizes=recv, input_split_sizes=send, group=group)
    lo, _ = backend.plan.owner_range(dist.get_rank(group))
    y_in = backend.forward_routed(rows_in, (gids_in - lo).to(torch.int32).contiguous())
    y_back = y_in.new_empty((rows.shape[0], y_in.shape[1]))
    dist.all_to_all_single(y_back, y_in, output_split_sizes=send, input_split_sizes=recv, group=group)
    return backend.combine(y_back, R)


def ep_forward_local(backends, xs):
    """The same forward for G ranks held in one process (each backend one
    rank): the all-to-alls become slices and concatenations.  Used to test
    the sharded path on one device and on the host."""
    G = len(backends)
    preps = [dispatch_prep(b, x) for b, x in zip(backends, xs)]
    starts = [np.concatenate([[0], np.cumsum(p[3])]) for p in preps]      # send offsets per source
    ys = []
    for q, b in enumerate(backends):
        rows_in = torch.cat([preps[s][1][starts[s][q]:starts[s][q + 1]] for s in range(G)])
        gids_in = torch.cat([preps[s][2][starts[s][q]:starts[s][q + 1]] for s in range(G)])
        lo, _ = b.plan.owner_range(q)
        ys.append(b.forward_routed(rows_in, (gids_in - lo).to(torch.int32).contiguous()))
    outs = []
    for s, b in enumerate(backends):
        parts = []
        for q in range(G):                    # rank q received, in source order, before s: sum of their sends
            base = sum(preps[src][3][q] for src in range(s))
            n = preps[s][3][q]
            parts.append(ys[q][base:base + n])
        outs.append(b.combine(torch.cat(parts), preps[s][0]))
    return outs
