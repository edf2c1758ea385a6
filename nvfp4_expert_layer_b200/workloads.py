"""Seeded synthetic workloads for the NVFP4 sparse-MoE layer forward.

This module only *generates inputs*: token activations, router weights and
NVFP4-encoded expert weights in the canonical layout that
``moe_fp4_load_experts`` accepts.  It holds none of the layer's arithmetic
(routing, dequantisation, the expert FFN, the combine); both the CPU oracle and
the CUDA path consume the arrays it returns.

Shapes follow the sparse-MoE layer described in "Optimizing Muse Spark Open on
TPU v7 with SGLang-TorchTPU" (Background: 256 experts, 8 routed per token,
NVFP4 experts with one scale per 16 values) and the workloads that page and
"Optimizing Models to Be Fast at Codegen" (section 2) describe: batch-1
decode, a batch of decode tokens, a block-draft verify step and a chunked
prefill.

Canonical NVFP4 layout (row-major, one matrix per expert):
  q   uint8 [rows][K/2]   two e2m1 codes per byte, element 2i in the low nibble
  sf  uint8 [rows][K/16]  e4m3fn block scale; block i covers elements 16i..16i+15
  gs  float32             one per-tensor scale per (expert, matrix)
gate/up matrices are [f][d] (K = d); the down matrix is [d][f] (K = f).

Expert weights are drawn as N(0, 0.02) and encoded to NVFP4 with the
generator's own nearest-value encoder.  Matrices with more than 2**22
elements are assembled from a seeded pool of 2**16 independently encoded
16-value blocks (block indices drawn per expert and matrix), with a per-tensor
scale jittered by a seeded factor in [0.75, 1.25): this keeps every block an
encoded draw of 16 i.i.d. N(0, 0.02) values while making the 6.3 GB of a
256-expert layer cheap to generate.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GATE, UP, DOWN = 0, 1, 2
_POOL_BLOCKS = 1 << 16
_DIRECT_LIMIT = 1 << 22
_W_STD = 0.02


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int          # tokens (rows of x)
    d: int          # model width
    E: int          # experts
    k: int          # experts per token
    f: int          # expert FFN width
    seed: int
    router: str     # 'gauss002' | 'unit' | 'zipf' | 'verify'
    requests: int = 0   # verify: number of requests (T = requests * draft)

    @property
    def pairs(self) -> int:
        return self.T * self.k


CONFIGS = {
    # Tiny layer: x ~ N(0,1), router ~ N(0, 0.02), seed 0.
    "tiny": LayerConfig("tiny", T=4, d=512, E=8, k=2, f=256, seed=0, router="gauss002"),
    # Batch-1 decode: router ~ N(0, 1/d) so logits ~ N(0,1); near-uniform routing.
    "decode1": LayerConfig("decode1", T=1, d=7168, E=256, k=8, f=2048, seed=1, router="unit"),
    # Decode batch 64 with Zipf(1.1)-biased routing.
    "decode64": LayerConfig("decode64", T=64, d=7168, E=256, k=8, f=2048, seed=2, router="zipf"),
    # Block-draft verify: 32 requests x 4 draft tokens, logits correlated 0.8 within a request.
    "verify": LayerConfig("verify", T=128, d=7168, E=256, k=8, f=2048, seed=3, router="verify",
                          requests=32),
    # Prefill 8 x 2048 tokens, near-uniform routing (~512 tokens per expert).
    "prefill": LayerConfig("prefill", T=16384, d=7168, E=256, k=8, f=2048, seed=4, router="unit"),
}


def custom_config(name="custom", T=4, d=512, E=8, k=2, f=256, seed=0, router="gauss002",
                  requests=0) -> LayerConfig:
    return LayerConfig(name, T=T, d=d, E=E, k=k, f=f, seed=seed, router=router, requests=requests)


# ----------------------------------------------------------------------------
# bf16 helpers (bit patterns stored as uint16; numpy has no bf16 dtype)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits_trunc(a: np.ndarray) -> np.ndarray:
    """Random-input helper: keep the top 16 bits of each float32 (truncation)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# The generator's own NVFP4 encoder (nearest representable value, ties to the
# code whose lowest bit is 0).  Only used to make weights.
# ----------------------------------------------------------------------------

def _e4m3_positive_grid():
    vals = []
    for code in range(0x7F):          # 0x7F is NaN
        e, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


_E4M3_GRID = _e4m3_positive_grid()
_E2M1_GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def _nearest_code(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to mag (mag >= 0), ties to the even index."""
    mag = np.minimum(mag, grid[-1])
    hi = np.clip(np.searchsorted(grid, mag, side="left"), 1, len(grid) - 1)
    lo = hi - 1
    dlo = mag - grid[lo]
    dhi = grid[hi] - mag
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo).astype(np.uint8)


def encode_nvfp4(w: np.ndarray):
    """Encode a float matrix [rows][K] (K % 16 == 0) to (q, sf, gs)."""
    w = np.asarray(w, dtype=np.float64)
    rows, K = w.shape
    amax = float(np.max(np.abs(w))) if w.size else 0.0
    gs = np.float32(amax / (6.0 * 448.0)) if amax > 0 else np.float32(1.0)
    blocks = w.reshape(rows, K // 16, 16)
    bmax = np.max(np.abs(blocks), axis=2)
    sf_code = _nearest_code(bmax / (6.0 * float(gs)), _E4M3_GRID)
    sf_val = _E4M3_GRID[sf_code]
    denom = (sf_val * float(gs))[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(denom > 0, blocks / np.where(denom > 0, denom, 1.0), 0.0)
    mag = _nearest_code(np.abs(ratio), _E2M1_GRID)
    codes = mag | np.where(ratio < 0, 8, 0).astype(np.uint8)
    codes = np.where(mag == 0, 0, codes).astype(np.uint8)       # no negative zero
    codes = codes.reshape(rows, K)
    q = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return q, sf_code.astype(np.uint8), gs


# ----------------------------------------------------------------------------
# Activations and router weights
# ----------------------------------------------------------------------------

def gen_x_router(cfg: LayerConfig):
    """Return (x_bf16_bits uint16 [T,d], router_w float32 [E,d])."""
    rng = np.random.default_rng([cfg.seed, 1])
    T, d, E = cfg.T, cfg.d, cfg.E
    if cfg.router == "verify":
        R = cfg.requests
        assert R > 0 and T % R == 0
        per = T // R
        u = rng.standard_normal((R, d), dtype=np.float32)
        z = rng.standard_normal((T, d), dtype=np.float32)
        x = np.sqrt(np.float32(0.8)) * np.repeat(u, per, axis=0) + np.sqrt(np.float32(0.2)) * z
    else:
        x = rng.standard_normal((T, d), dtype=np.float32)
    rrng = np.random.default_rng([cfg.seed, 2])
    if cfg.router == "gauss002":
        w = rrng.standard_normal((E, d), dtype=np.float32) * np.float32(0.02)
    elif cfg.router in ("unit", "verify"):
        w = rrng.standard_normal((E, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    elif cfg.router == "zipf":
        w = rrng.standard_normal((E, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d - 1))
        rank = rrng.permutation(E)
        p = (rank + 1.0) ** -1.1
        p /= p.sum()
        w[:, d - 1] = np.log(p).astype(np.float32)
        x[:, d - 1] = 1.0
    else:
        raise ValueError(cfg.router)
    return f32_to_bf16_bits_trunc(x), np.ascontiguousarray(w, dtype=np.float32)


# ----------------------------------------------------------------------------
# Expert weights
# ----------------------------------------------------------------------------

def _matrix_shape(cfg: LayerConfig, m: int):
    return (cfg.f, cfg.d) if m in (GATE, UP) else (cfg.d, cfg.f)


_pool_cache: dict = {}


def _pool_needed(cfg: LayerConfig, m: int) -> bool:
    rows, K = _matrix_shape(cfg, m)
    return rows * K > _DIRECT_LIMIT


def _pool(seed: int, m: int):
    key = (seed, m)
    if key not in _pool_cache:
        rng = np.random.default_rng([seed, 7777, m])
        vals = rng.standard_normal((_POOL_BLOCKS, 16), dtype=np.float32) * np.float32(_W_STD)
        q, sf, gs = encode_nvfp4(vals)               # rows = blocks, K = 16
        _pool_cache[key] = (q.reshape(_POOL_BLOCKS, 8).copy(), sf.reshape(_POOL_BLOCKS).copy(), gs)
    return _pool_cache[key]


def _fill_expert_matrix(cfg: LayerConfig, e: int, m: int, q_out: np.ndarray, sf_out: np.ndarray):
    """Write expert e, matrix m into q_out [rows][K/2] and sf_out [rows][K/16]; return gs."""
    rows, K = _matrix_shape(cfg, m)
    rng = np.random.default_rng([cfg.seed, e, m])
    if rows * K <= _DIRECT_LIMIT:
        w = rng.standard_normal((rows, K), dtype=np.float32) * np.float32(_W_STD)
        q, sf, gs = encode_nvfp4(w)
        q_out[...] = q
        sf_out[...] = sf
        return gs
    pq, psf, pgs = _pool(cfg.seed, m)
    nblk = rows * (K // 16)
    # one uniformly drawn pool block per 16-value block (pool size 2**16)
    idx = np.frombuffer(rng.bytes(2 * nblk), dtype=np.uint16).astype(np.intp)
    np.take(pq.view(np.uint64).reshape(-1), idx, out=q_out.view(np.uint64).reshape(-1))
    np.take(psf, idx, out=sf_out.reshape(-1))
    return np.float32(pgs * (0.75 + 0.5 * rng.random()))


def gen_expert_matrix(cfg: LayerConfig, e: int, m: int):
    """(q [rows][K/2], sf [rows][K/16], gs) of expert e, matrix m (GATE/UP/DOWN)."""
    rows, K = _matrix_shape(cfg, m)
    q = np.empty((rows, K // 2), np.uint8)
    sf = np.empty((rows, K // 16), np.uint8)
    gs = _fill_expert_matrix(cfg, e, m, q, sf)
    return q, sf, gs


@dataclasses.dataclass
class ExpertWeights:
    """Canonical NVFP4 expert arrays (host, numpy)."""
    gate_q: np.ndarray
    gate_sf: np.ndarray
    gate_gs: np.ndarray
    up_q: np.ndarray
    up_sf: np.ndarray
    up_gs: np.ndarray
    down_q: np.ndarray
    down_sf: np.ndarray
    down_gs: np.ndarray

    def expert(self, e: int):
        """Per-expert view: dict matrix -> (q, sf, gs)."""
        return {GATE: (self.gate_q[e], self.gate_sf[e], self.gate_gs[e]),
                UP: (self.up_q[e], self.up_sf[e], self.up_gs[e]),
                DOWN: (self.down_q[e], self.down_sf[e], self.down_gs[e])}


def gen_experts(cfg: LayerConfig) -> ExpertWeights:
    """All E experts in the canonical layout."""
    E, d, f = cfg.E, cfg.d, cfg.f
    out = {}
    for name, m in (("gate", GATE), ("up", UP), ("down", DOWN)):
        rows, K = _matrix_shape(cfg, m)
        q = np.empty((E, rows, K // 2), np.uint8)
        sf = np.empty((E, rows, K // 16), np.uint8)
        gs = np.empty((E,), np.float32)
        if _pool_needed(cfg, m):
            _pool(cfg.seed, m)           # build the shared pool once, before threads
        def fill(e, q=q, sf=sf, gs=gs, m=m):
            gs[e] = _fill_expert_matrix(cfg, e, m, q[e], sf[e])
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as pool:
            list(pool.map(fill, range(E)))
        out[name + "_q"], out[name + "_sf"], out[name + "_gs"] = q, sf, gs
    return ExpertWeights(**out)


class LazyExperts:
    """Per-expert generator with the same interface as ExpertWeights.expert().

    Regenerates expert e on demand from the same seeds, so the oracle can look
    at a few experts of a 256-expert layer without holding 6.3 GB."""

    def __init__(self, cfg: LayerConfig):
        self.cfg = cfg
        self._cache: dict = {}

    def expert(self, e: int):
        if e not in self._cache:
            if len(self._cache) > 16:
                self._cache.clear()
            self._cache[e] = {m: gen_expert_matrix(self.cfg, e, m) for m in (GATE, UP, DOWN)}
        return self._cache[e]


def gen_all(cfg: LayerConfig):
    x, rw = gen_x_router(cfg)
    return x, rw, gen_experts(cfg)
