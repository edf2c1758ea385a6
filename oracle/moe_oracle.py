"""CPU oracle for the NVFP4 sparse-MoE layer forward (test infrastructure).

This is the plain, slow, obviously-correct definition the CUDA path is checked
against.  It is *test infrastructure only*: tests, the smoke check and the
bench's CPU-baseline leg may call it; the library never does.  It shares no
code with the CUDA path and imports nothing from it.

Everything is numpy, float64 unless a step fixes another precision.  Each
function names the passage it restates:

  [P2-BG]  "Optimizing Muse Spark Open on TPU v7 with SGLang-TorchTPU",
           Background: every token is routed to 8 of 256 experts; expert
           weights are 4-bit with one scale per 16 values (microscaling).
  [P2-S5]  same page, section 5 (expert loop by per-expert row count; sort a
           step's experts by rows).
  [P2-S8]  same page, section 8 (gate/up, SwiGLU, down; one-pass combine;
           every output row written exactly once).
  [P3-S2]  "Optimizing Models to Be Fast at Codegen", section 2 (FP4 (e2m1)
           weights with a per-16 block scale, unpacked in registers).
  [P4]     "Mixture of Experts" topic page (256 experts, 8 selected per token).
  [P5-IP]  "Day-0 Inference Adaptation for Ultra-Large Sparse Models",
           section II, Index Pipeline (routing indexes built on the device).

Layer definition (the problem statement the library implements):
  NVFP4 weight = e2m1 value x e4m3fn block scale (one per 16 along K) x fp32
  per-tensor scale; fp32 router logits; softmax; top-k with ties to the lower
  expert index; weights renormalised over the selected experts; SwiGLU experts
  SiLU(gate) * up; down projection; routing-weighted sum; one bf16 rounding.

Readings where the pages are silent (each is stated where it is used):
  R1 e2m1: bit 3 sign, bits 2-1 exponent (bias 1), bit 0 mantissa;
     element 2i of a packed byte sits in the low nibble.
  R2 e4m3fn block scale: bias 7, no infinities, 0x7F/0xFF NaN, max 448,
     subnormals m * 2^-9; applied with its sign.
  R3 one fp32 tensor scale per (expert, matrix).
  R4 activation precision is chosen per expert by its row count n_e:
     n_e <  thr  -> activations stay unquantised (bf16 x, full-precision h);
     n_e >= thr  -> x and h are NVFP4-quantised along K with tensor scale 1.0:
                    sf = e4m3_rne_satfinite(fp32(amax / 6)),
                    q  = e2m1_rne_satfinite(fp32(v / sf))   (q = 0 if sf = 0),
                    both decisions taken in IEEE float32, as the kernel does.
  R5 ids are listed by (logit desc, expert asc); the permutation orders the
     (token, slot) pairs by (expert, token, slot).
  R6 a token whose k-th and (k+1)-th fp64 logits differ by less than 1e-6 is a
     near-tie and is excluded from id / output comparisons.
  R13 the optional dynamic activation tensor scale of the dense class: a
     power of two, gs = 2^e with e the smallest integer such that
     max|a| <= 6 * 448 * 2^e over the whole tensor of the call; a is quantised
     as a / gs by R4's rule and dequantised times gs.
  R14 the optional residual add: the block's input x joins the same fp64 sum
     as the expert outputs, out = bf16(x + sum_j w_j y_j), one rounding.
  R12 the optional per-expert output normalisation ([P2-S8]) is an RMS norm
     over the d outputs of each expert, y / sqrt(mean(y^2) + eps), with no
     learned gain and eps chosen by the caller (the pages give neither).
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# Formats  [P2-BG], [P3-S2], readings R1-R3
# ----------------------------------------------------------------------------

# e2m1 magnitudes for codes 0..7 (R1): exponent field e (bias 1), mantissa m:
#   e = 0: m * 0.5 (subnormal);  e > 0: 2^(e-1) * (1 + m/2)
E2M1_MAGNITUDE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit e2m1 codes (0..15) -> float64 values (R1)."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDE[codes & 7]
    return np.where(codes & 8, -mag, mag)


def e4m3fn_decode(b: np.ndarray) -> np.ndarray:
    """e4m3fn bytes -> float64 (R2): bias 7, 0x7F/0xFF NaN, subnormal m*2^-9."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    s = b >> 7
    e = (b >> 3) & 0xF
    m = b & 7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 0xF) & (m == 7), np.nan, val)
    return np.where(s == 1, -val, val)


def unpack_e2m1(q: np.ndarray) -> np.ndarray:
    """Packed bytes [..., K/2] -> codes [..., K]; element 2i = low nibble (R1)."""
    q = np.asarray(q, dtype=np.uint8)
    out = np.empty(q.shape[:-1] + (q.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = q & 0xF
    out[..., 1::2] = q >> 4
    return out


# Both e2m1 values of every packed byte (R1: element 2i in the low nibble):
# _BYTE_PAIRS[b] = (e2m1(b & 15), e2m1(b >> 4)).
_BYTE_PAIRS = np.stack([e2m1_decode(np.arange(256) & 15), e2m1_decode(np.arange(256) >> 4)], axis=-1)


def dequant_nvfp4(q: np.ndarray, sf: np.ndarray, gs) -> np.ndarray:
    """Exact NVFP4 dequantisation  W[n,k] = e2m1(q[n,k]) * e4m3(sf[n,k//16]) * gs.

    [P2-BG] 4-bit weights with one scale per 16 values; [P3-S2] e2m1 with a
    per-16 block scale; R3 fp32 per-tensor scale.  Float64 holds every product
    exactly (at most 3 + 4 + 24 significant bits), so the order of the two
    multiplications does not matter.  Each byte is decoded to its two values
    by table (the same values as e2m1_decode(unpack_e2m1(q)))."""
    q = np.asarray(q, dtype=np.uint8)
    vals = _BYTE_PAIRS[q].reshape(q.shape[:-1] + (q.shape[-1] // 8, 16))   # [..., K/16, 16]
    scale = e4m3fn_decode(sf)[..., None] * np.float64(np.float32(gs))      # [..., K/16, 1]
    return (vals * scale).reshape(q.shape[:-1] + (q.shape[-1] * 2,))


# ----------------------------------------------------------------------------
# Round-to-nearest-even onto a small float grid (R4's quantiser decisions)
# ----------------------------------------------------------------------------

def _rne_on_grid(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Code (index into the sorted non-negative grid) nearest to mag, ties to
    the code whose lowest bit (the mantissa lsb) is 0; saturates at the top."""
    mag = np.minimum(np.asarray(mag, dtype=np.float64), grid[-1])
    hi = np.clip(np.searchsorted(grid, mag, side="left"), 1, len(grid) - 1)
    lo = hi - 1
    dlo = mag - grid[lo]
    dhi = grid[hi] - mag
    take_hi = (dhi < dlo) | ((dhi == dlo) & ((hi & 1) == 0))
    return np.where(take_hi, hi, lo)


E4M3_POSITIVE = e4m3fn_decode(np.arange(0x7F, dtype=np.uint8))   # codes 0..126, increasing


def e4m3_rne_satfinite(v: np.ndarray) -> np.ndarray:
    """float -> e4m3fn value, nearest-even, clamped to +-448 (R2, R4)."""
    v = np.asarray(v, dtype=np.float64)
    code = _rne_on_grid(np.abs(v), E4M3_POSITIVE)
    return np.where(v < 0, -1.0, 1.0) * E4M3_POSITIVE[code]


def e2m1_rne_satfinite_codes(v: np.ndarray) -> np.ndarray:
    """float -> e2m1 code (0..15), nearest-even, clamped to +-6 (R1, R4)."""
    v = np.asarray(v, dtype=np.float64)
    mag = _rne_on_grid(np.abs(v), E2M1_MAGNITUDE).astype(np.uint8)
    return np.where((v < 0) & (mag != 0), mag | 8, mag).astype(np.uint8)


def quantize_act_nvfp4(v: np.ndarray):
    """R4 activation quantiser along the last axis, tensor scale 1.0.

    Decisions are taken in IEEE float32 exactly as stated in R4; returns
    (codes uint8 [..., K], sf_value float64 [..., K/16], dequantised float64)."""
    v32 = np.asarray(v, dtype=np.float32)
    K = v32.shape[-1]
    assert K % 16 == 0
    blk = v32.reshape(v32.shape[:-1] + (K // 16, 16))
    amax = np.max(np.abs(blk), axis=-1)                       # exact in fp32
    s32 = (amax / np.float32(6.0)).astype(np.float32)         # IEEE fp32 division
    sf = e4m3_rne_satfinite(s32)                              # exact e4m3 value
    sf32 = sf.astype(np.float32)                              # exact in fp32
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (blk / np.where(sf32 == 0, np.float32(1), sf32)[..., None]).astype(np.float32)
    codes = e2m1_rne_satfinite_codes(ratio)
    codes = np.where((sf32 == 0)[..., None], 0, codes).astype(np.uint8)
    deq = e2m1_decode(codes) * sf[..., None]
    return (codes.reshape(v32.shape), sf, deq.reshape(v32.shape))


def pow2_tensor_scale(amax: float) -> float:
    """Dynamic activation tensor scale (reading R13): 2^e for the smallest
    integer e with amax <= 6 * 448 * 2^e, so the largest 16-block's scale lands
    at the top of the e4m3 range; 1.0 when amax is 0.  Exact: amax <= 2^E
    for E = frexp exponent, and 2688 * 2^e is exact in binary floating point."""
    amax = float(amax)
    if not amax > 0:
        return 1.0
    _, E = np.frexp(amax)                       # amax = m 2^E, 0.5 <= m < 1
    e = int(E) - 12
    while amax > 2688.0 * 2.0 ** e:             # at most two steps
        e += 1
    while e > -1074 and amax <= 2688.0 * 2.0 ** (e - 1):
        e -= 1
    return 2.0 ** e


# ----------------------------------------------------------------------------
# bf16
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits_rne(v: np.ndarray) -> np.ndarray:
    """Round float64 directly to bf16 (8 significant bits, nearest-even).

    Normal range only (|v| >= 2^-126); overflow goes to inf.  Values below the
    normal range are rounded on the subnormal grid 2^-133."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros(v.shape, dtype=np.float64)
    nz = (v != 0) & np.isfinite(v)
    mant, ex = np.frexp(v[nz])                # v = mant * 2^ex, 0.5 <= |mant| < 1
    ex = np.maximum(ex, -125)                 # subnormal grid: quantum 2^-133
    scaled = np.ldexp(v[nz], 8 - ex)          # |scaled| < 2^8 (exact in fp64)
    out[nz] = np.ldexp(np.rint(scaled), ex - 8)   # np.rint: ties to even
    out[~np.isfinite(v)] = v[~np.isfinite(v)]
    f32 = out.astype(np.float32)              # exact: 8-bit significands
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    return bits


# ----------------------------------------------------------------------------
# Router  [P2-BG], [P4]: logits, softmax, top-k, renormalise
# ----------------------------------------------------------------------------

def router_logits(x_bits: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    """l[t,e] = sum_i x[t,i] * Wr[e,i], in float64 (exact up to fp64 rounding)."""
    x = bf16_bits_to_f64(x_bits)
    return x @ np.asarray(router_w, dtype=np.float64).T


def route(logits: np.ndarray, k: int):
    """Softmax -> top-k (ties to the lower expert index) -> renormalise (R5, R6).

    Returns ids [T,k] listed by (logit desc, expert asc), weights [T,k] with
    w_j = p_{S_j} / sum_S p, and the gap between the k-th and (k+1)-th logit."""
    T, E = logits.shape
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -logits), axis=1)
    ids = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(logits, ids, axis=1)
    m = np.max(logits, axis=1, keepdims=True)
    p = np.exp(logits - m)
    p /= p.sum(axis=1, keepdims=True)                      # softmax over all E
    ps = np.take_along_axis(p, ids, axis=1)
    w = ps / ps.sum(axis=1, keepdims=True)                 # renormalised over S
    if k < E:
        nxt = np.take_along_axis(logits, order[:, k:k + 1], axis=1)[:, 0]
        gap = sel[:, -1] - nxt
    else:
        gap = np.full(T, np.inf)
    return ids, w, gap


def near_tie_flags(gap: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """R6: tokens whose selection margin is below eps."""
    return np.asarray(gap) < eps


def fp32_logit_error_bound(x_bits: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    """Rigorous bound on |fl32(l) - l| for any fp32 summation order:
    gamma_{d+1} * sum_i |x_i w_i| (standard dot-product error bound)."""
    x = np.abs(bf16_bits_to_f64(x_bits))
    d = x.shape[1]
    u = 2.0 ** -24
    gamma = (d + 1) * u / (1 - (d + 1) * u)
    return gamma * (x @ np.abs(np.asarray(router_w, np.float64)).T) + 2 * u * np.abs(
        router_logits(x_bits, router_w))


# ----------------------------------------------------------------------------
# Permutation  [P5-IP], [P2-S5]
# ----------------------------------------------------------------------------

def permute(ids: np.ndarray, E: int):
    """Histogram, exclusive-scan offsets and the stable permutation (R5).

    perm[pos] = t*k + j for pairs sorted by (expert, t, j); inv[t*k+j] = pos."""
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)   # stable => (e, t, j)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, offsets, perm, inv


# ----------------------------------------------------------------------------
# Experts  [P2-S8] gate/up, SwiGLU, down; [P3-S2]
# ----------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z / (1 + e^-z)  (SwiGLU, [P2-S8])."""
    return z / (1.0 + np.exp(-z))


def expert_ffn(xrows: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray,
               quantized: bool, magnitudes: bool = False, scales=(1.0, 1.0)):
    """One expert on its rows.  Returns (h, y) in float64.

    quantized=False (R4, n_e < thr): h = SiLU(Wg x) * (Wu x); y = Wd h.
    quantized=True  (R4, n_e >= thr): x and h pass through quantize_act_nvfp4
    first; h is rounded to float32 before its quantiser (the kernel holds h
    in float32).  scales = (gs_x, gs_h): the activation tensor scales (R13;
    1.0 by default): a is quantised as a / gs and dequantised times gs.
    magnitudes=True also returns the absolute-value sums that bound rounding
    errors element by element (|Wg||x|, |Wu||x|, |Wd||h|, and g, u), and per
    row the largest row L1 norms of the expert's matrices (l1g, l1u, l1d:
    max_c sum_k |W[c,k]|) and max |x| of the row (xmax)."""
    gx, gh = scales
    xin = quantize_act_nvfp4(xrows / gx)[2] * gx if quantized else xrows
    g = xin @ Wg.T
    u = xin @ Wu.T
    h = silu(g) * u
    hin = quantize_act_nvfp4(h.astype(np.float32) / np.float32(gh))[2] * gh if quantized else h
    y = hin @ Wd.T
    if not magnitudes:
        return h, y
    ax = np.abs(xin)
    ones = np.ones((xrows.shape[0], 1))
    mag = dict(g=g, u=u, gabs=ax @ np.abs(Wg).T, uabs=ax @ np.abs(Wu).T,
               yabs=np.abs(hin) @ np.abs(Wd).T,
               l1g=ones * np.abs(Wg).sum(axis=1).max(), l1u=ones * np.abs(Wu).sum(axis=1).max(),
               l1d=ones * np.abs(Wd).sum(axis=1).max(), xmax=np.abs(xrows).max(axis=1, keepdims=True))
    return h, y, mag


def expert_rms_norm(y: np.ndarray, eps: float) -> np.ndarray:
    """Per-expert output normalisation  y / sqrt(mean_i y_i^2 + eps) over the
    d outputs of each row, with no learned gain ([P2-S8]: each expert's output
    is normalised before the weighted sum; reading R12: an RMS norm, eps given
    by the caller)."""
    return y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)


class PairRows:
    """Per-pair values of a forward, stored only for the pairs evaluated.

    Indexed like a [P, cols] array by permutation row (an int, an int array,
    or (rows, cols)); rows that were not evaluated read as NaN."""

    def __init__(self, P: int, cols: int):
        self.shape = (P, cols)
        self._index = np.full(P, -1, dtype=np.int64)
        self._blocks = []
        self._data = None

    def _put(self, pos: np.ndarray, values: np.ndarray):
        n0 = sum(b.shape[0] for b in self._blocks)
        self._index[pos] = n0 + np.arange(len(pos))
        self._blocks.append(np.asarray(values, dtype=np.float64))
        self._data = None

    def _rows(self, r):
        if self._data is None:
            self._data = np.concatenate(self._blocks + [np.full((1, self.shape[1]), np.nan)])
        return self._data[self._index[r]]          # index -1 -> the NaN row

    def __getitem__(self, key):
        if isinstance(key, tuple):
            return self._rows(key[0])[(Ellipsis,) + key[1:]]
        return self._rows(key)


def _expert_rows(task):
    """One expert on its selected rows (dequantise, then expert_ffn).
    task = (experts, e, xrows, quantized, magnitudes, scales); a top-level
    function so that a process pool can run it."""
    experts, e, xrows, quantized, magnitudes, scales = task
    mats = experts.expert(e)
    Wg = dequant_nvfp4(*mats[0])
    Wu = dequant_nvfp4(*mats[1])
    Wd = dequant_nvfp4(*mats[2])
    return expert_ffn(xrows, Wg, Wu, Wd, quantized=quantized, magnitudes=magnitudes, scales=scales)


def _expert_h_amax(task):
    """max |fp32(h)| of one dense-class expert over all its rows (R13's first
    pass).  task = (experts, e, xrows, gs_x)."""
    experts, e, xrows, gx = task
    mats = experts.expert(e)
    xin = quantize_act_nvfp4(xrows / gx)[2] * gx
    h = silu(xin @ dequant_nvfp4(*mats[0]).T) * (xin @ dequant_nvfp4(*mats[1]).T)
    return float(np.max(np.abs(h.astype(np.float32)))) if h.size else 0.0


def forward(x_bits: np.ndarray, router_w: np.ndarray, experts, E: int, k: int,
            thr: int = 128, token_subset=None, want_pairs: bool = True,
            magnitudes: bool = False, expert_norm_eps=None, map_fn=map, act_scale: str = "fixed",
            residual: bool = False):
    """The whole layer.  `experts.expert(e)` -> {0: (q,sf,gs) gate, 1: up, 2: down}.

    token_subset: if given, expert outputs are evaluated only for pairs of those
    tokens (routing and permutation are always computed for every token).
    expert_norm_eps: None for the plain weighted sum; a number eps >= 0 applies
    expert_rms_norm(y, eps) to every expert output before the weighted sum.
    map_fn: how the independent per-expert evaluations are mapped (the builtin
    map, or a process pool's map; results are assembled in expert order
    either way, so the output does not depend on it).
    residual: the block's input is added to its output before the one bf16
    rounding (R14: out = bf16(x + sum_j w_j y_j), a decoder layer's residual
    stream; rows outside token_subset then hold x).
    act_scale: "fixed" (R4: activation tensor scale 1.0) or "dynamic" (R13:
    gs_x from max|x| over all T tokens, gs_h from max|h| over every pair of
    every dense-class expert, each pow2_tensor_scale; h is evaluated for all
    dense pairs first, whatever token_subset is).
    Returns a dict with logits, ids, w, gap, counts, offsets, perm, inv, the
    per-pair h, y (the expert output Wd h) and partial (its contribution to
    the output; PairRows indexed by permutation row, NaN where not
    evaluated), out64 and the bf16 output bits (rows outside the subset are 0)."""
    T, d = x_bits.shape
    logits = router_logits(x_bits, router_w)
    ids, w, gap = route(logits, k)
    counts, offsets, perm, inv = permute(ids, E)
    x = bf16_bits_to_f64(x_bits)
    tokens = np.arange(T) if token_subset is None else np.unique(np.asarray(token_subset))
    want = np.zeros(T, dtype=bool)
    want[tokens] = True
    P = T * k
    # the (expert, rows) work list, in expert order
    work = []
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        pos = np.arange(lo, hi)
        pairs = perm[lo:hi]
        toks = pairs // k
        keep = want[toks]
        if not keep.any():
            continue
        # R4: the expert's class follows its full row count in the call
        work.append((e, pos[keep], pairs[keep], toks[keep], (hi - lo) >= thr))
    gs_x = gs_h = 1.0
    h_amax = None
    if act_scale == "dynamic":
        gs_x = pow2_tensor_scale(np.max(np.abs(x)) if x.size else 0.0)
        dense_all = [(experts, e, x[perm[offsets[e]:offsets[e + 1]] // k], gs_x) for e in range(E)
                     if offsets[e + 1] - offsets[e] >= thr and offsets[e + 1] > offsets[e]]
        h_amax = max(list(map_fn(_expert_h_amax, dense_all)) + [0.0])
        gs_h = pow2_tensor_scale(h_amax)
    elif act_scale != "fixed":
        raise ValueError(act_scale)
    results = list(map_fn(_expert_rows, [(experts, e, x[toks], q, magnitudes, (gs_x, gs_h))
                                         for e, _, _, toks, q in work]))
    h_all = partial_all = y_all = None
    out64 = np.zeros((T, d), dtype=np.float64)
    mags = None
    for (e, pos, pairs, toks, _), res in zip(work, results):
        h, y = res[0], res[1]
        if want_pairs and h_all is None:
            h_all, partial_all, y_all = PairRows(P, h.shape[1]), PairRows(P, d), PairRows(P, d)
        if magnitudes:
            if mags is None:
                mags = {n: PairRows(P, v.shape[1]) for n, v in res[2].items()}
            for n, v in res[2].items():
                mags[n]._put(pos, v)
        wj = w.reshape(-1)[pairs]
        yn = y if expert_norm_eps is None else expert_rms_norm(y, expert_norm_eps)
        contrib = wj[:, None] * yn
        if want_pairs:
            h_all._put(pos, h)
            y_all._put(pos, y)
            partial_all._put(pos, contrib)
        np.add.at(out64, toks, contrib)
    if residual:
        out64 = out64 + x
    out_bits = f64_to_bf16_bits_rne(out64)
    return dict(logits=logits, ids=ids, w=w, gap=gap, counts=counts, offsets=offsets,
                perm=perm, inv=inv, h=h_all, y=y_all, partial=partial_all, out64=out64,
                out_bits=out_bits, tokens=tokens, mags=mags, gs_x=gs_x, gs_h=gs_h, h_amax=h_amax)
