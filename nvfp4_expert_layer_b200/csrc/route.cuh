// Router logits, activation staging, top-k and the token -> expert permutation.
//
// Router: fp32 logits l[t,e] = sum_i x[t,i] * Wr[e,i] and softmax/top-k with
// ties to the lower expert index, weights renormalised over the selected
// experts ("Optimizing Muse Spark Open on TPU v7 with SGLang-TorchTPU",
// Background: each token picks 8 of 256 experts; section 2: experts are
// requested as soon as routing finishes).  The permutation is built on the
// device with no host synchronisation ("Day-0 Inference Adaptation for
// Ultra-Large Sparse Models", section II, Index Pipeline) and sorts a step's
// experts by row count (Muse Spark page, section 5).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "layout.cuh"

namespace moe {

constexpr int kJobRows = 16;   // rows per light job (two 8-wide MMA n-tiles)

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------------------------
// Per-row fp16 staging of x for the tensor-core GEMV: x16 = x * 2^s written in
// the B-fragment layout, xscale = 2^-s, with s chosen so max|x*2^s| lies in
// [2^14, 2^15).  bf16 -> fp16 is then exact for every element whose magnitude
// is at least 2^-17 of 2^14 (i.e. all but values ~2^-31 below the row max).
// ---------------------------------------------------------------------------
__device__ void stage_x_row(const uint16_t* __restrict__ xrow, int d, __half* __restrict__ x16row,
                            float* __restrict__ xscale_out, int* err, float* red) {
  float m = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) m = fmaxf(m, fabsf(bf16_bits_to_float(xrow[i])));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mm = fmaxf(mm, red[w]);
    red[32] = mm;
  }
  __syncthreads();
  const float mx = red[32];
  int s = 0;
  if (!(mx < INFINITY)) {                       // inf or NaN
    if (threadIdx.x == 0) set_error(err, kErrNumeric);
  } else if (mx > 0.f) {
    int e;
    frexpf(mx, &e);                             // mx = m * 2^e, m in [0.5, 1)
    s = 15 - e;
    s = max(-120, min(120, s));
  }
  const float up = ldexpf(1.f, s);
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const float v = bf16_bits_to_float(xrow[i]) * up;
    x16row[bfrag_offset(i)] = __float2half_rn(v);
  }
  if (threadIdx.x == 0) *xscale_out = ldexpf(1.f, -s);
  __syncthreads();
}

// Small-T router: one block per expert e; each warp handles tokens
// t = warp, warp + nwarps, ...  Block b < T also stages x row b (fp16).
// Requires d % 256 == 0 handled by the host (d % 128 == 0 -> 4-wide loads).
__global__ void __launch_bounds__(256) router_small_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ rw, int T, int d, int E,
    float* __restrict__ logits, __half* __restrict__ x16, float* __restrict__ xscale, int* err) {
  extern __shared__ __align__(16) float s_w[];   // d floats
  __shared__ float red[33];
  const int e = blockIdx.x;
  if (e < E) {
    const float4* src = reinterpret_cast<const float4*>(rw + (size_t)e * d);
    float4* dst = reinterpret_cast<float4*>(s_w);
    for (int i = threadIdx.x; i < d / 4; i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  if (e < E) {
    for (int t = warp; t < T; t += nwarps) {
      const uint16_t* xr = x + (size_t)t * d;
      float acc = 0.f;
      // lane handles 4 consecutive elements per 128-wide step
      for (int i = lane * 4; i < d; i += 128) {
        const uint2 xv = *reinterpret_cast<const uint2*>(xr + i);
        const float4 wv = *reinterpret_cast<const float4*>(s_w + i);
        acc = fmaf(__uint_as_float(xv.x << 16), wv.x, acc);
        acc = fmaf(__uint_as_float(xv.x & 0xffff0000u), wv.y, acc);
        acc = fmaf(__uint_as_float(xv.y << 16), wv.z, acc);
        acc = fmaf(__uint_as_float(xv.y & 0xffff0000u), wv.w, acc);
      }
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) logits[(size_t)t * E + e] = acc;
    }
  }
  for (int t = blockIdx.x; t < T; t += gridDim.x)
    stage_x_row(x + (size_t)t * d, d, x16 + (size_t)t * d, xscale + t, err, red);
}

// Stage x rows (used with the tiled router for large T): one block per row.
__global__ void __launch_bounds__(256) stage_x_kernel(const uint16_t* __restrict__ x, int T, int d,
                                                      __half* __restrict__ x16,
                                                      float* __restrict__ xscale, int* err) {
  __shared__ float red[33];
  for (int t = blockIdx.x; t < T; t += gridDim.x)
    stage_x_row(x + (size_t)t * d, d, x16 + (size_t)t * d, xscale + t, err, red);
}

// Large-T router: 64x64 output tile per block, fp32 FMA, K step 16.
__global__ void __launch_bounds__(256) router_tiled_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ rw, int T, int d, int E,
    float* __restrict__ logits) {
  __shared__ float sx[16][64 + 4];
  __shared__ float sw[16][64 + 4];
  const int t0 = blockIdx.x * 64, e0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i >> 4, kk = i & 15;
      const int t = t0 + r, e = e0 + r;
      sx[kk][r] = t < T ? bf16_bits_to_float(x[(size_t)t * d + k0 + kk]) : 0.f;
      sw[kk][r] = e < E ? rw[(size_t)e * d + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = sx[kk][ty * 4 + i]; b[i] = sw[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + ty * 4 + i, e = e0 + tx * 4 + j;
      if (t < T && e < E) logits[(size_t)t * E + e] = acc[i][j];
    }
}

// ---------------------------------------------------------------------------
// Top-k: one warp per token.  Lane l holds logits e = l + 32 i.  k rounds of a
// warp arg-max ordered by (logit desc, expert asc); weights are the softmax of
// the selected logits (equal to the renormalised full softmax).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int* __restrict__ ids,
                                                   float* __restrict__ wts) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[32];
  const int per = (E + 31) / 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    v[i] = (i < per && e < E) ? logits[(size_t)t * E + e] : -INFINITY;
  }
  float sel_l0 = 0.f, sum = 0.f;
  float my_l = 0.f;
  int my_e = 0;
  unsigned taken = 0u;            // bit i: element lane + 32 i already selected
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = lane + 32 * i;
      const bool cand = i < per && e < E && !((taken >> i) & 1u);
      if (cand && (be == 0x7fffffff || v[i] > bv || (v[i] == bv && e < be))) { bv = v[i]; be = e; }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      const bool better = (oe != 0x7fffffff) &&
                          (be == 0x7fffffff || ov > bv || (ov == bv && oe < be));
      if (better) { bv = ov; be = oe; }
    }
    if (be == 0x7fffffff) be = 0;       // unreachable for k <= E
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (j == 0) sel_l0 = bv;
    const float p = expf(bv - sel_l0);
    sum += p;
    if (lane == j) { my_l = p; my_e = be; }
  }
  if (lane < k) {
    ids[(size_t)t * k + lane] = my_e;
    wts[(size_t)t * k + lane] = my_l / sum;
  }
}

// ---------------------------------------------------------------------------
// Permutation, single block of 1024 threads (32 warps).
// Pairs p = t*k + j in [0, P) are cut into 32 contiguous warp chunks.  Each
// warp counts its chunk per expert (match_any groups equal experts inside a
// 32-pair step, so no atomics), the counts are scanned, and a second walk
// assigns positions in (expert, pair) order -- deterministic and stable.
// Then experts are classed by row count: light (0 < n < thr) experts are
// split into jobs of <= 16 rows, listed heavy-first; dense (n >= thr) experts
// are listed by n descending.
// Dynamic shared memory: 32*E + 3*E + 2 ints.
// ---------------------------------------------------------------------------
struct PermuteOut {
  int* counts;      // [E]
  int* offsets;     // [E+1]
  int* perm;        // [P]
  int* inv;         // [P]
  int4* light_jobs; // [E + P/16 + 1]  {expert, row0, nrows, 0}
  int* n_light_jobs;
  int4* dense_list; // [E]  {expert, row0, nrows, 0}
  int* n_dense;
  int* err;
};

__global__ void __launch_bounds__(1024) permute_kernel(const int* __restrict__ ids, int T, int k,
                                                       int E, int thr, int dense_supported,
                                                       PermuteOut o) {
  extern __shared__ int sm[];
  int* wc = sm;                 // [32][E]
  int* cnt = wc + 32 * E;       // [E]
  int* off = cnt + E;           // [E+1]
  int* jstart = off + E + 1;    // [E]
  __shared__ int s_nlight, s_ndense;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long P = (long long)T * k;
  const long long c0 = P * warp / 32, c1 = P * (warp + 1) / 32;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) wc[i] = 0;
  if (threadIdx.x == 0) { s_nlight = 0; s_ndense = 0; }
  __syncthreads();
  // pass 1: per-warp counts
  for (long long base = c0; base < c1; base += 32) {
    const long long idx = base + lane;
    const bool valid = idx < c1;
    const int e = valid ? ids[idx] : -1;
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    if (valid && lane == __ffs(mask) - 1 && e >= 0 && e < E) wc[warp * E + e] += __popc(mask);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int w = 0; w < 32; ++w) s += wc[w * E + e];
    cnt[e] = s;
  }
  __syncthreads();
  if (warp == 0) {   // exclusive scan of cnt by one warp
    int carry = 0;
    for (int b = 0; b < E; b += 32) {
      const int e = b + lane;
      int v = e < E ? cnt[e] : 0;
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (e < E) off[e] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) off[E] = carry;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = off[e];
    for (int w = 0; w < 32; ++w) {
      const int c = wc[w * E + e];
      wc[w * E + e] = run;
      run += c;
    }
    o.counts[e] = cnt[e];
    o.offsets[e] = off[e];
  }
  if (threadIdx.x == 0) o.offsets[E] = off[E];
  __syncthreads();
  // pass 2: positions
  const unsigned lt = (1u << lane) - 1u;
  for (long long base = c0; base < c1; base += 32) {
    const long long idx = base + lane;
    const bool valid = idx < c1;
    const int e = valid ? ids[idx] : -1;
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    int pos = 0;
    if (valid && e >= 0 && e < E) {
      pos = wc[warp * E + e] + __popc(mask & lt);
      o.perm[pos] = (int)idx;
      o.inv[idx] = pos;
    }
    __syncwarp();
    if (valid && e >= 0 && e < E && lane == __ffs(mask) - 1) wc[warp * E + e] += __popc(mask);
    __syncwarp();
  }
  // classes and job lists
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int n = cnt[e];
    jstart[e] = 0;
    if (n == 0) continue;
    const bool light = n < thr;
    int rank = 0, start = 0;
    for (int e2 = 0; e2 < E; ++e2) {
      const int n2 = cnt[e2];
      if (n2 == 0 || (n2 < thr) != light) continue;
      if (n2 > n || (n2 == n && e2 < e)) {
        ++rank;
        start += (n2 + kJobRows - 1) / kJobRows;
      }
    }
    if (light) {
      const int nj = (n + kJobRows - 1) / kJobRows;
      for (int q = 0; q < nj; ++q)
        o.light_jobs[start + q] = make_int4(e, off[e] + q * kJobRows, min(kJobRows, n - q * kJobRows), 0);
      atomicAdd(&s_nlight, nj);
    } else {
      o.dense_list[rank] = make_int4(e, off[e], n, 0);
      atomicAdd(&s_ndense, 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *o.n_light_jobs = s_nlight;
    *o.n_dense = s_ndense;
    if (s_ndense > 0 && !dense_supported) set_error(o.err, kErrUnsupported);
  }
}

}  // namespace moe
