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
#include <climits>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "layout.cuh"

namespace moe {

constexpr int kJobRows = 32;   // rows per light job (up to four 8-wide MMA n-tiles)

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
  // each thread owns up to 8 groups of 8 consecutive elements (d <= 16384)
  constexpr int kMaxG = 8;
  const int ngroups = d / 8;
  uint4 v[kMaxG];
  float m = 0.f;
#pragma unroll
  for (int q = 0; q < kMaxG; ++q) {
    const int gi = threadIdx.x + q * blockDim.x;
    v[q] = gi < ngroups ? *reinterpret_cast<const uint4*>(xrow + 8 * gi) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int q = 0; q < kMaxG; ++q) {
    const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xffff0000u))));
  }
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
    s = max(-120, min(120, 15 - e));
  }
  const float up = ldexpf(1.f, s);
#pragma unroll
  for (int q = 0; q < kMaxG; ++q) {
    const int gi = threadIdx.x + q * blockDim.x;
    if (gi < ngroups) {
      // elements 8gi..8gi+7: same chunk, step and slot; c = 0..3, half = 0..1
      const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
      const int base = bfrag_offset(8 * gi);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 h2 = __floats2half2_rn(__uint_as_float(w[i] << 16) * up,
                                             __uint_as_float(w[i] & 0xffff0000u) * up);
        *reinterpret_cast<__half2*>(x16row + base + 16 * i) = h2;
      }
    }
  }
  if (threadIdx.x == 0) *xscale_out = ldexpf(1.f, -s);
  __syncthreads();
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

// Rows routed by the caller (one expert per row, weight 1): the ids are
// copied into the workspace, the weights set to 1 and inv cleared to -1; an
// id outside [0, E) records MOE_FP4_ERR_INVALID_ARG in the device error word
// and is replaced by -1, which the permutation kernels skip (its inv stays -1).
__global__ void __launch_bounds__(256) preroute_kernel(const int* __restrict__ in_ids, int n, int E,
                                                       int* __restrict__ ids, float* __restrict__ wts,
                                                       int* __restrict__ inv, int* err) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    int e = in_ids[i];
    if (e < 0 || e >= E) {
      set_error(err, 1);
      e = -1;
    }
    ids[i] = e;
    wts[i] = 1.f;
    inv[i] = -1;            // the permutation writes the position of every valid row
  }
}

// ---------------------------------------------------------------------------
// Top-k: one warp per token.  Lane l holds logits e = l + 32 i.  k rounds of a
// warp arg-max ordered by (logit desc, expert asc); weights are the softmax of
// the selected logits (equal to the renormalised full softmax).
// ---------------------------------------------------------------------------
// Warp top-k over v[i] = logit of expert lane + 32 i (-inf beyond E).
// Lane j < k receives the j-th selected expert and its renormalised weight.
// PER = logits per lane rounded up to a power of two.  Each lane keeps its
// best untaken (logit, expert) as an order-preserving 32-bit key; a round is
// two warp reductions (the largest key, then the lowest expert among the
// lanes holding it) and only the winning lane rescans its PER values.
// Within a lane experts increase with i, so a strict comparison keeps the
// lower expert on ties.
// Order-preserving key of a logit: a > b as floats <=> key(a) > key(b); -0 and
// +0 share one key (they compare equal, so the lower expert wins), and every
// non-NaN logit has a key above 0.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

template <int PER>
__device__ __forceinline__ void topk_warp_t(const float (&v)[32], int E, int k, int lane, int& my_e,
                                            float& my_w) {
  float sel_l0 = 0.f, sum = 0.f, my_p = 0.f;
  my_e = 0;
  unsigned taken = 0u;            // bit i: element lane + 32 i already selected
  uint32_t lk = 0u;               // 0: no candidate left in this lane
  int le = 0;
  auto lane_best = [&]() {
    lk = 0u;
    le = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      const uint32_t key = (e < E && !((taken >> i) & 1u)) ? order_key(v[i]) : 0u;
      if (key > lk) { lk = key; le = e; }
    }
  };
  lane_best();
  for (int j = 0; j < k; ++j) {
    const uint32_t mk = __reduce_max_sync(0xffffffffu, lk);
    const int be = (int)__reduce_min_sync(0xffffffffu, lk == mk ? (uint32_t)le : 0xffffffffu);
    if ((be & 31) == lane) {
      taken |= 1u << (be >> 5);
      lane_best();
    }
    const float bv = order_key_value(mk);
    if (j == 0) sel_l0 = bv;
    const float p = expf(bv - sel_l0);
    sum += p;
    if (lane == j) { my_p = p; my_e = be; }
  }
  my_w = my_p / sum;
}

__device__ __forceinline__ void topk_warp(const float (&v)[32], int E, int k, int lane, int& my_e,
                                          float& my_w) {
  const int per = (E + 31) / 32;
  if (per <= 1) topk_warp_t<1>(v, E, k, lane, my_e, my_w);
  else if (per <= 2) topk_warp_t<2>(v, E, k, lane, my_e, my_w);
  else if (per <= 4) topk_warp_t<4>(v, E, k, lane, my_e, my_w);
  else if (per <= 8) topk_warp_t<8>(v, E, k, lane, my_e, my_w);
  else if (per <= 16) topk_warp_t<16>(v, E, k, lane, my_e, my_w);
  else topk_warp_t<32>(v, E, k, lane, my_e, my_w);
}

// Top-k for large T: one warp per token over the full logits.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int* __restrict__ ids,
                                                   float* __restrict__ wts) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? logits[(size_t)t * E + e] : -INFINITY;
  }
  int my_e;
  float my_w;
  topk_warp(v, E, k, lane, my_e, my_w);
  if (lane < k) {
    ids[(size_t)t * k + lane] = my_e;
    wts[(size_t)t * k + lane] = my_w;
  }
}

// ---------------------------------------------------------------------------
// Permutation: pairs p = t*k + j in [0, P) are placed in (expert, pair) order
// -- deterministic and stable -- and the active experts are classed by row
// count n:
//   light (n < thr): cut into jobs of 32 rows plus one remainder job; jobs of
//     <= 8 rows go to list 1 (one 8-wide MMA n-tile), jobs of 9..16 rows to
//     list 2 (two n-tiles), jobs of 17..32 rows to list 4 (four n-tiles);
//     each list is ordered heavy expert first;
//   dense (n >= thr): listed by n descending.
// At most 32 pairs: perm_small inside the routing kernel; otherwise three
// launches (perm_hist_kernel, perm_scan_kernel, perm_place_kernel).
// Shared memory of the scan (ints): 32*E + 4*E + 1 (counts, offsets, active
// list) + 8 scalars.
// ---------------------------------------------------------------------------
struct PermuteOut {
  int* counts;       // [E]
  int* offsets;      // [E+1]
  int* perm;         // [P]
  int* inv;          // [P]
  int4* jobs1;       // [E]            {expert, row0, nrows, 0}, 1 <= nrows <= 8
  int* n_jobs1;
  int4* jobs2;       // [E]            {expert, row0, nrows, 0}, 9 <= nrows <= 16
  int* n_jobs2;
  int4* jobs4;       // [E + P/32 + 1] {expert, row0, nrows, 0}, 17 <= nrows <= 32
  int* n_jobs4;
  int4* dense_list;  // [E]            {expert, row0, nrows, padded row0}
  int* n_dense;
  int* dense_ntoff;  // [2][E+1]       exclusive prefixes of ceil(nrows / 128) and ceil(nrows / 256)
                     //                over the dense list
  int* dense_pad_total;  // padded rows of the dense class (each expert rounded up to 256)
  int* err;
};

__host__ __device__ constexpr size_t permute_smem_ints(int E) { return (size_t)36 * E + 1 + 8; }

// Expert classes over the active experts (light jobs, dense list) from the
// counts, offsets and active list in shared memory (the layout of
// permute_smem_ints); writes the job lists, the dense list and the scalars.
__device__ void perm_classes(int E, int thr, int dense_supported, const PermuteOut& o, int* sm) {
  int* cnt = sm + 32 * E;
  int* off = cnt + E;
  int* act = off + E + 1;
  int* misc = act + E;
  // expert classes over the active experts only
  const int A = misc[0];
  for (int a = threadIdx.x; a < A; a += blockDim.x) {
    const int e = act[a];
    const int n = cnt[e];
    const bool light = n < thr;
    int rank = 0, s1 = 0, s2 = 0, s4 = 0, pad0 = 0, nt0 = 0, nt1 = 0;
    for (int b = 0; b < A; ++b) {
      const int e2 = act[b], n2 = cnt[e2];
      if ((n2 < thr) != light) continue;
      if (n2 > n || (n2 == n && e2 < e)) {
        ++rank;
        const int r2 = n2 % kJobRows;
        s1 += (r2 > 0 && r2 <= 8) ? 1 : 0;
        s2 += (r2 > 8 && r2 <= 16) ? 1 : 0;
        s4 += n2 / kJobRows + (r2 > 16 ? 1 : 0);
        pad0 += (n2 + 255) & ~255;
        nt0 += (n2 + 127) >> 7;
        nt1 += (n2 + 255) >> 8;
      }
    }
    if (light) {
      for (int r0 = 0; r0 < n; r0 += kJobRows) {
        const int nr = min(kJobRows, n - r0);
        const int4 jb = make_int4(e, off[e] + r0, nr, 0);
        if (nr <= 8) o.jobs1[s1] = jb; else if (nr <= 16) o.jobs2[s2] = jb; else o.jobs4[s4++] = jb;
      }
      const int r = n % kJobRows;
      atomicAdd(&misc[1], (r > 0 && r <= 8) ? 1 : 0);
      atomicAdd(&misc[2], (r > 8 && r <= 16) ? 1 : 0);
      atomicAdd(&misc[7], n / kJobRows + (r > 16 ? 1 : 0));
    } else {
      o.dense_list[rank] = make_int4(e, off[e], n, pad0);
      o.dense_ntoff[rank] = nt0;
      o.dense_ntoff[E + 1 + rank] = nt1;
      atomicAdd(&misc[3], 1);
      atomicAdd(&misc[4], (n + 127) >> 7);
      atomicAdd(&misc[5], (n + 255) & ~255);
      atomicAdd(&misc[6], (n + 255) >> 8);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *o.n_jobs1 = misc[1];
    *o.n_jobs2 = misc[2];
    *o.n_jobs4 = misc[7];
    *o.n_dense = misc[3];
    o.dense_ntoff[misc[3]] = misc[4];
    o.dense_ntoff[E + 1 + misc[3]] = misc[6];
    *o.dense_pad_total = misc[5];
    if (misc[3] > 0 && !dense_supported) set_error(o.err, kErrUnsupported);
  }
}

// ---------------------------------------------------------------------------
// Small batches (T * k <= 32 pairs, decode): top-k and permutation in the one
// block of 1024 threads, built from independent comparisons instead of k
// sequential arg-max rounds, so the latency is a few short phases.
// ---------------------------------------------------------------------------
// Shared-memory ints used by topk_small_block.
__host__ __device__ constexpr size_t topk_small_ints(int E, int T, int k) {
  const size_t G = (size_t)(E + 31) / 32, kk = (size_t)(k < 32 ? k : 32);
  return (size_t)T * G * 32 + 2 * (size_t)T * G * kk + 2 * (size_t)T * k + 2;
}

// Pair experts of the small path sit after the top-k scratch (and after the
// 64 ints the permutation exchanges through shared memory).
__host__ __device__ constexpr size_t route_small_ids_offset(int E, int T, int k) {
  return topk_small_ints(E, T, k) > 64 ? topk_small_ints(E, T, k) : 64;
}

// Top-k of T tokens (T <= 32; a block of 1024 threads) over the logits [T][E] with the order and the
// weights of topk_warp_t: (logit desc, expert asc), weights the softmax of the
// selected logits accumulated in selection order.  Phase 1 ranks every
// logit inside its group of 32 experts and keeps the best min(k, 32) of each
// group as candidates (a global top-k member has fewer than k better experts
// in its group); phase 2 ranks the candidates of a token against each other,
// several threads per candidate.  Candidates carry one 64-bit key, logit key
// above the complemented expert, so one comparison orders (logit, expert).
// Every loop has independent iterations (no load behind a branch): the
// phases are latency-bound, not issue-bound.
__device__ void topk_small_block(const float* logits, int T, int E, int k, int* ids_s, int* ids_out,
                                 float* wts, uint32_t* scratch) {
  const unsigned FULL = 0xffffffffu;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int ltp = 0;                                        // tokens rounded up to 2^ltp
  while ((1 << ltp) < T) ++ltp;
  const int ltpt = 10 - ltp;                          // threads per token 2^ltpt (>= 32)
  const int tpt = 1 << ltpt, wpt = tpt >> 5;
  const int t = tid >> ltpt, u = tid & (tpt - 1), wt = u >> 5;
  const int G = (E + 31) / 32, kk = min(k, 32), C = G * kk;
  uint32_t* s_key = scratch;                          // [T][G*32] keys, 0 beyond E
  uint64_t* c_key = reinterpret_cast<uint64_t*>(s_key + (((size_t)T * G * 32 + 1) & ~(size_t)1));   // [T][C]
  uint64_t* sel = c_key + (size_t)T * C;              // [T][k]
  for (int tt = 0; tt < T; ++tt)
    for (int e = tid; e < G * 32; e += blockDim.x) {
      float l = 0.f;
      if (e < E) asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(l) : "l"(logits + (size_t)tt * E + e));
      s_key[(size_t)tt * G * 32 + e] = e < E ? order_key(l) : 0u;
    }
  __syncthreads();
  if (t < T) {
    for (int g = wt; g < G; g += wpt) {
      const uint32_t* gk = s_key + ((size_t)t * G + g) * 32;
      const uint32_t mine = gk[lane];
      int r = 0;
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        const uint32_t o = gk[m];
        r += (o > mine || (o == mine && m < lane)) ? 1 : 0;
      }
      if (r < kk)
        c_key[(size_t)t * C + g * kk + r] = ((uint64_t)mine << 32) | (uint32_t)~(uint32_t)(g * 32 + lane);
    }
  }
  __syncthreads();
  if (t < T) {
    // 2^ls threads per candidate (at most 32), uniform trip counts per warp
    int ls = 0;
    while (ls < 5 && (C << (ls + 1)) <= tpt) ++ls;
    const int s = 1 << ls;
    const int per = tpt >> ls;                        // candidates per round
    const int q = u & (s - 1);
    const uint64_t* ck = c_key + (size_t)t * C;
    const int nm = (C + s - 1) >> ls;
    for (int c0 = 0; c0 < C; c0 += per) {
      const int c = c0 + (u >> ls);
      const uint64_t mine = c < C ? ck[c] : 0ull;
      int r = 0;
#pragma unroll 8
      for (int i = 0; i < nm; ++i) {
        const int m = q + i * s;
        const uint64_t o = m < C ? ck[m] : 0ull;
        r += o > mine ? 1 : 0;
      }
      for (int o = 1; o < s; o <<= 1) r += __shfl_xor_sync(FULL, r, o);
      if (c < C && q == 0 && r < k) sel[(size_t)t * k + r] = mine;
    }
  }
  __syncthreads();
  if (t < T && wt == 0 && lane < k) {
    const uint64_t* sk = sel + (size_t)t * k;
    const float l0 = order_key_value((uint32_t)(sk[0] >> 32));
    float sum = 0.f, my_p = 0.f;
    for (int j = 0; j < k; ++j) {
      const float p = expf(order_key_value((uint32_t)(sk[j] >> 32)) - l0);
      sum += p;
      if (j == lane) my_p = p;
    }
    const int e = (int)~(uint32_t)sk[lane];
    ids_s[t * k + lane] = e;
    ids_out[(size_t)t * k + lane] = e;
    wts[(size_t)t * k + lane] = my_p / sum;
  }
}

// Ascending bitonic sort of one 32-bit key per lane across a warp.
__device__ __forceinline__ uint32_t warp_sort_u32(uint32_t key, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint32_t other = __shfl_xor_sync(0xffffffffu, key, j);
      const bool keep_min = ((lane & j) == 0) == ((lane & k) == 0);
      key = keep_min ? min(key, other) : max(key, other);
    }
  }
  return key;
}

// Inclusive warp scan.
__device__ __forceinline__ uint32_t warp_scan_u32(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Permutation and classes of at most 32 pairs (ids in shared memory, padded
// with -1 to 32 entries), with the results of the three-launch permutation
// and perm_classes (E <= 1024, so an expert fits 10 bits).  Threads 32.. write
// the count and offset of every expert.  Warp 0 sorts the pair keys
// (expert, pair): lane i then holds permuted row i, so perm and inv follow
// directly, and the runs of equal experts give each active expert its row
// count n and offset.  A second sort orders the active experts by class
// (light before dense), n descending, expert ascending; exclusive warp scans
// over that order give every expert's job-list slots and dense-tile prefixes.
// A single warp runs at about one dependent instruction per several cycles,
// so this path is built from log-depth shuffle networks, not loops over 32.
__device__ void perm_small(const int* ids, int E, int thr, int dense_supported, const PermuteOut& o) {
  const unsigned FULL = 0xffffffffu;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int x = tid - 32; x >= 0 && x <= E; x += (int)blockDim.x - 32) {
    int cn = 0, before = 0;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const int eq = ids[q];
      const bool okq = eq >= 0 && eq < E;
      cn += (okq && eq == x) ? 1 : 0;
      before += (okq && eq < x) ? 1 : 0;
    }
    if (x < E) o.counts[x] = cn;
    o.offsets[x] = before;
  }
  if (warp != 0) return;
  const int e0 = ids[lane];
  const bool ok = e0 >= 0 && e0 < E;
  // 1. pairs in (expert, pair) order
  const uint32_t pk = warp_sort_u32(ok ? ((uint32_t)e0 << 5) | (uint32_t)lane : 0xffffffffu, lane);
  const bool valid = pk != 0xffffffffu;
  const int e = (int)(pk >> 5), pair = (int)(pk & 31u);
  if (valid) {
    o.perm[lane] = pair;
    o.inv[pair] = lane;
  }
  // 2. runs of equal experts: the first row of each run is the expert's offset
  const int e_prev = __shfl_up_sync(FULL, e, 1);
  const bool first = valid && (lane == 0 || e_prev != e);
  const unsigned fm = __ballot_sync(FULL, first);
  const int nvalid = __popc(__ballot_sync(FULL, valid));
  const unsigned later = fm & ~((2u << lane) - 1u);          // run starts after this lane
  const int n = first ? (later ? __ffs(later) - 1 : nvalid) - lane : 0;
  // 3. active experts by (class, n desc, expert asc); the row offset rides along
  const uint32_t cls = (first && n >= thr) ? 1u : 0u;
  const uint32_t ck = first ? (cls << 21) | ((uint32_t)(63 - n) << 15) | ((uint32_t)e << 5) | (uint32_t)lane
                            : 0xffffffffu;
  const uint32_t sk = warp_sort_u32(ck, lane);
  const bool act = sk != 0xffffffffu;
  const bool dense = act && ((sk >> 21) & 1u);
  const int ae = (int)((sk >> 5) & 1023u), an = act ? 63 - (int)((sk >> 15) & 63u) : 0;
  const int aoff = (int)(sk & 31u);
  // 4. exclusive scans over the class order: list-1, list-2 and list-4 jobs
  // (10 bits each), 128- and 256-row tiles (one byte each; at most 64 per
  // byte), padded rows / 256.  At most 32 pairs: an expert has at most 32
  // rows, so one job.
  const uint32_t c1 = (act && !dense && an <= 8) ? 1u : 0u;
  const uint32_t c2 = (act && !dense && an > 8 && an <= 16) ? 1u : 0u;
  const uint32_t c4 = (act && !dense && an > 16) ? 1u : 0u;
  const uint32_t t0 = dense ? (uint32_t)((an + 127) >> 7) : 0u;
  const uint32_t t1 = dense ? (uint32_t)((an + 255) >> 8) : 0u;
  const uint32_t packed = t0 | (t1 << 8);
  const uint32_t jpacked = c1 | (c2 << 10) | (c4 << 20);
  const uint32_t inc = warp_scan_u32(packed, lane), jinc = warp_scan_u32(jpacked, lane);
  const uint32_t exc = inc - packed, jexc = jinc - jpacked;
  const uint32_t tot = __shfl_sync(FULL, inc, 31), jtot = __shfl_sync(FULL, jinc, 31);
  const int nlight = __popc(__ballot_sync(FULL, act && !dense));
  if (act && !dense) {
    const int4 jb = make_int4(ae, aoff, an, 0);
    if (an <= 8) o.jobs1[jexc & 0x3ffu] = jb;
    else if (an <= 16) o.jobs2[(jexc >> 10) & 0x3ffu] = jb;
    else o.jobs4[(jexc >> 20) & 0x3ffu] = jb;
  } else if (dense) {
    const int crank = lane - nlight;
    o.dense_list[crank] = make_int4(ae, aoff, an, (int)((exc >> 8) & 0xffu) * 256);
    o.dense_ntoff[crank] = (int)(exc & 0xffu);
    o.dense_ntoff[E + 1 + crank] = (int)((exc >> 8) & 0xffu);
  }
  const int n_dense = __popc(__ballot_sync(FULL, dense));
  if (lane == 0) {
    *o.n_jobs1 = (int)(jtot & 0x3ffu);
    *o.n_jobs2 = (int)((jtot >> 10) & 0x3ffu);
    *o.n_jobs4 = (int)((jtot >> 20) & 0x3ffu);
    *o.n_dense = n_dense;
    o.dense_ntoff[n_dense] = (int)(tot & 0xffu);
    o.dense_ntoff[E + 1 + n_dense] = (int)((tot >> 8) & 0xffu);
    *o.dense_pad_total = (int)((tot >> 8) & 0xffu) * 256;
    if (n_dense > 0 && !dense_supported) set_error(o.err, kErrUnsupported);
  }
}

// ---------------------------------------------------------------------------
// The same permutation for large batches in three launches.  Block b of nb
// owns the contiguous pairs [P b / nb, P (b + 1) / nb):
//   perm_hist_kernel:  per-block expert counts bcnt[b][e];
//   perm_scan_kernel:  one block: counts, offsets, the active list and the
//                      classes, and bcnt turned into per-block bases
//                      off[e] + sum over earlier blocks;
//   perm_place_kernel: per block, per-warp counts on top of the block base,
//                      then positions in (expert, pair) order (match_any
//                      groups equal experts inside a 32-pair step).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) perm_hist_kernel(const int* __restrict__ ids, long long P, int E,
                                                         int* __restrict__ bcnt) {
  extern __shared__ int hist[];
  const int b = blockIdx.x, nb = gridDim.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const long long c0 = P * b / nb, c1 = P * (b + 1) / nb;
  for (long long i = c0 + threadIdx.x; i < c1; i += blockDim.x) {
    const int e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) bcnt[(size_t)b * E + e] = hist[e];
}

__global__ void __launch_bounds__(1024) perm_scan_kernel(int* __restrict__ bcnt, int nb, int E, int thr,
                                                         int dense_supported, PermuteOut o) {
  extern __shared__ int sm[];
  int* cnt = sm + 32 * E;
  int* off = cnt + E;
  int* act = off + E + 1;
  int* misc = act + E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < 8) misc[threadIdx.x] = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int b = 0; b < nb; ++b) s += bcnt[(size_t)b * E + e];
    cnt[e] = s;
  }
  __syncthreads();
  if (warp == 0) {              // exclusive scan of the counts; compaction of active experts
    int carry = 0, acarry = 0;
    for (int b = 0; b < E; b += 32) {
      const int e = b + lane;
      const int v = e < E ? cnt[e] : 0;
      int incl = v;
      for (int dd = 1; dd < 32; dd <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, dd);
        if (lane >= dd) incl += n;
      }
      if (e < E) off[e] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
      const unsigned am = __ballot_sync(0xffffffffu, v > 0);
      if (v > 0) act[acarry + __popc(am & ((1u << lane) - 1u))] = e;
      acarry += __popc(am);
    }
    if (lane == 0) { off[E] = carry; misc[0] = acarry; }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = off[e];
    for (int b = 0; b < nb; ++b) {
      const int c = bcnt[(size_t)b * E + e];
      bcnt[(size_t)b * E + e] = run;
      run += c;
    }
    o.counts[e] = cnt[e];
    o.offsets[e] = off[e];
  }
  if (threadIdx.x == 0) o.offsets[E] = off[E];
  perm_classes(E, thr, dense_supported, o, sm);
}

__global__ void __launch_bounds__(1024) perm_place_kernel(const int* __restrict__ ids, long long P, int E,
                                                          const int* __restrict__ bbase, PermuteOut o) {
  extern __shared__ int wc[];   // [32][E]
  const int b = blockIdx.x, nb = gridDim.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long b0 = P * b / nb, b1 = P * (b + 1) / nb, nbp = b1 - b0;
  const long long c0 = b0 + nbp * warp / 32, c1 = b0 + nbp * (warp + 1) / 32;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) wc[i] = 0;
  __syncthreads();
  for (long long base = c0; base < c1; base += 32) {          // per-warp counts
    const long long idx = base + lane;
    const bool valid = idx < c1;
    const int e = valid ? ids[idx] : -1;
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    if (valid && lane == __ffs(mask) - 1 && e >= 0 && e < E) wc[warp * E + e] += __popc(mask);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = bbase[(size_t)b * E + e];
    for (int w = 0; w < 32; ++w) {
      const int c = wc[w * E + e];
      wc[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (long long base = c0; base < c1; base += 32) {          // positions
    const long long idx = base + lane;
    const bool valid = idx < c1;
    const int e = valid ? ids[idx] : -1;
    const unsigned mask = __match_any_sync(0xffffffffu, e);
    const bool ok = valid && e >= 0 && e < E;
    if (ok) {
      const int pos = wc[warp * E + e] + __popc(mask & lt);
      o.perm[pos] = (int)idx;
      o.inv[idx] = pos;
    }
    __syncwarp();
    if (ok && lane == __ffs(mask) - 1) wc[warp * E + e] += __popc(mask);
    __syncwarp();
  }
}

// Small-T router logits (T <= 256) and x staging in one launch, plus the
// routing tail for at most 32 (token, expert) pairs.  With T <= 32 the grid
// may have extra blocks (on SMs the logit blocks leave free) that only stage
// x, in parallel with the logits.  Block b (1024 threads)
// computes the fp32 logits of experts EPB*b .. EPB*b + EPB-1 for every token:
// the router rows are staged in shared memory, thread i owns K = [8i, 8i+8)
// (and [8(i+1024), ...) when d > 8192, EPB = 1), so one x load feeds EPB
// experts; per token the 32 warp sums meet in shared memory.  Blocks also
// stage x rows t = b, b + grid, ... in fp16.  With tail != 0 the last block
// to finish (an atomic ticket; no grid barrier) runs the ranked top-k and the
// small permutation, then clears the ticket for the next launch.  Dynamic
// shared memory: the larger of EPB * (d + 1024) floats and, with the tail,
// route_small_ids_offset + 32 ints.
template <int EPB>
__global__ void __launch_bounds__(1024) route_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ rw, int T, int d, int E, int k,
    int thr, int dense_supported, int tail, float* __restrict__ logits, __half* __restrict__ x16,
    float* __restrict__ xscale, int* __restrict__ ids_out, float* __restrict__ wts,
    int* __restrict__ ticket, PermuteOut o) {
  constexpr int NG = 2 / EPB;                           // K groups of 8 per thread
  extern __shared__ __align__(16) int sm[];
  __shared__ float red[33];
  __shared__ int s_last;
  // blocks [0, nlb) compute logits; extra blocks, if any, only stage x (in
  // parallel with the logits); without them the logit blocks stage x
  const int nlb = (E + EPB - 1) / EPB;
  const bool stage_only = blockIdx.x >= nlb;
  const int e0 = stage_only ? E : blockIdx.x * EPB;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* s_w = reinterpret_cast<float*>(sm);
  float* s_part = s_w + (size_t)EPB * d;                // [EPB][32 tokens][32 warps]
  // each thread's router weights straight into registers: thread i owns
  // K = [8 i, 8 i + 8) (and [8 (i + 1024), ...) when NG = 2); every weight
  // is used from registers for all tokens, so no shared-memory staging
  float4 wa[EPB][NG], wb[EPB][NG];
  bool has[NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    const int kk = 8 * (threadIdx.x + q * blockDim.x);
    has[q] = kk < d;
#pragma unroll
    for (int j = 0; j < EPB; ++j) {
      const bool ok = has[q] && e0 + j < E;
      const float4* src = reinterpret_cast<const float4*>(rw + (size_t)(e0 + j) * d + kk);
      wa[j][q] = ok ? __ldg(src) : make_float4(0, 0, 0, 0);
      wb[j][q] = ok ? __ldg(src + 1) : make_float4(0, 0, 0, 0);
    }
  }
  for (int t0 = 0; t0 < (stage_only ? 0 : T); t0 += 32) {
    const int tn = min(32, T - t0);
    // four tokens per pass: their x loads are in flight together (the loop is
    // latency-bound, not issue-bound); each token's sum keeps the same order
    for (int tt = 0; tt < tn; tt += 4) {
      float acc[EPB][4];
#pragma unroll
      for (int j = 0; j < EPB; ++j)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[j][u] = 0.f;
#pragma unroll
      for (int q = 0; q < NG; ++q) {
        if (has[q]) {
          uint4 xv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            xv[u] = tt + u < tn ? *reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt + u) * d +
                                                                  8 * (threadIdx.x + q * blockDim.x))
                                : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int j = 0; j < EPB; ++j) {
              float a = acc[j][u];
              a = fmaf(__uint_as_float(xv[u].x << 16), wa[j][q].x, a);
              a = fmaf(__uint_as_float(xv[u].x & 0xffff0000u), wa[j][q].y, a);
              a = fmaf(__uint_as_float(xv[u].y << 16), wa[j][q].z, a);
              a = fmaf(__uint_as_float(xv[u].y & 0xffff0000u), wa[j][q].w, a);
              a = fmaf(__uint_as_float(xv[u].z << 16), wb[j][q].x, a);
              a = fmaf(__uint_as_float(xv[u].z & 0xffff0000u), wb[j][q].y, a);
              a = fmaf(__uint_as_float(xv[u].w << 16), wb[j][q].z, a);
              a = fmaf(__uint_as_float(xv[u].w & 0xffff0000u), wb[j][q].w, a);
              acc[j][u] = a;
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < EPB; ++j)
#pragma unroll
        for (int u = 0; u < 4; ++u)
          for (int off = 16; off > 0; off >>= 1) acc[j][u] += __shfl_xor_sync(0xffffffffu, acc[j][u], off);
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < EPB; ++j)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (tt + u < tn) s_part[((size_t)j * 32 + tt + u) * 32 + warp] = acc[j][u];
      }
    }
    __syncthreads();
    if (warp < tn) {                       // warp tt sums the 32 warp partials of token t0 + tt
#pragma unroll
      for (int j = 0; j < EPB; ++j) {
        float v = s_part[((size_t)j * 32 + warp) * 32 + lane];
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0 && e0 + j < E) logits[(size_t)(t0 + warp) * E + e0 + j] = v;
      }
    }
    __syncthreads();
  }
  if (gridDim.x > nlb) {
    if (stage_only)
      for (int t = blockIdx.x - nlb; t < T; t += gridDim.x - nlb)
        stage_x_row(x + (size_t)t * d, d, x16 + (size_t)t * d, xscale + t, o.err, red);
  } else {
    for (int t = blockIdx.x; t < T; t += gridDim.x)
      stage_x_row(x + (size_t)t * d, d, x16 + (size_t)t * d, xscale + t, o.err, red);
  }
  if (!tail) {
    pdl_launch_dependents();
    return;
  }
  // ---- last block: routing tail (at most 32 pairs)
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  // ranked top-k (scratch from the start of shared memory, the pair experts
  // after it), then the small permutation
  int* ids_small = sm + route_small_ids_offset(E, T, k);
  topk_small_block(logits, T, E, k, ids_small, ids_out, wts, reinterpret_cast<uint32_t*>(sm));
  if (threadIdx.x >= T * k && threadIdx.x < 32) ids_small[threadIdx.x] = -1;
  __syncthreads();
  perm_small(ids_small, E, thr, dense_supported, o);
  if (threadIdx.x == 0) *ticket = 0;
}

}  // namespace moe
