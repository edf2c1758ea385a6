// Combine and unpermute in a single pass over the per-pair partials.
//
// combine_kernel:       out[t] = bf16_rn( sum_j partial[inv[t,j]] ), slots
//                       j = 0..k-1 summed in order in fp32 (after x[t] when
//                       the residual add is on).
// combine_norm_kernel:  out[t] = bf16_rn( sum_j w[t,j] * y_j / sqrt(mean_i y_j[i]^2 + eps) ),
//                       y_j = partial[inv[t,j]] the unweighted expert output
//                       (the down epilogues skip the routing weight in this
//                       mode), an RMS normalisation of every expert's output
//                       with no learned gain, then the routing-weighted sum.
// Both read each partial row of a token once from HBM (the norm variant
// reads it a second time right after, from L2) and store each output row
// once, so the output needs no prior clearing.  Source: "Optimizing Muse
// Spark Open on TPU v7 with SGLang-TorchTPU", section 8 (the per-expert norm
// before the weighted sum, and the fused single-pass combine that replaced
// three separate passes).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace moe {

__device__ __forceinline__ uint4 pack_bf16x8(const float (&s)[8]) {
  uint4 o;
  uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(s[2 * i], s[2 * i + 1]);
    ow[i] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return o;
}

// grid (ceil(d / (8 * blockDim.x)), min(T, 65535)); tokens t = blockIdx.y,
// blockIdx.y + gridDim.y, ...; each thread owns 8 consecutive columns.
// resid (optional, bf16 [T][d]): the sum starts from resid[t] (a residual add
// in the same fp32 sum, one rounding).
__device__ __forceinline__ void load_resid8(const uint16_t* resid, size_t off, float (&s)[8]) {
  if (!resid) {
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] = 0.f;
    return;
  }
  const uint4 r = *reinterpret_cast<const uint4*>(resid + off);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s[2 * i] = __uint_as_float(w[i] << 16);
    s[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ partial,
                                                      const int* __restrict__ inv, int T, int k,
                                                      int d, const uint16_t* __restrict__ resid,
                                                      uint16_t* __restrict__ out) {
  pdl_wait();
  const int col = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  for (int t = blockIdx.y; t < T && col < d; t += gridDim.y) {
    float s[8];
    load_resid8(resid, (size_t)t * d + col, s);
    // slots in groups of 8: all index loads, then all row loads, then the sums
    for (int j0 = 0; j0 < k; j0 += 8) {
      int pos[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) pos[q] = j0 + q < k ? inv[(size_t)t * k + j0 + q] : -1;
      float4 a[8], b[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (pos[q] >= 0) {
          const float* src = partial + (size_t)pos[q] * d + col;
          a[q] = *reinterpret_cast<const float4*>(src);
          b[q] = *reinterpret_cast<const float4*>(src + 4);
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (pos[q] >= 0) {
          s[0] += a[q].x; s[1] += a[q].y; s[2] += a[q].z; s[3] += a[q].w;
          s[4] += b[q].x; s[5] += b[q].y; s[6] += b[q].z; s[7] += b[q].w;
        }
      }
    }
    *reinterpret_cast<uint4*>(out + (size_t)t * d + col) = pack_bf16x8(s);
  }
  pdl_launch_dependents();
}

constexpr int kNormThreads = 256;
constexpr int kNormMaxK = 32;

// One block per token (grid-stride over tokens).  Pass 1: each thread sums
// the squares of its columns of every slot's row; a block reduction gives
// ss_j.  Pass 2: scale_j = w_j / sqrt(ss_j / d + eps) (IEEE sqrt and
// division), out = sum_j y_j * scale_j in slot order.  wts is [T][k].
__global__ void __launch_bounds__(kNormThreads) combine_norm_kernel(
    const float* __restrict__ partial, const int* __restrict__ inv, const float* __restrict__ wts, int T,
    int k, int d, float eps, const uint16_t* __restrict__ resid, uint16_t* __restrict__ out) {
  __shared__ float red[kNormThreads / 32][kNormMaxK];
  __shared__ float scale[kNormMaxK];
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    float ss[kNormMaxK];
#pragma unroll
    for (int j = 0; j < kNormMaxK; ++j) ss[j] = 0.f;
    for (int col = threadIdx.x * 8; col < d; col += kNormThreads * 8) {
#pragma unroll
      for (int j = 0; j < kNormMaxK; ++j) {
        if (j < k) {
          const float* src = partial + (size_t)inv[(size_t)t * k + j] * d + col;
          const float4 a = *reinterpret_cast<const float4*>(src);
          const float4 b = *reinterpret_cast<const float4*>(src + 4);
          ss[j] += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w + b.x * b.x + b.y * b.y + b.z * b.z +
                   b.w * b.w;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kNormMaxK; ++j) {
      if (j < k) {
        float v = ss[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][j] = v;
      }
    }
    __syncthreads();
    if (threadIdx.x < k) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kNormThreads / 32; ++w) v += red[w][threadIdx.x];
      scale[threadIdx.x] = wts[(size_t)t * k + threadIdx.x] / sqrtf(v / (float)d + eps);
    }
    __syncthreads();
    for (int col = threadIdx.x * 8; col < d; col += kNormThreads * 8) {
      float s[8];
      load_resid8(resid, (size_t)t * d + col, s);
      for (int j = 0; j < k; ++j) {
        const float* src = partial + (size_t)inv[(size_t)t * k + j] * d + col;
        const float4 a = *reinterpret_cast<const float4*>(src);
        const float4 b = *reinterpret_cast<const float4*>(src + 4);
        const float c = scale[j];
        s[0] += a.x * c; s[1] += a.y * c; s[2] += a.z * c; s[3] += a.w * c;
        s[4] += b.x * c; s[5] += b.y * c; s[6] += b.z * c; s[7] += b.w * c;
      }
      *reinterpret_cast<uint4*>(out + (size_t)t * d + col) = pack_bf16x8(s);
    }
    __syncthreads();                     // red / scale reused by the next token
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// Pieces of an expert-parallel forward (the rows of a pair travel to the rank
// that owns its expert and its expert output travels back):
//   gather_rows_kernel:    rows[i] = x[perm[i] / k], the token row of each
//                          pair in permutation order (bf16, 16-byte moves);
//   unpermute_rows_kernel: y[i] = partial[inv[i]] for one expert per row
//                          (inv[i] outside [0, n): zeros);
//   combine_rows_kernel:   out[t] = bf16_rn( sum_j fl(w[t,j] * y[inv[t,j]]) ),
//                          slots j in order, fp32.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int* __restrict__ perm, int P, int k, int d,
                                                          uint16_t* __restrict__ rows) {
  const int n16 = d / 8;                         // 16-byte chunks per row
  for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < (long long)P * n16;
       c += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(c / n16), q = (int)(c - (long long)i * n16);
    const int t = perm[i] / k;
    reinterpret_cast<uint4*>(rows + (size_t)i * d)[q] = reinterpret_cast<const uint4*>(x + (size_t)t * d)[q];
  }
}

__global__ void __launch_bounds__(256) unpermute_rows_kernel(const float* __restrict__ partial,
                                                             const int* __restrict__ inv, int n, int d,
                                                             float* __restrict__ y) {
  const int n4 = d / 4;
  for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < (long long)n * n4;
       c += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(c / n4), q = (int)(c - (long long)i * n4);
    // a row whose expert id was rejected has no permuted position: zeros
    const int r = inv[i];
    reinterpret_cast<float4*>(y + (size_t)i * d)[q] =
        (r >= 0 && r < n) ? reinterpret_cast<const float4*>(partial + (size_t)r * d)[q]
                          : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// grid (ceil(d / (8 * blockDim.x)), min(T, 65535)), as combine_kernel
__global__ void __launch_bounds__(128) combine_rows_kernel(const float* __restrict__ y,
                                                           const int* __restrict__ inv,
                                                           const float* __restrict__ wts, int T, int k,
                                                           int d, uint16_t* __restrict__ out) {
  const int col = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  for (int t = blockIdx.y; t < T && col < d; t += gridDim.y) {
    float s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      const float w = wts[(size_t)t * k + j];
      const float* src = y + (size_t)inv[(size_t)t * k + j] * d + col;
      const float4 a = *reinterpret_cast<const float4*>(src);
      const float4 b = *reinterpret_cast<const float4*>(src + 4);
      s[0] += __fmul_rn(w, a.x); s[1] += __fmul_rn(w, a.y); s[2] += __fmul_rn(w, a.z); s[3] += __fmul_rn(w, a.w);
      s[4] += __fmul_rn(w, b.x); s[5] += __fmul_rn(w, b.y); s[6] += __fmul_rn(w, b.z); s[7] += __fmul_rn(w, b.w);
    }
    *reinterpret_cast<uint4*>(out + (size_t)t * d + col) = pack_bf16x8(s);
  }
}

}  // namespace moe
