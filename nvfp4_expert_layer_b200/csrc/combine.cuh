// One-pass combine and unpermute: out[t] = bf16_rn( sum_j partial[inv[t,j]] ),
// summed in slot order j = 0..k-1 in fp32, every output row written exactly
// once with no zero fill ("Optimizing Muse Spark Open on TPU v7 with
// SGLang-TorchTPU", section 8: a one-pass combine that reads the partials
// once; no zero fill, every output row written exactly once).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace moe {

// grid (ceil(d / (8 * blockDim.x)), T); each thread owns 8 consecutive columns.
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ partial,
                                                      const int* __restrict__ inv, int T, int k,
                                                      int d, uint16_t* __restrict__ out) {
  pdl_wait();
  const int t = blockIdx.y;
  const int col = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (t < T && col < d) {
    float s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
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
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(s[2 * i], s[2 * i + 1]);
      ow[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(out + (size_t)t * d + col) = o;
  }
  pdl_launch_dependents();
}

}  // namespace moe
