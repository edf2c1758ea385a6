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
    for (int j = 0; j < k; ++j) {
      const float* src = partial + (size_t)inv[(size_t)t * k + j] * d + col;
      const float4 a = *reinterpret_cast<const float4*>(src);
      const float4 b = *reinterpret_cast<const float4*>(src + 4);
      s[0] += a.x; s[1] += a.y; s[2] += a.z; s[3] += a.w;
      s[4] += b.x; s[5] += b.y; s[6] += b.z; s[7] += b.w;
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
