// Repack of canonical NVFP4 expert matrices into the fragment layout that the
// register-dequant expert kernel streams (layout described in layout.cuh).
#pragma once
#include <cstdint>
#include "layout.cuh"

namespace moe {

enum RepackMode { kGateUp = 0, kDown = 1 };

// ---------------------------------------------------------------------------
// Repack canonical NVFP4 matrices into the fragment layout (see layout.cuh).
// One thread per (expert, tile, chunk, lane).
// MODE kGateUp: rows A(g) = gate row 8t+g, rows B(g) = up row 8t+g, K = d.
// MODE kDown:   rows A(g) = down row 16t+g, rows B(g) = down row 16t+8+g, K = f.
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void repack_fragment_kernel(const uint8_t* __restrict__ qa, const uint8_t* __restrict__ sfa,
                                       const uint8_t* __restrict__ qb, const uint8_t* __restrict__ sfb,
                                       int E, int rows, int K, uint8_t* __restrict__ out) {
  const int tpe = (MODE == kGateUp) ? rows / 8 : rows / 16;
  const int cpt = K / kChunkK;
  const long long total = (long long)E * tpe * cpt * 32;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int lane = (int)(idx & 31);
    const long long rest = idx >> 5;
    const int ch = (int)(rest % cpt);
    const long long et = rest / cpt;
    const int t = (int)(et % tpe);
    const int e = (int)(et / tpe);
    const int g = lane >> 2, c = lane & 3;
    int rowA, rowB;
    const uint8_t *qA, *qB, *sA, *sB;
    if (MODE == kGateUp) {
      rowA = rowB = t * 8 + g;
      qA = qa; sA = sfa; qB = qb; sB = sfb;
    } else {
      rowA = t * 16 + g;
      rowB = rowA + 8;
      qA = qB = qa; sA = sB = sfa;
    }
    const size_t mat = (size_t)e * rows;
    const uint8_t* ra = qA + (mat + rowA) * (K / 2);
    const uint8_t* rb = qB + (mat + rowB) * (K / 2);
    uint8_t* dst = out + ((size_t)((size_t)e * tpe + t) * cpt + ch) * kChunkBytes;
    uint8_t b[16];
    for (int ks = 0; ks < 4; ++ks) {
      const int k0 = ch * kChunkK + ks * 16;
      b[4 * ks + 0] = ra[k0 / 2 + c];
      b[4 * ks + 1] = rb[k0 / 2 + c];
      b[4 * ks + 2] = ra[(k0 + 8) / 2 + c];
      b[4 * ks + 3] = rb[(k0 + 8) / 2 + c];
    }
    uint4 v;
    v.x = b[0] | (b[1] << 8) | (b[2] << 16) | ((uint32_t)b[3] << 24);
    v.y = b[4] | (b[5] << 8) | (b[6] << 16) | ((uint32_t)b[7] << 24);
    v.z = b[8] | (b[9] << 8) | (b[10] << 16) | ((uint32_t)b[11] << 24);
    v.w = b[12] | (b[13] << 8) | (b[14] << 16) | ((uint32_t)b[15] << 24);
    *reinterpret_cast<uint4*>(dst + lane * 16) = v;
    if (c == 0) {
      const uint8_t* fa = sA + (mat + rowA) * (K / 16);
      const uint8_t* fb = sB + (mat + rowB) * (K / 16);
      for (int ks = 0; ks < 4; ++ks) {
        dst[kChunkCodeBytes + g * 8 + ks] = fa[ch * 4 + ks];
        dst[kChunkCodeBytes + g * 8 + 4 + ks] = fb[ch * 4 + ks];
      }
    }
  }
}

}  // namespace moe
