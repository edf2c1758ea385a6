// Repack of canonical NVFP4 expert matrices into the fragment layout that the
// register-dequant expert kernel streams (layout described in layout.cuh).
#pragma once
#include <cstdint>
#include "layout.cuh"
#include "tc.cuh"

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
    const uint8_t* fa = sA + (mat + rowA) * (K / 16);
    const uint8_t* fb = sB + (mat + rowB) * (K / 16);
    uint8_t b[16];
    for (int ks = 0; ks < 4; ++ks) {
      const int k0 = ch * kChunkK + ks * 16;
      // a negative block scale is folded into its codes (sign flip, exact)
      const uint8_t xa = (fa[ch * 4 + ks] & 0x80u) ? 0x88u : 0u;
      const uint8_t xb = (fb[ch * 4 + ks] & 0x80u) ? 0x88u : 0u;
      b[4 * ks + 0] = ra[k0 / 2 + c] ^ xa;
      b[4 * ks + 1] = rb[k0 / 2 + c] ^ xb;
      b[4 * ks + 2] = ra[(k0 + 8) / 2 + c] ^ xa;
      b[4 * ks + 3] = rb[(k0 + 8) / 2 + c] ^ xb;
    }
    uint4 v;
    v.x = b[0] | (b[1] << 8) | (b[2] << 16) | ((uint32_t)b[3] << 24);
    v.y = b[4] | (b[5] << 8) | (b[6] << 16) | ((uint32_t)b[7] << 24);
    v.z = b[8] | (b[9] << 8) | (b[10] << 16) | ((uint32_t)b[11] << 24);
    v.w = b[12] | (b[13] << 8) | (b[14] << 16) | ((uint32_t)b[15] << 24);
    *reinterpret_cast<uint4*>(dst + lane * 16) = v;
    if (c == 0) {
      for (int ks = 0; ks < 4; ++ks) {
        dst[kChunkCodeBytes + g * 8 + ks] = fa[ch * 4 + ks] & 0x7Fu;
        dst[kChunkCodeBytes + g * 8 + 4 + ks] = fb[ch * 4 + ks] & 0x7Fu;
      }
    }
  }
}


// ---------------------------------------------------------------------------
// Largest row L1 norm of each expert's gate and up matrices, in units of
// e2m1 value x e4m3 block scale (the fp32 tensor scale is applied later):
//   l1[m * E + e] = max over rows c of sum_k |e2m1(q[c,k])| * |e4m3(sf[c,k/16])|
// for m = 0 (gate), 1 (up).  One warp per row; the per-expert maximum is taken
// with an integer atomicMax on the bits of the non-negative fp32 sums (order
// independent, so the result is deterministic).  l1 must be zero on entry.
// The light class uses it to bound |g| and |u| before any row is computed
// (see light_h_exp in experts.cuh).
// ---------------------------------------------------------------------------
__global__ void expert_l1_kernel(const uint8_t* __restrict__ gq, const uint8_t* __restrict__ gsf,
                                 const uint8_t* __restrict__ uq, const uint8_t* __restrict__ usf,
                                 int E, int f, int d, float* __restrict__ l1) {
  // twice the e2m1 magnitude of codes 0..7 (0, 1, 2, 3, 4, 6, 8, 12), one per nibble
  constexpr uint32_t kTwiceMag = 0xC8643210u;
  const int lane = threadIdx.x & 31;
  const long long rows = 2LL * E * f;
  const int nb = d / 16;
  for (long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < rows;
       w += ((long long)gridDim.x * blockDim.x) >> 5) {
    const int m = (int)(w / ((long long)E * f));
    const long long r = w - (long long)m * E * f;      // row of the [E*f] matrix
    const uint8_t* q = (m ? uq : gq) + r * (d / 2);
    const uint8_t* sf = (m ? usf : gsf) + r * nb;
    float acc = 0.f;
    for (int b = lane; b < nb; b += 32) {
      const uint2 v = *reinterpret_cast<const uint2*>(q + b * 8);
      uint32_t s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t byte = ((i < 4 ? v.x : v.y) >> (8 * (i & 3))) & 0xffu;
        s += ((kTwiceMag >> (4 * (byte & 7u))) & 15u) + ((kTwiceMag >> (4 * ((byte >> 4) & 7u))) & 15u);
      }
      acc += fabsf(e4m3_to_f32(sf[b])) * (0.5f * (float)s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) atomicMax(reinterpret_cast<int*>(l1) + (size_t)m * E + r / f, __float_as_int(acc));
  }
}

// hexp[e] = Eg + Eu with |gs_g| * l1_g < 2^Eg and |gs_u| * l1_u < 2^Eu
// (frexp exponents; 0 for a zero matrix).  gs: [3][E] tensor scales.
__global__ void expert_hexp_kernel(const float* __restrict__ l1, const float* __restrict__ gs, int E,
                                   int* __restrict__ hexp) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
    int eg = 0, eu = 0;
    frexpf(fabsf(gs[e]) * l1[e], &eg);
    frexpf(fabsf(gs[E + e]) * l1[E + e], &eu);
    hexp[e] = eg + eu;
  }
}

// ---------------------------------------------------------------------------
// Dense-class weight copies for the tensor cores.  The block-scaled MMA reads
// unsigned e4m3 scales, so a negative block scale is folded into the codes:
// the 16 codes of that block change sign and the scale's sign bit is cleared
// (exact).  One thread per (row, 16-value block).
// q: [rows][K/2] canonical codes, sf: [rows][K/16]; writes qd (same layout).
// ---------------------------------------------------------------------------
__global__ void dense_codes_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ sf,
                                   long long rows, int K, uint8_t* __restrict__ qd) {
  const int nb = K / 16;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < rows * nb;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / nb;
    const int blk = (int)(i - r * nb);
    uint2 v = *reinterpret_cast<const uint2*>(q + r * (K / 2) + blk * 8);
    if (sf[i] & 0x80u) { v.x ^= 0x88888888u; v.y ^= 0x88888888u; }
    *reinterpret_cast<uint2*>(qd + r * (K / 2) + blk * 8) = v;
  }
}

// Gate/up rows of the dense class are interleaved in groups of 32 so that one
// 32-lane TMEM quarter of a 128-row accumulator tile holds the gate rows
// (lanes 0-15) and the up rows (lanes 16-31) of the same 16 FFN channels:
// combined row rr of an expert (0 <= rr < 2f) is gate (rr & 16 == 0) or up
// row 16 * (rr / 32) + rr % 16.
__host__ __device__ __forceinline__ int gu_channel(int rr) { return 16 * (rr >> 5) + (rr & 15); }
__host__ __device__ __forceinline__ bool gu_is_up(int rr) { return (rr & 16) != 0; }

// Combined gate/up codes [E][2f][d/2] in the interleaved row order, signs of
// negative block scales folded into the codes.  One thread per (row, block).
__global__ void dense_gu_codes_kernel(const uint8_t* __restrict__ gq, const uint8_t* __restrict__ gsf,
                                      const uint8_t* __restrict__ uq, const uint8_t* __restrict__ usf,
                                      int E, int f, int d, uint8_t* __restrict__ qd) {
  const int nb = d / 16;
  const long long rows = (long long)E * 2 * f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < rows * nb;
       i += (long long)gridDim.x * blockDim.x) {
    const long long R = i / nb;
    const int blk = (int)(i - R * nb);
    const int e = (int)(R / (2 * f)), rr = (int)(R % (2 * f));
    const long long src = (long long)e * f + gu_channel(rr);
    const uint8_t* q = gu_is_up(rr) ? uq : gq;
    const uint8_t* sf = gu_is_up(rr) ? usf : gsf;
    uint2 v = *reinterpret_cast<const uint2*>(q + src * (d / 2) + blk * 8);
    if (sf[src * nb + blk] & 0x80u) { v.x ^= 0x88888888u; v.y ^= 0x88888888u; }
    *reinterpret_cast<uint2*>(qd + R * (d / 2) + blk * 8) = v;
  }
}

// Scales of the dense weights in the tensor-core layouts (gate/up:
// sf_rowpair_offset, 256-row N tiles; down: sf_pair_offset, 128-row M tiles),
// sign bit cleared.  One thread per (combined row, 16-block).
// MODE kGateUp: combined (interleaved) gate/up rows, rows = f per matrix, K = d.
// MODE kDown: down rows, rows = d, K = f.
template <int MODE>
__global__ void dense_sf_atoms_kernel(const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb,
                                      int E, int rows, int K, uint8_t* __restrict__ out) {
  const int nb = K / 16;
  const int crows = (MODE == kGateUp) ? 2 * rows : rows;     // combined rows per expert
  const long long total = (long long)E * crows * nb;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long R = i / nb;
    const int kb = (int)(i - R * nb);
    const int e = (int)(R / crows), rr = (int)(R % crows);
    const uint8_t* src = sfa;
    long long row = (long long)e * rows + rr;
    if (MODE == kGateUp) {
      src = gu_is_up(rr) ? sfb : sfa;
      row = (long long)e * rows + gu_channel(rr);
    }
    const uint8_t v = src[row * nb + kb] & 0x7Fu;
    // gate/up weights are the N = 256 operand, down weights the M = 128 one
    const size_t o = MODE == kGateUp ? sf_rowpair_offset(R, kb, K / 64) : sf_pair_offset(R, kb, K / 64);
    out[o] = v;
  }
}

}  // namespace moe
