// Dense expert class: experts that received at least `thr` rows run as
// grouped block-scaled NVFP4 GEMMs on the tcgen05 tensor cores, accumulating
// in TMEM ("Optimizing Models to Be Fast at Codegen", section 2: keep the
// weights 4-bit all the way to the tensor core and feed Blackwell's FP4
// tensor cores from shared memory; "Optimizing Muse Spark Open on TPU v7 with
// SGLang-TorchTPU", section 8: the fused MoE prefill kernel streams one
// expert's weights while the next prefetches, then gate/up, SwiGLU and down).
//
// Activations of the dense class are NVFP4 too (e2m1 values, one e4m3 scale
// per 16 along K, tensor scale 1): sf = e4m3_rn(amax / 6), q = e2m1_rn(v / sf),
// both decided in IEEE fp32.  Rows of every dense expert are padded to a
// multiple of 128 so each 128-token tile starts on a scale-unit boundary.
//
// Each MMA is D[128][N] += A[128][64] * B[N][64]^T (kind::mxf4nvf4, scale
// vector 16, N = 256, or 128 for a short last token tile of GEMM 2).
// GEMM 1 (kDenseGateUp): A = 128 tokens, B = 256 rows of the combined gate/up
//   matrix, gate and up interleaved in groups of 16 channels.  One TMEM lane
//   holds one token, and its 32 consecutive columns are the gate and the up
//   values of one 16-channel NVFP4 block of h: the epilogue forms
//   h = SiLU(g) * u, the block scale and the codes in registers and writes
//   the B operand of GEMM 2.
// GEMM 2 (kDenseDown): A = 128 rows of Wd, B = 256 tokens.  One TMEM lane
//   holds one output dimension, so for each token the 32 lanes of a warp write
//   128 contiguous bytes of the fp32 partial w * gs * D (permutation order).
// The A side is read as 128-row tiles with scales in the sf_pair_offset
// layout, the B side as 256-row tiles with scales in the sf_rowpair_offset
// layout; dense experts are padded to 256 rows.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "tc.cuh"

namespace moe {

constexpr int kDenseEpiWarps = 8;          // two per TMEM lane quarter, each on 128 of the 256 columns
constexpr int kDenseThreads = 64 + 32 * kDenseEpiWarps;   // warp 0 TMA, warp 1 MMA, warps 2.. epilogue
// K per pipeline stage: 256 fp4 values (128-byte rows, 128-byte swizzle) in
// three stages, or 128 (64-byte rows, 64-byte swizzle) in six.  Both keep the
// same bytes in flight; on B200 the 256 stages are faster (fewer barrier round
// trips and scale copies per MMA), 2.52 against 2.91 ms for the prefill gate/up.
constexpr int kDenseKStage = 256;
constexpr int kDenseRowBytes = kDenseKStage / 2;
constexpr int kDenseMmaPerStage = kDenseKStage / 64;
// Scale copies into TMEM, per GEMM (DenseStageCfg): a broadcast copy
// (tcgen05.cp .32x128b.warpx4) fills all four TMEM lane quarters from one
// 512-byte source, so shared memory holds every scale block once (6 KB a
// stage) and four stages fit; a .128x256b copy reads four replicas of a
// block (24 KB a stage, three stages) with half the copy instructions.  On
// B200 the down GEMM (8 stages per tile) gains from the fourth stage and the
// gate/up GEMM (28 stages per tile) from the fewer copies.
constexpr int kDenseN = 256;               // weight rows per tile (MMA N)
constexpr int kDenseABytes = 128 * kDenseRowBytes;       // 128 rows of the M operand
constexpr int kDenseBBytes = kDenseN * kDenseRowBytes;   // 256 rows of the N operand
// Scale blocks of a stage: one (tile, stage) block of device memory (2 KB M
// side, 4 KB N side), placed kDenseSfCopies times in a row in shared memory
constexpr int kSfaBlock = kSfPairUnitsPerStage * 4 * kSfGroupBytes;
constexpr int kSfbBlock = kSfRowpairUnitsPerStage * 4 * kSfGroupBytes;
constexpr uint32_t kDenseTmemCols = 512;
constexpr uint32_t kDenseSfCols = kDenseMmaPerStage * (4 + 8);   // per stage: 4 M-side + 8 N-side columns per MMA

enum DenseMode { kDenseGateUp = 0, kDenseDown = 1 };

template <int MODE>
struct DenseStageCfg {
  static constexpr bool kBcast = MODE == kDenseDown;
  static constexpr int kCopies = kBcast ? 1 : kSfReplicas;        // copies of each scale block in shared memory
  static constexpr int kStages = kBcast ? 4 : 3;
  static constexpr int kSfaBytes = kCopies * kSfaBlock;           // M-side pair layout
  static constexpr int kSfbBytes = kCopies * kSfbBlock;           // N-side rowpair layout
  static constexpr int kStageBytes = kDenseABytes + kDenseBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kBarBytes = (2 * kStages + 3) * 8 + 8;     // full[S] empty[S] accf acce done, padded
  static_assert(kDenseN + kDenseSfCols * kStages <= kDenseTmemCols, "accumulator + scales exceed TMEM");
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
};

// Dense list entry: {expert, row0 (permutation rows), rows, padded row0}.
struct DenseParams {
  CUtensorMap tmA;       // M side, box 128 B x 128 rows: gate/up x codes [pad rows][d/2]; down Wd [E*d][f/2]
  CUtensorMap tmB;       // N side, box 128 B x 256 rows: gate/up combined W [E*2f][d/2]; down h codes [pad rows][f/2]
  // CTA pairs (dense_gemm_pair_kernel): the N side in boxes of 128 rows, and
  // the scale blocks as 2-D byte tensors of 256-byte rows (a stage's M-side
  // block is 8 rows, its N-side block 16 rows)
  CUtensorMap tmB2;
  CUtensorMap tmSfa;
  CUtensorMap tmSfb;
  const uint8_t* sfA;    // M-side scales (sf_pair_offset layout)
  const uint8_t* sfB;    // N-side scales (sf_rowpair_offset layout)
  const int4* dense;     // dense list, ranked by rows descending
  const int* n_dense;
  const int* ntoff;      // [E+1] exclusive prefix over the dense list of the token tiles per expert
                         // (gate/up: ceil(rows / 128); down: ceil(rows / 256))
  int wt_per_expert;     // weight tiles per expert: gate/up 2f / 256, down d / 128
  int rows_per_expert;   // gate/up: 2f; down: d (rows of the weight copy per expert)
  int kstages;           // K / 256
  int kb64;              // K / 64
  int d, f, topk;
  const float* gs;       // [3][E]
  int E;
  const int* perm;
  const float* wts;      // routing weight per pair; null: partials unweighted
  // gate/up outputs
  uint8_t* hq;           // [P_pad][f/2]
  uint8_t* hsf;          // scales of hq (sf_rowpair_offset layout, K = f)
  float* h32;            // [P][f] or null
  // dynamic activation tensor scales (null: tensor scale 1):
  const int* x_amax;     // bits of max|x| of the call: gate/up results times gs_x
  int* h_amax;           // gate/up: write fp32 h to h32 and max|h| here, no NVFP4 h
  const int* h_amax_in;  // down: results times gs_h
  // down output
  float* partial;        // [P][d]
  int* err;
  int64_t wait_timeout_ns;
};

// ---------------------------------------------------------------------------
// Dynamic activation tensor scale (optional): gs = 2^e, e the smallest
// integer with amax <= 6 * 448 * 2^e, so the block scales of the largest
// block reach the top of the e4m3 range.  Found with exact comparisons
// (2688 * 2^e is exact in fp32): amax < 2^E (frexp) gives e = E - 12 when
// amax <= 2688 * 2^(E - 12) = 0.65625 * 2^E, else E - 11.  amax = 0 gives 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int pow2_tensor_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int E;
  frexpf(amax, &E);
  const int e = E - 12;
  return max(-100, min(100, amax <= ldexpf(2688.f, e) ? e : e + 1));
}
__device__ __forceinline__ float exp2i_f(int e) { return __int_as_float((e + 127) << 23); }

// ---------------------------------------------------------------------------
// Activation quantiser of the dense class, in two passes.
// quant_tok_kernel: one thread per (token, 16-value block): the bf16 row ->
//   NVFP4 codes [T][d/2] and one e4m3 scale byte per 16 values [T][d/16]
//   (plain layout).
// gather_x_dense_kernel: the codes and scales of token perm[row0 + i] / topk
//   copied into the padded permutation order, codes a warp per row over the
//   whole grid, scales a block per 128-row tile (assembled into whole
//   sf_pair_offset units, written with coalesced 16-byte stores).
//   Rows past an expert's count up to its next multiple of tile_rows -- the
//   rows a token tile of the gate/up GEMM reads (128, or 256 for CTA pairs)
//   -- are zeros; rows beyond are never read.
// Each token is quantised once, however many dense experts it is routed to.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int dense_rank_of_padrow(const int4* dense, int nd, int prow) {
  int lo = 0, hi = nd - 1;                       // pad0 increases with rank
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (dense[mid].w <= prow) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256) quant_tok_kernel(const uint16_t* __restrict__ x, int T, int d,
                                                        const int* __restrict__ n_dense,
                                                        const int* __restrict__ x_amax,
                                                        uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf) {
  pdl_wait();
  if (*n_dense == 0) { pdl_launch_dependents(); return; }
  const int nblk = d / 16;
  // dynamic tensor scale gs = 2^e: the values are quantised as v * 2^-e (exact)
  const float inv_gs = x_amax ? exp2i_f(-pow2_tensor_exp(__int_as_float(*x_amax))) : 1.f;
  // one thread per (token, 16-value block); consecutive threads take
  // consecutive blocks of a row (32-byte loads, 8-byte code stores)
  const long long units = (long long)T * nblk;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(u / nblk), blk = (int)(u - (long long)t * nblk);
    const uint16_t* src = x + (size_t)t * d + blk * 16;
    const uint4 a = *reinterpret_cast<const uint4*>(src);
    const uint4 b = *reinterpret_cast<const uint4*>(src + 8);
    const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float v[16];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      v[2 * q] = __uint_as_float(wv[q] << 16) * inv_gs;
      v[2 * q + 1] = __uint_as_float(wv[q] & 0xffff0000u) * inv_gs;
    }
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(v[q]));
    const uint32_t sfbyte = f32x2_to_e4m3x2(0.f, amax / 6.0f) & 0xffu;
    const float sf = e4m3_to_f32(sfbyte);
    uint2 codes = make_uint2(0, 0);
    if (sf > 0.f) {
      uint32_t c[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) c[q] = f32x2_to_e2m1x2(v[2 * q + 1] / sf, v[2 * q] / sf);
      codes.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
      codes.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
    }
    *reinterpret_cast<uint2*>(xq + (size_t)t * (d / 2) + blk * 8) = codes;
    xsf[(size_t)t * nblk + blk] = (uint8_t)sfbyte;
  }
  pdl_launch_dependents();
}

__global__ void __launch_bounds__(256) gather_x_dense_kernel(
    const uint8_t* __restrict__ xq_tok, const uint8_t* __restrict__ xsf_tok, const int4* __restrict__ dense,
    const int* __restrict__ n_dense, const int* __restrict__ pad_total, const int* __restrict__ perm, int topk,
    int d, int tile_rows, uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf) {
  __shared__ int s_tok[128];                     // token of each row of a tile, -1 for padding
  pdl_wait();
  const int nd = *n_dense;
  if (nd == 0) { pdl_launch_dependents(); return; }
  const int rows = *pad_total;
  const int n16 = d / 32;                        // 16-byte chunks of a code row
  const int npairs = d / 128;                    // scale units per 128-row tile
  const int lane = threadIdx.x & 31;
  // codes: a warp per padded row (every block takes part, however few the
  // rows), its lanes on consecutive 16-byte chunks
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nwarps) {
    const int4 de = dense[dense_rank_of_padrow(dense, nd, r)];
    const int i = r - de.w;
    if (i >= (de.z + tile_rows - 1) / tile_rows * tile_rows) continue;   // past the last token tile: never read
    const int t = i < de.z ? perm[de.y + i] / topk : -1;
    const uint4* src = reinterpret_cast<const uint4*>(xq_tok + (size_t)max(t, 0) * (d / 2));
    uint4* dst = reinterpret_cast<uint4*>(xq + (size_t)r * (d / 2));
    for (int ch = lane; ch < n16; ch += 32) dst[ch] = t >= 0 ? src[ch] : make_uint4(0, 0, 0, 0);
  }
  // scales: a block per 128-row tile; the 16 bytes of row slot l and 64-group
  // g hold the 4 scale bytes of rows l, l + 32, l + 64, l + 96 (see
  // sf_pair_offset), one 16-byte store per (pair, row slot, half)
  for (int tile = blockIdx.x; tile < rows / 128; tile += gridDim.x) {
    const int4 de = dense[dense_rank_of_padrow(dense, nd, tile * 128)];   // a tile lies inside one expert
    const int i0 = tile * 128 - de.w;
    if (i0 >= (de.z + tile_rows - 1) / tile_rows * tile_rows) continue;
    __syncthreads();                             // s_tok of the previous tile consumed
    if (threadIdx.x < 128) {
      const int i = i0 + threadIdx.x;
      s_tok[threadIdx.x] = i < de.z ? perm[de.y + i] / topk : -1;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < npairs * 64; c += blockDim.x) {
      const int pr = c >> 6, q = c & 63;
      const int l = q >> 1, h = q & 1;
      const int g = 2 * pr + h;                  // 64-wide K group
      uint32_t w[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int t = s_tok[l + 32 * m];
        w[m] = t >= 0 ? reinterpret_cast<const uint32_t*>(xsf_tok + (size_t)t * (d / 16))[g] : 0u;
      }
      *reinterpret_cast<uint4*>(xsf + sf_pair_offset((long long)tile * 128 + l, 4 * g, d / 64)) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  pdl_launch_dependents();
}

// max |x| of a bf16 tensor into *amax (int bits of a non-negative float;
// atomicMax is order independent, so the result is deterministic)
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint16_t* __restrict__ x, long long n,
                                                        const int* __restrict__ n_dense, int* __restrict__ amax) {
  pdl_wait();
  if (*n_dense == 0) { pdl_launch_dependents(); return; }
  float m = 0.f;
  for (long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n;
       i += (long long)gridDim.x * blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[q] << 16)), fabsf(__uint_as_float(w[q] & 0xffff0000u))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(amax, __float_as_int(m));
  pdl_launch_dependents();
}

// Dynamic h scale: the NVFP4 h of every padded dense row from the fp32 h the
// gate/up GEMM wrote (permutation rows), quantised as h * 2^-e_h with the R4
// rule; rows past an expert's count up to its next multiple of tile_rows
// (the token tile of the down GEMM: 128, or 256 for CTA pairs) are zeros.
// One warp per (padded row, 8 blocks of 16): codes and sf_rowpair_offset scales.
__global__ void __launch_bounds__(256) quant_h_dense_kernel(const float* __restrict__ h32, const int4* __restrict__ dense,
                                                            const int* __restrict__ n_dense,
                                                            const int* __restrict__ pad_total,
                                                            const int* __restrict__ h_amax, int f, int tile_rows,
                                                            uint8_t* __restrict__ hq, uint8_t* __restrict__ hsf) {
  pdl_wait();
  const int nd = *n_dense;
  if (nd == 0) { pdl_launch_dependents(); return; }
  const float inv_gs = exp2i_f(-pow2_tensor_exp(__int_as_float(*h_amax)));
  const int rows = *pad_total, nb = f / 16;
  const long long units = (long long)rows * nb;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(u / nb), kb = (int)(u - (long long)r * nb);
    const int4 de = dense[dense_rank_of_padrow(dense, nd, r)];
    const int i = r - de.w;
    if (i >= (de.z + tile_rows - 1) / tile_rows * tile_rows) continue;   // beyond the last token tile: never read
    uint32_t sfbyte = 0u;
    uint2 codes = make_uint2(0, 0);
    if (i < de.z) {
      const float4* src = reinterpret_cast<const float4*>(h32 + (size_t)(de.y + i) * f + kb * 16);
      float v[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 a = src[q];
        v[4 * q] = a.x * inv_gs; v[4 * q + 1] = a.y * inv_gs; v[4 * q + 2] = a.z * inv_gs; v[4 * q + 3] = a.w * inv_gs;
      }
      float am = 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q) am = fmaxf(am, fabsf(v[q]));
      sfbyte = f32x2_to_e4m3x2(0.f, am / 6.0f) & 0xffu;
      const float sf = e4m3_to_f32(sfbyte);
      if (sf > 0.f) {
        uint32_t c[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) c[q] = f32x2_to_e2m1x2(v[2 * q + 1] / sf, v[2 * q] / sf);
        codes.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
        codes.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
      }
    }
    *reinterpret_cast<uint2*>(hq + (size_t)r * (f / 2) + kb * 8) = codes;
    hsf[sf_rowpair_offset(r, kb, f / 64)] = (uint8_t)sfbyte;
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// Grouped block-scaled NVFP4 GEMM on tcgen05 (persistent, one block per SM).
// Tiles are (dense rank j, weight tile wt, token tile tt) with tt fastest, so
// the blocks working at the same time share a weight tile through L2.
// ---------------------------------------------------------------------------
struct DenseTile {
  int wt, tt;
  int4 de;      // {expert, row0, rows, padded row0}
};

__device__ __forceinline__ DenseTile dense_tile(const int4* __restrict__ dl, const int* __restrict__ ntoff,
                                                int nd, int wtpe, int i) {
  // rank j with wtpe * ntoff[j] <= i < wtpe * ntoff[j+1]
  int lo = 0, hi = nd - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (wtpe * __ldg(ntoff + mid) <= i) lo = mid; else hi = mid - 1;
  }
  DenseTile t;
  t.de = __ldg(dl + lo);
  const int n0 = __ldg(ntoff + lo);
  const int ntj = __ldg(ntoff + lo + 1) - n0;
  const int local = i - wtpe * n0;
  t.wt = local / ntj;
  t.tt = local - t.wt * ntj;
  return t;
}

// One epilogue warp's share of a drained accumulator: this lane's M-side
// row (m_row: an output dimension for down, a token index within the expert
// for gate/up) x the 128 accumulator columns 128 hf .. 128 hf + 127.  For
// down the columns are the tokens n_tok0 + 128 hf + c of the expert.
template <int MODE>
__device__ __forceinline__ void dense_epilogue(const DenseParams& p, const DenseTile& tl, const uint32_t (&r)[128],
                                               int m_row, int n_tok0, int hf, int lane) {
  const int e = tl.de.x;
  if (MODE == kDenseDown) {
    // lane = output dimension drow; columns = tokens 128 hf .. 128 hf + 127 of the tile
    const int drow = m_row;
    const int nrows = min(kDenseN, tl.de.z - n_tok0) - hf * 128;
    const int prow0 = tl.de.y + n_tok0 + hf * 128;               // permutation row of column 0
    const float gsd = p.gs[2 * p.E + e] *
                      (p.h_amax_in ? exp2i_f(pow2_tensor_exp(__int_as_float(*p.h_amax_in))) : 1.f);
#pragma unroll
    for (int c32 = 0; c32 < 4; ++c32) {
      if (32 * c32 >= nrows) break;                              // warp-uniform
      // routing weight x tensor scale of column 32 c32 + lane, broadcast below
      const float wl = 32 * c32 + lane < nrows
                           ? (p.wts ? p.wts[p.perm[prow0 + 32 * c32 + lane]] : 1.f) * gsd : 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float wv = __shfl_sync(0xffffffffu, wl, c);
        if (32 * c32 + c < nrows)
          p.partial[(size_t)(prow0 + 32 * c32 + c) * p.d + drow] = __uint_as_float(r[32 * c32 + c]) * wv;
      }
    }
  } else {
    // columns 32 bl .. 32 bl + 31: gate (first 16) and up (last 16) of the
    // channels chb + 16 bl .. chb + 16 bl + 15, one NVFP4 block of h each
    const int tok = m_row;                           // token of this lane within the expert
    const bool valid = tok < tl.de.z;
    const int prow = tl.de.y + tok;                  // permutation row
    const int hrow = tl.de.w + tok;                  // padded row
    const float gsx = p.x_amax ? exp2i_f(pow2_tensor_exp(__int_as_float(*p.x_amax))) : 1.f;
    const float gsg = p.gs[e] * gsx, gsu = p.gs[p.E + e] * gsx;
    float hmax = 0.f;
    const int chb = tl.wt * (kDenseN / 2) + hf * 64;
    uint32_t codes[8];
    uint32_t sfw = 0u;
#pragma unroll
    for (int bl = 0; bl < 4; ++bl) {
      float hv[16];
      float am = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float gv = __uint_as_float(r[32 * bl + i]) * gsg;
        const float uv = __uint_as_float(r[32 * bl + 16 + i]) * gsu;
        hv[i] = gv / (1.f + expf(-gv)) * uv;
        am = fmaxf(am, fabsf(hv[i]));
      }
      if (p.h32 && valid) {
        float4* dst = reinterpret_cast<float4*>(p.h32 + (size_t)prow * p.f + chb + 16 * bl);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
      }
      if (p.h_amax) {                 // dynamic h scale: quantised by quant_h_dense_kernel
        if (valid) hmax = fmaxf(hmax, am);
        continue;
      }
      const uint32_t sfbyte = f32x2_to_e4m3x2(0.f, am / 6.0f) & 0xffu;
      const float sf = e4m3_to_f32(sfbyte);
      uint32_t w0 = 0u, w1 = 0u;                    // channel i -> nibble i % 8 of word i / 8
      if (sf > 0.f) {
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          w0 |= f32x2_to_e2m1x2(hv[i + 1] / sf, hv[i] / sf) << (4 * i);
          w1 |= f32x2_to_e2m1x2(hv[i + 9] / sf, hv[i + 8] / sf) << (4 * i);
        }
      }
      codes[2 * bl] = w0;
      codes[2 * bl + 1] = w1;
      sfw |= sfbyte << (8 * bl);
    }
    if (p.h_amax) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
      if (lane == 0 && hmax > 0.f) atomicMax(p.h_amax, __float_as_int(hmax));
      return;
    }
    // padding rows (accumulators of zero activations) are written too: zeros
    uint4* dst = reinterpret_cast<uint4*>(p.hq + (size_t)hrow * (p.f / 2) + (chb >> 1));
    dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
    // the four blocks share one 64-wide K group: four consecutive scale bytes
    const size_t so = sf_rowpair_offset(hrow, chb >> 4, p.f / 64);
    *reinterpret_cast<uint32_t*>(p.hsf + so) = sfw;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kDenseThreads, 1) dense_gemm_kernel(const __grid_constant__ DenseParams p) {
  using C = DenseStageCfg<MODE>;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  // 1024-byte alignment (shared-window offset) for the 128-byte-swizzled tiles
  uint8_t* dsm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  uint8_t* meta = dsm + C::kStages * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta);                 // full[S] empty[S] accf acce done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + C::kBarBytes);
  int* svote = reinterpret_cast<int*>(meta + C::kBarBytes + 16);    // [8] epilogue wait outcomes

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  const int nd = *p.n_dense;
  if (nd == 0) { pdl_launch_dependents(); return; }
  const uint32_t bars_s = smem_u32(bars);
  auto full_b = [&](int s) { return bars_s + 8 * s; };
  auto empty_b = [&](int s) { return bars_s + 8 * (C::kStages + s); };
  const uint32_t accf_b = bars_s + 8 * (2 * C::kStages);
  const uint32_t acce_b = accf_b + 8;
  const uint32_t done_b = accf_b + 16;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) { mbar_init(full_b(s), 1); mbar_init(empty_b(s), 1); }
    mbar_init(accf_b, 1);
    mbar_init(acce_b, kDenseEpiWarps);
    mbar_init(done_b, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kDenseTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: the accumulator (256), then one set of scale columns per stage
  const uint32_t sf_t0 = tmem + kDenseN;

  const int ntiles = p.wt_per_expert * __ldg(p.ntoff + nd);
  const int G = gridDim.x, b = blockIdx.x;
  const int my_tiles = b < ntiles ? (ntiles - 1 - b) / G + 1 : 0;
  const uint64_t deadline = globaltimer_ns() + (uint64_t)p.wait_timeout_ns;
  const uint32_t stage0 = smem_u32(dsm);
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_normal(), pol_a = policy_evict_last();
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(&p.tmB);
      int k = 0;
      for (int it = 0; it < my_tiles && !failed; ++it) {
        const DenseTile tl = dense_tile(p.dense, p.ntoff, nd, p.wt_per_expert, b + it * G);
        const int wrow = tl.de.x * p.rows_per_expert + tl.wt * (MODE == kDenseGateUp ? kDenseN : 128);
        const int trow = tl.de.w + tl.tt * (MODE == kDenseGateUp ? 128 : kDenseN);   // padded token row
        const int arow = MODE == kDenseGateUp ? trow : wrow;
        const int brow = MODE == kDenseGateUp ? wrow : trow;
        const uint8_t* sfa = p.sfA + (size_t)(arow >> 7) * p.kstages * kSfaBlock;
        const uint8_t* sfb = p.sfB + (size_t)(brow >> 8) * p.kstages * kSfbBlock;
        for (int ks = 0; ks < p.kstages; ++ks, ++k) {
          const int s = k % C::kStages;
          if (!mbar_wait_spin(empty_b(s), ((k / C::kStages) & 1) ^ 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          const uint32_t st = stage0 + s * C::kStageBytes;
          mbar_arrive_expect_tx(full_b(s), C::kStageBytes);
          tma_load_2d(st, &p.tmA, ks * kDenseRowBytes, arow, full_b(s), pol_a);
          tma_load_2d(st + kDenseABytes, &p.tmB, ks * kDenseRowBytes, brow, full_b(s), pol_w);
          // scale blocks: each read from device memory once (replicas, if
          // any, come from L2)
          const uint8_t* sa = sfa + (size_t)ks * kSfaBlock;
          const uint8_t* sb = sfb + (size_t)ks * kSfbBlock;
          const uint32_t da = st + kDenseABytes + kDenseBBytes, db = da + C::kSfaBytes;
#pragma unroll
          for (int rep = 0; rep < C::kCopies; ++rep) {
            bulk_g2s(da + rep * kSfaBlock, sa, kSfaBlock, full_b(s), pol_a);
            bulk_g2s(db + rep * kSfbBlock, sb, kSfbBlock, full_b(s), pol_w);
          }
        }
      }
      // drain: every issued stage must land before the block exits
      for (int kk = max(0, k - C::kStages); kk < k; ++kk)
        mbar_wait_spin(full_b(kk % C::kStages), (kk / C::kStages) & 1,
                       globaltimer_ns() + (uint64_t)p.wait_timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int k = 0;
      bool issued_any = false;
      for (int it = 0; it < my_tiles && !failed; ++it) {
        // N = 256, or 128 when the down GEMM's token tile holds at most 128 rows
        uint32_t idesc = idesc_nvf4(kDenseN);
        if (MODE == kDenseDown) {
          const DenseTile tl = dense_tile(p.dense, p.ntoff, nd, p.wt_per_expert, b + it * G);
          if (tl.de.z - tl.tt * kDenseN <= 128) idesc = idesc_nvf4(128);
        }
        // the epilogue has drained the previous tile's accumulator
        if (!mbar_wait_spin(acce_b, (it & 1) ^ 1, deadline)) {
          failed = true; set_error(p.err, kErrTimeout); break;
        }
        tc_fence_after();
        for (int ks = 0; ks < p.kstages; ++ks, ++k) {
          const int s = k % C::kStages;
          if (!mbar_wait_spin(full_b(s), (k / C::kStages) & 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          tc_fence_after();
          const uint32_t st = stage0 + s * C::kStageBytes;
          const uint32_t sfa_s = st + kDenseABytes + kDenseBBytes, sfb_s = sfa_s + C::kSfaBytes;
          const uint32_t sfa_t = sf_t0 + kDenseSfCols * s, sfb_t = sfa_t + 4 * kDenseMmaPerStage;
          if (C::kBcast) {
            // MMA kb: M side unit kb / 2, 16-byte column kb % 2 -> 4 columns;
            // N side unit kb, columns h = 0, 1 (rows 0..127, 128..255) -> 8 columns
#pragma unroll
            for (int kb = 0; kb < kDenseMmaPerStage; ++kb) {
              tc_cp_32x128b_warpx4(sfa_t + 4 * kb,
                                   smem_desc_sf128(sfa_s + kSfGroupBytes * (kb >> 1) + 128 * (kb & 1),
                                                   kSfPairUnitsPerStage * kSfGroupBytes));
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tc_cp_32x128b_warpx4(sfb_t + 8 * kb + 4 * h,
                                     smem_desc_sf128(sfb_s + kSfGroupBytes * kb + 128 * h,
                                                     kSfRowpairUnitsPerStage * kSfGroupBytes));
            }
          } else {
#pragma unroll
            for (int pr = 0; pr < kDenseMmaPerStage / 2; ++pr)
              tc_cp_128x256b(sfa_t + 8 * pr, smem_desc_sf256(sfa_s + kSfGroupBytes * pr,
                                                             kSfPairUnitsPerStage * kSfGroupBytes));
#pragma unroll
            for (int kb = 0; kb < kDenseMmaPerStage; ++kb)
              tc_cp_128x256b(sfb_t + 8 * kb, smem_desc_sf256(sfb_s + kSfGroupBytes * kb,
                                                             kSfRowpairUnitsPerStage * kSfGroupBytes));
          }
          const uint64_t adesc = smem_desc_kmajor<kDenseRowBytes>(st);
          const uint64_t bdesc = smem_desc_kmajor<kDenseRowBytes>(st + kDenseABytes);
#pragma unroll
          for (int kb = 0; kb < kDenseMmaPerStage; ++kb)
            tc_mma_nvf4(tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc, sfa_t + 4 * kb, sfb_t + 8 * kb,
                        (ks > 0 || kb > 0) ? 1u : 0u);
          tc_commit(empty_b(s));
          issued_any = true;
        }
        if (failed) break;
        tc_commit(accf_b);
      }
      // every MMA issued must complete before TMEM is released
      if (issued_any) {
        tc_commit(done_b);
        mbar_wait_spin(done_b, 0, globaltimer_ns() + (uint64_t)p.wait_timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..)
    const int q = warp & 3;                              // TMEM lane quarter of this warp
    const int ew = warp - 2;                             // epilogue warp index
    const int hf = ew >> 2;                              // accumulator columns 128 hf .. 128 hf + 127
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    for (int it = 0; it < my_tiles && !failed; ++it) {
      const DenseTile tl = dense_tile(p.dense, p.ntoff, nd, p.wt_per_expert, b + it * G);
      // all epilogue warps take the same decision: each records whether its
      // bounded wait succeeded, then they meet at a barrier every warp reaches
      const bool ok = mbar_wait_spin(accf_b, it & 1, deadline);
      if (lane == 0) svote[ew] = ok ? 1 : 0;
      named_bar_sync(2, 32 * kDenseEpiWarps);
      bool all_ok = true;
#pragma unroll
      for (int i = 0; i < kDenseEpiWarps; ++i) all_ok = all_ok && svote[i];
      named_bar_sync(2, 32 * kDenseEpiWarps);
      if (!all_ok) {
        failed = true;
        if (lane == 0) set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      // drain this lane's 128 accumulator columns, then release the accumulator
      uint32_t r[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t (&rc)[32] = *reinterpret_cast<uint32_t (*)[32]>(r + 32 * c);
        tmem_ld_32x32b_x32(tmem + lane_base + hf * 128 + 32 * c, rc);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_b);
      // M side: an output dimension (down) or a token of the expert (gate/up)
      const int mrow = tl.wt * 128 + q * 32 + lane;
      const int mtok = tl.tt * 128 + q * 32 + lane;
      dense_epilogue<MODE>(p, tl, r, MODE == kDenseDown ? mrow : mtok, tl.tt * kDenseN, hf, lane);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDenseTmemCols);
  }
  pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// The same grouped GEMM on CTA pairs (clusters of two, tcgen05 cta_group::2).
// A pair computes a 256 x 256 tile: M = 256 (128 rows in each CTA: tokens
// for gate/up, rows of Wd for down), N = 256 (each CTA loads 128 of the B
// rows; the pair's tensor cores read both halves), so each CTA streams half
// of the B tile and the B operand bytes per MMA flop halve.  Each CTA loads
// its own A half, its B half, the scale block of its 128 A rows and the
// whole N-side scale block (every CTA's accumulator covers all 256 N
// columns); all loads of both CTAs complete on the even CTA's `full`
// barrier.  The even CTA's single MMA thread copies the scales into both
// CTAs' TMEM (each from its own shared memory) and issues the MMAs; its commits arrive on
// the `empty`, `accf` and `done` barriers of both CTAs.  Each CTA drains
// its own TMEM; the 16 epilogue warps of the pair release the accumulator
// on the even CTA's `acce` barrier.  Token tiles are 256 rows for both GEMMs
// (the dense rows are padded to 256).
// ---------------------------------------------------------------------------
constexpr int kPairABytes = 128 * kDenseRowBytes;
constexpr int kPairBBytes = 128 * kDenseRowBytes;
// Scale copies of the pair kernel: four replicas of each block in shared
// memory read by .128x256b copies (6 copy instructions a stage, 4 stages of
// 56 KB), or one copy read by .32x128b.warpx4 broadcasts (12 a stage, 5
// stages of 38 KB).  The tensor pipe spends about as long on a copy
// instruction of either shape, so the fewer, larger copies win on B200.
#ifndef MOE_PAIR_SF_BCAST
#define MOE_PAIR_SF_BCAST 0
#endif
struct PairStageCfg {
  static constexpr bool kBcast = MOE_PAIR_SF_BCAST != 0;
  static constexpr int kCopies = kBcast ? 1 : kSfReplicas;
  static constexpr int kStages = kBcast ? 5 : 4;
  static constexpr int kSfaBytes = kCopies * kSfaBlock;
  static constexpr int kSfbBytes = kCopies * kSfbBlock;
  static constexpr int kStageBytes = kPairABytes + kPairBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kBarBytes = (2 * kStages + 3) * 8 + 8;
  static_assert(kStageBytes % 1024 == 0, "pair stages keep the 1024-byte alignment of the swizzled tiles");
  static_assert(kDenseN + kDenseSfCols * kStages <= kDenseTmemCols, "pair accumulator + scales exceed TMEM");
};
constexpr int kPairStages = PairStageCfg::kStages;
constexpr int kPairStageBytes = PairStageCfg::kStageBytes;
constexpr int kPairBarBytes = PairStageCfg::kBarBytes;

template <int MODE>
__global__ void __launch_bounds__(kDenseThreads, 1) dense_gemm_pair_kernel(const __grid_constant__ DenseParams p) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  uint8_t* meta = dsm + kPairStages * kPairStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta);                 // full[S] empty[S] accf acce done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + kPairBarBytes);
  int* svote = reinterpret_cast<int*>(meta + kPairBarBytes + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  pdl_wait();
  const int nd = *p.n_dense;
  if (nd == 0) { pdl_launch_dependents(); return; }      // both CTAs of a pair read the same nd
  const uint32_t bars_s = smem_u32(bars);
  auto full_b = [&](int s) { return bars_s + 8 * s; };
  auto empty_b = [&](int s) { return bars_s + 8 * (kPairStages + s); };
  const uint32_t accf_b = bars_s + 8 * (2 * kPairStages);
  const uint32_t acce_b = accf_b + 8;
  const uint32_t done_b = accf_b + 16;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) { mbar_init(full_b(s), 1); mbar_init(empty_b(s), 1); }
    mbar_init(accf_b, 1);
    mbar_init(acce_b, 2 * kDenseEpiWarps);
    mbar_init(done_b, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), kDenseTmemCols);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();                  // both CTAs' barriers initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sf_t0 = tmem + kDenseN;

  const int ntiles = p.wt_per_expert * __ldg(p.ntoff + nd);
  const int G = gridDim.x >> 1, c = blockIdx.x >> 1;
  const int my_tiles = c < ntiles ? (ntiles - 1 - c) / G + 1 : 0;
  const uint64_t deadline = globaltimer_ns() + (uint64_t)p.wait_timeout_ns;
  const uint32_t stage0 = smem_u32(dsm);
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_normal(), pol_a = policy_evict_last();
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(&p.tmB2);
      tma_prefetch_desc(&p.tmSfa);
      tma_prefetch_desc(&p.tmSfb);
      int k = 0;
      for (int it = 0; it < my_tiles && !failed; ++it) {
        const DenseTile tl = dense_tile(p.dense, p.ntoff, nd, p.wt_per_expert, c + it * G);
        const int wrow = tl.de.x * p.rows_per_expert + tl.wt * 256;      // weight rows of the tile
        const int trow = tl.de.w + tl.tt * 256;                          // padded token rows
        const int arow = (MODE == kDenseGateUp ? trow : wrow) + 128 * (int)rank;
        const int brow = MODE == kDenseGateUp ? wrow : trow;
        const int sfa_y = ((arow >> 7) * p.kstages) * 8;                 // + 8 per stage
        const int sfb_y = ((brow >> 8) * p.kstages) * 16;                // + 16 per stage
        const int brow_mine = brow + 128 * (int)rank;
        for (int ks = 0; ks < p.kstages; ++ks, ++k) {
          const int s = k % kPairStages;
          if (!mbar_wait_spin(empty_b(s), ((k / kPairStages) & 1) ^ 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          const uint32_t st = stage0 + s * kPairStageBytes;
          const uint32_t fb = mapa_shared(full_b(s), 0);
          if (leader) mbar_arrive_expect_tx(full_b(s), 2 * kPairStageBytes);
          tma_load_2d_pair(st, &p.tmA, ks * kDenseRowBytes, arow, fb, pol_a);
          tma_load_2d_pair(st + kPairABytes, &p.tmB2, ks * kDenseRowBytes, brow_mine, fb, pol_w);
#pragma unroll
          for (int rep = 0; rep < PairStageCfg::kCopies; ++rep) {   // replicas after the first come from L2
            tma_load_2d_pair(st + kPairABytes + kPairBBytes + rep * kSfaBlock, &p.tmSfa, 0, sfa_y + 8 * ks, fb,
                             pol_a);
            tma_load_2d_pair(st + kPairABytes + kPairBBytes + PairStageCfg::kSfaBytes + rep * kSfbBlock, &p.tmSfb,
                             0, sfb_y + 16 * ks, fb, pol_w);
          }
        }
      }
      // drain: the even CTA's full barriers count the loads of both CTAs
      if (leader)
        for (int kk = max(0, k - kPairStages); kk < k; ++kk)
          mbar_wait_spin(full_b(kk % kPairStages), (kk / kPairStages) & 1,
                         globaltimer_ns() + (uint64_t)p.wait_timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_nvf4(kDenseN, 256);
      int k = 0;
      for (int it = 0; it < my_tiles && !failed; ++it) {
        if (!mbar_wait_cluster(acce_b, (it & 1) ^ 1, deadline)) {
          failed = true; set_error(p.err, kErrTimeout); break;
        }
        tc_fence_after();
        for (int ks = 0; ks < p.kstages; ++ks, ++k) {
          const int s = k % kPairStages;
          if (!mbar_wait_spin(full_b(s), (k / kPairStages) & 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          tc_fence_after();
          const uint32_t st = stage0 + s * kPairStageBytes;
          const uint32_t sfa_s = st + kPairABytes + kPairBBytes, sfb_s = sfa_s + PairStageCfg::kSfaBytes;
          const uint32_t sfa_t = sf_t0 + kDenseSfCols * s, sfb_t = sfa_t + 4 * kDenseMmaPerStage;
          if (PairStageCfg::kBcast) {
#pragma unroll
            for (int kb = 0; kb < kDenseMmaPerStage; ++kb) {
              tc_cp2_32x128b_warpx4(sfa_t + 4 * kb,
                                    smem_desc_sf128(sfa_s + kSfGroupBytes * (kb >> 1) + 128 * (kb & 1),
                                                    kSfPairUnitsPerStage * kSfGroupBytes));
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tc_cp2_32x128b_warpx4(sfb_t + 8 * kb + 4 * h,
                                      smem_desc_sf128(sfb_s + kSfGroupBytes * kb + 128 * h,
                                                      kSfRowpairUnitsPerStage * kSfGroupBytes));
            }
          } else {
#pragma unroll
            for (int pr = 0; pr < kDenseMmaPerStage / 2; ++pr)
              tc_cp2_128x256b(sfa_t + 8 * pr, smem_desc_sf256(sfa_s + kSfGroupBytes * pr,
                                                              kSfPairUnitsPerStage * kSfGroupBytes));
#pragma unroll
            for (int kb = 0; kb < kDenseMmaPerStage; ++kb)
              tc_cp2_128x256b(sfb_t + 8 * kb, smem_desc_sf256(sfb_s + kSfGroupBytes * kb,
                                                              kSfRowpairUnitsPerStage * kSfGroupBytes));
          }
          const uint64_t adesc = smem_desc_kmajor<kDenseRowBytes>(st);
          const uint64_t bdesc = smem_desc_kmajor<kDenseRowBytes>(st + kPairABytes);
#pragma unroll
          for (int kb = 0; kb < kDenseMmaPerStage; ++kb)
            tc_mma2_nvf4(tmem, adesc + 2 * kb, bdesc + 2 * kb, idesc, sfa_t + 4 * kb, sfb_t + 8 * kb,
                         (ks > 0 || kb > 0) ? 1u : 0u);
          tc_commit2_both(empty_b(s));
        }
        if (failed) break;
        tc_commit2_both(accf_b);
      }
      // both CTAs learn that every MMA issued (none, possibly) has completed
      tc_commit2_both(done_b);
    }
    if (lane == 0) mbar_wait_spin(done_b, 0, globaltimer_ns() + (uint64_t)p.wait_timeout_ns);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2.., both CTAs)
    const int q = warp & 3;
    const int ew = warp - 2;
    const int hf = ew >> 2;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const uint32_t acce_leader = mapa_shared(acce_b, 0);
    for (int it = 0; it < my_tiles && !failed; ++it) {
      const DenseTile tl = dense_tile(p.dense, p.ntoff, nd, p.wt_per_expert, c + it * G);
      const bool ok = mbar_wait_spin(accf_b, it & 1, deadline);
      if (lane == 0) svote[ew] = ok ? 1 : 0;
      named_bar_sync(2, 32 * kDenseEpiWarps);
      bool all_ok = true;
#pragma unroll
      for (int i = 0; i < kDenseEpiWarps; ++i) all_ok = all_ok && svote[i];
      named_bar_sync(2, 32 * kDenseEpiWarps);
      if (!all_ok) {
        failed = true;
        if (lane == 0) set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      uint32_t r[128];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t (&rc)[32] = *reinterpret_cast<uint32_t (*)[32]>(r + 32 * cc);
        tmem_ld_32x32b_x32(tmem + lane_base + hf * 128 + 32 * cc, rc);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_leader);
      const int m_in_tile = 128 * (int)rank + q * 32 + lane;
      const int mrow = tl.wt * 256 + m_in_tile;           // down: output dimension
      const int mtok = tl.tt * 256 + m_in_tile;           // gate/up: token of the expert
      dense_epilogue<MODE>(p, tl, r, MODE == kDenseDown ? mrow : mtok, tl.tt * 256, hf, lane);
    }
  }
  // no CTA leaves (or frees TMEM) while the other may still reach its shared
  // memory or TMEM: every MMA completed (done), both epilogues drained
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, kDenseTmemCols);
  }
  pdl_launch_dependents();
}

template <int MODE>
constexpr size_t dense_pair_smem_size() {
  return 1024 + (size_t)kPairStages * kPairStageBytes + kPairBarBytes + 48;
}

template <int MODE>
constexpr size_t dense_smem_size(int) {
  return 1024 + (size_t)DenseStageCfg<MODE>::kStages * DenseStageCfg<MODE>::kStageBytes +
         DenseStageCfg<MODE>::kBarBytes + 48;
}

}  // namespace moe
