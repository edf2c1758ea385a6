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
// multiple of 128 so each 128-token MMA tile starts on a scale-atom boundary.
//
// GEMM 1 (kDenseGateUp): D[128 rows of the combined gate/up matrix][128 tokens]
//   over K = d.  Gate and up rows are interleaved in groups of 16 channels, so
//   each 32-lane TMEM quarter holds gate (lanes 0-15) and up (lanes 16-31) of
//   the same 16 channels -- one NVFP4 block of h.  The epilogue transposes
//   each 32 x 32 chunk through shared memory so that one lane holds the 16
//   gate and 16 up values of one token, forms h = SiLU(g) * u, quantises the
//   block in registers and writes the B operand of GEMM 2.
// GEMM 2 (kDenseDown):   D[128 rows of Wd][128 tokens] over K = f; the
//   epilogue writes w * gs * D as fp32 partials (rows in permutation order).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "tc.cuh"

namespace moe {

constexpr int kDenseEpiWarps = 8;         // two per TMEM lane quarter, each on half of the columns
constexpr int kDenseThreads = 64 + 32 * kDenseEpiWarps;   // warp 0 TMA, warp 1 MMA, warps 2.. epilogue
constexpr int kDenseStages = 3;
constexpr int kDenseTileBytes = 128 * 128; // 128 rows x 128 bytes (256 fp4 along K)
constexpr int kDenseSfBytes = 2 * 4096;    // per operand per stage: 2 scale pair units (K = 256)
constexpr int kDenseStageBytes = 2 * kDenseTileBytes + 2 * kDenseSfBytes;
constexpr uint32_t kDenseTmemCols = 512;
static_assert(256 + 32 * kDenseStages <= kDenseTmemCols, "accumulators + per-stage scale factors exceed TMEM");
constexpr int kDenseBarBytes = (2 * kDenseStages + 6) * 8;   // mbarriers, padded to 16 bytes

enum DenseMode { kDenseGateUp = 0, kDenseDown = 1 };

// Dense list entry: {expert, row0 (permutation rows), rows, padded row0}.
struct DenseParams {
  CUtensorMap tmA;       // weights: combined gate/up rows [E][2f] or down rows [E][d]; box 128 B x 128 rows
  CUtensorMap tmB;       // activations (NVFP4, padded permutation order), box 128 B x 128 rows
  const uint8_t* sfA;    // weight scale atoms
  const uint8_t* sfB;    // activation scale atoms
  const int4* dense;     // dense list, ranked by rows descending
  const int* n_dense;
  const int* ntoff;      // [E+1] exclusive prefix of ceil(rows / 128) over the dense list
  int mt_per_expert;     // gate/up: f / 64; down: d / 128
  int rows_per_expert;   // gate/up: 2f; down: d (rows of the weight copy per expert)
  int kstages;           // K / 256
  int kb64;              // K / 64
  int d, f, topk;
  const float* gs;       // [3][E]
  int E;
  const int* perm;
  const float* wts;
  // gate/up outputs
  uint8_t* hq;           // [P_pad][f/2]
  uint8_t* hsf;          // scale atoms of hq
  float* h32;            // [P][f] or null
  // down output
  float* partial;        // [P][d]
  int* err;
  int64_t wait_timeout_ns;
};

// ---------------------------------------------------------------------------
// Activation quantiser: one warp per padded row of the dense class.
// src row (bf16) of token perm[row0 + i] / topk; rows past the expert's count
// are written as zeros.  Output: codes [rows][K/2], scales in atom layout.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int dense_rank_of_padrow(const int4* dense, int nd, int prow) {
  int lo = 0, hi = nd - 1;                       // pad0 increases with rank
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (dense[mid].w <= prow) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256) quant_x_dense_kernel(
    const uint16_t* __restrict__ x, const int4* __restrict__ dense, const int* __restrict__ n_dense,
    const int* __restrict__ pad_total, const int* __restrict__ perm, int topk, int d,
    uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf) {
  pdl_wait();
  const int nd = *n_dense;
  if (nd == 0) { pdl_launch_dependents(); return; }
  const int total = *pad_total;
  const int lane = threadIdx.x & 31;
  const int nblk = d / 16;
  for (int prow = blockIdx.x * 8 + (threadIdx.x >> 5); prow < total; prow += gridDim.x * 8) {
    const int j = dense_rank_of_padrow(dense, nd, prow);
    const int4 de = dense[j];
    const int i = prow - de.w;
    const bool valid = i < de.z;
    const uint16_t* src = valid ? x + (size_t)(perm[de.y + i] / topk) * d : nullptr;
    for (int blk = lane; blk < nblk; blk += 32) {
      uint2 codes = make_uint2(0, 0);
      uint32_t sfbyte = 0;
      if (valid) {
        const uint4 a = *reinterpret_cast<const uint4*>(src + blk * 16);
        const uint4 b = *reinterpret_cast<const uint4*>(src + blk * 16 + 8);
        const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float v[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          v[2 * q] = __uint_as_float(wv[q] << 16);
          v[2 * q + 1] = __uint_as_float(wv[q] & 0xffff0000u);
        }
        float amax = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) amax = fmaxf(amax, fabsf(v[q]));
        sfbyte = f32x2_to_e4m3x2(0.f, amax / 6.0f) & 0xffu;
        const float sf = e4m3_to_f32(sfbyte);
        if (sf > 0.f) {
          uint32_t c[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) c[q] = f32x2_to_e2m1x2(v[2 * q + 1] / sf, v[2 * q] / sf);
          codes.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
          codes.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
        }
      }
      *reinterpret_cast<uint2*>(xq + (size_t)prow * (d / 2) + blk * 8) = codes;
      const size_t so = sf_pair_offset(prow, blk, d / 64);
#pragma unroll
      for (int c = 0; c < kSfReplicas; ++c) xsf[so + 1024 * c] = (uint8_t)sfbyte;
    }
  }
  pdl_launch_dependents();
}


// ---------------------------------------------------------------------------
// Grouped block-scaled NVFP4 GEMM on tcgen05 (persistent, one block per SM).
// Tiles are (dense rank j, M tile mt, token tile nt) with nt fastest, so
// neighbouring blocks share the same weight tile through L2.
// ---------------------------------------------------------------------------
struct DenseTile {
  int j, mt, nt;
  int4 de;      // {expert, row0, rows, padded row0}
};

__device__ __forceinline__ DenseTile dense_tile(const int4* sd, const int* sntoff, int nd, int mtpe, int i) {
  // find rank j with mtpe * ntoff[j] <= i < mtpe * ntoff[j+1]
  int lo = 0, hi = nd - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (mtpe * sntoff[mid] <= i) lo = mid; else hi = mid - 1;
  }
  DenseTile t;
  t.j = lo;
  t.de = sd[lo];
  const int ntj = sntoff[lo + 1] - sntoff[lo];
  const int local = i - mtpe * sntoff[lo];
  t.mt = local / ntj;
  t.nt = local - t.mt * ntj;
  return t;
}

template <int MODE>
__global__ void __launch_bounds__(kDenseThreads, 1) dense_gemm_kernel(const __grid_constant__ DenseParams p) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  // 1024-byte alignment (shared-window offset) for the 128-byte-swizzled tiles
  uint8_t* dsm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  uint8_t* meta = dsm + kDenseStages * kDenseStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta);                 // full[S] empty[S] accf[2] acce[2] done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + kDenseBarBytes);
  int* svote = reinterpret_cast<int*>(meta + kDenseBarBytes + 16);    // [8] epilogue wait outcomes
  int4* sd = reinterpret_cast<int4*>(meta + kDenseBarBytes + 48);     // dense list (<= E entries)
  int* sntoff = reinterpret_cast<int*>(sd + p.E);                     // [E+1]
  float* tbuf = reinterpret_cast<float*>(sntoff + ((p.E + 4) & ~3));  // gate/up: [epilogue warps][32][33]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  const int nd = *p.n_dense;
  if (nd == 0) { pdl_launch_dependents(); return; }
  for (int i = threadIdx.x; i < nd; i += blockDim.x) sd[i] = p.dense[i];
  for (int i = threadIdx.x; i <= nd; i += blockDim.x) sntoff[i] = p.ntoff[i];
  const uint32_t bars_s = smem_u32(bars);
  auto full_b = [&](int s) { return bars_s + 8 * s; };
  auto empty_b = [&](int s) { return bars_s + 8 * (kDenseStages + s); };
  auto accf_b = [&](int a) { return bars_s + 8 * (2 * kDenseStages + a); };
  auto acce_b = [&](int a) { return bars_s + 8 * (2 * kDenseStages + 2 + a); };
  const uint32_t done_b = bars_s + 8 * (2 * kDenseStages + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDenseStages; ++s) { mbar_init(full_b(s), 1); mbar_init(empty_b(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(accf_b(a), 1); mbar_init(acce_b(a), kDenseEpiWarps); }
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
  // TMEM columns: accumulators 0-255 (two buffers of 128), then one set of
  // scale factors per shared-memory stage (16 columns for A, 16 for B).
  const uint32_t acc_t0 = tmem, sf_t0 = tmem + 256;

  const int ntiles = p.mt_per_expert * sntoff[nd];
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
        const DenseTile tl = dense_tile(sd, sntoff, nd, p.mt_per_expert, b + it * G);
        const int e = tl.de.x;
        const int brow = tl.de.w + tl.nt * 128;              // padded activation row
        for (int ks = 0; ks < p.kstages; ++ks, ++k) {
          const int s = k % kDenseStages;
          if (!mbar_wait_spin(empty_b(s), ((k / kDenseStages) & 1) ^ 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          const uint32_t st = stage0 + s * kDenseStageBytes;
          mbar_arrive_expect_tx(full_b(s), kDenseStageBytes);
          tma_load_2d(st, &p.tmA, ks * 128, e * p.rows_per_expert + tl.mt * 128, full_b(s), pol_w);
          tma_load_2d(st + kDenseTileBytes, &p.tmB, ks * 128, brow, full_b(s), pol_a);
          // scales: the two 4 KB pair units of this K stage (see sf_pair_offset)
          const uint8_t* sfa = p.sfA + ((size_t)(e * p.mt_per_expert + tl.mt) * (p.kb64 >> 1) + 2 * ks) * 4096;
          const uint8_t* sfb = p.sfB + ((size_t)(brow >> 7) * (p.kb64 >> 1) + 2 * ks) * 4096;
          bulk_g2s(st + 2 * kDenseTileBytes, sfa, kDenseSfBytes, full_b(s), pol_w);
          bulk_g2s(st + 2 * kDenseTileBytes + kDenseSfBytes, sfb, kDenseSfBytes, full_b(s), pol_a);
        }
      }
      // drain: every issued stage must land before the block exits
      for (int kk = max(0, k - kDenseStages); kk < k; ++kk)
        mbar_wait_spin(full_b(kk % kDenseStages), (kk / kDenseStages) & 1,
                        globaltimer_ns() + (uint64_t)p.wait_timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_nvf4(128);
      int k = 0;
      bool issued_any = false;
      for (int it = 0; it < my_tiles && !failed; ++it) {
        const int ab = it & 1;
        if (!mbar_wait_spin(acce_b(ab), ((it >> 1) & 1) ^ 1, deadline)) {
          failed = true; set_error(p.err, kErrTimeout); break;
        }
        tc_fence_after();
        const uint32_t acc = acc_t0 + ab * 128;
        for (int ks = 0; ks < p.kstages; ++ks, ++k) {
          const int s = k % kDenseStages;
          if (!mbar_wait_spin(full_b(s), (k / kDenseStages) & 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          tc_fence_after();
          const uint32_t st = stage0 + s * kDenseStageBytes;
          const uint32_t sfa_s = st + 2 * kDenseTileBytes, sfb_s = sfa_s + kDenseSfBytes;
          const uint32_t sfa_t = sf_t0 + 32 * s, sfb_t = sfa_t + 16;
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {                // one copy per pair of MMAs and operand
            tc_cp_128x256b(sfa_t + 8 * pr, smem_desc_sf256(sfa_s + 4096 * pr));
            tc_cp_128x256b(sfb_t + 8 * pr, smem_desc_sf256(sfb_s + 4096 * pr));
          }
          const uint64_t adesc = smem_desc_sw128(st), bdesc = smem_desc_sw128(st + kDenseTileBytes);
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            tc_mma_nvf4(acc, adesc + 2 * kb, bdesc + 2 * kb, idesc, sfa_t + 4 * kb, sfb_t + 4 * kb,
                        (ks > 0 || kb > 0) ? 1u : 0u);
          tc_commit(empty_b(s));
          issued_any = true;
        }
        if (failed) break;
        tc_commit(accf_b(ab));
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
    const int chalf = (ew >> 2) * 32;                    // first 32-column chunk of this warp
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    for (int it = 0; it < my_tiles && !failed; ++it) {
      const int ab = it & 1;
      const DenseTile tl = dense_tile(sd, sntoff, nd, p.mt_per_expert, b + it * G);
      // all epilogue warps take the same decision: each records whether its
      // bounded wait succeeded, then they meet at a barrier every warp reaches
      const bool ok = mbar_wait_spin(accf_b(ab), (it >> 1) & 1, deadline);
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
      const uint32_t acc = acc_t0 + ab * 128 + lane_base;
      const int e = tl.de.x, ncols = min(128, tl.de.z - tl.nt * 128);
      const int prow0 = tl.de.y + tl.nt * 128;           // permutation row of column 0
      const int hrow0 = tl.de.w + tl.nt * 128;           // padded row of column 0
      if (MODE == kDenseDown) {
        const float gsd = p.gs[2 * p.E + e];
        const int drow = tl.mt * 128 + q * 32 + lane;
        for (int c0 = chalf; c0 < ncols; c0 += 64) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(acc + c0, r);
          // routing weight x tensor scale of column c0 + lane, broadcast below
          const float wl = c0 + lane < ncols ? p.wts[p.perm[prow0 + c0 + lane]] * gsd : 0.f;
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float wv = __shfl_sync(0xffffffffu, wl, c);
            if (c0 + c < ncols) p.partial[(size_t)(prow0 + c0 + c) * p.d + drow] = __uint_as_float(r[c]) * wv;
          }
        }
      } else {
        // Lanes 0-15 hold the gate rows and lanes 16-31 the up rows of channels
        // ch0 .. ch0 + 15.  Each 32-column chunk is transposed through shared
        // memory so that lane L owns token column c0 + L: its 16 h values, their
        // NVFP4 block scale and 8 bytes of codes then need no cross-lane traffic.
        const float gsg = p.gs[e], gsu = p.gs[p.E + e];
        const int ch0 = tl.mt * 64 + q * 16;
        float* tb = tbuf + ew * (32 * 33);
        for (int c0 = chalf; c0 < ncols; c0 += 64) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(acc + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) tb[lane * 33 + c] = __uint_as_float(r[c]);
          __syncwarp();
          float hv[16];
          float am = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float gv = tb[i * 33 + lane] * gsg;
            const float uv = tb[(16 + i) * 33 + lane] * gsu;
            hv[i] = gv / (1.f + expf(-gv)) * uv;
            am = fmaxf(am, fabsf(hv[i]));
          }
          __syncwarp();                                   // tb is rewritten by the next chunk
          const int n = c0 + lane;                        // < 128: inside the expert's padded rows
          if (p.h32 && n < ncols) {
            float4* dst = reinterpret_cast<float4*>(p.h32 + (size_t)(prow0 + n) * p.f + ch0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
          }
          const uint32_t sfbyte = f32x2_to_e4m3x2(0.f, am / 6.0f) & 0xffu;
          const float sf = e4m3_to_f32(sfbyte);
          uint32_t w0 = 0u, w1 = 0u;                      // channel i -> nibble i % 8 of word i / 8
          if (sf > 0.f) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              w0 |= f32x2_to_e2m1x2(hv[i + 1] / sf, hv[i] / sf) << (4 * i);
              w1 |= f32x2_to_e2m1x2(hv[i + 9] / sf, hv[i + 8] / sf) << (4 * i);
            }
          }
          const int hr = hrow0 + n;
          *reinterpret_cast<uint2*>(p.hq + (size_t)hr * (p.f / 2) + (ch0 >> 1)) = make_uint2(w0, w1);
          const size_t so = sf_pair_offset(hr, ch0 >> 4, p.f / 64);
#pragma unroll
          for (int c = 0; c < kSfReplicas; ++c) p.hsf[so + 1024 * c] = (uint8_t)sfbyte;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_b(ab));
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

template <int MODE>
constexpr size_t dense_smem_size(int E) {
  return 1024 + (size_t)kDenseStages * kDenseStageBytes + kDenseBarBytes + 48 + (size_t)E * 16 +
         (size_t)((E + 4) & ~3) * 4 + (MODE == kDenseGateUp ? kDenseEpiWarps * 32 * 33 * 4 : 0);
}

}  // namespace moe
