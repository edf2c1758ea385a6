// Router logits for large token counts on the tcgen05 tensor cores.
//
// The router computes fp32 logits l[t,e] = sum_i x[t,i] * Wr[e,i] with x in
// bf16 and Wr in fp32.  Wr is split exactly into three bf16 matrices,
// Wr = W1 + W2 + W3 (W1 = bf16_rn(Wr), W2 = bf16_rn(Wr - W1), W3 = Wr - W1 - W2,
// which has at most 8 significant bits and is therefore a bf16 value), so
// every product x_i * Wj_i is exact in fp32 and the kind::f16 MMA (bf16
// operands, fp32 accumulation in TMEM) sums the 3d exact products in fp32:
// the same arithmetic class as an fp32 dot product, at tensor-core speed.
//
// Tile: 128 experts (M, rows of one W part) x 128 tokens (N) per accumulator,
// K chunk of 64 (one 128-byte swizzled row); per chunk the three W parts are
// issued against the same x tile.  Warp 0 loads (TMA), warp 1 issues the MMA,
// warps 2-5 drain TMEM into logits[t][e] (lanes = experts: coalesced rows).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "tc.cuh"

namespace moe {

constexpr int kRtThreads = 192;
constexpr int kRtStages = 3;
constexpr int kRtTile = 128 * 128;                    // 128 rows x 64 bf16
constexpr int kRtStageBytes = 4 * kRtTile;            // W1, W2, W3 tiles + the x tile
constexpr uint32_t kRtTmemCols = 256;                 // two 128-column accumulators
constexpr int kRtBarBytes = (2 * kRtStages + 5) * 8;

struct RouterParams {
  CUtensorMap tmW;     // [3E][d] bf16 (the three parts stacked), box 64 x 128
  CUtensorMap tmX;     // [T][d] bf16, box 64 x 128
  int T, d, E;
  float* logits;       // [T][E]
  int* err;
  int64_t wait_timeout_ns;
};

// kind::f16 instruction descriptor: bf16 A and B, fp32 accumulator, M = 128,
// N = 128, both K-major.
constexpr uint32_t kRtIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// Wr (fp32 [E][d]) -> three exact bf16 parts, stacked [3][E][d].
__global__ void router_split_kernel(const float* __restrict__ rw, long long n, __nv_bfloat16* __restrict__ out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const float w = rw[i];
    const __nv_bfloat16 w1 = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(w1);           // exact
    const __nv_bfloat16 w2 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(w2);          // exact, <= 8 significant bits
    out[i] = w1;
    out[n + i] = w2;
    out[2 * n + i] = __float2bfloat16_rn(r2);            // exact
  }
}

__global__ void __launch_bounds__(kRtThreads, 1) router_tc_kernel(const __grid_constant__ RouterParams p) {
  extern __shared__ __align__(1024) uint8_t rsm_raw[];
  uint8_t* sm = rsm_raw + ((1024u - (smem_u32(rsm_raw) & 1023u)) & 1023u);
  uint8_t* meta = sm + kRtStages * kRtStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta);   // full[S] empty[S] accf[2] acce[2] done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + kRtBarBytes);
  int* svote = reinterpret_cast<int*>(meta + kRtBarBytes + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  const uint32_t bars_s = smem_u32(bars);
  auto full_b = [&](int s) { return bars_s + 8 * s; };
  auto empty_b = [&](int s) { return bars_s + 8 * (kRtStages + s); };
  auto accf_b = [&](int a) { return bars_s + 8 * (2 * kRtStages + a); };
  auto acce_b = [&](int a) { return bars_s + 8 * (2 * kRtStages + 2 + a); };
  const uint32_t done_b = bars_s + 8 * (2 * kRtStages + 4);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) { mbar_init(full_b(s), 1); mbar_init(empty_b(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(accf_b(a), 1); mbar_init(acce_b(a), 4); }
    mbar_init(done_b, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kRtTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_mt = (p.E + 127) / 128, n_nt = (p.T + 127) / 128;
  const int ntiles = n_mt * n_nt, kchunks = p.d / 64;
  const int G = gridDim.x, b = blockIdx.x;
  const int my_tiles = b < ntiles ? (ntiles - 1 - b) / G + 1 : 0;
  const uint64_t deadline = globaltimer_ns() + (uint64_t)p.wait_timeout_ns;
  const uint32_t stage0 = smem_u32(sm);
  bool failed = false;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      tma_prefetch_desc(&p.tmW);
      tma_prefetch_desc(&p.tmX);
      int k = 0;
      for (int it = 0; it < my_tiles && !failed; ++it) {
        const int tile = b + it * G;
        const int mt = tile % n_mt, nt = tile / n_mt;     // both expert tiles of a token tile back to back
        for (int kc = 0; kc < kchunks; ++kc, ++k) {
          const int s = k % kRtStages;
          if (!mbar_wait_spin(empty_b(s), ((k / kRtStages) & 1) ^ 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          const uint32_t st = stage0 + s * kRtStageBytes;
          mbar_arrive_expect_tx(full_b(s), kRtStageBytes);
#pragma unroll
          for (int j = 0; j < 3; ++j)
            tma_load_2d(st + j * kRtTile, &p.tmW, kc * 64, j * p.E + mt * 128, full_b(s), pol);
          tma_load_2d(st + 3 * kRtTile, &p.tmX, kc * 64, nt * 128, full_b(s), pol);
        }
      }
      for (int kk = max(0, k - kRtStages); kk < k; ++kk)
        mbar_wait_spin(full_b(kk % kRtStages), (kk / kRtStages) & 1,
                        globaltimer_ns() + (uint64_t)p.wait_timeout_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int k = 0;
      bool issued_any = false;
      for (int it = 0; it < my_tiles && !failed; ++it) {
        const int ab = it & 1;
        if (!mbar_wait_spin(acce_b(ab), ((it >> 1) & 1) ^ 1, deadline)) {
          failed = true; set_error(p.err, kErrTimeout); break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + ab * 128;
        for (int kc = 0; kc < kchunks; ++kc, ++k) {
          const int s = k % kRtStages;
          if (!mbar_wait_spin(full_b(s), (k / kRtStages) & 1, deadline)) {
            failed = true; set_error(p.err, kErrTimeout); break;
          }
          tc_fence_after();
          const uint32_t st = stage0 + s * kRtStageBytes;
          const uint64_t bdesc = smem_desc_sw128(st + 3 * kRtTile);
#pragma unroll
          for (int j = 0; j < 3; ++j) {
            const uint64_t adesc = smem_desc_sw128(st + j * kRtTile);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)       // K = 16 bf16 = 32 bytes per MMA
              tc_mma_f16(acc, adesc + 2 * kk, bdesc + 2 * kk, kRtIdesc, (kc | j | kk) ? 1u : 0u);
          }
          tc_commit(empty_b(s));
          issued_any = true;
        }
        if (failed) break;
        tc_commit(accf_b(ab));
      }
      if (issued_any) {
        tc_commit(done_b);
        mbar_wait_spin(done_b, 0, globaltimer_ns() + (uint64_t)p.wait_timeout_ns);
      }
    }
  } else {
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    for (int it = 0; it < my_tiles && !failed; ++it) {
      const int ab = it & 1;
      const int tile = b + it * G;
      const int mt = tile % n_mt, nt = tile / n_mt;
      const bool ok = mbar_wait_spin(accf_b(ab), (it >> 1) & 1, deadline);
      if (lane == 0) svote[q] = ok ? 1 : 0;
      named_bar_sync(2, 128);
      const bool all_ok = svote[0] && svote[1] && svote[2] && svote[3];
      named_bar_sync(2, 128);
      if (!all_ok) {
        failed = true;
        if (lane == 0) set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const int e = mt * 128 + q * 32 + lane;
      const int t0 = nt * 128, ncols = min(128, p.T - t0);
      for (int c0 = 0; c0 < ncols; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ab * 128 + lane_base + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c0 + c < ncols && e < p.E) p.logits[(size_t)(t0 + c0 + c) * p.E + e] = __uint_as_float(r[c]);
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
    tmem_dealloc(tmem, kRtTmemCols);
  }
  pdl_launch_dependents();
}

constexpr size_t router_tc_smem_size() { return 1024 + (size_t)kRtStages * kRtStageBytes + kRtBarBytes + 32; }

}  // namespace moe
