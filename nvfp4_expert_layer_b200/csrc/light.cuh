// Light expert class: experts that received fewer rows than the dense
// threshold.  The weights stay 4-bit in HBM and in shared memory; each warp
// unpacks e2m1 codes and their e4m3 block scale in registers into exact fp16
// MMA operands ("Optimizing Models to Be Fast at Codegen", section 2: stream
// the packed weights through TMA, unpack e2m1 and the per-16 block scale in
// registers, grouped over only the active experts) and multiplies them with
// up to 16 token rows on m16n8k16 tensor-core MMAs.  The few-row loop has its
// own kernel, apart from the dense class, so its registers stay small
// ("Optimizing Muse Spark Open on TPU v7 with SGLang-TorchTPU", section 5).
//
// Work decomposition: a job is (expert, up to 16 consecutive rows of the
// permutation); a tile is 16 weight rows of one job's expert over the full K.
// A block of 4 warps owns one tile at a time and splits its K range into four
// contiguous quarters; each warp streams its quarter through a private ring
// of shared-memory stages filled by untiled bulk copies (cp.async.bulk, one
// elected lane, mbarrier completion), so up to kRing stages per warp are in
// flight.  The four partial accumulators meet in shared memory at the end of
// the tile.  Blocks are persistent: block b handles tiles b, b + grid, ...
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "layout.cuh"

namespace moe {

constexpr int kLightWarps = 4;
constexpr int kLightThreads = kLightWarps * 32;
constexpr int kLightNT = 2;              // 8-wide n-tiles per job (16 rows)

enum LightMode { kGateUp = 0, kDown = 1 };

struct LightParams {
  const uint8_t* frag;      // fragment-layout weights of all experts
  int tpe;                  // tiles per expert
  int cpt;                  // 64-wide K chunks per tile
  const int4* jobs;         // {expert, row0, nrows, 0}
  const int* njobs;         // device count of jobs
  const int* perm;          // permutation (pair index per row)
  int topk;
  const __half* bsrc;       // gate/up: x16 [T][K] ; down: h16 [P][K]  (B-fragment layout)
  int bk;                   // K of a B row (halves)
  const float* xscale;      // gate/up: per-token 2^-s
  const float* gs0;         // gate/up: gate gs ; down: down gs
  const float* gs1;         // gate/up: up gs
  const float* wts;         // down: routing weight per pair
  float* h32;               // gate/up output [P][f] (fp32)
  __half* h16;              // gate/up output [P][f] (B-fragment layout)
  int f;                    // gate/up: f
  float* partial;           // down output [P][d] (fp32)
  int d;                    // down: d
  int* err;
  int64_t wait_timeout_ns;  // bound on every mbarrier wait of a launch
};

template <int MODE, int RING>
__global__ void __launch_bounds__(kLightThreads, 1)
light_expert_kernel(LightParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring_all = smem;
  uint64_t* bars_all = reinterpret_cast<uint64_t*>(smem + kLightWarps * RING * kStageBytes);
  float* red = reinterpret_cast<float*>(bars_all + kLightWarps * RING);   // [4][NT][32][4]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  pdl_wait();                                    // routing outputs of the previous kernels
  const int njobs = *p.njobs;
  const int ntiles = njobs * p.tpe;
  if ((int)blockIdx.x >= ntiles) { pdl_launch_dependents(); return; }
  const int my_tiles = (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1;
  const int spt = (p.cpt + kStageChunks - 1) / kStageChunks;      // stages per tile
  const int slo = warp * spt / kLightWarps, shi = (warp + 1) * spt / kLightWarps;
  const int nw = shi - slo;                                         // my stages per tile
  const int total = my_tiles * nw;

  uint8_t* ring = ring_all + warp * RING * kStageBytes;
  uint64_t* bars = bars_all + warp * RING;
  const uint32_t ring_s = smem_u32(ring);
  const uint32_t bars_s = smem_u32(bars);
  const uint64_t pol = policy_evict_first();

  if (lane == 0) {
    for (int i = 0; i < RING; ++i) mbar_init(bars_s + 8 * i, 1);
    fence_mbar_init();
  }
  __syncwarp();

  auto issue = [&](int j) {
    const int i = j / nw, s = slo + j % nw;
    const int tile = (int)blockIdx.x + i * (int)gridDim.x;
    const int job = tile / p.tpe, t = tile - job * p.tpe;
    const int e = p.jobs[job].x;
    const int nch = min(kStageChunks, p.cpt - kStageChunks * s);
    const uint8_t* src = p.frag + ((size_t)((size_t)e * p.tpe + t) * p.cpt + (size_t)kStageChunks * s) * kChunkBytes;
    const uint32_t bytes = nch * kChunkBytes;
    const int slot = j % RING;
    mbar_arrive_expect_tx(bars_s + 8 * slot, bytes);
    bulk_g2s(ring_s + slot * kStageBytes, src, bytes, bars_s + 8 * slot, pol);
  };

  if (lane == 0)
    for (int j = 0; j < min(RING, total); ++j) issue(j);
  int issued = min(RING, total);     // stages issued so far (warp-uniform)

  const uint64_t deadline = globaltimer_ns() + (uint64_t)p.wait_timeout_ns;
  bool failed = false;
  int j_fail = 0;
  int j = 0;
  for (int it = 0; it < my_tiles; ++it) {
    const int tile = (int)blockIdx.x + it * (int)gridDim.x;
    const int job = tile / p.tpe, t = tile - job * p.tpe;
    const int4 jb = p.jobs[job];
    const int e = jb.x, row0 = jb.y, nrows = jb.z;
    const int ntu = (nrows + 7) >> 3;

    // B rows for this lane: n = nt*8 + g
    const __half* brow[kLightNT];
#pragma unroll
    for (int nt = 0; nt < kLightNT; ++nt) {
      const int n = nt * 8 + g;
      brow[nt] = nullptr;
      if (n < nrows) {
        const int r = row0 + n;
        const int brow_idx = (MODE == kGateUp) ? (p.perm[r] / p.topk) : r;
        brow[nt] = p.bsrc + (size_t)brow_idx * p.bk;
      }
    }

    float acc[kLightNT][4];
#pragma unroll
    for (int nt = 0; nt < kLightNT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[nt][q] = 0.f;

    for (int ss = 0; ss < nw; ++ss, ++j) {
      const int s = slo + ss;
      const int nch = min(kStageChunks, p.cpt - kStageChunks * s);
      // activation fragments for this stage (L2-resident, issued before the wait)
      uint4 bf[kLightNT][kStageChunks][2];
#pragma unroll
      for (int nt = 0; nt < kLightNT; ++nt)
#pragma unroll
        for (int ch = 0; ch < kStageChunks; ++ch) {
          if (brow[nt] != nullptr && ch < nch) {
            const __half* bp = brow[nt] + (size_t)(kStageChunks * s + ch) * kChunkK + c * 16;
            bf[nt][ch][0] = ldg_nc_v4(bp);
            bf[nt][ch][1] = ldg_nc_v4(bp + 8);
          } else {
            bf[nt][ch][0] = make_uint4(0, 0, 0, 0);
            bf[nt][ch][1] = make_uint4(0, 0, 0, 0);
          }
        }
      const int slot = j % RING;
      if (!failed && !mbar_wait_until(bars_s + 8 * slot, (j / RING) & 1, deadline)) {
        failed = true;
        j_fail = j;
        set_error(p.err, kErrTimeout);
      }
      if (!failed) {
        const uint32_t st = ring_s + slot * kStageBytes;
#pragma unroll
        for (int ch = 0; ch < kStageChunks; ++ch) {
          if (ch < nch) {
            const uint4 codes = ld_shared_v4(st + ch * kChunkBytes + lane * 16);
            const uint2 sc = ld_shared_v2(st + ch * kChunkBytes + kChunkCodeBytes + g * 8);
            const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
            const uint32_t bw[8] = {bf[0][ch][0].x, bf[0][ch][0].y, bf[0][ch][0].z, bf[0][ch][0].w,
                                    bf[0][ch][1].x, bf[0][ch][1].y, bf[0][ch][1].z, bf[0][ch][1].w};
            const uint32_t bw1[8] = {bf[1][ch][0].x, bf[1][ch][0].y, bf[1][ch][0].z, bf[1][ch][0].w,
                                     bf[1][ch][1].x, bf[1][ch][1].y, bf[1][ch][1].z, bf[1][ch][1].w};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint32_t pair = ((ks < 2 ? sc.x : sc.y) >> (16 * (ks & 1))) & 0xffffu;
              const uint32_t s2 = e4m3x2_to_f16x2(pair);
              const uint32_t sA = dup_lo(s2), sB = dup_hi(s2);
              uint32_t a[4];
              e2m1x8_to_f16x2x4(cw[ks], a);
              a[0] = hmul2_u32(a[0], sA);
              a[1] = hmul2_u32(a[1], sB);
              a[2] = hmul2_u32(a[2], sA);
              a[3] = hmul2_u32(a[3], sB);
              mma_16816_f16(acc[0], a, bw[2 * ks], bw[2 * ks + 1]);
              if (ntu > 1) mma_16816_f16(acc[1], a, bw1[2 * ks], bw1[2 * ks + 1]);
            }
          }
        }
      }
      __syncwarp();
      if (!failed && j + RING < total) {
        if (lane == 0) issue(j + RING);
        issued = j + RING + 1;
      }
    }

    // cross-warp reduction of the tile
#pragma unroll
    for (int nt = 0; nt < kLightNT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) red[((warp * kLightNT + nt) * 32 + lane) * 4 + q] = acc[nt][q];
    __syncthreads();
    if (warp < ntu) {
      const int nt = warp;
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kLightWarps; ++w) s += red[((w * kLightNT + nt) * 32 + lane) * 4 + q];
        v[q] = s;
      }
      if (MODE == kGateUp) {
        const float gsg = p.gs0[e], gsu = p.gs1[e];
        const int fidx = t * 8 + g;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int n = nt * 8 + 2 * c + q;
          if (n < nrows) {
            const int r = row0 + n;
            const int tok = p.perm[r] / p.topk;
            const float xs = p.xscale[tok];
            const float gv = v[q] * gsg * xs;
            const float uv = v[2 + q] * gsu * xs;
            const float hv = gv / (1.f + expf(-gv)) * uv;
            p.h32[(size_t)r * p.f + fidx] = hv;
            if (!(fabsf(hv) <= 65504.f)) set_error(p.err, kErrNumeric);
            p.h16[(size_t)r * p.f + bfrag_offset(fidx)] = __float2half_rn(hv);
          }
        }
      } else {
        const float gsd = p.gs0[e];
        const int drow = t * 16 + g;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int n = nt * 8 + 2 * c + q;
          if (n < nrows) {
            const int r = row0 + n;
            const float wv = p.wts[p.perm[r]] * gsd;
            p.partial[(size_t)r * p.d + drow] = v[q] * wv;
            p.partial[(size_t)r * p.d + drow + 8] = v[2 + q] * wv;
          }
        }
      }
    }
    __syncthreads();
  }
  // Drain: if a wait failed, give the copies already issued a bounded chance
  // to land before the block's shared memory is released.
  if (failed) {
    const uint64_t drain = globaltimer_ns() + (uint64_t)p.wait_timeout_ns;
    for (int jj = j_fail; jj < issued; ++jj)
      if (!mbar_wait_until(bars_s + 8 * (jj % RING), (jj / RING) & 1, drain)) break;
  }
  pdl_launch_dependents();
}

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
        dst[kChunkCodeBytes + g * 8 + 2 * ks] = fa[ch * 4 + ks];
        dst[kChunkCodeBytes + g * 8 + 2 * ks + 1] = fb[ch * 4 + ks];
      }
    }
  }
}

}  // namespace moe
