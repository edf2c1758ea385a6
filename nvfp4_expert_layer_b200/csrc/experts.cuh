// Light-class expert phase as one persistent kernel: gate/up + SwiGLU and
// down (x routing weight) into per-pair fp32 partials, for every job whose
// expert received fewer rows than the dense threshold (the combine /
// unpermute is the next kernel).
//
// The weights stay 4-bit in HBM and shared memory; each warp unpacks e2m1
// codes and their e4m3 block scales in registers into exact fp16 MMA operands
// ("Optimizing Models to Be Fast at Codegen", section 2: stream the packed
// weights through TMA, unpack e2m1 and the per-16 block scale in registers, a
// grouped GEMM over only the active experts, a persistent kernel so every SM
// stays busy at batch 1, split-K to fill the machine) and multiplies them with
// up to 16 token rows on m16n8k16 tensor-core MMAs.
//
// One uninterrupted weight stream ("Optimizing Muse Spark Open on TPU v7 with
// SGLang-TorchTPU", section 1-2: a decode step should be one stream of weights
// with every transfer in flight before it is needed): block b owns tiles
// b, b + G, b + 2G, ... of one list that holds every gate/up tile followed by
// every down tile.  A warp's bulk-copy ring therefore runs straight from its
// gate/up tiles into its down tiles, so down weights are fetched while other
// blocks finish gate/up.  A down tile waits (bounded) for the gate/up tiles of
// its job through a per-job completion counter before it reads h.
//
// Tile = 16 weight rows of one job over the full K.  The 4 warps of a block
// split K into quarters and meet in shared memory at the end of the tile
// (split-K inside the block).  Gate/up tile t pairs gate rows f = 8t+g with up
// rows 8t+g, so one accumulator holds g and u of the same f and the SwiGLU
// epilogue stays in registers.
//
// Counters reset themselves: the last block to leave clears the per-job
// counters, so a CUDA graph can replay the kernel without a memset.  The
// permutation guarantees that every job has 1..16 rows.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "layout.cuh"

namespace moe {

constexpr int kExpWarps = 4;
constexpr int kExpThreads = kExpWarps * 32;
#ifndef MOE_EXP_SC
#define MOE_EXP_SC 4
#endif
#ifndef MOE_EXP_RING
#define MOE_EXP_RING 4
#endif
constexpr int kExpSC = MOE_EXP_SC;      // 64-wide K chunks per bulk-copy stage (4: 2304 bytes)
constexpr int kExpRing = MOE_EXP_RING;  // bulk-copy stage slots per warp (RT row tiles share RT slots)
static_assert(kExpSC % 2 == 0 && (kExpRing & (kExpRing - 1)) == 0 && kExpRing >= 4, "ring shape");
constexpr int kExpSB = kExpSC * kChunkBytes;
// Resident blocks per SM of the 1- and 2-n-tile kernels (registers capped by
// __launch_bounds__ at 96); with 5 the job table and the reduction buffer
// shrink so that five blocks' shared memory fits an SM.  The kernel is
// latency-bound: on B200 five blocks (20 warps per SM, 96 registers) beat
// four (16 warps, 115 registers) by about 1 %.
#ifndef MOE_EXP_BLOCKS
#define MOE_EXP_BLOCKS 5
#endif
constexpr int kExpBlocks = MOE_EXP_BLOCKS;
constexpr int kExpSmemJobs = kExpBlocks > 4 ? 64 : 512;  // job table copied to shared memory when it fits
constexpr int kExpRedBufs = kExpBlocks > 4 ? 1 : 2;      // cross-warp reduction buffers (by tile parity)
// fp32 MMA accumulators per (row tile, n-tile): the four K steps of a chunk
// chain into one (the chains of the row tiles and n-tiles interleave).
constexpr int kAccK = 1;

struct ExpertParams {
  const uint8_t* gu_frag;     // gate/up fragment layout [E][f/8 tiles][d/64 chunks]
  const uint8_t* dn_frag;     // down fragment layout    [E][d/16 tiles][f/64 chunks]
  int tpe_gu, cpt_gu;         // f/8, d/64
  int tpe_dn, cpt_dn;         // d/16, f/64
  const int4* jobs;           // {expert, row0, nrows, 0}, 1 <= nrows <= 16
  const int* njobs;
  const int* perm;            // pair index per permuted row
  const int* inv;             // permuted row per pair
  int topk, T, d, f, E;
  const __half* x16;          // [T][d] B-fragment layout, x * 2^s
  const float* xscale;        // [T] 2^-s
  __half* h16;                // [P][f] B-fragment layout
  float* h32;                 // [P][f]
  const float* gs;            // [3][E] gate, up, down tensor scales
  const int* hexp;            // [E] exponent bound of |g| * |u| per expert (light_h_exp)
  const float* wts;           // [P] routing weight per pair; null: partials unweighted
  float* partial;             // [P][d]
  int* gu_done;               // [max jobs] gate/up tiles finished per job
  int* exit_cnt;              // blocks that left
  int* err;
  int64_t wait_timeout_ns;
  int wait_extra;             // test hook: added to every down tile's completion target (0)
  const uint8_t* l2_next;     // bytes to prefetch into L2 (the next layer's router weights) or null
  long long l2_next_bytes;    // a multiple of 16
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// fp16 staging exponent of h for one (token, expert) row of the light class.
// h enters the down projection as fp16, so it is held as h * 2^e_h with e_h
// chosen before any gate/up tile of the row runs, from a bound that every
// tile can compute alike:
//   the staged x row has max |x * 2^s| < 2^15, xs = 2^-s (stage_x_row), so
//   max |x| < 2^(15 - s);  |g| <= |gs_g| * L1_g * max|x| < 2^(Eg + 15 - s) and
//   |u| < 2^(Eu + 15 - s) (hexp = Eg + Eu, expert_hexp_kernel);  |SiLU(g)| <= |g|,
//   so |h| < 2^(Eg + Eu + 30 - 2s).
// e_h = 2s - 15 - hexp keeps |h| * 2^e_h below 2^15 (half of the fp16 range,
// room for the fp32 rounding of g and u) whatever the magnitudes of x and the
// weights, so h never overflows fp16, and values far below the bound lose
// only absolute precision 2^-25 * 2^-e_h.  The exponent is clamped to +-120
// (fp32 range); beyond that the overflow check still reports
// MOE_FP4_ERR_NUMERIC.
__device__ __forceinline__ int light_h_exp(float xs, int hexp_e) {
  const int s = 127 - (int)((__float_as_uint(xs) >> 23) & 0xffu);   // xs = 2^-s, a normal float
  return max(-120, min(120, 2 * s - 15 - hexp_e));
}
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

__device__ __forceinline__ uint4 ldg_cg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Everything a warp needs to know about one tile of the list.
struct TileInfo {
  int down;       // 0 gate/up, 1 down
  int job, t;     // job index, tile index within the expert
  int e, row0, nrows;
  int cpt;        // chunks per tile
  int slo, nw;    // this warp's first stage and stage count
  const uint8_t* base;
};

// RT = 16-row tiles of the fragment layout per work tile (consecutive tiles
// t, t + 1 of one expert matrix); ti.t is the first of them.
template <int RT>
__device__ __forceinline__ TileInfo tile_info(const ExpertParams& p, const int4* jobs, int i, int ngu,
                                              int warp) {
  TileInfo ti;
  ti.down = i >= ngu;
  const int tpe = ti.down ? p.tpe_dn : p.tpe_gu;
  const int wtpe = tpe / RT;
  const int li = ti.down ? i - ngu : i;
  ti.job = li / wtpe;
  ti.t = (li - ti.job * wtpe) * RT;
  const int4 jb = jobs[ti.job];
  ti.e = jb.x;
  ti.row0 = jb.y;
  ti.nrows = jb.z;
  ti.cpt = ti.down ? p.cpt_dn : p.cpt_gu;
  const int spt = (ti.cpt + kExpSC - 1) / kExpSC;
  ti.slo = warp * spt / kExpWarps;
  ti.nw = (warp + 1) * spt / kExpWarps - ti.slo;
  ti.base = (ti.down ? p.dn_frag : p.gu_frag) + (size_t)((size_t)ti.e * tpe + ti.t) * ti.cpt * kChunkBytes;
  return ti;
}

// Two non-negative e4m3 block scales as f16x2, each times 2^-8, on the
// integer pipes: {a_k, b_k} (byte k of `a` in the low half, byte k of `b` in
// the high half).  A byte's 7 bits placed at f16 bit 7 give 2^(E-15) (1 + M/8)
// for exponent field E >= 1 and 2^-14 M/8 for E = 0, i.e. exactly 2^-8 times
// the e4m3 value in both cases (f16 subnormals cover the e4m3 subnormals);
// the 2^-8 is undone on the fp32 accumulators.  One byte permute puts the two
// bytes in the low byte of each half (the other bytes come from the
// sign-replicate mode of a byte whose top bit is clear, i.e. zero), one shift
// moves them to f16 bit 7.  (The PTX prmt default mode honours the selector's
// sign-replicate bit; __byte_perm keeps only the low three bits of each
// selector nibble.)
constexpr float kScaleUndo = 256.f;

template <int K>
__device__ __forceinline__ uint32_t e4m3_pair_f16x2(uint32_t a, uint32_t b) {
  constexpr uint32_t sel = (uint32_t)K | ((8u | K) << 4) | ((4u + K) << 8) | ((12u + K) << 12);
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "n"(sel));
  return r << 7;
}

// a * {lo(s), lo(s)} and a * {hi(s), hi(s)}: the half broadcast is an operand
// modifier of the f16x2 multiply.
__device__ __forceinline__ uint32_t hmul2_bcast_lo(uint32_t a, uint32_t s) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), __low2half2(*reinterpret_cast<const __half2*>(&s)));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hmul2_bcast_hi(uint32_t a, uint32_t s) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), __high2half2(*reinterpret_cast<const __half2*>(&s)));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Activation fragment of one 64-wide chunk for lane c and one n-tile: the two
// 16-byte halves holding b0, b1 of the chunk's four K steps (zero beyond the
// job's rows).
struct BPair {
  uint4 lo, hi;
};

// Units of a work tile: RT row tiles x NT n-tiles (two for NT = 1, 2; four for NT = 4).
template <int NT>
struct TileShape {
  static constexpr int RT = NT == 1 ? 2 : 1;       // 16-row tiles per work tile
  static constexpr int U = RT * NT;                // (row tile, n-tile) units, one per epilogue warp
  static constexpr int NR = NT < 2 ? 2 : NT;       // B row pointers held per lane
};

template <int NT, int NR, bool COHERENT>
__device__ __forceinline__ void load_bchunk(const __half* const (&brow)[NR], int chunk, int c, BPair (&b)[NT]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if (brow[nt] == nullptr) {
      b[nt].lo = make_uint4(0, 0, 0, 0);
      b[nt].hi = b[nt].lo;
    } else {
      const __half* bp = brow[nt] + (size_t)chunk * kChunkK + c * 16;
      b[nt].lo = COHERENT ? ldg_cg_v4(bp) : ldg_nc_v4(bp);
      b[nt].hi = COHERENT ? ldg_cg_v4(bp + 8) : ldg_nc_v4(bp + 8);
    }
  }
}

// One stage of a work tile: RT row tiles x NT n-tiles.  The activation
// fragments are not held a stage ahead (64 NT registers) but one chunk ahead:
// `be` holds chunk0's on entry and the next chunk's on exit when `more` says
// the warp's next stage of this tile follows.  FULL: all kExpSC chunks
// present (no per-chunk bounds).  The fragments of even chunks live in `be`,
// those of odd chunks in `bo`: each chunk prefetches the next one into the
// other set, so a full stage ends with the next stage's first chunk in `be`
// and nothing is copied.  The codes and scales of the next (chunk, row tile)
// unit are loaded before the current one is converted.
template <int NT, int RT, int NR, bool COHERENT, bool FULL>
__device__ __forceinline__ void mma_stage_jit(uint32_t st, int nch, int lane, int g, const __half* const (&brow)[NR],
                                              int chunk0, int c, bool more, int nrows, BPair (&be)[NT],
                                              float (&acc)[RT][kAccK][NT][4]) {
  constexpr int NU = kExpSC * RT;
  auto unit_addr = [&](int u) { return st + (u % RT) * kExpSB + (u / RT) * kChunkBytes; };
  uint4 codes_n = ld_shared_v4(unit_addr(0) + lane * 16);
  uint2 sc_n = ld_shared_v2(unit_addr(0) + kChunkCodeBytes + g * 8);
  BPair bo[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) { bo[nt].lo = make_uint4(0, 0, 0, 0); bo[nt].hi = bo[nt].lo; }
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const int ch = u / RT, rt = u % RT;
    if (!FULL && ch >= nch) break;
    if (rt == 0) {
      const bool pf = FULL ? (ch + 1 < kExpSC || more) : (ch + 1 < nch || more);
      if (pf) {
        if (ch & 1) load_bchunk<NT, NR, COHERENT>(brow, chunk0 + ch + 1, c, be);
        else load_bchunk<NT, NR, COHERENT>(brow, chunk0 + ch + 1, c, bo);
      }
    }
    const BPair (&bb)[NT] = (ch & 1) ? bo : be;
    const uint4 codes = codes_n;
    const uint2 sc = sc_n;
    if (u + 1 < NU && (FULL || (u + 1) / RT < nch)) {
      codes_n = ld_shared_v4(unit_addr(u + 1) + lane * 16);
      sc_n = ld_shared_v2(unit_addr(u + 1) + kChunkCodeBytes + g * 8);
    }
    const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
    // scales: sc.x = row A(g) for K steps 0..3, sc.y = row B(g); non-negative
    // e4m3 bytes (signs are folded into the codes)
    const uint32_t sAB[4] = {e4m3_pair_f16x2<0>(sc.x, sc.y), e4m3_pair_f16x2<1>(sc.x, sc.y),
                             e4m3_pair_f16x2<2>(sc.x, sc.y), e4m3_pair_f16x2<3>(sc.x, sc.y)};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t a[4];
      e2m1x8_to_f16x2x4(cw[ks], a);
      a[0] = hmul2_bcast_lo(a[0], sAB[ks]);
      a[1] = hmul2_bcast_hi(a[1], sAB[ks]);
      a[2] = hmul2_bcast_lo(a[2], sAB[ks]);
      a[3] = hmul2_bcast_hi(a[3], sAB[ks]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint4& lo = bb[nt].lo;
        const uint4& hi = bb[nt].hi;
        const uint32_t b0 = ks == 0 ? lo.x : ks == 1 ? lo.z : ks == 2 ? hi.x : hi.z;
        const uint32_t b1 = ks == 0 ? lo.y : ks == 1 ? lo.w : ks == 2 ? hi.y : hi.w;
        if (NT == 1 || nt * 8 < nrows) mma_16816_f16(acc[rt][ks % kAccK][nt], a, b0, b1);
      }
    }
  }
}

// NT = 8-wide n-tiles per job: expert_kernel<1> runs jobs of <= 8 rows,
// expert_kernel<2> jobs of 9..16 rows, expert_kernel<4> jobs of 17..32 rows;
// each has its own job list and counters.  With one n-tile a work tile is
// two 16-row tiles (RT = 2) that share the activation fragments, the loop
// control and the epilogue barrier.  A job's weights are streamed once per
// job, so the 32-row jobs stream an expert with up to 32 rows once.
template <int NT>
__global__ void __launch_bounds__(kExpThreads, NT == 4 ? 3 : kExpBlocks) expert_kernel(ExpertParams p) {
  constexpr int RT = TileShape<NT>::RT;
  constexpr int U = TileShape<NT>::U;
  constexpr int NR = TileShape<NT>::NR;
  constexpr int RING = kExpRing / RT;          // stages in flight per warp (same bytes)
  constexpr int SLOT = RT * kExpSB;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars_all = reinterpret_cast<uint64_t*>(smem + kExpWarps * RING * SLOT);
  float* red_all = reinterpret_cast<float*>(bars_all + kExpWarps * RING);   // [2][4 warps][U][32][4]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int G = (int)gridDim.x, b = (int)blockIdx.x;

  pdl_wait();                                   // routing results of the previous kernel
  // the next layer's router weights go to L2 while this layer streams its
  // experts: each block asks for its slice (a hint; nothing waits on it)
  if (p.l2_next && threadIdx.x == 0) {
    const long long per = ((p.l2_next_bytes / G + 15) / 16) * 16;
    const long long lo = per * b;
    for (long long o = lo; o < lo + per && o < p.l2_next_bytes; o += 32768)
      bulk_prefetch_l2(p.l2_next + o, (uint32_t)min(32768LL, min(lo + per, p.l2_next_bytes) - o));
  }
  const int njobs = *p.njobs;
  const int ngu = njobs * (p.tpe_gu / RT);
  const int ntot = ngu + njobs * (p.tpe_dn / RT);
  const int my_tiles = b < ntot ? (ntot - 1 - b) / G + 1 : 0;
  const uint64_t deadline = globaltimer_ns() + (uint64_t)p.wait_timeout_ns;
  __shared__ int4 s_jobs[kExpSmemJobs];
  const int4* jobs = p.jobs;
  if (njobs <= kExpSmemJobs) {
    for (int i = threadIdx.x; i < njobs; i += blockDim.x) s_jobs[i] = p.jobs[i];
    jobs = s_jobs;
  }
  __syncthreads();

  const uint32_t ring_s = smem_u32(smem + warp * RING * SLOT);
  const uint32_t bars_s = smem_u32(bars_all + warp * RING);
  const uint64_t pol = policy_evict_first();
  if (lane == 0) {
    for (int i = 0; i < RING; ++i) mbar_init(bars_s + 8 * i, 1);
    fence_mbar_init();
  }
  __syncwarp();

  // ---- producer state (lane 0 of each warp): walks this warp's stages in order.
  // Per tile: the source of the warp's next stage (row tile 0), the distance
  // between row tiles, the stages left and the chunk count of the last one.
  static_assert((RING & (RING - 1)) == 0, "ring slots: a power of two");
  int c_it = 0, c_left = 0, c_nch_last = 0, issued = 0;
  const uint8_t* c_src = nullptr;
  size_t c_rt_stride = 0;
  auto cursor_ready = [&]() -> bool {
    while (c_left == 0) {
      if (c_it >= my_tiles) return false;
      const TileInfo t = tile_info<RT>(p, jobs, b + c_it * G, ngu, warp);
      ++c_it;
      c_left = t.nw;
      c_src = t.base + (size_t)kExpSC * t.slo * kChunkBytes;
      c_rt_stride = (size_t)t.cpt * kChunkBytes;
      c_nch_last = t.cpt - kExpSC * (t.slo + t.nw - 1);
      if (c_nch_last > kExpSC) c_nch_last = kExpSC;
    }
    return true;
  };
  auto produce = [&](int consumed) {          // keep RING stages in flight
    while (issued < consumed + RING && cursor_ready()) {
      const int nch = c_left == 1 ? c_nch_last : kExpSC;
      const int slot = issued & (RING - 1);
      mbar_arrive_expect_tx(bars_s + 8 * slot, RT * nch * kChunkBytes);
#pragma unroll
      for (int rt = 0; rt < RT; ++rt)
        bulk_g2s(ring_s + slot * SLOT + rt * kExpSB, c_src + rt * c_rt_stride, nch * kChunkBytes,
                 bars_s + 8 * slot, pol);
      c_src += kExpSC * kChunkBytes;
      --c_left;
      ++issued;
    }
  };
  if (lane == 0) produce(0);

  bool failed = false;
  int consumed = 0;

  // B rows of this lane (row n = nt*8 + g of the job), resolved one tile ahead
  auto tile_rows = [&](const TileInfo& t, const __half* (&row)[NR]) {
#pragma unroll
    for (int nt = 0; nt < NR; ++nt) {
      const int n = nt * 8 + g;
      row[nt] = nullptr;
      if (n < t.nrows) {
        const int r = t.row0 + n;
        row[nt] = t.down ? p.h16 + (size_t)r * p.f : p.x16 + (size_t)(p.perm[r] / p.topk) * p.d;
      }
    }
  };
  TileInfo ti_next{};
  const __half* row_next[NR] = {};
  if (my_tiles > 0) {
    ti_next = tile_info<RT>(p, jobs, b, ngu, warp);
    tile_rows(ti_next, row_next);
  }

  for (int it = 0; it < my_tiles; ++it) {
    const TileInfo ti = ti_next;
    const int nt_used = (ti.nrows + 7) >> 3;
    const __half* row[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) row[i] = row_next[i];
    if (it + 1 < my_tiles) {
      ti_next = tile_info<RT>(p, jobs, b + (it + 1) * G, ngu, warp);
      tile_rows(ti_next, row_next);
    }
    if (ti.down && ti.nw > 0 && !failed) {      // h of this job must be complete
      int ok = 1;
      if (lane == 0) {
        uint32_t n = 0;
        // every gate/up tile of the job is published once per writer warp (n-tile)
        const int target = p.tpe_gu * ((ti.nrows + 7) >> 3) + p.wait_extra;
        while (ld_acquire(p.gu_done + ti.job) < target) {
          __nanosleep(128);
          if ((++n & 15u) == 0 && globaltimer_ns() > deadline) { ok = 0; break; }
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        failed = true;
        if (lane == 0) set_error(p.err, kErrTimeout);
      }
    }

    float part[U][4];                    // this warp's partial sums, per unit u = rt * NT + nt
    {
      float acc[RT][kAccK][NT][4];
#pragma unroll
      for (int rt = 0; rt < RT; ++rt)
#pragma unroll
        for (int a = 0; a < kAccK; ++a)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[rt][a][nt][q] = 0.f;
      BPair be[NT];
      if (ti.nw > 0) {
        if (ti.down) load_bchunk<NT, NR, true>(row, kExpSC * ti.slo, c, be);
        else load_bchunk<NT, NR, false>(row, kExpSC * ti.slo, c, be);
      }
      for (int ss = 0; ss < ti.nw; ++ss) {
        const int s = ti.slo + ss;
        const int nch = min(kExpSC, ti.cpt - kExpSC * s);
        const bool more = ss + 1 < ti.nw;
        const int slot = consumed & (RING - 1);
        if (!failed && !mbar_wait_until(bars_s + 8 * slot, ((unsigned)consumed / RING) & 1u, deadline)) {
          failed = true;
          set_error(p.err, kErrTimeout);
        }
        if (!failed) {
          const uint32_t sp = ring_s + slot * SLOT;
          const int k0 = kExpSC * s, nr = ti.nrows;
          if (nch == kExpSC) {
            if (ti.down) mma_stage_jit<NT, RT, NR, true, true>(sp, nch, lane, g, row, k0, c, more, nr, be, acc);
            else mma_stage_jit<NT, RT, NR, false, true>(sp, nch, lane, g, row, k0, c, more, nr, be, acc);
          } else {
            if (ti.down) mma_stage_jit<NT, RT, NR, true, false>(sp, nch, lane, g, row, k0, c, more, nr, be, acc);
            else mma_stage_jit<NT, RT, NR, false, false>(sp, nch, lane, g, row, k0, c, more, nr, be, acc);
          }
        }
        __syncwarp();
        ++consumed;
        if (lane == 0 && !failed) produce(consumed);
      }
      // units: NT == 1 -> (row tile u, n-tile 0); NT >= 2 -> (row tile 0, n-tile u)
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int rt = NT == 1 ? u : 0, nt = NT == 1 ? 0 : u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v = acc[rt][0][nt][q];
#pragma unroll
          for (int a = 1; a < kAccK; ++a) v += acc[rt][a][nt][q];
          part[u][q] = v;
        }
      }
    }

    // ---- cross-warp reduction of the tile (buffer alternates by tile parity;
    // with one buffer the previous tile's readers finish first)
    if (kExpRedBufs == 1 && it > 0) __syncthreads();
    float* red = red_all + (kExpRedBufs == 1 ? 0 : (it & 1)) * (kExpWarps * U * 32 * 4);
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        red[((warp * U + u) * 32 + lane) * 4 + q] = part[u][q];
    __syncthreads();
    const int units_used = RT * nt_used;
    if (warp < units_used) {
      const int nt = NT == 1 ? 0 : warp;           // unit u = warp: row tile rt, n-tile nt
      const int rt = NT == 1 ? warp : 0;
      const int red_u = warp;
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kExpWarps; ++w) sum += red[((w * U + red_u) * 32 + lane) * 4 + q];
        v[q] = sum;
      }
      if (!ti.down) {
        const float gsg = p.gs[ti.e] * kScaleUndo, gsu = p.gs[p.E + ti.e] * kScaleUndo;
        const int fidx = (ti.t + rt) * 8 + g;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int n = nt * 8 + 2 * c + q;
          if (n < ti.nrows) {
            const int r = ti.row0 + n;
            const float xs = p.xscale[p.perm[r] / p.topk];
            const float gv = v[q] * gsg * xs;
            const float uv = v[2 + q] * gsu * xs;
            const float hv = gv / (1.f + expf(-gv)) * uv;
            p.h32[(size_t)r * p.f + fidx] = hv;
            const float hs = hv * exp2i(light_h_exp(xs, p.hexp[ti.e]));
            if (!(fabsf(hs) <= 65504.f)) set_error(p.err, kErrNumeric);
            p.h16[(size_t)r * p.f + bfrag_offset(fidx)] = __float2half_rn(hs);
          }
        }
      } else {
        const float gsd = p.gs[2 * p.E + ti.e];
        const int drow = (ti.t + rt) * 16 + g;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int n = nt * 8 + 2 * c + q;
          if (n < ti.nrows) {
            const int r = ti.row0 + n;
            const int pr = p.perm[r];
            const float hinv = exp2i(-light_h_exp(p.xscale[pr / p.topk], p.hexp[ti.e]));
            const float wv = (p.wts ? p.wts[pr] : 1.f) * gsd * kScaleUndo * hinv;
            p.partial[(size_t)r * p.d + drow] = v[q] * wv;
            p.partial[(size_t)r * p.d + drow + 8] = v[2 + q] * wv;
          }
        }
      }
      // publish this (row tile, n-tile) of a gate/up work tile (release, no round trip)
      __syncwarp();
      if (!ti.down && lane == 0) red_release_add(p.gu_done + ti.job, 1);
    }
  }

  // Drain: after a failed wait, give the copies already issued a bounded chance
  // to land before the block's shared memory is released.
  if (failed && lane == 0) {
    const uint64_t drain = globaltimer_ns() + (uint64_t)p.wait_timeout_ns;
    for (int jj = consumed; jj < issued; ++jj)
      if (!mbar_wait_until(bars_s + 8 * (jj & (RING - 1)), ((unsigned)jj / RING) & 1u, drain)) break;
  }
  // ---- exit protocol: the last block clears the per-job counters
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(p.exit_cnt, 1);
    if (old == G - 1) {
      for (int jb = 0; jb < njobs; ++jb) p.gu_done[jb] = 0;
      *p.exit_cnt = 0;
      __threadfence();
    }
  }
  pdl_launch_dependents();
}

template <int NT>
constexpr size_t expert_smem_size() {
  return (size_t)kExpWarps * kExpRing * kExpSB + (size_t)kExpWarps * kExpRing * 8 +
         (size_t)kExpRedBufs * kExpWarps * TileShape<NT>::U * 32 * 4 * 4;
}

}  // namespace moe
