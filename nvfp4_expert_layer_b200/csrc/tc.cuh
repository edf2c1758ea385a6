// tcgen05 / TMEM / tensor-TMA wrappers for the dense expert class (sm_100a).
#pragma once
#include <cstdint>
#include <cuda.h>
#include "ptx.cuh"

namespace moe {

// ---------------------------------------------------------------- TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_result), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on an mbarrier once every tcgen05 operation issued so far by this thread completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}
// Shared memory (descriptor) -> TMEM: 128 lanes x 256 bits (8 columns), lane L
// from source row L.
__device__ __forceinline__ void tc_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
// Shared memory (descriptor) -> TMEM: 32 rows x 128 bits (4 columns), row L
// to lane L of every one of the four lane quarters.
__device__ __forceinline__ void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
// D[128 x N] (+)= A[128 x 64] * B[N x 64]^T, NVFP4 operands with e4m3 scales per 16 (in TMEM).
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// 32 lanes x 32 columns of 32-bit words: this thread's lane, columns taddr.col .. +31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(n) : "memory");
}

// ---------------------------------------------------------------- descriptors
// K-major operand with 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);          // start address
  d |= (uint64_t)1 << 16;                           // leading byte offset (unused with swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;                 // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                           // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                           // layout: SWIZZLE_128B
  return d;
}
// K-major operand with rows of ROW_BYTES (128: 128-byte swizzle; 64: 64-byte
// swizzle), 8-row atoms of 8 * ROW_BYTES bytes.
template <int ROW_BYTES>
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t saddr) {
  static_assert(ROW_BYTES == 128 || ROW_BYTES == 64, "row bytes");
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)((8 * ROW_BYTES) >> 4) << 32;      // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(ROW_BYTES == 128 ? 2 : 4) << 61;  // SWIZZLE_128B / SWIZZLE_64B
  return d;
}

// Scale-factor copy source: 128 rows x 32 bytes, no swizzle, as core matrices
// of 8 rows x 16 bytes; the two 16-byte halves of a row group are 128 bytes
// apart (leading byte offset), row groups `sbo` bytes apart (stride byte
// offset: 256 times the units per stage of the interleaved scale layouts).
__device__ __forceinline__ uint64_t smem_desc_sf256(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)(128 >> 4) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  return d;                                         // layout: SWIZZLE_NONE
}
// Scale-factor copy source of 32 rows x 16 bytes, no swizzle: four core
// matrices of 8 rows x 16 bytes, `sbo` bytes apart (the leading byte offset
// is unused with one 16-byte column).
__device__ __forceinline__ uint64_t smem_desc_sf128(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)(128 >> 4) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  return d;                                         // layout: SWIZZLE_NONE
}
// Instruction descriptor: kind::mxf4nvf4, A/B e2m1, e4m3 scales, fp32 accumulate, K-major;
// M = 128 (one CTA) or 256 (a CTA pair).
__host__ __device__ constexpr uint32_t idesc_nvf4(int N, int M = 128) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (0u << 23) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- tensor TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar), "l"(policy) : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(map) : "memory");
}

// ---------------------------------------------------------------- CTA pairs (cta_group::2)
// A cluster of two CTAs runs one MMA of M = 256 (128 rows in each CTA's
// TMEM and shared memory) x N (each CTA holding N / 2 rows of B); the even
// CTA of the pair issues the MMAs and the scale copies for both.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// every thread of both CTAs: release this CTA's prior work to the cluster, wait for the other CTA
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_result), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
// arrive on the mbarrier at `bar` (a shared::cluster address: this CTA's or
// the other CTA's of the pair) once the MMAs issued so far complete
__device__ __forceinline__ void tc_commit2(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}
// the same arrival on the barrier at offset `bar` in both CTAs of the pair
__device__ __forceinline__ void tc_commit2_both(uint32_t bar) {
  tc_commit2(bar);
  tc_commit2(mapa_shared(bar, 1));
}
__device__ __forceinline__ void tc_cp2_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_cp2_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma2_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// Tensor load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (`bar` a shared::cluster address);
// no multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar), "l"(policy) : "memory");
}
// arrive (release, cluster scope) on an mbarrier of any CTA of the cluster
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(bar_cluster) : "memory");
}
// try_wait with acquire at cluster scope (arrivals from the other CTA)
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(bar), "r"(phase) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t phase, uint64_t deadline_ns) {
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, phase)) return true;
    if ((i & 63u) == 0 && globaltimer_ns() > deadline_ns) return false;
  }
}

// ---------------------------------------------------------------- NVFP4 conversions
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float hi, float lo) {   // lo -> low byte
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float hi, float lo) {   // lo -> low nibble
  uint32_t r;
  asm("{\n .reg .b8 b;\n cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n cvt.u32.u8 %0, b;\n}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  const uint32_t h2 = e4m3x2_to_f16x2(byte & 0xffu);
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// Scale layouts of the tensor-core operands.  The scale bytes of one MMA
// (K = 64, four 16-blocks) for 128 rows form a "unit" of 32 row slots
// l = r % 32 in four 8-row groups g = l / 8, a group being 256 bytes:
//   h * 128 + (l % 8) * 16 + (r % 128 / 32) * 4 + kb % 4,
// where h picks one of two 16-byte columns.  A tcgen05.cp .128x256b copies
// 128 rows x 32 bytes (16 groups, the two 16-byte columns 128 bytes apart)
// and fills every TMEM lane quarter with the same 32 x 8 columns when its
// source is a unit four times over (groups 4i..4i+3 = replica i).  So that
// one bulk copy moves one replica of all the units of a K-stage (K = 256),
// the units of a (row tile, stage) are interleaved by group in memory:
//   block (tile, stage) = [group g (4)][unit j (U)][256 bytes],  U units per stage,
// and the copy of unit j reads groups at j * 256 + g * U * 256 (the
// descriptor's stride).  Device memory holds each block once; for the
// .128x256b copies shared memory holds it four times in a row (kSfReplicas),
// while a .32x128b.warpx4 copy reads one 16-byte column h of a unit's four
// groups and broadcasts it to the four lane quarters itself.
constexpr int kSfReplicas = 4;
constexpr int kSfGroupBytes = 256;

// M side, 128-row tiles (pair layout): a unit covers two 64-wide K groups
// (h = which one), two units per stage; column 4h + (r % 128) / 32 of lane
// r % 32 holds the four scales of row r for the MMA of 64-group h.
// Size: rows / 128 * (K / 128) * 1024 bytes.
constexpr int kSfPairUnitsPerStage = 2;
__host__ __device__ __forceinline__ size_t sf_pair_offset(long long r, int kb, int kblocks64) {
  const long long tile = r >> 7;
  const int rr = (int)(r & 127), l = rr & 31, kg = kb >> 2, pr = kg >> 1;
  const int stage = pr >> 1, j = pr & 1, nstages = kblocks64 >> 2;
  return (((size_t)tile * nstages + stage) * 4 + (l >> 3)) * (kSfPairUnitsPerStage * kSfGroupBytes) +
         (size_t)(j * kSfGroupBytes + (kg & 1) * 128 + (l & 7) * 16 + (rr >> 5) * 4 + (kb & 3));
}
__host__ __device__ constexpr size_t sf_pair_bytes(long long rows, int K) {
  return (size_t)(rows / 128) * (K / 128) * 1024;
}

// N side, 256-row groups (rowpair layout): a unit covers one 64-wide K group
// for 256 rows (h = (r % 256) / 128), four units per stage; one copy fills
// the 8 scale columns one N = 256 MMA reads: column (r % 256) / 32 of lane
// r % 32.  Size: rows / 256 * (K / 64) * 1024 bytes.
constexpr int kSfRowpairUnitsPerStage = 4;
__host__ __device__ __forceinline__ size_t sf_rowpair_offset(long long r, int kb, int kblocks64) {
  const long long grp = r >> 8;
  const int rr = (int)(r & 255), h = rr >> 7, r128 = rr & 127, l = r128 & 31, kg = kb >> 2;
  const int stage = kg >> 2, j = kg & 3, nstages = kblocks64 >> 2;
  return (((size_t)grp * nstages + stage) * 4 + (l >> 3)) * (kSfRowpairUnitsPerStage * kSfGroupBytes) +
         (size_t)(j * kSfGroupBytes + h * 128 + (l & 7) * 16 + (r128 >> 5) * 4 + (kb & 3));
}
__host__ __device__ constexpr size_t sf_rowpair_bytes(long long rows, int K) {
  return (size_t)(rows / 256) * (K / 64) * 1024;
}

}  // namespace moe
