// Library-owned data layouts (device side).
//
// "Fragment layout" of an NVFP4 matrix for the register-dequant GEMV path.
// A matrix is cut into tiles of 16 rows; a tile is a sequence of 64-element K
// chunks; a chunk is 576 bytes:
//   bytes [0, 512)   32 lanes x 16 B of e2m1 codes.  Lane L = 4*g + c holds,
//                    for the four 16-wide K steps ks of the chunk, the four
//                    bytes that make its m16n8k16 A fragment:
//                      byte 4ks+0: row A(g),  K = 16ks + 2c, +1   (a0:a1)
//                      byte 4ks+1: row B(g),  same K               (a2:a3)
//                      byte 4ks+2: row A(g),  K = 16ks + 8 + 2c, +1 (a4:a5)
//                      byte 4ks+3: row B(g),  same K               (a6:a7)
//                    (low nibble = lower K, as in the canonical layout; the
//                    codes of a block whose scale is negative have their
//                    signs flipped, which is exact)
//   bytes [512, 576) 8 groups g x 8 B of e4m3 scales with the sign bit
//                    cleared: bytes 0..3 = scales of row A(g) for steps
//                    ks = 0..3, bytes 4..7 = row B(g).
// Tile rows: gate/up tile t pairs gate rows f = 8t+g (A) with up rows 8t+g
// (B), so one MMA accumulator holds g and u of the same f; down tile t holds
// rows 16t+g (A) and 16t+8+g (B).
//
// "B-fragment layout" of an fp16 activation row of length K: per 64-element
// chunk, 4 lanes c x 4 steps ks x {b0, b1} x 2 halves:
//   half offset = 64*chunk + 16*c + 4*ks + 2*slot + half,
//   for K index 64*chunk + 16*ks + r:  slot = r / 8, c = (r % 8) / 2, half = r % 2.
#pragma once
#include <cstdint>

namespace moe {

constexpr int kChunkK = 64;
constexpr int kChunkBytes = 576;
constexpr int kChunkCodeBytes = 512;

__host__ __device__ __forceinline__ int bfrag_offset(int kidx) {
  const int chunk = kidx >> 6, kk = kidx & 63;
  const int ks = kk >> 4, r = kk & 15;
  const int slot = r >> 3, c = (r & 7) >> 1, half = r & 1;
  return (chunk << 6) + (c << 4) + (ks << 2) + (slot << 1) + half;
}

}  // namespace moe
