// Physical layout of the StagQ plane-major stream and the bit manipulations
// that read it. Shared by the host packer / host level re-read and by the
// sm_100a kernels, so the two can only agree.
//
// The StagQ paper (arXiv 2610.05977, Section 3.3) fixes the plane order --
// base first, then refinement planes in order of k, so a p_M read fetches only
// the base and planes 3..M -- and leaves the layout inside a plane open.
// This library's choice:
//
//  * every plane is row-major over the out x in matrix; a row of the base
//    takes in/4 bytes, a row of a refinement plane in/8 bytes;
//  * inside a row, weights come in 64-weight "lane chunks" (one GPU lane
//    reads one chunk of one row: 16 base bytes + 8 bytes per plane);
//  * inside a chunk, weight t = 16 i + 4 s + j  (word i = 0..3, slot s = 0..3,
//    byte j = 0..3). Its base digit q sits in base word i, bits
//    [8j+2s+1 : 8j+2s]. A mask 0x03030303 << 2s of word i therefore yields the
//    four weights (i, s, 0..3) as bytes holding q * 4^s, ready for an integer
//    dot-product instruction against four 16-bit activations.
//  * planes 3 and 4 are placed so that a handful of bit operations fuse
//    (q, b3, b4) of a word pair into 4-bit "nibble composites"
//    4q + 2 b3 + b4 = u_4 (Eq. 8 at M = 4; with b4 absent it is 2 u_3), one
//    nibble per weight, grouped exactly like the base slots;
//  * planes 5 and 6 keep bit (8j + 4(i&1) + s) of chunk word i>>1.
//
// None of this changes what is stored (the digits of Eq. 8), only where.
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define STAGQ_HD __host__ __device__ __forceinline__
#else
#define STAGQ_HD inline
#endif

namespace stagq {

constexpr int kChunk = 64;          // weights per lane chunk
constexpr int kBaseChunkBytes = 16; // base bytes per chunk
constexpr int kPlaneChunkBytes = 8; // bytes per chunk of one refinement plane

STAGQ_HD uint32_t rotl32(uint32_t v, int n) { return (v << n) | (v >> (32 - n)); }

// (a & m) | (b & ~m): a bitwise select, one LOP3.
STAGQ_HD uint32_t bsel(uint32_t a, uint32_t b, uint32_t m) { return (a & m) | (b & ~m); }

// Position of weight t = 16i + 4s + j inside its chunk.
struct ChunkPos {
  int i, s, j;
};
STAGQ_HD ChunkPos chunk_pos(int t) { return ChunkPos{t >> 4, (t >> 2) & 3, t & 3}; }

// Base digit: word i, bit offset 8j + 2s.
STAGQ_HD int base_bit(const ChunkPos& p) { return 8 * p.j + 2 * p.s; }

// Plane 3 / plane 4 bit offset inside chunk word (i >> 1). Derived from the
// composite construction in nibble_words(): nibble n = 2j + (s >> 1) of the
// E (odd s) or O (even s) word of base word i.
STAGQ_HD int plane3_bit(const ChunkPos& p) {
  const int n = 2 * p.j + (p.s >> 1);
  if ((p.i & 1) == 0) return (p.s & 1) ? 4 * n + 1 : (4 * n - 1) & 31;
  return (p.s & 1) ? 4 * n + 2 : 4 * n;
}
STAGQ_HD int plane4_bit(const ChunkPos& p) {
  const int n = 2 * p.j + (p.s >> 1);
  if ((p.i & 1) == 0) return (p.s & 1) ? 4 * n : (4 * n - 2) & 31;
  return (p.s & 1) ? 4 * n + 1 : (4 * n - 1) & 31;
}
// Planes 5 and 6.
STAGQ_HD int plane56_bit(const ChunkPos& p) { return 8 * p.j + 4 * (p.i & 1) + p.s; }

// Fuse base words B0 (chunk word 2w) and B1 (word 2w+1) with plane-3 / plane-4
// words P3, P4 (chunk word w; P4 = 0 for a p3 read) into four nibble-composite
// words. Nibble n = 2j + h of
//   E0 : weight (2w,   s = 2h+1, j)     O0 : weight (2w,   s = 2h, j)
//   E1 : weight (2w+1, s = 2h+1, j)     O1 : weight (2w+1, s = 2h, j)
// holds 4q + 2 b3 + b4.
STAGQ_HD void nibble_words(uint32_t B0, uint32_t B1, uint32_t P3, uint32_t P4, uint32_t& E0,
                           uint32_t& O0, uint32_t& E1, uint32_t& O1) {
  const uint32_t T0 = bsel(P3, P4, 0x22222222u);
  E0 = bsel(B0, T0, 0xCCCCCCCCu);
  const uint32_t T1 = bsel(P3, P4, 0x88888888u);
  O0 = rotl32(bsel(B0, T1, 0x33333333u), 2);
  const uint32_t T2 = bsel(P3, P4, 0x44444444u);
  E1 = bsel(B1, T2 >> 1, 0xCCCCCCCCu);
  const uint32_t T3 = bsel(P3, P4, 0x11111111u);
  O1 = bsel(rotl32(B1, 2), rotl32(T3, 1), 0xCCCCCCCCu);
}

// u_M (Eq. 8) of weight t of a chunk, read through the same composites as the
// GEMV kernels. base: 4 words; p[k-3]: the 2 chunk words of plane k.
STAGQ_HD int chunk_level(const uint32_t* base, const uint32_t (*p)[2], int M, int t) {
  const ChunkPos c = chunk_pos(t);
  if (M == 2) return (base[c.i] >> base_bit(c)) & 3;
  const int w = c.i >> 1;
  uint32_t E0, O0, E1, O1;
  nibble_words(base[2 * w], base[2 * w + 1], p[0][w], M >= 4 ? p[1][w] : 0u, E0, O0, E1, O1);
  const uint32_t C = (c.i & 1) ? ((c.s & 1) ? E1 : O1) : ((c.s & 1) ? E0 : O0);
  const int n = 2 * c.j + (c.s >> 1);
  const int v = (C >> (4 * n)) & 15;  // 4q + 2b3 + b4 (b4 = 0 when M = 3)
  if (M == 3) return v >> 1;
  if (M == 4) return v;
  const int b5 = (p[2][w] >> plane56_bit(c)) & 1;
  if (M == 5) return 2 * v + b5;
  const int b6 = (p[3][w] >> plane56_bit(c)) & 1;
  return 4 * v + 2 * b5 + b6;
}

// Byte offsets of a chunk inside its plane.
STAGQ_HD int64_t base_chunk_offset(int64_t row, int64_t in, int64_t chunk) {
  return row * (in / 4) + chunk * kBaseChunkBytes;
}
STAGQ_HD int64_t plane_chunk_offset(int64_t row, int64_t in, int64_t chunk) {
  return row * (in / 8) + chunk * kPlaneChunkBytes;
}
STAGQ_HD int64_t plane_region_offset(int64_t out, int64_t in, int k /* 3.. */) {
  return out * in / 4 + (int64_t)(k - 3) * (out * in / 8);
}

}  // namespace stagq
