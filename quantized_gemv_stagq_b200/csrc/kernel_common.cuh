// Device helpers shared by the GEMV kernels (gemv.cu: any number of
// activation vectors; gemv1.cu: one vector): PTX wrappers for mbarriers, bulk
// copies and programmatic dependent launch, the integer dot products of the
// code bytes / nibble composites (layout.cuh), and the shared-memory order of
// the fixed-point activations.
#pragma once
#include <cuda_fp16.h>

#include <cstdint>

#include "device_matrix.hpp"
#include "layout.cuh"

namespace stagq {
namespace kernels {

constexpr unsigned kFull = 0xFFFFFFFFu;

// x~ in shared memory: see xq_piece_index / xq_slot_of_column (device_matrix.hpp).
__device__ __forceinline__ int xq_piece(int c, int p) { return xq_piece_index(c, p); }
__device__ __forceinline__ int xq_elem(int col) { return xq_slot_of_column(col); }


// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait until the phase of `bar` with the given parity has completed, for at
// most `limit_ns`; false on expiry.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0 && global_timer() - t0 > limit_ns) return false;
  }
}
// mbar_wait that also gives up as soon as *stop is nonzero (another thread of
// the CTA gave up).
__device__ __forceinline__ bool mbar_wait_unless(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                                 const volatile uint32_t* stop) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*stop) return false;
    if ((i & 15u) == 0 && global_timer() - t0 > limit_ns) return false;
  }
}
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src and bytes are multiples of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ int dp2a_lo(uint32_t xpair, uint32_t codes, int acc) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(xpair), "r"(codes), "r"(acc));
  return d;
}
__device__ __forceinline__ int dp2a_hi(uint32_t xpair, uint32_t codes, int acc) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(xpair), "r"(codes), "r"(acc));
  return d;
}

// Four weights (i, s, j = 0..3) whose code bytes are `m`, against their
// fixed-point activations X[8i+2s] (j = 0, 1) and X[8i+2s+1] (j = 2, 3).
__device__ __forceinline__ int dot4(const uint32_t (&X)[32], int i, int s, uint32_t m, int acc) {
  acc = dp2a_lo(X[8 * i + 2 * s], m, acc);
  return dp2a_hi(X[8 * i + 2 * s + 1], m, acc);
}

// Sums of v_t X_t over the G groups of one 64-weight chunk, v = u_M (v = 2 u_3
// at M = 3). G = 1, 2 or 4: a group is 64 / G weights, i.e. 4 / G consecutive
// chunk words (word i holds weights 16 i .. 16 i + 15). B: the 4 base words;
// P[k]: the 2 chunk words of plane k+3. Exact in int32.
template <int M, int G>
__device__ __forceinline__ void chunk_dot_g(const uint32_t (&X)[32], const uint32_t (&B)[4], const uint2* P,
                                            int (&tot)[G]) {
  static_assert(G == 1 || G == 2 || G == 4, "groups per chunk");
  constexpr int WPG = 4 / G;  // chunk words per group
  if constexpr (M == 2) {
    int a[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) a[g][0] = a[g][1] = a[g][2] = a[g][3] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int g = i / WPG;
      a[g][0] = dot4(X, i, 0, B[i] & 0x03030303u, a[g][0]);
      a[g][1] = dot4(X, i, 1, B[i] & 0x0C0C0C0Cu, a[g][1]);
      a[g][2] = dot4(X, i, 2, B[i] & 0x30303030u, a[g][2]);
      a[g][3] = dot4(X, i, 3, B[i] & 0xC0C0C0C0u, a[g][3]);
    }
    // slot s carries q * 4^s, so every product in a[g][s] is a multiple of 4^s
#pragma unroll
    for (int g = 0; g < G; ++g) tot[g] = a[g][0] + (a[g][1] >> 2) + (a[g][2] >> 4) + (a[g][3] >> 6);
  } else {
    int lo[G], hi[G];
#pragma unroll
    for (int g = 0; g < G; ++g) lo[g] = hi[g] = 0;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint32_t p3 = w ? P[0].y : P[0].x;
      uint32_t p4 = 0u;
      if constexpr (M >= 4) p4 = w ? P[1].y : P[1].x;
      uint32_t E0, O0, E1, O1;
      nibble_words(B[2 * w], B[2 * w + 1], p3, p4, E0, O0, E1, O1);
      const int i0 = 2 * w, i1 = 2 * w + 1, g0 = i0 / WPG, g1 = i1 / WPG;
      lo[g0] = dot4(X, i0, 1, E0 & 0x0F0F0F0Fu, lo[g0]);
      hi[g0] = dot4(X, i0, 3, E0 & 0xF0F0F0F0u, hi[g0]);
      lo[g0] = dot4(X, i0, 0, O0 & 0x0F0F0F0Fu, lo[g0]);
      hi[g0] = dot4(X, i0, 2, O0 & 0xF0F0F0F0u, hi[g0]);
      lo[g1] = dot4(X, i1, 1, E1 & 0x0F0F0F0Fu, lo[g1]);
      hi[g1] = dot4(X, i1, 3, E1 & 0xF0F0F0F0u, hi[g1]);
      lo[g1] = dot4(X, i1, 0, O1 & 0x0F0F0F0Fu, lo[g1]);
      hi[g1] = dot4(X, i1, 2, O1 & 0xF0F0F0F0u, hi[g1]);
    }
    int nib[G];
#pragma unroll
    for (int g = 0; g < G; ++g) nib[g] = lo[g] + (hi[g] >> 4);  // high-nibble products are multiples of 16
    if constexpr (M <= 4) {
#pragma unroll
      for (int g = 0; g < G; ++g) tot[g] = nib[g];
    } else {
      int a5[G], a6[G];
#pragma unroll
      for (int g = 0; g < G; ++g) a5[g] = a6[g] = 0;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const uint32_t p5 = w ? P[2].y : P[2].x;
        uint32_t p6 = 0u;
        if constexpr (M >= 6) p6 = w ? P[3].y : P[3].x;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int g = (2 * w + h) / WPG;
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const int sh = 4 * h + s;
            a5[g] = dot4(X, 2 * w + h, s, (p5 >> sh) & 0x01010101u, a5[g]);
            if constexpr (M >= 6) a6[g] = dot4(X, 2 * w + h, s, (p6 >> sh) & 0x01010101u, a6[g]);
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) tot[g] = M == 5 ? 2 * nib[g] + a5[g] : 4 * nib[g] + 2 * a5[g] + a6[g];
    }
  }
}

// Decoding and dot product of chunk_dot_g split in two, for launches with
// several activation vectors (M <= 4): chunk_codes turns the chunk's base /
// plane words into its 16 masked code words once, and chunk_dot_codes dots
// them with one vector's x~ (the same dp2a sequence as chunk_dot_g, so the
// integer result is identical).
//   M = 2:     cw[4 i + s] = base word i & (0x03030303 << 2 s)  (bytes q 4^s)
//   M = 3, 4:  per word pair w, the low / high nibbles of the composites
//              E0, O0, E1, O1 (layout.cuh: nibble 4q + 2 b3 + b4)
template <int M>
__device__ __forceinline__ void chunk_codes(const uint32_t (&B)[4], const uint2* P, uint32_t (&cw)[16]) {
  static_assert(M >= 2 && M <= 4, "codes of up to two planes");
  if constexpr (M == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int s = 0; s < 4; ++s) cw[4 * i + s] = B[i] & (0x03030303u << (2 * s));
  } else {
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint32_t p3 = w ? P[0].y : P[0].x;
      uint32_t p4 = 0u;
      if constexpr (M >= 4) p4 = w ? P[1].y : P[1].x;
      uint32_t E0, O0, E1, O1;
      nibble_words(B[2 * w], B[2 * w + 1], p3, p4, E0, O0, E1, O1);
      cw[8 * w + 0] = E0 & 0x0F0F0F0Fu; cw[8 * w + 1] = E0 & 0xF0F0F0F0u;
      cw[8 * w + 2] = O0 & 0x0F0F0F0Fu; cw[8 * w + 3] = O0 & 0xF0F0F0F0u;
      cw[8 * w + 4] = E1 & 0x0F0F0F0Fu; cw[8 * w + 5] = E1 & 0xF0F0F0F0u;
      cw[8 * w + 6] = O1 & 0x0F0F0F0Fu; cw[8 * w + 7] = O1 & 0xF0F0F0F0u;
    }
  }
}
template <int M, int G>
__device__ __forceinline__ void chunk_dot_codes(const uint32_t (&X)[32], const uint32_t (&cw)[16], int (&tot)[G]) {
  constexpr int WPG = 4 / G;  // chunk words per group
  if constexpr (M == 2) {
    int a[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) a[g][0] = a[g][1] = a[g][2] = a[g][3] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int g = i / WPG;
#pragma unroll
      for (int s = 0; s < 4; ++s) a[g][s] = dot4(X, i, s, cw[4 * i + s], a[g][s]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) tot[g] = a[g][0] + (a[g][1] >> 2) + (a[g][2] >> 4) + (a[g][3] >> 6);
  } else {
    int lo[G], hi[G];
#pragma unroll
    for (int g = 0; g < G; ++g) lo[g] = hi[g] = 0;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int i0 = 2 * w, i1 = 2 * w + 1, g0 = i0 / WPG, g1 = i1 / WPG;
      lo[g0] = dot4(X, i0, 1, cw[8 * w + 0], lo[g0]);
      hi[g0] = dot4(X, i0, 3, cw[8 * w + 1], hi[g0]);
      lo[g0] = dot4(X, i0, 0, cw[8 * w + 2], lo[g0]);
      hi[g0] = dot4(X, i0, 2, cw[8 * w + 3], hi[g0]);
      lo[g1] = dot4(X, i1, 1, cw[8 * w + 4], lo[g1]);
      hi[g1] = dot4(X, i1, 3, cw[8 * w + 5], hi[g1]);
      lo[g1] = dot4(X, i1, 0, cw[8 * w + 6], lo[g1]);
      hi[g1] = dot4(X, i1, 2, cw[8 * w + 7], hi[g1]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) tot[g] = lo[g] + (hi[g] >> 4);
  }
}

// The whole chunk as one group (groups of 64 weights or more).
template <int M>
__device__ __forceinline__ int chunk_dot(const uint32_t (&X)[32], const uint32_t (&B)[4], const uint2* P) {
  int t[1];
  chunk_dot_g<M, 1>(X, B, P, t);
  return t[0];
}

// One task of the conversion of x to 16-bit fixed point: 16 values of one
// 64-element chunk (the chunk's 4 tasks sit in adjacent lanes, every lane of
// the warp calls this). raw: the 16 fp16 values; SC: times the run-time
// inverse activation scale s (16 fp32 values; the quantiser saw W diag(a), so
// channel c of x is multiplied by 1/a_c, Appendix E), rounded to fp32.
// Scale 2^e with max|x| 2^e in [2^14, 2^15) over the chunk, so the largest
// entries of fp16 x convert exactly; rounding to nearest even goes through the
// 1.5 * 2^23 shifter (the low 16 bits of the sum are the two's-complement
// integer). With SC the largest scaled fp32 product can round up to 2^15, so
// the result is clamped to 2^15 - 1.
// Out: Q (8 pairs of int16), xs = 2^-e, sum16 = the task's sum of x~, sumq =
// the chunk's.
template <bool SC>
__device__ __forceinline__ void convert_x_task(const uint4 (&raw)[2], const float4 (&s)[4], uint32_t (&Q)[8], float& xs,
                                               int& sum16, int& sumq) {
  constexpr float kShift = 12582912.0f;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(raw);
  float2 f[8];
  float mx = 0.f;
  if constexpr (SC) {
    const float* sv = reinterpret_cast<const float*>(s);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      f[k] = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      f[k].x *= sv[2 * k];
      f[k].y *= sv[2 * k + 1];
      mx = fmaxf(mx, fmaxf(fabsf(f[k].x), fabsf(f[k].y)));
    }
  } else {
    __half2 m2 = __habs2(*reinterpret_cast<const __half2*>(&w[0]));
#pragma unroll
    for (int k = 1; k < 8; ++k) m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __half2*>(&w[k])));
    mx = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
    for (int k = 0; k < 8; ++k) f[k] = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
  }
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
  int e = mx > 0.f ? 14 - ((int)((__float_as_uint(mx) >> 23) & 0xFF) - 127) : 0;
  if constexpr (SC) e = max(-126, min(126, e));  // 2^e and 2^-e stay normal floats
  const float sc = __int_as_float((127 + e) << 23);
  sumq = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float vx = fmaf(f[k].x, sc, kShift), vy = fmaf(f[k].y, sc, kShift);
    if constexpr (SC) {  // |x s| 2^e < 2^15 before rounding; keep the rounded value inside int16
      vx = fminf(fmaxf(vx, kShift - 32768.f), kShift + 32767.f);
      vy = fminf(fmaxf(vy, kShift - 32768.f), kShift + 32767.f);
    }
    Q[k] = __byte_perm(__float_as_uint(vx), __float_as_uint(vy), 0x5410);
    sumq = dp2a_lo(Q[k], 0x0101u, sumq);
  }
  sum16 = sumq;
  sumq += __shfl_xor_sync(kFull, sumq, 1);
  sumq += __shfl_xor_sync(kFull, sumq, 2);
  xs = __int_as_float((127 - e) << 23);
}

// Groups per 64-weight chunk for a group size of 2^group_shift (>= 16).
__host__ __device__ inline int groups_per_chunk(int group_shift) {
  return group_shift >= 6 ? 1 : 1 << (6 - group_shift);
}

// G pair bytes of one row, starting at p (aligned to G bytes), as an integer
// whose byte g is the pair of the chunk's group g.
template <int G>
__device__ __forceinline__ uint32_t load_pairs(const uint8_t* p) {
  if constexpr (G == 1) return *p;
  else if constexpr (G == 2) return *reinterpret_cast<const uint16_t*>(p);
  else return *reinterpret_cast<const uint32_t*>(p);
}

}  // namespace kernels
}  // namespace stagq
