// sm_100a kernels of the StagQ batch-one GEMV y = W_hat^(M) x.
//
// What is computed (StagQ paper, arXiv 2610.05977): for every row i,
//   y_i = sum_groups [ s_M(g) * sum_{j in g} u_M,j x_j + lo_M(g) * sum_{j in g} x_j ]
//         + sum_{held-out (i,c)} x_c (v_ic - lo_M(g(i,c)))
// -- the affine map of Eq. (10) applied once per group, with u_M from Eq. (8),
// and the side record of Eq. (4) fused into the epilogue (held-out digits are
// zero, so the main stream decoded lo_M there and the correction is v - lo_M).
//
// How (design for B200; batch-one GEMV is bound by HBM, so no tensor cores):
//  * one CTA per SM owns a contiguous, balanced range of rows; its warps are
//    KW "K slices" (2048 weights of K each: 32 lanes x one 64-weight chunk)
//    times RG row groups, and each warp walks its rows UP at a time;
//  * the CTA's pair bytes and side-record entries are staged in shared memory
//    once, up front; every lane streams its own chunk bytes -- 16 base bytes
//    + 8 bytes per read plane (a p_M read never touches deeper planes) -- with
//    cp.async into its own shared-memory ring, several batches ahead, so the
//    loop has no barrier: cp.async.wait_group is the only ordering;
//  * x is converted once per CTA to 16-bit fixed point with a power-of-two
//    scale per 64-element chunk (|error| <= 2^-16 max|x_chunk|); each lane
//    keeps its chunk's 64 activations in registers for every row;
//  * a lane turns its chunk into code bytes / nibble composites (layout.cuh)
//    and feeds them to dp2a integer dot products (exact in int32); the group
//    affine is applied once per chunk in fp32 and a transposed shuffle reduces
//    the batch's rows to one partial per (row, K slice) in shared memory;
//  * a final pass per row adds the held-out entries, x_c (v - lo_M), and the
//    KW partials in a fixed order and stores y -- deterministic, no atomics,
//    no workspace, no second launch (the K split of Appendix G's atomic-add
//    kernel becomes this reduction).
#include <cuda_fp16.h>

#include <cstdint>
#include <mutex>

#include "device_matrix.hpp"
#include "layout.cuh"

namespace stagq {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
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

// sum over one 64-weight chunk of v_t X_t with v = u_M (v = 2 u_3 at M = 3).
// B: the 4 base words; P[k]: the 2 chunk words of plane k+3. Exact in int32.
template <int M>
__device__ __forceinline__ int chunk_dot(const uint32_t (&X)[32], const uint32_t (&B)[4], const uint2* P) {
  if constexpr (M == 2) {
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a0 = dot4(X, i, 0, B[i] & 0x03030303u, a0);
      a1 = dot4(X, i, 1, B[i] & 0x0C0C0C0Cu, a1);
      a2 = dot4(X, i, 2, B[i] & 0x30303030u, a2);
      a3 = dot4(X, i, 3, B[i] & 0xC0C0C0C0u, a3);
    }
    // slot s carries q * 4^s, so every product in a_s is a multiple of 4^s
    return a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
  } else {
    int lo = 0, hi = 0;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint32_t p3 = w ? P[0].y : P[0].x;
      uint32_t p4 = 0u;
      if constexpr (M >= 4) p4 = w ? P[1].y : P[1].x;
      uint32_t E0, O0, E1, O1;
      nibble_words(B[2 * w], B[2 * w + 1], p3, p4, E0, O0, E1, O1);
      const int i0 = 2 * w, i1 = 2 * w + 1;
      lo = dot4(X, i0, 1, E0 & 0x0F0F0F0Fu, lo);
      hi = dot4(X, i0, 3, E0 & 0xF0F0F0F0u, hi);
      lo = dot4(X, i0, 0, O0 & 0x0F0F0F0Fu, lo);
      hi = dot4(X, i0, 2, O0 & 0xF0F0F0F0u, hi);
      lo = dot4(X, i1, 1, E1 & 0x0F0F0F0Fu, lo);
      hi = dot4(X, i1, 3, E1 & 0xF0F0F0F0u, hi);
      lo = dot4(X, i1, 0, O1 & 0x0F0F0F0Fu, lo);
      hi = dot4(X, i1, 2, O1 & 0xF0F0F0F0u, hi);
    }
    const int nib = lo + (hi >> 4);  // high-nibble products are multiples of 16
    if constexpr (M <= 4) {
      return nib;
    } else {
      int a5 = 0, a6 = 0;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const uint32_t p5 = w ? P[2].y : P[2].x;
        uint32_t p6 = 0u;
        if constexpr (M >= 6) p6 = w ? P[3].y : P[3].x;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const int sh = 4 * h + s;
            a5 = dot4(X, 2 * w + h, s, (p5 >> sh) & 0x01010101u, a5);
            if constexpr (M >= 6) a6 = dot4(X, 2 * w + h, s, (p6 >> sh) & 0x01010101u, a6);
          }
        }
      }
      if constexpr (M == 5) return 2 * nib + a5;
      else return 4 * nib + 2 * a5 + a6;
    }
  }
}

// Sum v[0..UP-1] over the 32 lanes; afterwards lanes [u*32/UP, (u+1)*32/UP)
// hold the total of v[u]. UP - 1 + log2(32) - log2(UP) shuffles.
template <int UP>
__device__ __forceinline__ float transposed_reduce(float (&v)[UP], int lane) {
  if constexpr (UP == 1) {
    float s = v[0];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
    return s;
  } else if constexpr (UP == 2) {
    const bool hi = lane & 16;
    float s = (hi ? v[1] : v[0]) + __shfl_xor_sync(kFull, hi ? v[0] : v[1], 16);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
    return s;
  } else {  // UP == 4
    const bool h16 = lane & 16, h8 = lane & 8;
    const float k0 = h16 ? v[2] : v[0], k1 = h16 ? v[3] : v[1];
    const float s0 = k0 + __shfl_xor_sync(kFull, h16 ? v[0] : v[2], 16);
    const float s1 = k1 + __shfl_xor_sync(kFull, h16 ? v[1] : v[3], 16);
    float s = (h8 ? s1 : s0) + __shfl_xor_sync(kFull, h8 ? s0 : s1, 8);
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
    return s;
  }
}

struct GemvKernelArgs {
  DeviceMatrix m;
  GemvPlan plan;
  const float2* table;  // (lo_M, s_M c_M) of this precision
  const __half* x;
  void* y;
  int y_f32;
};

// Copies of 16 / 8 bytes that read `n` of them (0 or all) and zero-fill
// the rest, so a predicate needs no branch. `src` must be a valid address.
__device__ __forceinline__ void cp_async16z(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async8z(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Shared-memory carve-up, identical on host (plan) and device.
struct SmemLayout {
  uint32_t xq, xh, xscale, xsum, tab, rp, pairs, ents, partial, ring;
  uint32_t warp_ring;  // bytes of one warp's ring
  uint32_t total;
};

__host__ __device__ inline uint32_t align_up_u32(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout smem_layout(const GemvPlan& p, int in, int M) {
  SmemLayout L;
  const uint32_t nchunk = in / kChunk, R = p.max_rows_per_cta, W = p.KW * p.RG;
  uint32_t o = 0;
  L.xq = o; o += 2 * in;
  L.xh = o; o += 2 * in;
  L.xscale = o; o += 4 * nchunk;
  L.xsum = o; o += 4 * nchunk;
  o = align_up_u32(o, 16);
  L.tab = o; o += 256 * 8;
  L.rp = o; o += 4 * (R + 1);
  o = align_up_u32(o, 16);
  L.pairs = o; o += R * p.pair_stride;
  o = align_up_u32(o, 16);
  L.ents = o; o += 4 * (p.ent_cap + 4);
  L.partial = o; o += 4 * p.KW * R;
  o = align_up_u32(o, 128);
  L.ring = o;
  L.warp_ring = (uint32_t)(p.depth + 1) * p.up * 32u * (16 + 8 * (M - 2));
  o += W * L.warp_ring;
  L.total = o;
  return L;
}

template <int M, int UP, int D>
__global__ void __launch_bounds__(kMaxConsumerWarps * 32, 1) gemv_kernel(const GemvKernelArgs a) {
  constexpr int NS = D + 1;                         // ring slots: D in flight + the one read
  constexpr uint32_t RB = 32u * (16 + 8 * (M - 2));  // one row: base | planes, over 32 lanes
  constexpr uint32_t SLOT = UP * RB;
  extern __shared__ __align__(128) uint8_t smem[];
  const GemvPlan& P = a.plan;
  const int in = a.m.in;
  const int nchunk = in / kChunk;
  const SmemLayout L = smem_layout(P, in, M);
  int16_t* xq = reinterpret_cast<int16_t*>(smem + L.xq);
  __half* xh = reinterpret_cast<__half*>(smem + L.xh);
  float* xscale = reinterpret_cast<float*>(smem + L.xscale);
  float* xsum = reinterpret_cast<float*>(smem + L.xsum);
  float2* tab = reinterpret_cast<float2*>(smem + L.tab);
  int* rp = reinterpret_cast<int*>(smem + L.rp);                // [rows + 1] row_ptr
  uint8_t* pairs = smem + L.pairs;                              // [rows][pair_stride]
  uint32_t* ents = reinterpret_cast<uint32_t*>(smem + L.ents);  // staged side record
  float* partial = reinterpret_cast<float*>(smem + L.partial);  // [rows][KW]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthreads = blockDim.x;
  const int KW = P.KW, RG = P.RG, ps = P.pair_stride;
  const int kw = warp % KW, rg = warp / KW;
  const int c = kw * 32 + lane;  // this lane's 64-weight chunk
  const bool active = c < nchunk;
  const int gidx = (c * kChunk) >> P.group_shift;
  const int r0 = (int)((int64_t)blockIdx.x * a.m.out / gridDim.x);
  const int rows = (int)((int64_t)(blockIdx.x + 1) * a.m.out / gridDim.x) - r0;
  const int rows_rg = rows > rg ? (rows - rg + RG - 1) / RG : 0;  // rows of this row group
  const int nb = (rows_rg + UP - 1) / UP;                         // batches
  const uint32_t ring = smem_addr(smem + L.ring) + (uint32_t)warp * L.warp_ring;  // shared address
  const uint8_t* const ring_g = smem + L.ring + (size_t)warp * L.warp_ring;       // same, generic

  // Issue state: the next row (index mi within the row group) to prefetch.
  const int64_t stride_b = (int64_t)RG * (in / 4), stride_p = (int64_t)RG * (in / 8);
  const uint8_t* ib = a.m.base + (int64_t)(r0 + rg) * (in / 4) + c * kBaseChunkBytes;
  const uint8_t* ip[M > 2 ? M - 2 : 1];
#pragma unroll
  for (int k = 0; k < M - 2; ++k) ip[k] = a.m.plane[k] + (int64_t)(r0 + rg) * (in / 8) + c * kPlaneChunkBytes;
  const uint8_t* const safe = a.m.base;  // a valid address for zero-byte copies
  int left = active ? rows_rg : 0;        // rows still to prefetch
  uint32_t slot_i = 0;

#define STAGQ_ISSUE_BATCH()                                                                    \
  {                                                                                            \
    uint32_t rec = ring + slot_i * SLOT + lane * 16;                                           \
    _Pragma("unroll") for (int u = 0; u < UP; ++u) {                                           \
      const bool ok = u < left;                                                                \
      cp_async16z(rec, ok ? ib : safe, ok ? 16u : 0u);                                         \
      _Pragma("unroll") for (int k = 0; k < M - 2; ++k)                                        \
        cp_async8z(rec - lane * 8 + 512 + k * 256, ok ? ip[k] : safe, ok ? 8u : 0u);           \
      ib += stride_b;                                                                          \
      _Pragma("unroll") for (int k = 0; k < M - 2; ++k) ip[k] += stride_p;                     \
      rec += RB;                                                                               \
    }                                                                                          \
    left -= UP;                                                                                \
    slot_i = slot_i + 1 == NS ? 0 : slot_i + 1;                                                \
    cp_async_commit();                                                                         \
  }

  // Copy order (cp.async groups): this CTA's pair bytes, the weights of
  // batches 0..D-1, then its side record -- so batch b can start as soon as
  // the pair bytes and its own weights have landed.
  {
    const uint32_t pdst = smem_addr(pairs);
    const uint8_t* psrc = a.m.pair + (int64_t)r0 * ps;
    for (int i = tid * 16; i < rows * ps; i += nthreads * 16) cp_async16z(pdst + i, psrc + i, 16u);
    cp_async_commit();
  }
#pragma unroll
  for (int b = 0; b < D; ++b) STAGQ_ISSUE_BATCH();
  grid_launch_dependents();
  if (tid < 256) tab[tid] = a.table[tid];
  for (int i = tid; i <= rows; i += nthreads) rp[i] = __ldg(a.m.row_ptr + r0 + i);
  const int e_begin = __ldg(a.m.row_ptr + r0), e_end = __ldg(a.m.row_ptr + r0 + rows);
  const int e_base = e_begin & ~3;  // staged from a 16-byte boundary
  const bool staged = (e_end - e_base) <= P.ent_cap;
  {
    if (staged) {
      const uint32_t edst = smem_addr(ents);
      const uint32_t* esrc = a.m.entries + e_base;
      const int n16 = (e_end - e_base + 3) >> 2;  // 16-byte chunks; the entries array is padded
      for (int i = tid; i < n16; i += nthreads) cp_async16z(edst + 16 * i, esrc + 4 * i, 16u);
    }
    cp_async_commit();
  }
  grid_dependency_wait();  // x may come from the previous kernel
  {
    // x -> 16-bit fixed point; a task is 8 values, 8 tasks form a 64-value chunk.
    const int n8 = in / 8;
    for (int i0 = warp * 32; i0 < n8; i0 += nthreads) {
      const int i = i0 + lane;
      const bool v = i < n8;
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (v) raw = __ldg(reinterpret_cast<const uint4*>(a.x) + i);
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
      float f[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 t = __half22float2(h2[k]);
        f[2 * k] = t.x;
        f[2 * k + 1] = t.y;
      }
      float mx = 0.f, sm = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        mx = fmaxf(mx, fabsf(f[k]));
        sm += f[k];
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
        sm += __shfl_xor_sync(kFull, sm, off);
      }
      // e with max|x| 2^e in [2^14, 2^15): the largest entries convert exactly
      const int e = mx > 0.f ? 14 - (((__float_as_int(mx) >> 23) & 0xFF) - 127) : 0;
      const float sc = __int_as_float((127 + e) << 23);
      uint32_t packed[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int lo16 = __float2int_rn(f[2 * k] * sc);
        const int hi16 = __float2int_rn(f[2 * k + 1] * sc);
        packed[k] = (uint32_t)(lo16 & 0xFFFF) | ((uint32_t)hi16 << 16);
      }
      if (v) {
        reinterpret_cast<uint4*>(xh)[i] = raw;
        reinterpret_cast<uint4*>(xq)[i] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        if ((i & 7) == 0) {
          xscale[i >> 3] = __int_as_float((127 - e) << 23);
          xsum[i >> 3] = sm;
        }
      }
    }
  }
  // Pair bytes are group 0: with D + 1 newer groups allowed pending it has landed.
  cp_async_wait_group<D + 1>();
  __syncthreads();

  uint32_t X[32];
  float xs, xsm;
  {
    const uint4* src = reinterpret_cast<const uint4*>(xq + (active ? c : 0) * kChunk);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 t = src[k];
      X[4 * k] = t.x;
      X[4 * k + 1] = t.y;
      X[4 * k + 2] = t.z;
      X[4 * k + 3] = t.w;
    }
    xs = active ? xscale[c] : 0.f;
    xsm = active ? xsum[c] : 0.f;
  }

  uint32_t slot_c = 0;
  const uint8_t* pr = pairs + rg * ps + gidx;  // pair byte of the row being consumed
  const int pr_step = RG * ps;
  float* pw_out = partial + rg * KW + kw;
  for (int b = 0; b < nb; ++b) {
    // Groups so far: pairs, batches 0..D-1, side record, then one refill per
    // iteration. Batch b < D is group b + 1, batch b >= D group b + 2.
    if (b < D) cp_async_wait_group<D>();
    else cp_async_wait_group<D - 1>();
    const uint8_t* rec = ring_g + slot_c * SLOT + lane * 16;
    const int valid = rows_rg - UP * b;  // rows of this batch that exist
    float v[UP];
#pragma unroll
    for (int u = 0; u < UP; ++u) {
      const uint4 b4 = *reinterpret_cast<const uint4*>(rec + u * RB);
      const uint32_t B[4] = {b4.x, b4.y, b4.z, b4.w};
      uint2 Pw[M > 2 ? M - 2 : 1];
#pragma unroll
      for (int k = 0; k < M - 2; ++k)
        Pw[k] = *reinterpret_cast<const uint2*>(rec - lane * 8 + u * RB + 512 + k * 256);
      const int tot = chunk_dot<M>(X, B, Pw);
      const float2 lm = tab[u < valid ? pr[u * pr_step] : 0];
      v[u] = fmaf(lm.y, (float)tot * xs, lm.x * xsm);
    }
    slot_c = slot_c + 1 == NS ? 0 : slot_c + 1;
    STAGQ_ISSUE_BATCH();  // batch b + D refills the slot read one batch ago

    const float s = transposed_reduce<UP>(v, lane);
    const int uu = lane / (32 / UP);
    if ((lane & (32 / UP - 1)) == 0 && uu < valid) pw_out[uu * RG * KW] = s;
    pr += UP * pr_step;
    pw_out += UP * RG * KW;
  }
#undef STAGQ_ISSUE_BATCH
  cp_async_wait_all();
  __syncthreads();

  // Per row: held-out entries add x_c (v - lo_M(g(r, c))); then the K-slice
  // partials in order; one warp per row, lanes over the row's entries.
  const int nwarps = nthreads >> 5;
  for (int lr = warp; lr < rows; lr += nwarps) {
    const int e0 = rp[lr], e1 = rp[lr + 1];
    float cs = 0.f;
    for (int e = e0 + lane; e < e1; e += 32) {
      const uint32_t en = staged ? ents[e - e_base] : __ldg(a.m.entries + e);
      const int col = (int)(en & 0xFFFFu);
      const float lo = tab[pairs[lr * ps + (col >> P.group_shift)]].x;
      cs = fmaf(__half2float(xh[col]), __half2float(__ushort_as_half((unsigned short)(en >> 16))) - lo, cs);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cs += __shfl_xor_sync(kFull, cs, off);
    if (lane == 0) {
      float acc = 0.f;
      for (int k = 0; k < KW; ++k) acc += partial[lr * KW + k];
      acc += cs;
      if (a.y_f32) reinterpret_cast<float*>(a.y)[r0 + lr] = acc;
      else reinterpret_cast<__half*>(a.y)[r0 + lr] = __float2half_rn(acc);
    }
  }
}

template <int M>
__global__ void decode_levels_kernel(const DeviceMatrix m, uint8_t* u) {
  const int64_t in = m.in, nchunk = in / kChunk, total = (int64_t)m.out * nchunk;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = t / nchunk, c = t % nchunk;
    const uint4 b = *reinterpret_cast<const uint4*>(m.base + base_chunk_offset(r, in, c));
    const uint32_t base[4] = {b.x, b.y, b.z, b.w};
    uint32_t pw[4][2] = {};
#pragma unroll
    for (int k = 0; k < M - 2; ++k) {
      const uint2 p = *reinterpret_cast<const uint2*>(m.plane[k] + plane_chunk_offset(r, in, c));
      pw[k][0] = p.x;
      pw[k][1] = p.y;
    }
    for (int q = 0; q < kChunk; ++q) u[r * in + c * kChunk + q] = (uint8_t)chunk_level(base, pw, M, q);
  }
}

// Opt a kernel into `smem` bytes of dynamic shared memory on the current
// device, once per (device, kernel) and only when it grows.
cudaError_t ensure_smem(const void* kern, int key, size_t smem) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static size_t granted[kMaxDev][64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDev || key < 0 || key >= 64) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lock(mu);
  if (granted[dev][key] >= smem) return cudaSuccess;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess) granted[dev][key] = smem;
  return err;
}

template <int M, int UP, int D>
cudaError_t launch_gemv_mud(const DeviceMatrix& m, const GemvPlan& plan, const void* x, void* y, int y_f32,
                            cudaStream_t stream) {
  GemvKernelArgs a;
  a.m = m;
  a.plan = plan;
  a.table = m.tables + 256 * (M - 2);
  a.x = reinterpret_cast<const __half*>(x);
  a.y = y;
  a.y_f32 = y_f32;
  const SmemLayout L = smem_layout(plan, m.in, M);
  auto kern = gemv_kernel<M, UP, D>;
  cudaError_t err = ensure_smem(reinterpret_cast<const void*>(kern), ((M - 2) * 3 + (UP == 4 ? 2 : UP - 1)) * 4 + D - 1, L.total);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)plan.grid);
  cfg.blockDim = dim3((unsigned)(32 * plan.KW * plan.RG));
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = plan.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int M, int UP>
cudaError_t launch_gemv_mu(const DeviceMatrix& m, const GemvPlan& plan, const void* x, void* y, int y_f32,
                           cudaStream_t stream) {
  switch (plan.depth) {
    case 1: return launch_gemv_mud<M, UP, 1>(m, plan, x, y, y_f32, stream);
    case 2: return launch_gemv_mud<M, UP, 2>(m, plan, x, y, y_f32, stream);
    case 3: return launch_gemv_mud<M, UP, 3>(m, plan, x, y, y_f32, stream);
    case 4: return launch_gemv_mud<M, UP, 4>(m, plan, x, y, y_f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int M>
cudaError_t launch_gemv_m(const DeviceMatrix& m, const GemvPlan& plan, const void* x, void* y, int y_f32,
                          cudaStream_t stream) {
  switch (plan.up) {
    case 1: return launch_gemv_mu<M, 1>(m, plan, x, y, y_f32, stream);
    case 2: return launch_gemv_mu<M, 2>(m, plan, x, y, y_f32, stream);
    case 4: return launch_gemv_mu<M, 4>(m, plan, x, y, y_f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int M>
cudaError_t launch_decode_m(const DeviceMatrix& m, uint8_t* u, cudaStream_t stream) {
  const int64_t total = (int64_t)m.out * (m.in / kChunk);
  int grid = (int)((total + 255) / 256);
  if (grid > 65535) grid = 65535;
  decode_levels_kernel<M><<<grid, 256, 0, stream>>>(m, u);
  return cudaGetLastError();
}

}  // namespace

uint32_t gemv_smem_bytes(const GemvPlan& plan, int in, int bits) { return smem_layout(plan, in, bits).total; }

int gemv_grid(int out, int num_sms) {
  int g = out < num_sms ? out : num_sms;
  if ((out + g - 1) / g > kMaxRowsPerCta) g = (out + kMaxRowsPerCta - 1) / kMaxRowsPerCta;
  return g;
}

int k_slices(int in) { return (in / kChunk + 31) / 32; }

bool make_plan(const DeviceMatrix& m, int bits, GemvPlan* p) {
  p->KW = k_slices(m.in);
  if (p->KW > kMaxConsumerWarps) return false;
  p->RG = kMaxConsumerWarps / p->KW;
  p->grid = gemv_grid(m.out, m.num_sms);
  p->max_rows_per_cta = (m.out + p->grid - 1) / p->grid;
  p->pair_stride = m.pair_stride;
  p->group_shift = 0;
  while ((1 << p->group_shift) < m.group) ++p->group_shift;
  p->pdl = 1;
  // Stage the side record in shared memory when it fits beside a ring of at
  // least two batches, else read it from global memory in the final pass.
  for (int stage_ents = 1; stage_ents >= 0; --stage_ents) {
    p->ent_cap = stage_ents ? m.max_cta_entries + 4 : 0;
    for (int up = 4; up >= 1; up /= 2) {
      p->up = up;
      for (int d = kPrefetchGroups; d >= 2; --d) {
        p->depth = d;
        if (smem_layout(*p, m.in, bits).total <= (uint32_t)m.smem_limit) return true;
      }
    }
  }
  return false;
}

cudaError_t launch_gemv(const DeviceMatrix& m, const GemvPlan& plan, int bits, const void* x, void* y, int y_f32,
                        cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_gemv_m<2>(m, plan, x, y, y_f32, stream);
    case 3: return launch_gemv_m<3>(m, plan, x, y, y_f32, stream);
    case 4: return launch_gemv_m<4>(m, plan, x, y, y_f32, stream);
    case 5: return launch_gemv_m<5>(m, plan, x, y, y_f32, stream);
    case 6: return launch_gemv_m<6>(m, plan, x, y, y_f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_levels(const DeviceMatrix& m, int bits, uint8_t* u, cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_decode_m<2>(m, u, stream);
    case 3: return launch_decode_m<3>(m, u, stream);
    case 4: return launch_decode_m<4>(m, u, stream);
    case 5: return launch_decode_m<5>(m, u, stream);
    case 6: return launch_decode_m<6>(m, u, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace stagq
