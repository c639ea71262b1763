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
//  * one CTA per SM owns a contiguous, balanced range of rows, cut into
//    "stages" of R_s consecutive rows. Because every plane is row-major, a
//    stage is one contiguous byte range per plane: a producer warp streams
//    base + planes 3..M (only those: a p_M read never touches deeper planes)
//    + pair bytes with 1-D bulk copies (cp.async.bulk, mbarrier completion)
//    into a ring of shared-memory slots, as far ahead as the ring allows, and
//    prefetches each stage's side-record entries with cp.async;
//  * x is converted once per CTA to 16-bit fixed point with a power-of-two
//    scale per 64-element chunk (|error| <= 2^-16 max|x_chunk|); each consumer
//    lane keeps its chunk's 64 activations in registers for every row;
//  * consumer warps = KW "K-warps" (2048 weights of K each) x RG row groups.
//    A lane turns 16 base bytes (+ 8 bytes per plane) of one 64-weight chunk
//    into code bytes / nibble composites (layout.cuh) and feeds them to dp2a
//    integer dot products (exact in int32); the group affine is applied once
//    per chunk in fp32; rows are reduced across lanes by a transposed shuffle;
//  * each stage row's side-record correction is computed by one consumer warp
//    (lanes over entries); the producer warp then adds the K-warp partials in
//    a fixed order, adds the correction and stores y -- deterministic, no
//    atomics, no workspace, no second launch (the K split of Appendix G's
//    atomic-add kernel becomes a fixed-order shared-memory reduction);
//  * every mbarrier wait is bounded in time; on expiry the kernel records an
//    error in the handle's status word and returns.
#include <cuda_fp16.h>

#include <cstdint>
#include <mutex>

#include "device_matrix.hpp"
#include "layout.cuh"

namespace stagq {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait, then give up

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if ((i & 63u) == 0 && global_timer() - t0 > kWaitLimitNs) return false;
  }
}
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* b) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(b)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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

// Shared-memory carve-up, identical on host (plan) and device.
struct SmemLayout {
  uint32_t full, ent, empty;        // mbarrier arrays [S]
  uint32_t xq, xh, xscale, xsum, tab, rp, partial, corr, slots;
  uint32_t slot_bytes, s_base, s_plane, s_pair, s_ent;
  uint32_t total;
};

__host__ __device__ inline uint32_t align_up_u32(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout smem_layout(const GemvPlan& p, int in, int M) {
  SmemLayout L;
  const uint32_t S = p.slots, Rs = p.rows_per_stage, nchunk = in / kChunk;
  uint32_t o = 0;
  L.full = o; o += 8 * S;
  L.ent = o; o += 8 * S;
  L.empty = o; o += 8 * S;
  o = align_up_u32(o, 16);
  L.xq = o; o += 2 * in;
  L.xh = o; o += 2 * in;
  L.xscale = o; o += 4 * nchunk;
  L.xsum = o; o += 4 * nchunk;
  o = align_up_u32(o, 16);
  L.tab = o; o += 256 * 8;
  L.rp = o; o += 4 * (p.max_rows_per_cta + 1);
  o = align_up_u32(o, 16);
  L.partial = o; o += 4 * S * p.KW * Rs;
  L.corr = o; o += 4 * S * Rs;
  o = align_up_u32(o, 128);
  L.slots = o;
  L.s_base = 0;
  L.s_plane = Rs * (in / 4);
  L.s_pair = L.s_plane + (M - 2) * Rs * (in / 8);
  L.s_ent = align_up_u32(L.s_pair + Rs * p.pair_stride, 16);
  L.slot_bytes = align_up_u32(L.s_ent + 4 * p.ecap, 128);
  o += S * L.slot_bytes;
  L.total = o;
  return L;
}

template <int M, int UP>
__global__ void __launch_bounds__(kMaxConsumerWarps * 32 + 32, 1) gemv_kernel(const GemvKernelArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const GemvPlan& P = a.plan;
  const int in = a.m.in;
  const int nchunk = in / kChunk;
  const SmemLayout L = smem_layout(P, in, M);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.full);
  uint64_t* ent_full = reinterpret_cast<uint64_t*>(smem + L.ent);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L.empty);
  int16_t* xq = reinterpret_cast<int16_t*>(smem + L.xq);
  __half* xh = reinterpret_cast<__half*>(smem + L.xh);
  float* xscale = reinterpret_cast<float*>(smem + L.xscale);
  float* xsum = reinterpret_cast<float*>(smem + L.xsum);
  float2* tab = reinterpret_cast<float2*>(smem + L.tab);
  int* rp = reinterpret_cast<int*>(smem + L.rp);
  float* partial = reinterpret_cast<float*>(smem + L.partial);  // [S][KW][Rs]
  float* corr = reinterpret_cast<float*>(smem + L.corr);        // [S][Rs]
  uint8_t* slots = smem + L.slots;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int KW = P.KW, RG = P.RG, Wc = KW * RG, Rs = P.rows_per_stage, S = P.slots;
  const bool producer = warp == Wc;
  const int64_t r0 = (int64_t)blockIdx.x * a.m.out / gridDim.x;
  const int64_t r1 = (int64_t)(blockIdx.x + 1) * a.m.out / gridDim.x;
  const int rows = (int)(r1 - r0);
  const int nst = (rows + Rs - 1) / Rs;
  const uint32_t plane_row = in / 8, base_row = in / 4;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ent_full[s], 32);
      mbar_init(&empty[s], Wc);
    }
    fence_barrier_init();
  }
  __syncthreads();

  // Producer: bulk copies of one stage's planes + pair bytes into its slot.
  auto issue_planes = [&](int st) {
    const int slot = st % S;
    const int64_t row0 = r0 + (int64_t)st * Rs;
    const uint32_t n = (uint32_t)min(Rs, rows - st * Rs);
    uint8_t* dst = slots + (size_t)slot * L.slot_bytes;
    const uint32_t bb = n * base_row, pb = n * plane_row, qb = n * P.pair_stride;
    mbar_arrive_expect_tx(&full[slot], bb + (M - 2) * pb + qb);
    bulk_load(dst + L.s_base, a.m.base + row0 * base_row, bb, &full[slot]);
#pragma unroll
    for (int k = 0; k < M - 2; ++k)
      bulk_load(dst + L.s_plane + k * Rs * plane_row, a.m.plane[k] + row0 * plane_row, pb, &full[slot]);
    bulk_load(dst + L.s_pair, a.m.pair + row0 * P.pair_stride, qb, &full[slot]);
  };
  // Producer warp: side-record entries of one stage (first ecap of them).
  auto issue_entries = [&](int st) {
    const int slot = st % S;
    const int lr0 = st * Rs, lr1 = min(lr0 + Rs, rows);
    const int e0 = rp[lr0], n = min(rp[lr1] - e0, P.ecap);
    uint32_t* dst = reinterpret_cast<uint32_t*>(slots + (size_t)slot * L.slot_bytes + L.s_ent);
    for (int e = lane; e < n; e += 32) cp_async4(dst + e, a.m.entries + e0 + e);
    cp_async_arrive_noinc(&ent_full[slot]);
  };

  if (producer) {
    if (lane == 0)
      for (int st = 0; st < min(S, nst); ++st) issue_planes(st);
    for (int i = lane; i <= rows; i += 32) rp[i] = __ldg(a.m.row_ptr + r0 + i);
    __syncwarp();
    for (int st = 0; st < min(S, nst); ++st) issue_entries(st);
  }
  // Let the next kernel in the stream start its own prologue early; x (which a
  // previous kernel may have produced) is read only after the dependency wait.
  grid_launch_dependents();
  grid_dependency_wait();

  if (!producer) {
    for (int i = tid; i < 256; i += Wc * 32) tab[i] = a.table[i];
    // x -> fixed point; a task is 8 consecutive values, 8 tasks form a chunk.
    const int n8 = in / 8;
    for (int i0 = warp * 32; i0 < n8; i0 += Wc * 32) {
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
  __syncthreads();

  if (!producer) {
    // ------------------------------------------------------------ consumers
    const int kw = warp % KW, rg = warp / KW;
    const int c = kw * 32 + lane;  // this lane's 64-weight chunk
    const bool active = c < nchunk;
    const int gidx = (c * kChunk) / a.m.group;
    uint32_t X[32];
    float xs = 0.f, xsm = 0.f;
    if (active) {
      const uint4* src = reinterpret_cast<const uint4*>(xq + c * kChunk);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint4 t = src[k];
        X[4 * k] = t.x;
        X[4 * k + 1] = t.y;
        X[4 * k + 2] = t.z;
        X[4 * k + 3] = t.w;
      }
      xs = xscale[c];
      xsm = xsum[c];
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) X[k] = 0u;
    }

    for (int st = 0; st < nst; ++st) {
      const int slot = st % S;
      const uint32_t par = (uint32_t)(st / S) & 1u;
      const int n = min(Rs, rows - st * Rs);
      const uint8_t* sd = slots + (size_t)slot * L.slot_bytes;
      if (!mbar_wait(&full[slot], par)) {
        if (lane == 0) atomicOr(a.m.status, 1u);
        return;
      }
      float v[UP];
#pragma unroll
      for (int u = 0; u < UP; ++u) {
        const int row = rg + RG * u;  // stage-local
        v[u] = 0.f;
        if (row < n && active) {
          const uint4 b4 = *reinterpret_cast<const uint4*>(sd + L.s_base + row * base_row + c * kBaseChunkBytes);
          const uint32_t B[4] = {b4.x, b4.y, b4.z, b4.w};
          uint2 Pw[M > 2 ? M - 2 : 1];
#pragma unroll
          for (int k = 0; k < M - 2; ++k)
            Pw[k] = *reinterpret_cast<const uint2*>(sd + L.s_plane + (k * Rs + row) * plane_row +
                                                   c * kPlaneChunkBytes);
          const int tot = chunk_dot<M>(X, B, Pw);
          const float2 lm = tab[sd[L.s_pair + row * P.pair_stride + gidx]];
          v[u] = fmaf(lm.y, (float)tot * xs, lm.x * xsm);
        }
      }
      const float s = transposed_reduce<UP>(v, lane);
      const int u_of_lane = lane / (32 / UP);
      if ((lane & (32 / UP - 1)) == 0) {
        const int row = rg + RG * u_of_lane;
        if (row < n) partial[(slot * KW + kw) * Rs + row] = s;
      }
      // side-record corrections of the stage rows assigned to this warp
      const int first = (st * Rs) % Wc;
      int j = warp - first;
      if (j < 0) j += Wc;
      if (j < n) {
        if (!mbar_wait(&ent_full[slot], par)) {
          if (lane == 0) atomicOr(a.m.status, 2u);
          return;
        }
        const uint32_t* se = reinterpret_cast<const uint32_t*>(sd + L.s_ent);
        const int est = rp[st * Rs];
        for (; j < n; j += Wc) {
          const int e0 = rp[st * Rs + j], e1 = rp[st * Rs + j + 1];
          float cs = 0.f;
          for (int e = e0 + lane; e < e1; e += 32) {
            const int le = e - est;
            const uint32_t en = le < P.ecap ? se[le] : __ldg(a.m.entries + e);
            const int col = (int)(en & 0xFFFFu);
            const float val = __half2float(__ushort_as_half((unsigned short)(en >> 16)));
            const float lo = tab[sd[L.s_pair + j * P.pair_stride + col / a.m.group]].x;
            cs = fmaf(__half2float(xh[col]), val - lo, cs);
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) cs += __shfl_xor_sync(kFull, cs, off);
          if (lane == 0) corr[slot * Rs + j] = cs;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  } else {
    // ------------------------------------------------------------- producer
    for (int st = 0; st < nst; ++st) {
      const int slot = st % S;
      const uint32_t par = (uint32_t)(st / S) & 1u;
      const int n = min(Rs, rows - st * Rs);
      if (!mbar_wait(&empty[slot], par)) {
        if (lane == 0) atomicOr(a.m.status, 4u);
        break;
      }
      if (lane < n) {
        float acc = 0.f;
        for (int k = 0; k < KW; ++k) acc += partial[(slot * KW + k) * Rs + lane];
        acc += corr[slot * Rs + lane];
        const int64_t r = r0 + (int64_t)st * Rs + lane;
        if (a.y_f32) reinterpret_cast<float*>(a.y)[r] = acc;
        else reinterpret_cast<__half*>(a.y)[r] = __float2half_rn(acc);
      }
      __syncwarp();
      if (st + S < nst) {
        if (lane == 0) issue_planes(st + S);
        issue_entries(st + S);
      }
    }
    // Nothing may still be landing in shared memory when the CTA exits.
    cp_async_wait_all();
    for (int st = max(0, nst - S); st < nst; ++st)
      mbar_wait(&full[st % S], (uint32_t)(st / S) & 1u);
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
  static size_t granted[kMaxDev][32] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDev || key < 0 || key >= 32) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lock(mu);
  if (granted[dev][key] >= smem) return cudaSuccess;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess) granted[dev][key] = smem;
  return err;
}

template <int M, int UP>
cudaError_t launch_gemv_mu(const DeviceMatrix& m, const GemvPlan& plan, const void* x, void* y, int y_f32,
                           cudaStream_t stream) {
  GemvKernelArgs a;
  a.m = m;
  a.plan = plan;
  a.table = m.tables + 256 * (M - 2);
  a.x = reinterpret_cast<const __half*>(x);
  a.y = y;
  a.y_f32 = y_f32;
  const SmemLayout L = smem_layout(plan, m.in, M);
  auto kern = gemv_kernel<M, UP>;
  cudaError_t err = ensure_smem(reinterpret_cast<const void*>(kern), M * 4 + UP, L.total);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)plan.grid);
  cfg.blockDim = dim3((unsigned)(32 * (plan.KW * plan.RG + 1)));
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = plan.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
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

void stage_partition(int out, int in, int num_sms, int* grid, int* rows_per_stage) {
  const int KW = (in / kChunk + 31) / 32;
  const int RG = KW >= kMaxConsumerWarps ? 1 : kMaxConsumerWarps / KW;
  const int up = RG * 2 <= kMaxStageRows ? 2 : 1;
  int g = out < num_sms ? out : num_sms;
  if ((out + g - 1) / g > kMaxRowsPerCta) g = (out + kMaxRowsPerCta - 1) / kMaxRowsPerCta;
  *grid = g;
  *rows_per_stage = RG * up;
}

bool make_plan(const DeviceMatrix& m, int bits, GemvPlan* p) {
  const int nchunk = m.in / kChunk;
  p->KW = (nchunk + 31) / 32;
  if (p->KW > kMaxConsumerWarps) return false;
  p->RG = p->KW >= kMaxConsumerWarps ? 1 : kMaxConsumerWarps / p->KW;
  int grid = 0, rs = 0;
  stage_partition(m.out, m.in, m.num_sms, &grid, &rs);
  p->grid = grid;
  p->max_rows_per_cta = (m.out + grid - 1) / grid;
  p->pair_stride = m.pair_stride;
  p->ecap = m.ecap;
  p->pdl = 1;
  // Two rows per row group and stage if the ring can still hold >= 3 stages,
  // else one; the ring then takes as many slots as shared memory allows.
  for (int up = rs / p->RG; up >= 1; --up) {
    p->up = up;
    p->rows_per_stage = p->RG * up;
    const int nst = (p->max_rows_per_cta + p->rows_per_stage - 1) / p->rows_per_stage;
    int S = 0;
    for (int t = 1; t <= nst; ++t) {
      p->slots = t;
      if (smem_layout(*p, m.in, bits).total > (uint32_t)m.smem_limit) break;
      S = t;
    }
    if (S == 0) continue;
    p->slots = S;
    if (S >= (nst < 3 ? nst : 3) || up == 1) return true;
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
