// sm_100a kernels of the StagQ batch-one GEMV y = W_hat^(M) x.
//
// What is computed (StagQ paper, arXiv 2610.05977): for every row i,
//   y_i = sum_groups [ s_M(g) * sum_{j in g} u_M,j x_j + lo_M(g) * sum_{j in g} x_j ]
//         + sum_{held-out (i,c)} x_c (v_ic - lo_M(g(i,c)))
// -- the affine map of Eq. (10) applied once per group, with u_M from Eq. (8),
// and the side record of Eq. (4) fused into the epilogue (held-out digits are
// zero, so the main stream decoded lo_M there and the correction is v - lo_M).
//
// How (design for B200):
//  * batch-one GEMV is bound by HBM, so no tensor cores: each lane streams
//    16 base bytes + 8 bytes per read plane of one 64-weight chunk with
//    128/64-bit non-allocating loads; a p_M read touches only planes 3..M;
//  * x is converted once per CTA to 16-bit fixed point with a power-of-two
//    scale per 64-element chunk (|error| <= 2^-16 max|x_chunk|) and kept in
//    registers for every row the lane visits;
//  * the composite level is never materialised: code bytes (base slots, or
//    the nibble composites of layout.cuh) go straight into dp2a integer dot
//    products, exact in int32; the group affine is applied once per chunk in
//    fp32;
//  * K is split across the warps of one CTA (up to 16 x 2048 weights); their
//    partial sums are added in a fixed order through shared memory, so
//    results are deterministic and no second pass or atomics are needed.
#include <cuda_fp16.h>

#include <cstdint>

#include "device_matrix.hpp"
#include "layout.cuh"

namespace stagq {
namespace {

constexpr int kMaxWarps = 16;
constexpr unsigned kFull = 0xFFFFFFFFu;

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

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int M>
struct RowRegs {
  uint4 b;                         // base chunk
  uint2 p[M > 2 ? M - 2 : 1];      // planes 3..M
  uint32_t pair;                   // 8-bit pair of the chunk's group
  int e0, e1;                      // side-record range of the row
};

// sum over the chunk of v_t X_t, with v = u_M (v = 2 u_3 at M = 3). Exact.
template <int M>
__device__ __forceinline__ int chunk_dot(const uint32_t (&X)[32], const RowRegs<M>& r) {
  const uint32_t B[4] = {r.b.x, r.b.y, r.b.z, r.b.w};
  if constexpr (M == 2) {
    int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a0 = dot4(X, i, 0, B[i] & 0x03030303u, a0);
      a1 = dot4(X, i, 1, B[i] & 0x0C0C0C0Cu, a1);
      a2 = dot4(X, i, 2, B[i] & 0x30303030u, a2);
      a3 = dot4(X, i, 3, B[i] & 0xC0C0C0C0u, a3);
    }
    // slot s carries q * 4^s; every product of a_s is a multiple of 4^s
    return a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);
  } else {
    int lo = 0, hi = 0;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint32_t p3 = w ? r.p[0].y : r.p[0].x;
      uint32_t p4 = 0u;
      if constexpr (M >= 4) p4 = w ? r.p[1].y : r.p[1].x;
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
        const uint32_t p5 = w ? r.p[2].y : r.p[2].x;
        uint32_t p6 = 0u;
        if constexpr (M >= 6) p6 = w ? r.p[3].y : r.p[3].x;
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

struct GemvKernelArgs {
  DeviceMatrix m;
  const float2* table;  // (lo_M, s_M c_M) of this precision
  const __half* x;
  void* y;
  int y_f32;
  int KW, RG;
};

template <int M, int U>
__device__ __forceinline__ void load_rows(const GemvKernelArgs& a, RowRegs<M> (&R)[U], int64_t r_begin,
                                          int rg, int m0, int nrows, int c, bool active, int gidx) {
  const int64_t in = a.m.in;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (m0 + u < nrows) {
      const int64_t r = r_begin + rg + (int64_t)a.RG * (m0 + u);
      if (active) {
        R[u].b = ld_stream16(a.m.base + r * (in / 4) + (int64_t)c * kBaseChunkBytes);
#pragma unroll
        for (int k = 0; k < M - 2; ++k)
          R[u].p[k] = ld_stream8(a.m.plane[k] + r * (in / 8) + (int64_t)c * kPlaneChunkBytes);
        R[u].pair = __ldg(a.m.pair + r * (in / a.m.group) + gidx);
      }
      R[u].e0 = __ldg(a.m.row_ptr + r);
      R[u].e1 = __ldg(a.m.row_ptr + r + 1);
    }
  }
}

template <int M, int U>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) gemv_kernel(const GemvKernelArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int in = a.m.in, out = a.m.out;
  const int nchunk = in / kChunk;
  int16_t* xq = reinterpret_cast<int16_t*>(smem);                 // [in] fixed-point x
  __half* xh = reinterpret_cast<__half*>(smem + 2 * in);          // [in] fp16 x
  float* xscale = reinterpret_cast<float*>(smem + 4 * in);        // [nchunk]
  float* xsum = xscale + nchunk;                                  // [nchunk]
  float2* tab = reinterpret_cast<float2*>(xsum + nchunk);         // [256]
  float* partial = reinterpret_cast<float*>(tab + 256);           // [2][RG][KW][U]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int KW = a.KW, RG = a.RG;
  const int kw = warp % KW, rg = warp / KW;
  const int64_t r_begin = (int64_t)blockIdx.x * out / gridDim.x;
  const int64_t r_end = (int64_t)(blockIdx.x + 1) * out / gridDim.x;
  const int nrows = (int)((r_end - r_begin - rg + RG - 1) / RG);  // rows of this row group
  const int c = kw * 32 + lane;                                   // this lane's chunk
  const bool active = c < nchunk;
  const int gidx = (c * kChunk) / a.m.group;

  // Weight loads do not depend on x: start the first batch now.
  RowRegs<M> cur[U];
  load_rows<M, U>(a, cur, r_begin, rg, 0, nrows, c, active, gidx);

  for (int i = tid; i < 256; i += blockDim.x) tab[i] = a.table[i];
  // x -> fixed point. A task is 8 consecutive values; 8 tasks form a chunk.
  const int n8 = in / 8;
  for (int i0 = warp * 32; i0 < n8; i0 += nwarps * 32) {
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
    // e such that max|x| * 2^e lies in [2^14, 2^15): the scaled fp16 values
    // fit int16 and the largest ones convert exactly.
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
  __syncthreads();

  uint32_t X[32];
  float xs = 0.f, xsm = 0.f;
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(xq + (int64_t)c * kChunk);
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

  int buf = 0;
  for (int m0 = 0; m0 < nrows; m0 += U) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float p = 0.f;
      if (m0 + u < nrows) {  // warp-uniform
        float lo_own = 0.f;
        if (active) {
          const int tot = chunk_dot<M>(X, cur[u]);
          const float2 lm = tab[cur[u].pair];
          p = fmaf(lm.y, (float)tot * xs, lm.x * xsm);
          lo_own = lm.x;
        }
        // side record: this K-warp corrects the held-out entries in its columns
        const int e0 = cur[u].e0, e1 = cur[u].e1;
        for (int e = e0; e < e1; e += 32) {
          const int ee = e + lane;
          const uint32_t ent = ee < e1 ? __ldg(a.m.entries + ee) : 0xFFFFFFFFu;
          const int col = (int)(ent & 0xFFFFu);
          const float lo = __shfl_sync(kFull, lo_own, (col >> 6) & 31);
          if (ee < e1 && (col >> 11) == kw) {
            const float v = __half2float(__ushort_as_half((unsigned short)(ent >> 16)));
            p = fmaf(__half2float(xh[col]), v - lo, p);
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(kFull, p, off);
      }
      if (lane == 0) partial[((buf * RG + rg) * KW + kw) * U + u] = p;
    }
    if (KW > 1) named_barrier(1 + rg, KW * 32);
    else __syncwarp();
    if (kw == 0 && lane < U && m0 + lane < nrows) {
      const int64_t r = r_begin + rg + (int64_t)RG * (m0 + lane);
      float acc = 0.f;
      for (int k = 0; k < KW; ++k) acc += partial[((buf * RG + rg) * KW + k) * U + lane];
      if (a.y_f32) reinterpret_cast<float*>(a.y)[r] = acc;
      else reinterpret_cast<__half*>(a.y)[r] = __float2half_rn(acc);
    }
    buf ^= 1;
    if (m0 + U < nrows) load_rows<M, U>(a, cur, r_begin, rg, m0 + U, nrows, c, active, gidx);
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

template <int M>
cudaError_t launch_gemv_m(const DeviceMatrix& m, const void* x, void* y, int y_f32, cudaStream_t stream) {
  constexpr int U = M <= 4 ? 4 : 2;
  const int nchunk = m.in / kChunk;
  const int KW = (nchunk + 31) / 32;
  if (KW > kMaxWarps) return cudaErrorInvalidValue;
  const int RG = KW == 1 ? kMaxWarps : kMaxWarps / KW;  // named barriers 1..RG when KW > 1
  GemvKernelArgs a;
  a.m = m;
  a.table = m.tables + 256 * (M - 2);
  a.x = reinterpret_cast<const __half*>(x);
  a.y = y;
  a.y_f32 = y_f32;
  a.KW = KW;
  a.RG = RG;
  const int threads = 32 * KW * RG;
  const int grid = m.out < m.num_sms ? m.out : m.num_sms;
  const size_t smem = (size_t)4 * m.in + (size_t)8 * nchunk + 256 * sizeof(float2) +
                      (size_t)2 * RG * KW * U * sizeof(float);
  auto kern = gemv_kernel<M, U>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<grid, threads, smem, stream>>>(a);
  return cudaGetLastError();
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

cudaError_t launch_gemv(const DeviceMatrix& m, int bits, const void* x, void* y, int y_f32,
                        cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_gemv_m<2>(m, x, y, y_f32, stream);
    case 3: return launch_gemv_m<3>(m, x, y, y_f32, stream);
    case 4: return launch_gemv_m<4>(m, x, y, y_f32, stream);
    case 5: return launch_gemv_m<5>(m, x, y, y_f32, stream);
    case 6: return launch_gemv_m<6>(m, x, y, y_f32, stream);
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
