// sm_100a kernels of the StagQ batch-one GEMV y = W_hat^(M) x.
//
// What is computed (StagQ paper, arXiv 2610.05977): for every row i,
//   y_i = sum_groups [ s_M(g) * sum_{j in g} u_M,j x_j + lo_M(g) * sum_{j in g} x_j ]
//         + sum_{held-out (i,c)} x_c (v_ic - lo_M(g(i,c)))
// -- the affine map of Eq. (10) applied once per group, with u_M from Eq. (8),
// and the side record of Eq. (4) fused in (held-out digits are zero, so the
// main stream decoded lo_M there and the correction is v - lo_M).
//
// How (design for B200; batch-one GEMV is bound by HBM, so no tensor cores):
//  * one CTA per SM owns a contiguous, balanced range of rows. It is cut into
//    blocks of BR rows; a block's base rows, read-plane rows (a p_M read never
//    touches deeper planes) and pair bytes are contiguous in HBM, so one
//    thread moves a block into a shared-memory ring slot with 2 + (M - 2)
//    bulk copies (cp.async.bulk, completion on the slot's mbarrier). The
//    CTA's side record (cut per CTA at load time) and the precision's pair
//    table arrive the same way;
//  * the CTA is small (<= 8 warps, <= 113 KB of shared memory, <= 128
//    registers a thread) so the next GEMV's CTA fits beside it on the SM:
//    with programmatic dependent launch it starts early and its copies are in
//    flight while this GEMV computes;
//  * warps are KW "K slices" (2048 weights of K each: 32 lanes x one
//    64-weight chunk) times RG row groups; in every block each warp takes UP
//    rows, as straight-line code so their dot products interleave;
//  * x is converted once per CTA to 16-bit fixed point with a power-of-two
//    scale per 64-element chunk (|error| <= 2^-16 max|x_chunk|); each lane
//    keeps its chunk's 64 activations in registers; code bytes / nibble
//    composites (layout.cuh) feed dp2a integer dot products (exact in int32)
//    and the group affine is applied once per chunk in fp32;
//  * the held-out entries of the warp's rows in its K slice add
//    x~_c (v - lo_M) with the same fixed-point x~, so the result is exactly
//    W_hat x~ up to fp32 rounding;
//  * a transposed shuffle reduces the UP rows to one partial per (row, K
//    slice); the warp that finishes a block last (a shared-memory counter)
//    adds the block's KW partials in a fixed order, stores y and refills the
//    slot -- deterministic, no atomics on data, no workspace, no second
//    launch (the K split of Appendix G's atomic-add kernel becomes this);
//  * every mbarrier wait is bounded in time; on expiry the kernel records it
//    in the handle's status word, waits (bounded) for its own copies and
//    returns.
#include <cuda_fp16.h>

#include <cstdint>
#include <mutex>

#include "device_matrix.hpp"
#include "kernel_common.cuh"
#include "layout.cuh"

namespace stagq {
namespace {

using namespace kernels;

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
  const float* dlo;     // lo - lo_M of this precision (post-grid entries)
  const __half* x;
  const float* in_scale;  // SC: per-channel multiplier of x (the inverse activation scale)
  void* y;
  int y_f32;
};

// What a post-grid entry needs beside its residual: the pair byte of its
// group (row u's pair bytes start at prow + u * pstep in the slot) and
// lo - lo_M of that pair.
struct PostCtx {
  const uint8_t* prow;
  uint32_t pstep;
  const float* dlo;
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // a copy that has not landed in 2 s never will
constexpr uint64_t kDrainLimitNs = 100000000ull;   // after a failure: wait for own copies, 0.1 s

// Shared-memory carve-up, identical on host (plan) and device.
struct SmemLayout {
  uint32_t bar, cnt, last, tab, xq, xscale, xsum, xsum16, lo, partial, side, ring;
  uint32_t slot;                 // bytes of one ring slot
  uint32_t plane_piece, pair_piece;  // offsets inside a slot (base rows at 0)
  uint32_t total;
};

__host__ __device__ inline uint32_t align_up_u32(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline SmemLayout smem_layout(const GemvPlan& p, int in, int M) {
  SmemLayout L;
  const uint32_t nchunk = in / kChunk, BR = p.br;
  uint32_t o = 0;
  L.bar = o; o += 8 * (kMaxSlots + 2);  // full[slot] + side/table barrier + a test barrier nothing completes
  L.cnt = o; o += 4 * kMaxSlots;         // warps done with the slot's blocks so far
  L.last = o; o += 4 * kMaxSlots;        // last block issued into the slot
  o = align_up_u32(o, 16);
  L.tab = o; o += 256 * 8 * (uint32_t)p.nmem;  // the pair table of each stacked member
  L.xq = o; o += 2u * in * p.nb;        // x~ of each of the nb vectors
  L.xscale = o; o += 4u * nchunk * p.nb;
  L.xsum = o; o += 4u * nchunk * p.nb;
  L.xsum16 = o; o += p.group_shift < 6 ? 16u * nchunk * p.nb : 0u;  // per 16 values, for groups < 64
  o = align_up_u32(o, 16);
  // per warp: lo_M of each of a lane's groups per row of a block
  L.lo = o; o += 4u * 32 * p.up * p.NW * (uint32_t)groups_per_chunk(p.group_shift);
  L.partial = o; o += 4u * p.ns * BR * p.KW * p.nb;  // [slot][BR][KW][nb]
  o = align_up_u32(o, 128);
  L.side = o; o += p.stage_side ? (uint32_t)p.side_stride : 0u;
  o = align_up_u32(o, 128);
  L.ring = o;
  L.plane_piece = BR * (in / 4);
  L.pair_piece = L.plane_piece + (uint32_t)(M - 2) * BR * (in / 8);
  L.slot = align_up_u32(L.pair_piece + BR * p.pair_stride, 128);
  o += p.ns * L.slot;
  L.total = o;
  return L;
}

// Dot products of NR rows of one block for this lane's chunk, with the group
// affine: v[u] = sum over the chunk's G groups of s_M c_M sum(v x~) + lo_M
// sum(x~) (xsg[g]: sum of x~ over group g), and the lane's lo_M per row and
// group (for the side record). Row u of the warp sits at offsets off.b + u *
// step.b (base), off.p + u * step.p (first read plane; plane k at + k *
// plane_stride) and off.g + u * step.g (its G pair bytes) in the slot.
struct RowOffsets {
  uint32_t b, p, g;
};

// v = sum_g s_M c_M tot[g] xs + lo_M xsg[g] for the G pair bytes in `pairs`
// (byte g = group g); lo[g] = lo_M of group g.
template <int G>
__device__ __forceinline__ float group_affine(const float2* tab, uint32_t pairs, const int (&tot)[G], float xs,
                                              const float (&xsg)[G], float (&lo)[G]) {
  if constexpr (G == 1) {
    const float2 l = tab[pairs];
    lo[0] = l.x;
    return fmaf(l.y, (float)tot[0] * xs, l.x * xsg[0]);
  } else {
    float acc = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float2 l = tab[(pairs >> (8 * g)) & 0xFFu];
      lo[g] = l.x;
      acc = fmaf(l.y, (float)tot[g] * xs, fmaf(l.x, xsg[g], acc));
    }
    return acc;
  }
}

template <int M, int NR, int G>
__device__ __forceinline__ void rows_dot(const uint32_t (&X)[32], float xs, const float (&xsg)[G], const uint8_t* sb,
                                         RowOffsets off, RowOffsets step, uint32_t plane_stride,
                                         const float2* const (&tb)[NR], float (&v)[NR], float (&lo)[NR][G]) {
#pragma unroll
  for (int u = 0; u < NR; ++u) {
    const uint4 b4 = *reinterpret_cast<const uint4*>(sb + off.b + u * step.b);
    const uint32_t B[4] = {b4.x, b4.y, b4.z, b4.w};
    uint2 Pw[M > 2 ? M - 2 : 1];
#pragma unroll
    for (int k = 0; k < M - 2; ++k)
      Pw[k] = *reinterpret_cast<const uint2*>(sb + off.p + u * step.p + k * plane_stride);
    int tot[G];
    chunk_dot_g<M, G>(X, B, Pw, tot);
    v[u] = group_affine<G>(tb[u], load_pairs<G>(sb + off.g + u * step.g), tot, xs, xsg, lo[u]);
  }
}

// As rows_dot for NB activation vectors (NB > 1): the slot's code words are
// read once and dotted with each vector's x~, which is taken from shared
// memory vector by vector (x~ of vector j at xq + j * in, its chunk scales at
// xscale / xsum + j * nchunk, its 16-value sums at xsum16 + 4 j nchunk). v[j][u]
// is row u against vector j.
template <int M, int NR, int NB, int G>
__device__ __forceinline__ void rows_dot_nb(const int16_t* xq, const float* xscale, const float* xsum,
                                            const float* xsum16, int in, int nchunk, int cc, bool active,
                                            const uint8_t* sb, RowOffsets off, RowOffsets step, uint32_t plane_stride,
                                            const float2* const (&tb)[NR], float (&v)[NB][NR], float (&lo)[NR][G]) {
  uint32_t B[NR][4];
  uint2 Pw[NR][M > 2 ? M - 2 : 1];
  uint32_t pr[NR];
  // up to two planes: the code words are decoded once for all NB vectors
  constexpr bool kCodes = M <= 4;
  uint32_t cw[kCodes ? NR : 1][16];
#pragma unroll
  for (int u = 0; u < NR; ++u) {
    const uint4 b4 = *reinterpret_cast<const uint4*>(sb + off.b + u * step.b);
    B[u][0] = b4.x; B[u][1] = b4.y; B[u][2] = b4.z; B[u][3] = b4.w;
#pragma unroll
    for (int k = 0; k < M - 2; ++k)
      Pw[u][k] = *reinterpret_cast<const uint2*>(sb + off.p + u * step.p + k * plane_stride);
    pr[u] = load_pairs<G>(sb + off.g + u * step.g);
    if constexpr (kCodes) chunk_codes<M>(B[u], Pw[u], cw[u]);
  }
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    uint32_t X[32];
    const uint4* src = reinterpret_cast<const uint4*>(xq + j * in);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 t = src[xq_piece(cc, k)];
      X[4 * k] = t.x;
      X[4 * k + 1] = t.y;
      X[4 * k + 2] = t.z;
      X[4 * k + 3] = t.w;
    }
    const float xs = active ? xscale[j * nchunk + cc] : 0.f;
    float xsg[G];
    if constexpr (G == 1) {
      xsg[0] = active ? xsum[j * nchunk + cc] : 0.f;
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < 4 / G; ++q) t += xsum16[4 * (j * nchunk + cc) + (4 / G) * g + q];
        xsg[g] = active ? t : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < NR; ++u) {
      int tot[G];
      if constexpr (kCodes) chunk_dot_codes<M, G>(X, cw[u], tot);
      else chunk_dot_g<M, G>(X, B[u], Pw[u], tot);
      v[j][u] = group_affine<G>(tb[u], pr[u], tot, xs, xsg, lo[u]);
    }
  }
}

// Where lo_M of column `col`'s group sits among a row's per-lane lo values
// (G per lane: lane (col >> 6) & 31, group (col >> gs) within its chunk).
template <int G>
__device__ __forceinline__ int lo_index(int col, int gs) {
  if constexpr (G == 1) return (col >> 6) & 31;
  else return ((col >> 6) & 31) * G + ((col >> gs) & (G - 1));
}

// Held-out entries of NR consecutive rows of the warp's row class in its K
// slice: row u owns entries [o_lo, o_hi) of the CTA's side record, handled by
// the 32 / NR lanes of group u (lane / (32 / NR)). Adds x~_c (v - lo_M) to
// v[u]; lo_M of column c's group is read from lo_s[u][c's lane][group], where
// every lane of the warp left its own lo_M per row and group.
// The correction factor of entry `en` of row ur: v - lo_M for a pre-grid
// entry, r + (lo - lo_M) for a post-grid one (bit 15), Eq. (4).
// Kernels of a matrix with post-grid entries (POST) use it; the others keep
// the plain pre-grid expression (bit 15 is never set there).
template <int G>
__device__ __forceinline__ float entry_delta(uint32_t en, int col, const float* lo_row, int gs, const PostCtx& pc,
                                             int ur) {
  const float v = __half2float(__ushort_as_half((unsigned short)(en >> 16)));
  if (en & 0x8000u) return v + __ldg(pc.dlo + pc.prow[ur * pc.pstep + (col >> gs)]);
  return v - lo_row[lo_index<G>(col, gs)];
}

template <int NR, int G, bool POST>
__device__ __forceinline__ void side_record(int o_lo, int o_hi, const uint32_t* ents, const int16_t* xq,
                                            const float* xscale, const float* lo_s, int lane, int gs,
                                            const PostCtx& pc, float (&v)[NR]) {
  constexpr int LPR = 32 / NR;  // lanes per row
  const int ur = lane / LPR;
  const float* lo_row = lo_s + ur * 32 * G;
  float cs = 0.f;
  for (int j = o_lo + lane % LPR; __any_sync(kFull, j < o_hi); j += LPR) {
    if (j < o_hi) {
      const uint32_t en = ents[j];
      const int col = (int)(en & (POST ? 0x7FFFu : 0xFFFFu));  // bit 15: post-grid flag
      const float xv = (float)xq[xq_elem(col)] * xscale[col >> 6];
      if constexpr (POST) cs = fmaf(xv, entry_delta<G>(en, col, lo_row, gs, pc, ur), cs);
      else cs = fmaf(xv, __half2float(__ushort_as_half((unsigned short)(en >> 16))) - lo_row[lo_index<G>(col, gs)], cs);
    }
  }
#pragma unroll
  for (int i = 0; i < NR; ++i) v[i] += ur == i ? cs : 0.f;
}

// As side_record for NB activation vectors: v[j][u] += x~_j,c (v - lo_M).
template <int NR, int NB, int G, bool POST>
__device__ __forceinline__ void side_record_nb(int o_lo, int o_hi, const uint32_t* ents, const int16_t* xq,
                                               const float* xscale, int in, int nchunk, const float* lo_s, int lane,
                                               int gs, const PostCtx& pc, float (&v)[NB][NR]) {
  constexpr int LPR = 32 / NR;  // lanes per row
  const int ur = lane / LPR;
  const float* lo_row = lo_s + ur * 32 * G;
  float cs[NB];
#pragma unroll
  for (int j = 0; j < NB; ++j) cs[j] = 0.f;
  for (int e = o_lo + lane % LPR; __any_sync(kFull, e < o_hi); e += LPR) {
    if (e < o_hi) {
      const uint32_t en = ents[e];
      const int col = (int)(en & (POST ? 0x7FFFu : 0xFFFFu));  // bit 15: post-grid flag
      float d;
      if constexpr (POST) d = entry_delta<G>(en, col, lo_row, gs, pc, ur);
      else d = __half2float(__ushort_as_half((unsigned short)(en >> 16))) - lo_row[lo_index<G>(col, gs)];
      const int xe = xq_elem(col);
#pragma unroll
      for (int j = 0; j < NB; ++j) cs[j] = fmaf((float)xq[j * in + xe] * xscale[j * nchunk + (col >> 6)], d, cs[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < NB; ++j)
#pragma unroll
    for (int i = 0; i < NR; ++i) v[j][i] += ur == i ? cs[j] : 0.f;
}

// The UP rows (or, for a short block, `mine` rows one at a time) of one block
// for this lane's chunk: dot products, side record, and the cross-lane sums
// into pout[u * pstep + j] (row u, vector j).
template <int M, int NR, int NB, int G, bool POST>
__device__ __forceinline__ void block_rows(const uint32_t (&X)[32], float xs, const float (&xsg)[G], const int16_t* xq,
                                           const float* xscale, const float* xsum, const float* xsum16, int in,
                                           int nchunk, int cc, bool active, const uint8_t* sb, RowOffsets off,
                                           RowOffsets step, uint32_t plane_stride, const float2* tab, int mine,
                                           const int32_t* o, const uint32_t* ents, float* lo_w, int lane, int gs,
                                           const float* dlo, float* pout, int pstep,
                                           const int32_t (&mem_row)[kMaxStack], int grow0, int rstep) {
  // global row of the warp's row u: grow0 + rstep u; each row reads its member's pair table
  const float2* tb[NR];
#pragma unroll
  for (int u = 0; u < NR; ++u) tb[u] = tab + member_table_offset(mem_row, grow0 + rstep * u);
  float v[NB][NR], lo[NR][G];
  if constexpr (NB == 1) {
    rows_dot<M, NR, G>(X, xs, xsg, sb, off, step, plane_stride, tb, v[0], lo);
  } else {
    rows_dot_nb<M, NR, NB, G>(xq, xscale, xsum, xsum16, in, nchunk, cc, active, sb, off, step, plane_stride, tb, v,
                              lo);
  }
#pragma unroll
  for (int u = 0; u < NR; ++u)
#pragma unroll
    for (int g = 0; g < G; ++g) lo_w[(u * 32 + lane) * G + g] = lo[u][g];
  __syncwarp();
  const int ur = lane / (32 / NR);
  PostCtx pc = {nullptr, 0u, nullptr};
  if constexpr (POST)  // read by post-grid entries only; lane group ur holds row ur
    pc = {sb + off.g - ((cc * kChunk) >> gs), step.g, dlo + member_table_offset(mem_row, grow0 + rstep * ur)};
  if constexpr (NB == 1) {
    side_record<NR, G, POST>(o[ur < mine ? ur : mine], o[ur + 1 < mine ? ur + 1 : mine], ents, xq, xscale, lo_w, lane, gs,
                       pc, v[0]);
  } else {
    side_record_nb<NR, NB, G, POST>(o[ur < mine ? ur : mine], o[ur + 1 < mine ? ur + 1 : mine], ents, xq, xscale, in,
                              nchunk, lo_w, lane, gs, pc, v);
  }
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    const float s = transposed_reduce<NR>(v[j], lane);
    if ((lane & (32 / NR - 1)) == 0 && ur < mine) pout[ur * pstep + j] = s;
  }
}

template <int M, int UP, int NB, int G, bool POST, bool SC>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) gemv_kernel(const GemvKernelArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const GemvPlan& P = a.plan;
  const int in = a.m.in;
  const int nchunk = in / kChunk;
  const SmemLayout L = smem_layout(P, in, M);
  const uint32_t sbase = smem_addr(smem);
  float2* tab = reinterpret_cast<float2*>(smem + L.tab);
  int16_t* xq = reinterpret_cast<int16_t*>(smem + L.xq);
  float* xscale = reinterpret_cast<float*>(smem + L.xscale);
  float* xsum = reinterpret_cast<float*>(smem + L.xsum);
  float* xsum16 = reinterpret_cast<float*>(smem + L.xsum16);
  float* partial = reinterpret_cast<float*>(smem + L.partial);  // [slot][BR][KW]
  float* lo_w = reinterpret_cast<float*>(smem + L.lo) + 32 * UP * G * (threadIdx.x >> 5);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + L.cnt);
  int* last = reinterpret_cast<int*>(smem + L.last);
  const uint32_t full0 = sbase + L.bar, side_bar = sbase + L.bar + 8 * kMaxSlots;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthreads = blockDim.x;
  const int KW = P.KW, RG = P.RG, NW = P.NW, NS = P.ns, BR = P.br, ps = P.pair_stride;
  const int kw = warp % KW, rg = warp / KW;
  const int c = kw * 32 + lane;  // this lane's 64-weight chunk
  const bool active = c < nchunk;
  const int cc = active ? c : 0;  // reads of inactive lanes stay inside the row
  const int r0 = (int)((int64_t)blockIdx.x * a.m.out / gridDim.x);
  const int rows = (int)((int64_t)(blockIdx.x + 1) * a.m.out / gridDim.x) - r0;
  const int nblk = (rows + BR - 1) / BR;
  const int rb = in / 4, rp = in / 8;
  const uint8_t* side_g = a.m.side + (int64_t)blockIdx.x * a.m.side_stride;
  const uint8_t* side = P.stage_side ? smem + L.side : side_g;
  // (row class rg, K slice kw) run offsets: row m of the class starts at seg[m]
  const int32_t* seg = reinterpret_cast<const int32_t*>(side) + (rg * KW + kw) * (P.class_rows + 1);
  const uint32_t* ents = reinterpret_cast<const uint32_t*>(side + a.m.side_ent_off);

  // Block b of the CTA's rows -> slot b % NS (one thread).
  auto issue_block = [&](int b, int slot) {
    const int lr0 = b * BR;
    const int nr = min(BR, rows - lr0);
    const uint32_t dst = sbase + L.ring + slot * L.slot, bar = full0 + 8 * slot;
    mbar_arrive_expect_tx(bar, (uint32_t)nr * (rb + (M - 2) * rp + ps));
    bulk_load(dst, a.m.base + (int64_t)(r0 + lr0) * rb, nr * rb, bar);
#pragma unroll
    for (int k = 0; k < M - 2; ++k)
      bulk_load(dst + L.plane_piece + k * BR * rp, a.m.plane[k] + (int64_t)(r0 + lr0) * rp, nr * rp, bar);
    bulk_load(dst + L.pair_piece, a.m.pair + (int64_t)(r0 + lr0) * ps, nr * ps, bar);
    last[slot] = b;
  };

  // Thread 0 sets up the barriers and starts the copies that do not depend
  // on the previous kernel: the pair table, the side record and block 0. The
  // other blocks follow once this CTA's x loads are on their way, so that x
  // does not queue behind them. (Every thread passes the barrier after the x
  // conversion before it waits on an mbarrier.)
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      cnt[s] = 0;
      last[s] = -1;
    }
    mbar_init(side_bar, 1);
    mbar_init(side_bar + 8, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(side_bar, 256 * 8 * (uint32_t)P.nmem + (P.stage_side ? (uint32_t)a.m.side_stride : 0u));
    bulk_load(sbase + L.tab, a.table, 256 * 8 * (uint32_t)P.nmem, side_bar);
    if (P.stage_side) bulk_load(sbase + L.side, side_g, (uint32_t)a.m.side_stride, side_bar);
    issue_block(0, 0);
  }
  grid_launch_dependents();
  grid_dependency_wait();  // x may come from the previous kernel; y may be read by it

  // x -> 16-bit fixed point, once per CTA: a task is a quarter chunk (16
  // values) and the 4 tasks of a chunk sit in adjacent lanes. Scale 2^e with
  // max|x| 2^e in [2^14, 2^15) per chunk, so the largest entries convert
  // exactly; rounding to nearest even goes through the 1.5 * 2^23 shifter (the
  // low 16 bits of the sum are the two's-complement integer).
  {
    constexpr int kBatch = 4;
    const int tpv = 4 * nchunk;  // tasks per vector
    const int ntask = tpv * NB;
    const uint4* x4 = reinterpret_cast<const uint4*>(a.x);
    const float4* s4 = reinterpret_cast<const float4*>(a.in_scale);
    for (int t0 = 0; t0 < ntask; t0 += kBatch * nthreads) {
      uint4 raw[kBatch][2];
      float4 sv[kBatch][4];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int t = t0 + q * nthreads + tid;
        raw[q][0] = raw[q][1] = make_uint4(0u, 0u, 0u, 0u);
        if (t < ntask) {  // x is [NB][in]: task t of the flat list reads 16 values from 16 t on
          raw[q][0] = __ldg(x4 + 2 * t);
          raw[q][1] = __ldg(x4 + 2 * t + 1);
        }
        if constexpr (SC) {  // the scale of the task's channels (16 (t mod tpv) on)
          const int ts = t < ntask ? t % tpv : 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) sv[q][k] = __ldg(s4 + 4 * ts + k);
        }
      }
      if (t0 == 0 && tid == 0)
        for (int b = 1; b < NS && b < nblk; ++b) issue_block(b, b);
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int tw = t0 + q * nthreads + warp * 32;  // first task of this warp
        if (tw >= ntask) break;                         // warp-uniform
        const int t = tw + lane;
        uint32_t Q[8];
        float xs_c;
        int sum16, sumq;
        convert_x_task<SC>(raw[q], sv[q], Q, xs_c, sum16, sumq);
        if (t < ntask) {
          const int j = t / tpv, tt = t - j * tpv;  // vector, task within it
          uint4* dst = reinterpret_cast<uint4*>(xq + j * in);
          dst[xq_piece(tt >> 2, 2 * (tt & 3))] = make_uint4(Q[0], Q[1], Q[2], Q[3]);
          dst[xq_piece(tt >> 2, 2 * (tt & 3) + 1)] = make_uint4(Q[4], Q[5], Q[6], Q[7]);
          if constexpr (G > 1) xsum16[t] = xs_c * (float)sum16;  // t = 4 (j nchunk + c) + q
          if ((tt & 3) == 0) {
            xscale[j * nchunk + (tt >> 2)] = xs_c;
            xsum[j * nchunk + (tt >> 2)] = xs_c * (float)sumq;
          }
        }
      }
    }
  }
  __syncthreads();
  uint32_t X[32];  // one vector: this lane's x~ stays in registers (more vectors: read per block)
  float xs = 0.f, xsg[G];
#pragma unroll
  for (int g = 0; g < G; ++g) xsg[g] = 0.f;
  if constexpr (NB == 1) {
    const uint4* src = reinterpret_cast<const uint4*>(xq);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 t = src[xq_piece(cc, k)];
      X[4 * k] = t.x;
      X[4 * k + 1] = t.y;
      X[4 * k + 2] = t.z;
      X[4 * k + 3] = t.w;
    }
    xs = active ? xscale[cc] : 0.f;
    if constexpr (G == 1) {
      xsg[0] = active ? xsum[cc] : 0.f;
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < 4 / G; ++q) t += xsum16[4 * cc + (4 / G) * g + q];  // exact: multiples of one 2^-e
        xsg[g] = active ? t : 0.f;
      }
    }
  }

  // Where this warp's rows sit in a slot (row u of the warp = block row rg + RG u).
  const RowOffsets off = {(uint32_t)(rg * rb + cc * 16), (uint32_t)(L.plane_piece + rg * rp + cc * 8),
                          (uint32_t)(L.pair_piece + rg * ps + ((cc * kChunk) >> P.group_shift))};
  const RowOffsets step = {(uint32_t)(RG * rb), (uint32_t)(RG * rp), (uint32_t)(RG * ps)};
  const uint32_t plane_stride = BR * rp;

  // The lanes of a warp leave together: the block code below uses full-warp
  // shuffles and __syncwarp.
  bool ok = __all_sync(kFull, mbar_wait(side_bar, 0, kWaitLimitNs));
  // Test hook (stagq_debug_stall): every warp takes one bounded wait that runs
  // out, so that the give-up path below runs on a healthy launch.
  if (a.m.debug_stall_ns && !__all_sync(kFull, mbar_wait(side_bar + 8, 0, a.m.debug_stall_ns))) ok = false;
  const uint8_t* ring_g = smem + L.ring;
  int slot = 0;
  uint32_t phase = 0, round = 0;
  for (int b = 0; ok && b < nblk; ++b) {
    if (!__all_sync(kFull, mbar_wait(full0 + 8 * slot, phase, kWaitLimitNs))) {
      ok = false;
      break;
    }
    const uint8_t* sb = ring_g + slot * L.slot;
    const int nr = min(BR, rows - b * BR);
    float* pout = partial + ((slot * BR + rg) * KW + kw) * NB;
    const int pstep = RG * KW * NB;
    const int32_t* o = seg + UP * b;  // this block's rows of the class
    // my rows in this block; a short block runs as a full one with the
    // missing rows masked, unless fewer than half of them are there
    const int mine = nr == BR ? UP : (nr > rg ? (nr - rg + RG - 1) / RG : 0);
    if (mine == UP || 2 * mine > UP) {
      block_rows<M, UP, NB, G, POST>(X, xs, xsg, xq, xscale, xsum, xsum16, in, nchunk, cc, active, sb, off, step,
                               plane_stride, tab, mine, o, ents, lo_w, lane, P.group_shift, a.dlo, pout, pstep,
                               a.m.mem_row, r0 + b * BR + rg, RG);
    } else {
      for (int u = 0; u < mine; ++u) {
        const RowOffsets ou = {off.b + u * step.b, off.p + u * step.p, off.g + u * step.g};
        block_rows<M, 1, NB, G, POST>(X, xs, xsg, xq, xscale, xsum, xsum16, in, nchunk, cc, active, sb, ou, step,
                                plane_stride, tab, 1, o + u, ents, lo_w, lane, P.group_shift, a.dlo, pout + u * pstep,
                                pstep, a.m.mem_row, r0 + b * BR + rg + RG * u, RG);
        __syncwarp();  // lo_w is rewritten by the next row
      }
    }
    __syncwarp();  // lo_w is rewritten by the next block
    // Done with the slot: the warp that finishes it last stores the block's
    // rows of y and refills the slot.
    __syncwarp();
    uint32_t done = 0;
    if (lane == 0) {
      __threadfence_block();
      done = atomicAdd(cnt + slot, 1u) + 1u;
    }
    done = __shfl_sync(kFull, done, 0);
    if (done == (uint32_t)NW * (round + 1)) {
      __threadfence_block();
      if (lane < nr) {
        const float* pr = partial + (slot * BR + lane) * KW * NB;
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          float acc = 0.f;
          for (int k = 0; k < KW; ++k) acc += pr[k * NB + j];
          const int64_t yi = (int64_t)j * a.m.out + r0 + b * BR + lane;
          if (a.y_f32) reinterpret_cast<float*>(a.y)[yi] = acc;
          else reinterpret_cast<__half*>(a.y)[yi] = __float2half_rn(acc);
        }
      }
      __syncwarp();
      if (lane == 0 && b + NS < nblk) issue_block(b + NS, slot);
    }
    if (++slot == NS) {
      slot = 0;
      phase ^= 1u;
      ++round;
    }
  }
  if (!ok && lane == 0) atomicOr(a.m.status, 1u);
  if (__syncthreads_or(!ok) && tid == 0) {
    // Gave up: let this CTA's copies in flight land before it exits.
    mbar_wait(side_bar, 0, kDrainLimitNs);
    for (int s = 0; s < NS; ++s)
      if (last[s] >= 0) mbar_wait(full0 + 8 * s, (uint32_t)(last[s] / NS) & 1u, kDrainLimitNs);
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
  static size_t granted[kMaxDev][768] = {};  // key < 720: (M - 2, rows per warp, vectors, groups, post, scaled)
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDev || key < 0 || key >= 768) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lock(mu);
  if (granted[dev][key] >= smem) return cudaSuccess;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  // The largest shared-memory carve-out, as the single-vector kernel asks:
  // consecutive GEMVs of either kernel then run under one L1 / shared split
  // and can share an SM without reconfiguring it.
  if (err == cudaSuccess) err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (err == cudaSuccess) granted[dev][key] = smem;
  return err;
}

template <int M, int UP, int NB, int G, bool SC>
cudaError_t launch_gemv_mu(const DeviceMatrix& m, const GemvPlan& plan, const void* x, const float* in_scale, void* y,
                           int y_f32, cudaStream_t stream) {
  GemvKernelArgs a;
  a.m = m;
  a.plan = plan;
  a.table = m.tables + 256 * m.nmem * (M - 2);
  a.dlo = m.dlo + 256 * m.nmem * (M - 2);
  a.x = reinterpret_cast<const __half*>(x);
  a.in_scale = in_scale;
  a.y = y;
  a.y_f32 = y_f32;
  const SmemLayout L = smem_layout(plan, m.in, M);
  // every region that bulk copies fill or 16-byte accesses read starts on 16 bytes
  if ((L.tab | L.xq | L.side | L.ring | L.slot | L.plane_piece | L.pair_piece) & 15u) return cudaErrorInvalidValue;
  auto kern = m.has_post ? gemv_kernel<M, UP, NB, G, true, SC> : gemv_kernel<M, UP, NB, G, false, SC>;
  const int key = (((((M - 2) * 3 + (UP == 4 ? 2 : UP - 1)) * 4 + (NB - 1)) * 3 + (G == 4 ? 2 : G - 1)) * 2 +
                   (m.has_post ? 1 : 0)) * 2 + (SC ? 1 : 0);
  cudaError_t err = ensure_smem(reinterpret_cast<const void*>(kern), key, L.total);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)plan.grid);
  cfg.blockDim = dim3((unsigned)(32 * plan.NW));
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = plan.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int M, bool SC>
cudaError_t launch_gemv_m(const DeviceMatrix& m, const GemvPlan& plan, const void* x, const float* in_scale, void* y,
                          int y_f32, cudaStream_t stream) {
  // Instances the planner can select (see make_plan): more vectors or deeper
  // reads take fewer rows per warp, so that the registers do not spill;
  // groups below 64 weights take one row per warp.
  const int G = groups_per_chunk(plan.group_shift);
  if (G > 1) {
    if (plan.up != 1) return cudaErrorInvalidValue;
    switch (G * 8 + plan.nb) {
      case 16 + 1: return launch_gemv_mu<M, 1, 1, 2, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 16 + 2: return launch_gemv_mu<M, 1, 2, 2, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 16 + 3: return launch_gemv_mu<M, 1, 3, 2, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 16 + 4: return launch_gemv_mu<M, 1, 4, 2, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 32 + 1: return launch_gemv_mu<M, 1, 1, 4, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 32 + 2: return launch_gemv_mu<M, 1, 2, 4, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 32 + 3: return launch_gemv_mu<M, 1, 3, 4, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 32 + 4: return launch_gemv_mu<M, 1, 4, 4, SC>(m, plan, x, in_scale, y, y_f32, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (plan.nb == 1) {
    if (plan.up == 1) return launch_gemv_mu<M, 1, 1, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
    if (plan.up == 2) return launch_gemv_mu<M, 2, 1, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
    if (plan.up == 4) return launch_gemv_mu<M, 4, 1, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
    return cudaErrorInvalidValue;
  }
  if constexpr (M >= 5) {
    if (plan.up != 1) return cudaErrorInvalidValue;
    switch (plan.nb) {
      case 2: return launch_gemv_mu<M, 1, 2, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 3: return launch_gemv_mu<M, 1, 3, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 4: return launch_gemv_mu<M, 1, 4, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      default: return cudaErrorInvalidValue;
    }
  } else {
    const int k = (plan.up == 4 ? 2 : plan.up - 1) * 4 + plan.nb;
    switch (k) {
      case 2: return launch_gemv_mu<M, 1, 2, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 3: return launch_gemv_mu<M, 1, 3, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 4: return launch_gemv_mu<M, 1, 4, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 6: return launch_gemv_mu<M, 2, 2, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 7: return launch_gemv_mu<M, 2, 3, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 8: return launch_gemv_mu<M, 2, 4, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      case 10: return launch_gemv_mu<M, 4, 2, 1, SC>(m, plan, x, in_scale, y, y_f32, stream);
      default: return cudaErrorInvalidValue;
    }
  }
}

template <int M>
cudaError_t launch_gemv_m(const DeviceMatrix& m, const GemvPlan& plan, const void* x, const float* in_scale, void* y,
                          int y_f32, cudaStream_t stream) {
  return in_scale ? launch_gemv_m<M, true>(m, plan, x, in_scale, y, y_f32, stream)
                  : launch_gemv_m<M, false>(m, plan, x, nullptr, y, y_f32, stream);
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

int k_slices(int in) { return (in / kChunk + 31) / 32; }

int gemv_grid(int out, int in, int num_sms) {
  // Large matrices: two CTAs per SM (while a CTA has <= 8 warps), so one
  // computes while the other starts or finishes. Small ones: one CTA per SM,
  // which leaves room for the next GEMV's CTA to start early beside it.
  const bool two = k_slices(in) <= kMaxWarps / 2 && (int64_t)out * in >= kTwoCtaWeightsPerSm * (int64_t)num_sms;
  const int per_sm = two ? 2 : 1;
  int g = out < per_sm * num_sms ? out : per_sm * num_sms;
  if ((out + g - 1) / g > kMaxRowsPerCta) g = (out + kMaxRowsPerCta - 1) / kMaxRowsPerCta;
  return g;
}

bool make_plan(const DeviceMatrix& m, int bits, int nb, GemvPlan* p) {
  GemvPlan q = {};
  if (nb < 1 || nb > 4) return false;
  q.nb = nb;
  q.KW = k_slices(m.in);
  if (q.KW < 1 || q.KW > kMaxWarps) return false;
  q.RG = row_groups(q.KW);
  q.NW = q.KW * q.RG;
  q.grid = m.side_grid;
  q.rows_cap = (m.out + q.grid - 1) / q.grid;
  q.class_rows = (q.rows_cap + q.RG - 1) / q.RG;
  q.pair_stride = m.pair_stride;
  q.side_stride = m.side_stride;
  q.group_shift = 0;
  while ((1 << q.group_shift) < m.group) ++q.group_shift;
  q.pdl = 1;
  q.nmem = m.nmem;
  // Rows per warp per block: up to 4, but no more than the CTA's rows call for.
  const int per_rg = (q.rows_cap + q.RG - 1) / q.RG;
  int up_max = per_rg >= 4 ? 4 : per_rg >= 2 ? 2 : 1;
  // registers: rows x vectors x planes (the instances launch_gemv_m provides)
  if (nb >= 2 && bits >= 5) up_max = 1;
  else if (nb >= 3 && up_max > 2) up_max = 2;
  if (q.group_shift < 6) up_max = 1;  // groups below 64 weights: G pairs and lo values per row
  // Shared memory: small enough for two CTAs per SM when the CTA has <= 8
  // warps, else (or if nothing fits) the per-block maximum. Prefer the side
  // record staged, then at least three slots (or one per block), then more
  // rows per warp.
  const int budgets[2] = {q.NW <= kMaxWarps / 2 ? m.smem_pair_budget : m.smem_limit, m.smem_limit};
  for (int bi = 0; bi < 2; ++bi) {
    for (int stage = 1; stage >= 0; --stage) {
      bool have = false;
      GemvPlan best = q;
      for (int up = up_max; up >= 1; up /= 2) {
        GemvPlan t = q;
        t.up = up;
        t.br = q.RG * up;
        t.stage_side = stage;
        const int nblk = (q.rows_cap + t.br - 1) / t.br;
        t.ns = nblk < kMaxSlots ? nblk : kMaxSlots;
        while (t.ns >= 1 && smem_layout(t, m.in, bits).total > (uint32_t)budgets[bi]) --t.ns;
        if (t.ns < 1) continue;
        if (t.ns >= (nblk < 3 ? nblk : 3)) {
          *p = t;
          return true;
        }
        if (!have || t.ns > best.ns) {
          best = t;
          have = true;
        }
      }
      if (have) {
        *p = best;
        return true;
      }
    }
  }
  return false;
}

cudaError_t launch_gemv(const DeviceMatrix& m, const GemvPlan& plan, int bits, const void* x, const float* in_scale,
                        void* y, int y_f32, cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_gemv_m<2>(m, plan, x, in_scale, y, y_f32, stream);
    case 3: return launch_gemv_m<3>(m, plan, x, in_scale, y, y_f32, stream);
    case 4: return launch_gemv_m<4>(m, plan, x, in_scale, y, y_f32, stream);
    case 5: return launch_gemv_m<5>(m, plan, x, in_scale, y, y_f32, stream);
    case 6: return launch_gemv_m<6>(m, plan, x, in_scale, y, y_f32, stream);
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
