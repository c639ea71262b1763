// sm_100a kernel of the StagQ GEMV for one activation vector, y = W_hat^(M) x.
//
// What is computed (StagQ paper, arXiv 2610.05977): for every row i,
//   y_i = sum_groups [ s_M(g) * sum_{j in g} u_M,j x_j + lo_M(g) * sum_{j in g} x_j ]
//         + sum_{held-out (i,c)} x_c (v_ic - lo_M(g(i,c)))
// -- the affine map of Eq. (10) applied once per group, with u_M from Eq. (8),
// and the side record of Eq. (4) (held-out digits are zero, so the main
// stream decoded lo_M there and the correction is v - lo_M).
//
// How (for B200; batch-one GEMV is bound by HBM and by the SM's integer issue
// rate, so no tensor cores):
//  * One CTA per SM owns a contiguous, balanced range of rows, cut into blocks
//    of BR rows. Warp 0 is the producer: it moves each block's base rows and
//    read-plane rows (a p_M read never touches deeper planes) into a shared-
//    memory ring slot with 1 + (M - 2) bulk copies. Warps 1..NW are consumers:
//    KW K slices (2048 weights: 32 lanes x one 64-weight chunk) x RG row
//    groups; in every block a consumer takes UP rows of its group in its slice.
//  * The CTA has the SM to itself, with as many consumer warps as the
//    register file holds (make_plan1); with programmatic dependent launch it
//    starts as soon as the previous launch's CTA on its SM has left, and its
//    copies -- weights, pair table, the CTA's pair bytes and side record, none
//    of which depend on earlier kernels -- are in flight while the previous
//    grid drains.
//  * x is converted once per CTA to 16-bit fixed point with a power-of-two
//    scale per 64-element chunk (|error| <= 2^-16 max|x_chunk|); each lane keeps
//    its chunk's 64 activations in registers; code bytes / nibble composites
//    (layout.cuh) feed dp2a integer dot products (exact in int32) and the group
//    affine is applied once per chunk in fp32.
//  * Two shuffle stages leave 8 partial sums per (row, K slice) in shared
//    memory, and the slot goes back to the producer.
//  * The held-out entries are taken apart from the blocks, where they would
//    add a chain of dependent shared-memory reads to every block. T lanes per
//    row (T = 32 / rows per warp, as many as the CTA's threads allow) each sum
//    a share of the row's terms x~_c (v - lo_M), and a fixed shuffle tree adds
//    the shares: right after the x conversion, into one float per row, where
//    the CTA refills ring slots (the later slots land meanwhile); otherwise in
//    the final pass.
//  * Finally T lanes per row add the row's partials the same way, with the
//    row's held-out terms, and the row's first lane stores y: deterministic,
//    no atomics on data, no workspace, one launch.
//  * x is read before the copies of all but the first block are issued: those
//    copies would otherwise delay the L2 reads of x that every warp waits for.
//  * Every mbarrier wait is bounded in time; on expiry the kernel records it
//    in the handle's status word, waits (bounded) for its own copies and
//    returns.
#include <cuda_fp16.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "device_matrix.hpp"
#include "kernel_common.cuh"
#include "layout.cuh"

namespace stagq {
namespace {

using namespace kernels;

constexpr int kRegs1 = 128;            // registers per thread: one CTA of up to 16 warps per SM
constexpr int kParts1 = 8;             // partial sums per (row, K slice), each over 4 lanes

struct Gemv1Args {
  DeviceMatrix m;
  Gemv1Plan plan;
  const float2* table;  // (lo_M, s_M c_M) of this precision
  const float* dlo;     // lo - lo_M of this precision (post-grid entries)
  const __half* x;
  const float* in_scale;  // SC: per-channel multiplier of x (the inverse activation scale)
  void* y;
  int y_f32;
};

constexpr uint64_t kWaitLimit1Ns = 2000000000ull;  // a copy that has not landed in 2 s never will
constexpr uint64_t kDrainLimit1Ns = 100000000ull;  // after a failure: wait for own copies, 0.1 s

// Floats per row of K-slice partials. One vector: KW x 8 padded to an odd
// multiple of 4, so that 8 threads reading consecutive rows with 16-byte loads
// hit 8 different bank groups. nb vectors: one float per (K slice, vector),
// padded to an odd count.
__host__ __device__ inline int part_stride1(int KW, int nb) {
  return nb == 1 ? KW * kParts1 + 4 : (KW * nb) | 1;
}

struct Smem1 {
  uint32_t full, empty, side_bar, flag, stall, tab, xq, xscale, xsum, xsum16, pairs, side, part, rowterm, ring;
  uint32_t slot;         // bytes of one ring slot
  uint32_t plane_piece;  // offset of the first read plane inside a slot (base rows at 0)
  uint32_t total;
};

__host__ __device__ inline uint32_t up16(uint32_t v) { return (v + 15u) & ~15u; }

__host__ __device__ inline Smem1 smem1(const Gemv1Plan& p, int in, int M) {
  Smem1 L;
  const uint32_t nchunk = in / kChunk, BR = p.br, rc = (uint32_t)p.rows_cap, nb = (uint32_t)p.nb;
  uint32_t o = 0;
  L.full = o; o += 8 * kMaxSlots;    // block landed in the slot (producer arrive + bytes)
  L.empty = o; o += 8 * kMaxSlots;   // every consumer warp is done with the slot
  L.side_bar = o; o += 8;            // pair table, pair bytes and side record landed
  L.flag = o; o += 8;                // a wait gave up (any thread)
  L.stall = o; o += 8;               // test hook: a barrier nothing completes
  o = up16(o);                       // bulk-copy destinations and 16-byte accesses from here on
  L.tab = o; o += 256 * 8 * (uint32_t)p.nmem;  // the pair table of each stacked member
  L.xq = o; o += 2 * in * nb;        // x~ of every vector, vector-major
  L.xscale = o; o += 4 * nchunk * nb;
  L.xsum = o; o += 4 * nchunk * nb;
  // per 16 values: groups < 64, or half chunks (several vectors)
  L.xsum16 = o; o += (p.group_shift < 6 || nb > 1) ? 16 * nchunk * nb : 0u;
  o = up16(o);
  L.pairs = o; o += up16(rc * (uint32_t)p.pair_stride);
  L.side = o; o += p.stage_side ? (uint32_t)p.side_stride : 0u;
  o = up16(o);
  L.part = o; o += 4u * rc * (uint32_t)part_stride1(p.KW, p.nb);
  L.rowterm = o; o += 4u * rc * nb;  // each row's sum of x~_c (v - lo_M) over its held-out entries, per vector
  o = (o + 127u) & ~127u;
  L.ring = o;
  L.plane_piece = BR * (in / 4);
  L.slot = (L.plane_piece + (uint32_t)(M - 2) * BR * (in / 8) + 127u) & ~127u;
  o += p.ns * L.slot;
  L.total = o;
  return L;
}

__device__ __forceinline__ void mbar_arrive1(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Cross-lane sums of the UP rows of a block: afterwards lane l holds, for row
// reduced_row1<UP>(l), the sum of its 4 lanes {l, l^8, l^16, l^24}; lanes with
// keeps_partial1<UP>(l) store it (8 partials per row).
template <int UP>
__device__ __forceinline__ float partial_reduce1(const float (&v)[UP], int lane) {
  const bool h16 = lane & 16, h8 = lane & 8;
  if constexpr (UP == 4) {
    const float s0 = (h16 ? v[2] : v[0]) + __shfl_xor_sync(kFull, h16 ? v[0] : v[2], 16);
    const float s1 = (h16 ? v[3] : v[1]) + __shfl_xor_sync(kFull, h16 ? v[1] : v[3], 16);
    return (h8 ? s1 : s0) + __shfl_xor_sync(kFull, h8 ? s0 : s1, 8);
  } else if constexpr (UP == 2) {
    const float s = (h16 ? v[1] : v[0]) + __shfl_xor_sync(kFull, h16 ? v[0] : v[1], 16);
    return s + __shfl_xor_sync(kFull, s, 8);
  } else {
    const float s = v[0] + __shfl_xor_sync(kFull, v[0], 16);
    return s + __shfl_xor_sync(kFull, s, 8);
  }
}
template <int UP>
__device__ __forceinline__ int reduced_row1(int lane) {
  return UP == 4 ? ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1) : UP == 2 ? (lane >> 4) & 1 : 0;
}
template <int UP>
__device__ __forceinline__ bool keeps_partial1(int lane) {
  return UP == 4 ? true : UP == 2 ? (lane & 8) == 0 : lane < 8;
}

// ---- several activation vectors: a lane takes half a chunk (32 weights) ----
// Half h of a chunk is base words 2h, 2h + 1 and word h of every plane
// (layout.cuh), so the code words below are those of chunk_codes for the word
// pair w = h, and the x~ of the half are chunk words 16 h .. 16 h + 15.

// The half chunk's masked code words, decoded once for every vector:
// cw[0..7] as chunk_codes for one word pair (M = 2: the bytes q of base word i,
// slot s, (word >> 2 s) & 0x03030303, at 4 i + s; M >= 3: the nibble
// composites' low / high nibbles), and
// for M >= 5 the plane-5 / plane-6 bits of base word i, slot s, at 4 i + s.
template <int M>
__device__ __forceinline__ void half_codes(uint2 B, const uint32_t* P, uint32_t (&cw)[8], uint32_t (&c5)[8],
                                           uint32_t (&c6)[8]) {
  if constexpr (M == 2) {  // shifted down to bytes q, so that one sum serves every slot
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      cw[s] = (B.x >> (2 * s)) & 0x03030303u;
      cw[4 + s] = (B.y >> (2 * s)) & 0x03030303u;
    }
  } else {
    uint32_t E0, O0, E1, O1;
    nibble_words(B.x, B.y, P[0], M >= 4 ? P[1] : 0u, E0, O0, E1, O1);
    cw[0] = E0 & 0x0F0F0F0Fu; cw[1] = E0 & 0xF0F0F0F0u;
    cw[2] = O0 & 0x0F0F0F0Fu; cw[3] = O0 & 0xF0F0F0F0u;
    cw[4] = E1 & 0x0F0F0F0Fu; cw[5] = E1 & 0xF0F0F0F0u;
    cw[6] = O1 & 0x0F0F0F0Fu; cw[7] = O1 & 0xF0F0F0F0u;
    if constexpr (M >= 5) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          c5[4 * i + s] = (P[2] >> (4 * i + s)) & 0x01010101u;
          if constexpr (M >= 6) c6[4 * i + s] = (P[3] >> (4 * i + s)) & 0x01010101u;
        }
    }
  }
}

// Four weights (local word i, slot s, j = 0..3) against X[8 i + 2 s] (j = 0, 1)
// and X[8 i + 2 s + 1] (j = 2, 3) of a half chunk's x~.
__device__ __forceinline__ int hdot4(const uint32_t (&X)[16], int i, int s, uint32_t m, int acc) {
  acc = dp2a_lo(X[8 * i + 2 * s], m, acc);
  return dp2a_hi(X[8 * i + 2 * s + 1], m, acc);
}

// sum of u_M x~ over the half chunk (the dp2a sequence of chunk_dot_g for one
// word pair), exact in int32.
template <int M>
__device__ __forceinline__ int half_dot(const uint32_t (&X)[16], const uint32_t (&cw)[8], const uint32_t (&c5)[8],
                                        const uint32_t (&c6)[8]) {
  if constexpr (M == 2) {
    int a0 = 0, a1 = 0;  // two chains for latency
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      a0 = hdot4(X, 0, s, cw[s], a0);
      a1 = hdot4(X, 1, s, cw[4 + s], a1);
    }
    return a0 + a1;
  } else {
    int lo = 0, hi = 0;
    lo = hdot4(X, 0, 1, cw[0], lo);
    hi = hdot4(X, 0, 3, cw[1], hi);
    lo = hdot4(X, 0, 0, cw[2], lo);
    hi = hdot4(X, 0, 2, cw[3], hi);
    lo = hdot4(X, 1, 1, cw[4], lo);
    hi = hdot4(X, 1, 3, cw[5], hi);
    lo = hdot4(X, 1, 0, cw[6], lo);
    hi = hdot4(X, 1, 2, cw[7], hi);
    const int nib = lo + (hi >> 4);  // high-nibble products are multiples of 16
    if constexpr (M <= 4) {
      return nib;
    } else {
      int a5 = 0, a6 = 0;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          a5 = hdot4(X, i, s, c5[4 * i + s], a5);
          if constexpr (M >= 6) a6 = hdot4(X, i, s, c6[4 * i + s], a6);
        }
      return M == 5 ? 2 * nib + a5 : 4 * nib + 2 * a5 + a6;
    }
  }
}

// Sums over the 32 lanes of N values per lane (N a power of two <= 32), in a
// fixed order: afterwards lane l holds the full sum of value l / (32 / N).
template <int N>
__device__ __forceinline__ float lane_sums(float (&v)[N], int lane) {
  int n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool up = lane & o;
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        if (k < n / 2) {
          const float send = up ? v[k] : v[k + n / 2], keep = up ? v[k + n / 2] : v[k];
          v[k] = keep + __shfl_xor_sync(kFull, send, o);
        }
      }
      n /= 2;
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], o);
    }
  }
  return v[0];
}

template <int M, int UP, int G, bool SC, int NB>
__global__ void __maxnreg__(kRegs1) gemv1_kernel(const Gemv1Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Gemv1Plan& P = a.plan;
  const int in = a.m.in;
  const int nchunk = in / kChunk;
  const Smem1 L = smem1(P, in, M);
  const uint32_t sbase = smem_addr(smem);
  const float2* tab = reinterpret_cast<const float2*>(smem + L.tab);
  int16_t* xq = reinterpret_cast<int16_t*>(smem + L.xq);
  float* xscale = reinterpret_cast<float*>(smem + L.xscale);
  float* xsum = reinterpret_cast<float*>(smem + L.xsum);
  float* xsum16 = reinterpret_cast<float*>(smem + L.xsum16);
  float* part = reinterpret_cast<float*>(smem + L.part);  // [row][part_stride1(KW)]: [KW][8] used
  float* rowterm = reinterpret_cast<float*>(smem + L.rowterm);
  volatile uint32_t* flag = reinterpret_cast<volatile uint32_t*>(smem + L.flag);
  const uint32_t full0 = sbase + L.full, empty0 = sbase + L.empty, side_bar = sbase + L.side_bar;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthreads = blockDim.x;
  const int KW = P.KW, NW = P.NW, NS = P.ns, BR = P.br, ps = P.pair_stride, gs = P.group_shift;
  const int nvec = NB == 1 ? 1 : P.nb;  // activation vectors (NB >= nvec registers' worth)
  const int PST = part_stride1(KW, nvec);
  // rows [b out / grid, (b + 1) out / grid) of CTA b, without a 64-bit division
  const uint32_t bx = blockIdx.x, gx = gridDim.x;
  const int f0 = (int)(bx * (uint32_t)P.rows_rem / gx), f1 = (int)((bx + 1) * (uint32_t)P.rows_rem / gx);
  const int r0 = (int)bx * P.rows_q + f0;
  const int rows = P.rows_q + f1 - f0;
  const int nblk = (rows + BR - 1) / BR;
  const int rb = in / 4, rp = in / 8;
  const uint8_t* side_g = a.m.side1 + (int64_t)blockIdx.x * P.side_stride;
  const uint8_t* pair_g = a.m.pair + (int64_t)r0 * ps;
  // Parameters of the later phases, read here with the first ones: the first
  // read of a parameter's cache line in a launch waits about as long as a
  // load from L2, and this way those waits overlap instead of adding up.
  const uint4* const x4 = reinterpret_cast<const uint4*>(a.x);
  const float4* const s4 = reinterpret_cast<const float4*>(a.in_scale);
  void* const yout = a.y;
  const float* const dlo = a.dlo;
  const int y_f32 = a.y_f32, has_post = a.m.has_post, out_rows = a.m.out;
  const uint32_t side_ent_off = (uint32_t)P.side_ent_off;
  asm volatile("" ::"l"(x4), "l"(s4), "l"(yout), "l"(dlo), "r"(y_f32), "r"(has_post), "r"(side_ent_off));
  const uint8_t* pairs = smem + L.pairs;
  const uint8_t* side = P.stage_side ? smem + L.side : side_g;

  int issued = 0;  // blocks issued so far (producer lane 0 = thread 0)
  // Block b of the CTA's rows -> slot b % NS (producer lane 0).
  auto issue_block = [&](int b, int slot) {
    const int lr0 = b * BR;
    const int nr = min(BR, rows - lr0);
    const uint32_t dst = sbase + L.ring + slot * L.slot, bar = full0 + 8 * slot;
    mbar_arrive_expect_tx(bar, (uint32_t)nr * (rb + (M - 2) * rp));
    bulk_load(dst, a.m.base + (int64_t)(r0 + lr0) * rb, nr * rb, bar);
#pragma unroll
    for (int k = 0; k < M - 2; ++k)
      bulk_load(dst + L.plane_piece + k * BR * rp, a.m.plane[k] + (int64_t)(r0 + lr0) * rp, nr * rp, bar);
    issued = b + 1;
  };

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, (uint32_t)NW);
    }
    mbar_init(side_bar, 1);
    mbar_init(sbase + L.stall, 1);
    *flag = 0u;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    // Nothing of this depends on earlier kernels: fill the ring before
    // waiting for them.
    const uint32_t pb = (uint32_t)(rows * ps);
    const uint32_t sb = P.stage_side ? (uint32_t)P.side_stride : 0u;
    mbar_arrive_expect_tx(side_bar, 256 * 8 * (uint32_t)P.nmem + pb + sb);
    bulk_load(sbase + L.tab, a.table, 256 * 8 * (uint32_t)P.nmem, side_bar);
    bulk_load(sbase + L.pairs, pair_g, pb, side_bar);
    if (sb) bulk_load(sbase + L.side, side_g, sb, side_bar);
    // Only the first block before x: the copies of later blocks would delay
    // the L2 reads of x that every warp waits for.
    if (nblk > 0) issue_block(0, 0);
  }
  grid_launch_dependents();
  grid_dependency_wait();  // x may come from the previous kernel; y may be read by it

  // x -> 16-bit fixed point, once per CTA (every warp): a task is a quarter
  // chunk (16 values) and the 4 tasks of a chunk sit in adjacent lanes. Scale
  // 2^e with max|x| 2^e in [2^14, 2^15) per chunk, so the largest entries
  // convert exactly; rounding to nearest even goes through the 1.5 * 2^23
  // shifter (the low 16 bits of the sum are the two's-complement integer).
  // With several vectors, task t is task t mod 4 nchunk of vector t / (4 nchunk)
  // and the chunks are numbered on across the vectors.
  {
    constexpr int kBatch = 4;
    const int tpv = 4 * nchunk, ntask = nvec * tpv;
    for (int t0 = 0; t0 < ntask; t0 += kBatch * nthreads) {
      uint4 raw[kBatch][2];
      float4 sv[kBatch][4];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int t = t0 + q * nthreads + tid;
        raw[q][0] = raw[q][1] = make_uint4(0u, 0u, 0u, 0u);
        if (t < ntask) {
          raw[q][0] = __ldg(x4 + 2 * t);
          raw[q][1] = __ldg(x4 + 2 * t + 1);
        }
        if constexpr (SC) {
#pragma unroll
          for (int k = 0; k < 4; ++k) sv[q][k] = t < ntask ? __ldg(s4 + 4 * (t % tpv) + k) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
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
          uint4* dst = reinterpret_cast<uint4*>(xq);
          dst[xq_piece(t >> 2, 2 * (t & 3))] = make_uint4(Q[0], Q[1], Q[2], Q[3]);
          dst[xq_piece(t >> 2, 2 * (t & 3) + 1)] = make_uint4(Q[4], Q[5], Q[6], Q[7]);
          if constexpr (G > 1 || NB > 1) xsum16[t] = xs_c * (float)sum16;
          if ((t & 3) == 0) {
            xscale[t >> 2] = xs_c;
            xsum[t >> 2] = xs_c * (float)sumq;
          }
        }
      }
    }
  }
  // x~ is complete; every warp takes the same branch on the pair table, pair
  // bytes and side record having landed.
  bool ok = __syncthreads_and(mbar_wait(side_bar, 0, kWaitLimit1Ns)) != 0;
  if (tid == 0)
    for (int b = issued; b < NS && b < nblk; ++b) issue_block(b, b);

  // T lanes per row (as many as the CTA's threads allow, up to a warp) for the
  // per-row passes below; rpw rows per warp at a time.
  int T = 32;
  while (T > 1 && rows * T > nthreads) T >>= 1;
  const int sub = lane & (T - 1), rpw = 32 / T;
  // ------------------------------------------------ per-row passes
  // Lane sub of a row's group takes the row's partials (float4) sub, sub + T,
  // ... (final pass) and its held-out entries sub, sub + T, ... (terms); a
  // pre-grid entry adds x~_c (v - lo_M), a post-grid entry (bit 15)
  // x~_c (r + lo - lo_M), Eq. (4). A fixed shuffle tree sums the T shares.
  // Where the CTA refills ring slots, the terms are summed before the blocks,
  // while the later slots are landing, into one float per row; otherwise in
  // the final pass, where they cost less than delaying the only blocks.
  const bool terms_first = nblk > NS;
  const int32_t* offs = reinterpret_cast<const int32_t*>(side);
  const uint32_t* ents = reinterpret_cast<const uint32_t*>(side + side_ent_off);
  auto row_pass = [&](auto with_post, bool terms, bool final) {
    if constexpr (NB == 1) {
      for (int rb = warp * rpw; rb < rows; rb += (nthreads / 32) * rpw) {  // warp-uniform trip count
        const int r = rb + lane / T;
        float t0 = 0.f, t1 = 0.f, t2 = 0.f, t3 = 0.f;
        if (r < rows && final) {
          const float4* pr = reinterpret_cast<const float4*>(part + r * PST);
          for (int k = sub; k < KW * kParts1 / 4; k += T) {
            const float4 q = pr[k];
            t0 += q.x; t1 += q.y; t2 += q.z; t3 += q.w;
          }
        }
        if (r < rows && terms) {
          const uint8_t* prow = pairs + r * ps;
          const int moff = member_table_offset(a.m.mem_row, r0 + r);
          auto term = [&](int j) {
            const uint32_t en = ents[j];
            const int col = (int)(en & 0x7FFFu);
            const int e = xq_elem(col);  // the column's x~ slot (same 64-chunk as the column)
            const int pb = prow[col >> gs] + moff;
            const float v = __half2float(__ushort_as_half((unsigned short)(en >> 16)));
            float d;
            if constexpr (decltype(with_post)::value) d = (en & 0x8000u) ? v + __ldg(dlo + pb) : v - tab[pb].x;
            else d = v - tab[pb].x;
            return (float)xq[e] * xscale[e >> 6] * d;
          };
          const int e1 = offs[r + 1];
          int j = offs[r] + sub;
          for (; j + 3 * T < e1; j += 4 * T) {
            t0 += term(j); t1 += term(j + T); t2 += term(j + 2 * T); t3 += term(j + 3 * T);
          }
          for (; j < e1; j += T) t0 += term(j);
        }
        float t = (t0 + t1) + (t2 + t3);
        for (int o = T >> 1; o >= 1; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
        if (sub == 0 && r < rows) {
          if (!final) {
            rowterm[r] = t;
          } else {
            if (!terms) t += rowterm[r];
            if (y_f32) reinterpret_cast<float*>(yout)[r0 + r] = t;
            else reinterpret_cast<__half*>(yout)[r0 + r] = __float2half_rn(t);
          }
        }
      }
    } else {
      // several vectors: one sum per vector, d computed once per entry
      for (int rb = warp * rpw; rb < rows; rb += (nthreads / 32) * rpw) {  // warp-uniform trip count
        const int r = rb + lane / T;
        float t[NB];
#pragma unroll
        for (int jv = 0; jv < NB; ++jv) t[jv] = 0.f;
        if (r < rows && final) {
          const float* pr = part + r * PST;
          for (int k = sub; k < KW; k += T) {
#pragma unroll
            for (int jv = 0; jv < NB; ++jv)
              if (jv < nvec) t[jv] += pr[k * nvec + jv];
          }
        }
        if (r < rows && terms) {
          const uint8_t* prow = pairs + r * ps;
          const int moff = member_table_offset(a.m.mem_row, r0 + r);
          const int e1 = offs[r + 1];
          for (int j = offs[r] + sub; j < e1; j += T) {
            const uint32_t en = ents[j];
            const int col = (int)(en & 0x7FFFu);
            const int pb = prow[col >> gs] + moff;
            const float v = __half2float(__ushort_as_half((unsigned short)(en >> 16)));
            float d;
            if constexpr (decltype(with_post)::value) d = (en & 0x8000u) ? v + __ldg(dlo + pb) : v - tab[pb].x;
            else d = v - tab[pb].x;
#pragma unroll
            for (int jv = 0; jv < NB; ++jv) {
              if (jv < nvec) {
                const int cg = jv * in + col;  // column of vector jv in the x~ of all vectors
                t[jv] += (float)xq[xq_elem(cg)] * xscale[cg >> 6] * d;
              }
            }
          }
        }
#pragma unroll
        for (int jv = 0; jv < NB; ++jv)
          for (int o = T >> 1; o >= 1; o >>= 1) t[jv] += __shfl_xor_sync(kFull, t[jv], o);
        if (sub == 0 && r < rows) {
#pragma unroll
          for (int jv = 0; jv < NB; ++jv) {
            if (jv >= nvec) break;
            if (!final) {
              rowterm[r * nvec + jv] = t[jv];
            } else {
              const float tt = terms ? t[jv] : t[jv] + rowterm[r * nvec + jv];
              const int64_t yo = (int64_t)jv * out_rows + r0 + r;
              if (y_f32) reinterpret_cast<float*>(yout)[yo] = tt;
              else reinterpret_cast<__half*>(yout)[yo] = __float2half_rn(tt);
            }
          }
        }
      }
    }
  };
  if (ok && terms_first) {
    if (has_post) row_pass(std::true_type{}, true, false);
    else row_pass(std::false_type{}, true, false);
  }

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    for (int b = 0; ok && b + NS < nblk; ++b) {
      // stops early when a consumer has given up (it releases no more slots)
      if (!__all_sync(kFull, mbar_wait_unless(empty0 + 8 * (b % NS), (uint32_t)(b / NS) & 1u, kWaitLimit1Ns, flag))) {
        ok = false;
        break;
      }
      if (lane == 0) issue_block(b + NS, b % NS);
      __syncwarp();
    }
  } else if (ok) {
    // ---------------------------------------------------------- consumers
    if constexpr (NB == 1) {
      const int cw = warp - 1;                 // consumer warp index
      const int kw = cw % KW, rg = cw / KW, RG = P.RG;
      const int c = kw * 32 + lane;            // this lane's 64-weight chunk
      const bool active = c < nchunk;
      const int cc = active ? c : 0;           // reads of inactive lanes stay inside the row
      uint32_t X[32];
      float xs, xsm;
      float xsg[G];  // sum of x~ over each of the chunk's groups (G > 1)
      {
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
        xsm = active ? xsum[cc] : 0.f;
        if constexpr (G > 1) {
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
      const uint32_t off_b = (uint32_t)(rg * rb + cc * kBaseChunkBytes);
      const uint32_t off_p = L.plane_piece + (uint32_t)(rg * rp + cc * kPlaneChunkBytes);
      const uint32_t step_b = (uint32_t)(RG * rb), step_p = (uint32_t)(RG * rp), plane_stride = (uint32_t)(BR * rp);
      const int pcol = (cc * kChunk) >> gs;    // this lane's pair byte within a row
      const int urow = reduced_row1<UP>(lane);
      const bool keep = keeps_partial1<UP>(lane);
      const uint8_t* ring = smem + L.ring;
      int slot = 0;
      uint32_t phase = 0;
      // Test hook (stagq_debug_stall): one bounded wait that runs out, so that
      // the give-up path below runs on a healthy launch.
      if (a.m.debug_stall_ns && !__all_sync(kFull, mbar_wait(sbase + L.stall, 0, a.m.debug_stall_ns))) {
        ok = false;
        if (lane == 0) *flag = 1u;
      }
      for (int b = 0; ok && b < nblk; ++b) {
        if (!__all_sync(kFull, mbar_wait(full0 + 8 * slot, phase, kWaitLimit1Ns))) {
          ok = false;
          if (lane == 0) *flag = 1u;
          break;
        }
        const uint8_t* sb = ring + slot * L.slot;
        const int lr = b * BR + rg;            // local row of this warp's row 0 in the block
        uint32_t B[UP][4];
        uint2 Pw[UP][M > 2 ? M - 2 : 1];
        float2 lm[UP];
        const float2* tb[UP];  // the pair table of each row's member
        uint32_t pw[UP];  // G > 1: the row's G pair bytes of this chunk
  #pragma unroll
        for (int u = 0; u < UP; ++u) {
          const uint4 b4 = *reinterpret_cast<const uint4*>(sb + off_b + u * step_b);
          B[u][0] = b4.x; B[u][1] = b4.y; B[u][2] = b4.z; B[u][3] = b4.w;
  #pragma unroll
          for (int k = 0; k < M - 2; ++k)
            Pw[u][k] = *reinterpret_cast<const uint2*>(sb + off_p + u * step_p + k * plane_stride);
          const int row = min(lr + RG * u, rows - 1);  // rows past the CTA's end read a valid pair byte
          tb[u] = tab + member_table_offset(a.m.mem_row, r0 + row);
          if constexpr (G == 1) lm[u] = tb[u][pairs[row * ps + pcol]];
          else pw[u] = load_pairs<G>(pairs + row * ps + pcol);
        }
        float v[UP];
  #pragma unroll
        for (int u = 0; u < UP; ++u) {
          if constexpr (G == 1) {
            const int tot = chunk_dot<M>(X, B[u], Pw[u]);
            v[u] = fmaf(lm[u].y, (float)tot * xs, lm[u].x * xsm);
          } else {
            int tot[G];
            chunk_dot_g<M, G>(X, B[u], Pw[u], tot);
            float acc = 0.f;
  #pragma unroll
            for (int g = 0; g < G; ++g) {
              const float2 l = tb[u][(pw[u] >> (8 * g)) & 0xFFu];
              acc = fmaf(l.y, (float)tot[g] * xs, fmaf(l.x, xsg[g], acc));
            }
            v[u] = acc;
          }
        }
        const float s = partial_reduce1<UP>(v, lane);
        const int row = lr + RG * urow;
        if (keep && row < rows) part[row * PST + kw * kParts1 + (lane & 7)] = s;
        __syncwarp();  // every lane has read the slot before it is released
        if (lane == 0) mbar_arrive1(empty0 + 8 * slot);
        if (++slot == NS) {
          slot = 0;
          phase ^= 1u;
        }
      }
    } else {
      // Several vectors: lane l takes half chunk kw * 32 + l (32 weights) of
      // every row, with the x~ of all vectors in registers; a row's code words
      // are decoded once and dotted with each vector.
      const int cwi = warp - 1;                // consumer warp index
      const int kw = cwi % KW, rg = cwi / KW, RG = P.RG;
      const int hc = kw * 32 + lane;           // this lane's half chunk
      const bool active = hc < 2 * nchunk;
      const int cc = active ? hc >> 1 : 0, hh = active ? hc & 1 : 0;  // reads of inactive lanes stay inside the row
      uint32_t X[NB][16];
      float xs[NB], xsh[NB];                   // chunk scale; sum of x~ times it over the half
      {
        const uint4* src = reinterpret_cast<const uint4*>(xq);
#pragma unroll
        for (int jv = 0; jv < NB; ++jv) {
          const bool on = active && jv < nvec;
          const int gc = (jv < nvec ? jv : 0) * nchunk + cc;  // chunk index across the vectors
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 t = src[xq_piece(gc, 4 * hh + k)];
            X[jv][4 * k] = on ? t.x : 0u;
            X[jv][4 * k + 1] = on ? t.y : 0u;
            X[jv][4 * k + 2] = on ? t.z : 0u;
            X[jv][4 * k + 3] = on ? t.w : 0u;
          }
          xs[jv] = on ? xscale[gc] : 0.f;
          xsh[jv] = on ? xsum16[4 * gc + 2 * hh] + xsum16[4 * gc + 2 * hh + 1] : 0.f;  // exact: multiples of one 2^-e
        }
      }
      const uint32_t off_b = (uint32_t)(rg * rb + cc * kBaseChunkBytes + 8 * hh);
      const uint32_t off_p = L.plane_piece + (uint32_t)(rg * rp + cc * kPlaneChunkBytes + 4 * hh);
      const uint32_t step_b = (uint32_t)(RG * rb), step_p = (uint32_t)(RG * rp), plane_stride = (uint32_t)(BR * rp);
      const int pcol = (cc * kChunk) >> gs;    // this lane's pair byte within a row (groups of 64 or more)
      constexpr int NV = NB * UP;              // values per lane and block: (vector, row)
      const uint8_t* ring = smem + L.ring;
      int slot = 0;
      uint32_t phase = 0;
      // Test hook (stagq_debug_stall), as for one vector.
      if (a.m.debug_stall_ns && !__all_sync(kFull, mbar_wait(sbase + L.stall, 0, a.m.debug_stall_ns))) {
        ok = false;
        if (lane == 0) *flag = 1u;
      }
      for (int b = 0; ok && b < nblk; ++b) {
        if (!__all_sync(kFull, mbar_wait(full0 + 8 * slot, phase, kWaitLimit1Ns))) {
          ok = false;
          if (lane == 0) *flag = 1u;
          break;
        }
        const uint8_t* sb = ring + slot * L.slot;
        const int lr = b * BR + rg;            // local row of this warp's row 0 in the block
        uint32_t cw[UP][8], c5[UP][8], c6[UP][8];
        float2 lm[UP];
#pragma unroll
        for (int u = 0; u < UP; ++u) {
          const uint2 B = *reinterpret_cast<const uint2*>(sb + off_b + u * step_b);
          uint32_t Pw[M > 2 ? M - 2 : 1];
#pragma unroll
          for (int k = 0; k < M - 2; ++k)
            Pw[k] = *reinterpret_cast<const uint32_t*>(sb + off_p + u * step_p + k * plane_stride);
          half_codes<M>(B, Pw, cw[u], c5[u], c6[u]);
          const int row = min(lr + RG * u, rows - 1);  // rows past the CTA's end read a valid pair byte
          lm[u] = (tab + member_table_offset(a.m.mem_row, r0 + row))[pairs[row * ps + pcol]];
        }
        float v[NV];
#pragma unroll
        for (int jv = 0; jv < NB; ++jv)
#pragma unroll
          for (int u = 0; u < UP; ++u) {
            const int tot = half_dot<M>(X[jv], cw[u], c5[u], c6[u]);
            v[jv * UP + u] = fmaf(lm[u].y, (float)tot * xs[jv], lm[u].x * xsh[jv]);
          }
        const float sres = lane_sums<NV>(v, lane);
        const int idx = lane / (32 / NV), jv = idx / UP, row = lr + RG * (idx % UP);
        if ((lane & (32 / NV - 1)) == 0 && jv < nvec && row < rows) part[row * PST + kw * nvec + jv] = sres;
        __syncwarp();  // every lane has read the slot before it is released
        if (lane == 0) mbar_arrive1(empty0 + 8 * slot);
        if (++slot == NS) {
          slot = 0;
          phase ^= 1u;
        }
      }
    }
  }

  if (!ok && lane == 0) *flag = 1u;
  __syncthreads();

  if (*flag == 0u) {
    // ---------------------------------------------------------- y
    if (has_post) row_pass(std::true_type{}, !terms_first, true);
    else row_pass(std::false_type{}, !terms_first, true);
  } else if (tid == 0) {
    atomicOr(a.m.status, 1u);
    // Gave up: let this CTA's copies in flight land before it exits.
    mbar_wait(side_bar, 0, kDrainLimit1Ns);
    for (int b = issued - 1; b >= 0 && b >= issued - NS; --b)
      mbar_wait(full0 + 8 * (b % NS), (uint32_t)(b / NS) & 1u, kDrainLimit1Ns);
  }
}

// Opt a kernel into `smem` bytes of dynamic shared memory (and the largest
// shared-memory carve-out) on the current device, once per (device, kernel).
cudaError_t ensure_smem1(const void* kern, int key, size_t smem) {
  constexpr int kMaxDev = 64, kKeys = 384;
  static std::mutex mu;
  static size_t granted[kMaxDev][kKeys] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDev || key < 0 || key >= kKeys) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lock(mu);
  if (granted[dev][key] >= smem) return cudaSuccess;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess) err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (err == cudaSuccess) granted[dev][key] = smem;
  return err;
}

template <int M, int UP, int G, bool SC, int NB>
cudaError_t launch1_mu(const DeviceMatrix& m, const Gemv1Plan& plan, const void* x, const float* in_scale, void* y,
                       int y_f32, cudaStream_t stream) {
  Gemv1Args a;
  a.m = m;
  a.plan = plan;
  a.table = m.tables + 256 * m.nmem * (M - 2);
  a.dlo = m.dlo + 256 * m.nmem * (M - 2);
  a.x = reinterpret_cast<const __half*>(x);
  a.in_scale = in_scale;
  a.y = y;
  a.y_f32 = y_f32;
  const Smem1 L = smem1(plan, m.in, M);
  // every region that bulk copies fill or 16-byte accesses read starts on 16 bytes
  if ((L.tab | L.xq | L.pairs | L.side | L.part | L.ring | L.slot | L.plane_piece) & 15u) return cudaErrorInvalidValue;
  auto kern = gemv1_kernel<M, UP, G, SC, NB>;
  const int key = ((((M - 2) * 3 + (UP == 4 ? 2 : UP - 1)) * 3 + (G == 4 ? 2 : G - 1)) * 2 + (SC ? 1 : 0)) * 3 +
                  (NB == 1 ? 0 : NB == 2 ? 1 : 2);
  cudaError_t err = ensure_smem1(reinterpret_cast<const void*>(kern), key, L.total);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)plan.grid);
  cfg.blockDim = dim3((unsigned)(32 * (plan.NW + 1)));
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
cudaError_t launch1_m(const DeviceMatrix& m, const Gemv1Plan& plan, const void* x, const float* in_scale, void* y,
                      int y_f32, cudaStream_t stream) {
  if (plan.nb > 1) {  // several vectors: groups of 64 or more, 1 or 2 rows per warp per block
    if (groups_per_chunk(plan.group_shift) != 1) return cudaErrorInvalidValue;
    const bool four = plan.nb > 2;
    switch (plan.up) {
      case 1: return four ? launch1_mu<M, 1, 1, SC, 4>(m, plan, x, in_scale, y, y_f32, stream)
                          : launch1_mu<M, 1, 1, SC, 2>(m, plan, x, in_scale, y, y_f32, stream);
      case 2: return four ? launch1_mu<M, 2, 1, SC, 4>(m, plan, x, in_scale, y, y_f32, stream)
                          : launch1_mu<M, 2, 1, SC, 2>(m, plan, x, in_scale, y, y_f32, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (groups_per_chunk(plan.group_shift) * 8 + plan.up) {
    case 8 + 1: return launch1_mu<M, 1, 1, SC, 1>(m, plan, x, in_scale, y, y_f32, stream);
    case 8 + 2: return launch1_mu<M, 2, 1, SC, 1>(m, plan, x, in_scale, y, y_f32, stream);
    case 8 + 4: return launch1_mu<M, 4, 1, SC, 1>(m, plan, x, in_scale, y, y_f32, stream);
    case 16 + 1: return launch1_mu<M, 1, 2, SC, 1>(m, plan, x, in_scale, y, y_f32, stream);  // groups of 32
    case 16 + 2: return launch1_mu<M, 2, 2, SC, 1>(m, plan, x, in_scale, y, y_f32, stream);
    case 32 + 1: return launch1_mu<M, 1, 4, SC, 1>(m, plan, x, in_scale, y, y_f32, stream);  // groups of 16
    case 32 + 2: return launch1_mu<M, 2, 4, SC, 1>(m, plan, x, in_scale, y, y_f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int M>
cudaError_t launch1_m(const DeviceMatrix& m, const Gemv1Plan& plan, const void* x, const float* in_scale, void* y,
                      int y_f32, cudaStream_t stream) {
  return in_scale ? launch1_m<M, true>(m, plan, x, in_scale, y, y_f32, stream)
                  : launch1_m<M, false>(m, plan, x, nullptr, y, y_f32, stream);
}

}  // namespace

int gemv1_grid(int out, int num_sms) {
  int g = out < num_sms ? out : num_sms;
  if ((out + g - 1) / g > kMaxRowsPerCta) g = (out + kMaxRowsPerCta - 1) / kMaxRowsPerCta;
  return g;
}

// Launch shape (measured on B200 over the Llama-3.1-8B, Phi-4 and OLMo-2
// linears at 2..6 bits, alone and as a layer's chain of launches):
//  * One CTA per SM that has the SM to itself, with as many consumer warps
//    as the register file holds at kRegs1 registers (14-15 for the Llama
//    shapes). Every single-vector launch having the same shape keeps a chain
//    of launches evenly placed: a CTA starts only where its predecessor's CTA
//    has left, one per SM, and its ring fills while the predecessor grid
//    drains (programmatic dependent launch). Plans that let a CTA share its
//    SM with the next launch's measured faster alone but slower in chains
//    that mix shapes: an SM freed early could take two of the next launch's
//    CTAs while another took none.
//  * About 60 KB of weights in flight per SM hide the HBM latency: the ring
//    grows to that from 3 slots where the shared memory allows.
//  * Larger blocks (UP = 4) amortise the per-block waits and sums, as long as
//    the CTA's rows still make about 5 blocks to pipeline; with fewer rows, 2
//    rows per warp while that makes at least 3 blocks (measured on q/k/v
//    stacked, 41 rows per CTA: 2 rows in 3 blocks beat 4 rows in 2 by up to
//    0.8 us), else 4.
constexpr uint32_t kInflightTarget = 60u * 1024u;
constexpr int kMinBlocks = 5;   // 4 rows per warp per block from this many blocks up
constexpr int kMinBlocks2 = 3;  // below it, 2 rows from this many blocks up (else 4, fewer blocks)

// The ring for given row groups: false if nothing fits the shared memory.
bool plan1_fit(const DeviceMatrix& m, int bits, const Gemv1Plan& q, Gemv1Plan* out) {
  const uint32_t budget = (uint32_t)m.smem_limit;
  const int nblk4 = (q.rows_cap + 4 * q.RG - 1) / (4 * q.RG);
  const int nblk2 = (q.rows_cap + 2 * q.RG - 1) / (2 * q.RG);
  // groups below 64 weights (several pairs per chunk): at most 2 rows per warp per block;
  // several vectors: 2 rows (1 with more than two planes), for the registers
  int up0 = q.group_shift < 6 ? 2 : (nblk4 >= kMinBlocks || nblk2 < kMinBlocks2) ? 4 : 2;
  if (q.nb > 1) up0 = bits > 4 ? 1 : 2;
  for (int stage = 1; stage >= 0; --stage) {   // side record staged in shared memory where it fits
    for (int up = up0; up >= 1; up /= 2) {
      Gemv1Plan t = q;
      t.up = up;
      t.br = q.RG * up;
      t.stage_side = stage;
      const int nblk = (q.rows_cap + t.br - 1) / t.br;
      const int ns_min = nblk < 3 ? nblk : 3;
      const int ns_max = nblk < kMaxSlots ? nblk : kMaxSlots;
      t.ns = 0;
      for (int ns = ns_min; ns <= ns_max; ++ns) {
        t.ns = ns;
        if (smem1(t, m.in, bits).total > budget) {
          t.ns = ns - 1;
          break;
        }
        if ((uint32_t)ns * smem1(t, m.in, bits).slot >= kInflightTarget) break;
      }
      if (t.ns < ns_min) continue;
      *out = t;
      return true;
    }
  }
  return false;
}

bool make_plan1(const DeviceMatrix& m, int bits, int nb, Gemv1Plan* p) {
  // warps the register file holds at kRegs1 registers a thread (a sub-partition: 16384 registers)
  constexpr int kRegFileWarps = 4 * (16384 / (32 * kRegs1));
  Gemv1Plan q = {};
  if (nb < 1 || nb > 4) return false;
  q.nb = nb;
  // a K slice is 32 lanes x one chunk, or x half a chunk for several vectors
  // (groups of 64 weights or more)
  if (nb > 1 && m.group < kChunk) return false;
  q.KW = nb == 1 ? (m.in / kChunk + 31) / 32 : (2 * (m.in / kChunk) + 31) / 32;
  if (q.KW < 1 || q.KW + 1 > kRegFileWarps) return false;
  q.grid = m.side1_grid;
  if (q.grid < 1) return false;
  q.rows_cap = (m.out + q.grid - 1) / q.grid;
  q.rows_q = m.out / q.grid;
  q.rows_rem = m.out % q.grid;
  q.pair_stride = m.pair_stride;
  q.side_stride = m.side1_stride;
  q.side_ent_off = m.side1_ent_off;
  q.side_max = m.side1_max;
  q.group_shift = 0;
  while ((1 << q.group_shift) < m.group) ++q.group_shift;
  q.pdl = 1;
  q.nmem = m.nmem;
  // row groups: as many as the register file holds beside the producer warp
  q.RG = (kRegFileWarps - 1) / q.KW;
  q.NW = q.KW * q.RG;
  return plan1_fit(m, bits, q, p);
}

cudaError_t launch_gemv1(const DeviceMatrix& m, const Gemv1Plan& plan, int bits, const void* x, const float* in_scale,
                         void* y, int y_f32, cudaStream_t stream) {
  switch (bits) {
    case 2: return launch1_m<2>(m, plan, x, in_scale, y, y_f32, stream);
    case 3: return launch1_m<3>(m, plan, x, in_scale, y, y_f32, stream);
    case 4: return launch1_m<4>(m, plan, x, in_scale, y, y_f32, stream);
    case 5: return launch1_m<5>(m, plan, x, in_scale, y, y_f32, stream);
    case 6: return launch1_m<6>(m, plan, x, in_scale, y, y_f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace stagq
