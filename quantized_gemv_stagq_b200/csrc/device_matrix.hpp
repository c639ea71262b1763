// Device-side view of a loaded StagQ matrix, the GEMV launch plan and the
// kernel launchers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace stagq {

constexpr int kMaxConsumerWarps = 16;   // warps per CTA
constexpr int kMaxRowsPerCta = 2048;    // a CTA's row_ptr / slice offsets live in shared memory
constexpr int kPrefetchGroups = 4;      // deepest cp.async prefetch (batches in flight per lane)
constexpr int kSliceWeights = 2048;     // K weights per K slice (one warp: 32 lanes x 64)

struct DeviceMatrix {
  int32_t out, in, group, n_planes;
  int64_t nnz;
  const uint8_t* base;        // base plane, out*in/4 bytes
  const uint8_t* plane[4];    // planes 3..6, out*in/8 bytes each (null when absent)
  const uint8_t* pair;        // 8-bit pairs, row stride pair_stride (in/group padded to 16)
  int32_t pair_stride;
  const int32_t* row_ptr;     // [out+1]
  const uint32_t* entries;    // [nnz]: column | (fp16 value << 16), then 16 bytes of padding
  int32_t max_cta_entries;    // most side-record entries in one CTA's row range
  const float2* tables;       // [n_planes+1][256]: (lo_M, s_M * c_M) for M = 2..2+n_planes
  int num_sms;
  int smem_limit;             // opt-in shared memory per block
};

// How one GEMV is laid out over the GPU (see gemv.cu).
struct GemvPlan {
  int grid;              // CTAs (one per SM unless rows per CTA would exceed kMaxRowsPerCta)
  int KW, RG, up;        // K slices, row groups, rows per batch
  int depth;             // batches each lane keeps in flight (2..kPrefetchGroups)
  int ent_cap;           // side-record entries staged per CTA (0: read from global memory)
  int group_shift;       // log2(group)
  int pair_stride;
  int max_rows_per_cta;
  int pdl;               // launch with programmatic dependent launch
};

// Plan for a GEMV at `bits`; returns false if the shape cannot be planned.
bool make_plan(const DeviceMatrix& m, int bits, GemvPlan* plan);
int k_slices(int in);
int gemv_grid(int out, int num_sms);
uint32_t gemv_smem_bytes(const GemvPlan& plan, int in, int bits);

// y = W_hat^(bits) x for n = 1. y is fp16 (y_f32 = 0) or fp32.
cudaError_t launch_gemv(const DeviceMatrix& m, const GemvPlan& plan, int bits, const void* x, void* y,
                        int y_f32, cudaStream_t stream);

// u_M per weight into u (device [out*in]).
cudaError_t launch_decode_levels(const DeviceMatrix& m, int bits, uint8_t* u, cudaStream_t stream);

// Composite factor c_M folded into the stored step: the kernels accumulate
// sum(v x) with v = 2 u_3 at M = 3 and v = u_M otherwise.
inline double composite_factor(int M) { return M == 3 ? 0.5 : 1.0; }

}  // namespace stagq
