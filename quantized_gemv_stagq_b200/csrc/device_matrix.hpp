// Device-side view of a loaded StagQ matrix, the GEMV launch plan and the
// kernel launchers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace stagq {

constexpr int kMaxConsumerWarps = 16;   // + 1 producer warp per CTA
constexpr int kMaxStageRows = 32;       // rows per stage (one producer lane per row)
constexpr int kMaxRowsPerCta = 2048;    // row_ptr of a CTA's range is cached in shared memory
constexpr int kMaxEntryCap = 2048;      // side-record entries prefetched per stage

struct DeviceMatrix {
  int32_t out, in, group, n_planes;
  int64_t nnz;
  const uint8_t* base;        // base plane, out*in/4 bytes
  const uint8_t* plane[4];    // planes 3..6, out*in/8 bytes each (null when absent)
  const uint8_t* pair;        // 8-bit pairs, row stride pair_stride (in/group padded to 16)
  int32_t pair_stride;
  const int32_t* row_ptr;     // [out+1]
  const uint32_t* entries;    // [nnz]: column | (fp16 value << 16), 16 bytes of padding after
  const float2* tables;       // [n_planes+1][256]: (lo_M, s_M * c_M) for M = 2..2+n_planes
  uint32_t* status;           // device word: nonzero if a kernel gave up on a wait
  int num_sms;
  int smem_limit;             // opt-in shared memory per block
  int ecap;                   // side-record entries to prefetch per stage
};

// How one GEMV is laid out over the GPU (see gemv.cu).
struct GemvPlan {
  int grid;              // CTAs (one per SM unless rows per CTA would exceed kMaxRowsPerCta)
  int KW, RG, up;        // K-warps, row groups, rows per row group per stage
  int rows_per_stage;    // RG * up (<= kMaxStageRows)
  int slots;             // shared-memory ring depth
  int ecap;              // entries prefetched per stage
  int pair_stride;
  int max_rows_per_cta;
  int pdl;               // launch with programmatic dependent launch
};

// Plan for a GEMV at `bits`; returns false if the shape cannot be planned.
bool make_plan(const DeviceMatrix& m, int bits, GemvPlan* plan);
// Rows per stage / grid of the plan used for every precision (entry cap sizing).
void stage_partition(int out, int in, int num_sms, int* grid, int* rows_per_stage);
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
