// Device-side view of a loaded StagQ matrix and the kernel launchers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace stagq {

struct DeviceMatrix {
  int32_t out, in, group, n_planes;
  int64_t nnz;
  const uint8_t* base;        // base plane, out*in/4 bytes
  const uint8_t* plane[4];    // planes 3..6, out*in/8 bytes each (null when absent)
  const uint8_t* pair;        // [out, in/group] 8-bit pairs
  const int32_t* row_ptr;     // [out+1]
  const uint32_t* entries;    // [nnz]: column | (fp16 value << 16)
  const float2* tables;       // [n_planes+1][256]: (lo_M, s_M * c_M) for M = 2..2+n_planes
  int num_sms;
};

// y = W_hat^(bits) x for n = 1. y is fp16 (y_f32 = 0) or fp32.
cudaError_t launch_gemv(const DeviceMatrix& m, int bits, const void* x, void* y, int y_f32,
                        cudaStream_t stream);

// u_M per weight into u (device [out*in]).
cudaError_t launch_decode_levels(const DeviceMatrix& m, int bits, uint8_t* u, cudaStream_t stream);

// Composite factor c_M folded into the stored step: the kernels accumulate
// sum(v x) with v = 2 u_3 at M = 3 and v = u_M otherwise.
inline double composite_factor(int M) { return M == 3 ? 0.5 : 1.0; }

}  // namespace stagq
