// Device-side view of a loaded StagQ matrix, the GEMV launch plan and the
// kernel launchers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace stagq {

constexpr int kMaxWarps = 16;           // warps per CTA (K slices x row groups)
constexpr int kMaxSlots = 8;            // shared-memory ring slots
constexpr int kMaxRowsPerCta = 2048;    // rows of one CTA
constexpr int kSliceWeights = 2048;     // K weights per K slice (one warp: 32 lanes x 64)
constexpr int64_t kTwoCtaWeightsPerSm = 256 * 1024;  // from this many weights per SM on, two GEMV CTAs per SM
constexpr int kMaxStack = 4;            // member matrices of a stacked handle (STAGQ_MAX_STACK)

// Row groups of a CTA with KW K slices: up to 8 warps in all, at least one group.
inline int row_groups(int KW) { return KW <= 4 ? 8 / KW : 1; }

// Shared-memory order of the fixed-point activations x~ inside a GEMV CTA:
// chunk c (64 int16) is 8 pieces of 16 bytes, piece p stored at piece slot
// (p + c) mod 8, so that 32 lanes reading piece p of their own chunks hit 8
// different 16-byte bank groups instead of one.
__host__ __device__ inline int xq_piece_index(int c, int p) { return c * 8 + ((p + c) & 7); }
// Element slot of column `col` (its chunk is slot >> 6, as for the column).
__host__ __device__ inline int xq_slot_of_column(int col) {
  const int c = col >> 6, e = col & 63;
  return xq_piece_index(c, e >> 3) * 8 + (e & 7);
}
// The column whose element slot is `slot` (inverse of xq_slot_of_column).
__host__ __device__ inline int column_of_xq_slot(int slot) {
  const int c = slot >> 6, piece_slot = (slot >> 3) & 7;
  return c * 64 + ((piece_slot - c) & 7) * 8 + (slot & 7);
}

struct DeviceMatrix;
// Offset of the pair table of the member that holds global row `row` (a
// multiple of 256 entries).
__host__ __device__ inline int member_table_offset(const int32_t (&mem_row)[kMaxStack], int row) {
  return 256 * ((row >= mem_row[1]) + (row >= mem_row[2]) + (row >= mem_row[3]));
}

struct DeviceMatrix {
  int32_t out, in, group, n_planes;
  int64_t nnz;
  const uint8_t* base;        // base plane, out*in/4 bytes
  const uint8_t* plane[4];    // planes 3..6, out*in/8 bytes each (null when absent)
  const uint8_t* pair;        // 8-bit pairs, row stride pair_stride (in/group padded to 16)
  int32_t pair_stride;
  // Side record cut per CTA of the GEMV grid (side_grid CTAs over the rows as
  // gemv_grid splits them), side_stride bytes each. A CTA's rows fall in RG
  // classes (local row mod RG); its entries are ordered by (class, K slice,
  // row, column), and int32 offsets [RG][KW][class_rows + 1] give where each
  // row of a class starts within its (class, K slice) run, plus the run's end.
  // The entries (column | fp16 value << 16; bit 15 marks a post-grid entry,
  // whose value is the residual r) start at side_ent_off.
  const uint8_t* side;
  int32_t side_stride, side_ent_off, side_grid;
  // The same side record cut for the single-vector kernel (gemv1.cu): per
  // CTA of its grid (side1_grid CTAs, one per SM), side1_stride bytes: int32
  // offsets [rows + 1] (where each local row's entries start, then the end),
  // and from side1_ent_off the entries (column | post-grid flag << 15 | fp16
  // value << 16) in (row, column) order; side1_max entries at most per CTA.
  const uint8_t* side1;
  int32_t side1_stride, side1_ent_off, side1_grid, side1_max;
  const float2* tables;       // [n_planes+1][nmem][256]: (lo_M, s_M * c_M) for M = 2..2+n_planes
  const float* dlo;           // [n_planes+1][nmem][256]: lo - lo_M, the correction of a post-grid entry beside r
  // A stacked handle holds nmem member matrices (their rows in order, each
  // with its own codebooks); mem_row[j] is member j's first row (INT32_MAX for
  // j >= nmem), so a row's member is the number of mem_row[1..] <= row.
  int32_t nmem;
  int32_t mem_row[kMaxStack];
  int32_t has_post;           // the side record holds post-grid entries (bit 15 of the column / slot)
  uint32_t* status;           // nonzero once a kernel gave up waiting for its copies
  uint32_t debug_stall_ns;    // test hook: launches include one bounded wait of this length that runs out
  int num_sms;
  int smem_limit;             // opt-in shared memory per block
  int smem_pair_budget;       // shared memory per block that still lets two blocks share an SM (general kernel)
};

// How one GEMV is laid out over the GPU (see gemv.cu).
struct GemvPlan {
  int grid;              // CTAs (= side_grid)
  int KW, RG, NW;        // K slices, row groups, warps (KW * RG)
  int up, br;            // rows per warp per block, rows per block (RG * up)
  int ns;                // ring slots
  int stage_side;        // the CTA's side record is copied into shared memory
  int side_stride;
  int rows_cap;          // most rows of one CTA
  int class_rows;        // most rows of one row class (ceil(rows_cap / RG))
  int group_shift;       // log2(group)
  int pair_stride;
  int pdl;               // launch with programmatic dependent launch
  int nmem;              // stacked members (pair tables)
  int nb;                // activation vectors per launch (1..4; the weights are read once)
};

// Launch plan of the single-vector kernel (gemv1.cu).
struct Gemv1Plan {
  int nb;                // activation vectors (1..4); above 1 a lane takes half a chunk
  int grid;              // CTAs (= side1_grid, at most one per SM)
  int KW, RG, NW;        // K slices, row groups, consumer warps (KW * RG); one producer warp more
  int up, br;            // rows per warp per block, rows per block (RG * up)
  int ns;                // ring slots
  int rows_cap;          // most rows of one CTA
  int rows_q, rows_rem;  // out = rows_q * grid + rows_rem: CTA b starts at row b rows_q + floor(b rows_rem / grid)
  int stage_side;        // the CTA's side record is copied into shared memory
  int side_stride, side_ent_off, side_max;
  int group_shift;       // log2(group)
  int pair_stride;
  int pdl;               // launch with programmatic dependent launch
  int nmem;              // stacked members (pair tables)
};

// Plan for the single-vector kernel at `bits` with `nb` activation vectors;
// false if it cannot be planned (the general kernel then serves the call).
bool make_plan1(const DeviceMatrix& m, int bits, int nb, Gemv1Plan* plan);
int gemv1_grid(int out, int num_sms);
// in_scale: null, or device fp32 [in] multiplying x channel by channel first.
cudaError_t launch_gemv1(const DeviceMatrix& m, const Gemv1Plan& plan, int bits, const void* x, const float* in_scale,
                         void* y, int y_f32, cudaStream_t stream);

// Plan for a GEMV at `bits` with `nb` activation vectors; false if the shape
// cannot be planned.
bool make_plan(const DeviceMatrix& m, int bits, int nb, GemvPlan* plan);
int k_slices(int in);
int gemv_grid(int out, int in, int num_sms);
uint32_t gemv_smem_bytes(const GemvPlan& plan, int in, int bits);

// y = W_hat^(bits) x for plan.nb vectors (x [nb][in], y [nb][out]). y is fp16
// (y_f32 = 0) or fp32.
cudaError_t launch_gemv(const DeviceMatrix& m, const GemvPlan& plan, int bits, const void* x, const float* in_scale,
                        void* y, int y_f32, cudaStream_t stream);

// u_M per weight into u (device [out*in]).
cudaError_t launch_decode_levels(const DeviceMatrix& m, int bits, uint8_t* u, cudaStream_t stream);

// Composite factor c_M folded into the stored step: the kernels accumulate
// sum(v x) with v = 2 u_3 at M = 3 and v = u_M otherwise.
inline double composite_factor(int M) { return M == 3 ? 0.5 : 1.0; }

}  // namespace stagq
