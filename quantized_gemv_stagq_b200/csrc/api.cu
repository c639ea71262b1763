// C ABI of libstagq.so: handle lifecycle, loading a stream onto a GPU, and the
// GEMV entry points. See include/stagq.h for the contract of each function.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "device_matrix.hpp"
#include "host_common.hpp"
#include "layout.cuh"
#include "stream.hpp"

struct stagq_matrix {
  int device = -1;
  stagq::DeviceMatrix dm{};
  stagq::GemvPlan plan[7][STAGQ_MAX_BATCH + 1]{};  // per precision (bits) and vector count
  bool plan_ok[7][STAGQ_MAX_BATCH + 1]{};
  stagq::Gemv1Plan plan1[7][STAGQ_MAX_BATCH + 1]{};  // single-vector kernel, per precision and vector count
  bool plan1_ok[7][STAGQ_MAX_BATCH + 1]{};
  bool prefer1[7]{};             // the single-vector kernel serves the calls it can plan by default
  void* d_mem = nullptr;
  size_t d_bytes = 0;
  void* d_stage = nullptr;      // x / y staging for stagq_gemv_host
  size_t stage_bytes = 0;
};

namespace stagq {
namespace {

int cuda_fail(cudaError_t e, const char* what) {
  return fail(STAGQ_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) ok = true;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Per-precision (lo_M, s_M c_M) for the 256 pairs of each stacked member
// (its own two codebooks, Section 3.1), Eq. (10) in fp64, stored fp32; and per
// precision and member lo - lo_M of every pair: at a post-grid entry the main
// stream decodes lo_M + s q (zero planes), the reconstruction is lo + s q + r,
// so the correction is r + (lo - lo_M). Layout [M - 2][member][pair].
void build_tables(const stagq_host_stream* const* members, int nmem, std::vector<float2>& t,
                  std::vector<float>& dlo) {
  const int N = 2 + members[0]->n_planes;
  t.assign((size_t)(N - 1) * nmem * 256, make_float2(0.f, 0.f));
  dlo.assign((size_t)(N - 1) * nmem * 256, 0.f);
  for (int M = 2; M <= N; ++M) {
    for (int j = 0; j < nmem; ++j) {
      const stagq_host_stream* s = members[j];
      for (int p = 0; p < 256; ++p) {
        const double sp = std::exp2(half_to_double(s->codebook_log2s[p >> 4]));
        const double lo = half_to_double(s->codebook_lo_over_s[p & 15]) * sp;
        const double sM = sp / std::ldexp(1.0, M - 2);
        const double loM = lo - sp * (std::ldexp(1.0, M - 2) - 1.0) / std::ldexp(1.0, M - 1);
        const size_t i = ((size_t)(M - 2) * nmem + j) * 256 + p;
        t[i] = make_float2((float)loM, (float)(sM * composite_factor(M)));
        dlo[i] = (float)(lo - loM);
      }
    }
  }
}

int check_handle_bits(stagq_handle h, int bits) {
  if (!h) return fail(STAGQ_EINVAL, "null handle");
  if (bits < 2 || bits > 2 + h->dm.n_planes) return fail(STAGQ_EINVAL, "bits outside 2..2+n_planes");
  return STAGQ_OK;
}

}  // namespace
}  // namespace stagq

using namespace stagq;

namespace {
constexpr uint16_t kColMask = 0x7FFF;  // side-record column without the post-grid flag
}

namespace {

// Copies a (possibly stacked) stream to the device. `s` is the whole stream
// (members' rows stacked in order); members[j] are the member streams, whose
// codebooks give each member its own pair tables (nmem = 1: s itself).
int load_impl(const stagq_host_stream* s, const stagq_host_stream* const* members, int nmem, int device,
              stagq_handle* out) {
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess || ndev == 0) return fail(STAGQ_ENODEV, "no CUDA device");
  if (device < 0 || device >= ndev) return fail(STAGQ_EINVAL, "device index out of range");
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10) return fail(STAGQ_ENODEV, std::string("kernels are built for sm_100a; device is ") + prop.name);

  DeviceGuard guard(device);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");

  const int64_t out_ = s->out, in = s->in;
  const int np = s->n_planes;
  const size_t base_bytes = (size_t)(out_ * in / 4), plane_bytes = (size_t)(out_ * in / 8);
  const size_t pair_row = (size_t)(in / s->group), pair_stride = align_up(pair_row, 16);
  const size_t pair_bytes = (size_t)out_ * pair_stride;
  const size_t tab_bytes = (size_t)(np + 1) * nmem * 256 * sizeof(float2);
  const size_t dlo_bytes = (size_t)(np + 1) * nmem * 256 * sizeof(float);
  int has_post = 0;
  for (int64_t e = 0; e < s->nnz; ++e) has_post |= (s->col[e] & STAGQ_SIDE_POST) != 0;
  // Side record cut per CTA of the GEMV grid (see DeviceMatrix::side).
  const int grid = gemv_grid(s->out, s->in, prop.multiProcessorCount);
  const int KW = k_slices(s->in), RG = row_groups(KW);
  const int rows_cap = (int)((out_ + grid - 1) / grid);
  const int class_rows = (rows_cap + RG - 1) / RG;
  int64_t max_cta = 0;
  for (int b = 0; b < grid; ++b) {
    const int64_t ra = (int64_t)b * out_ / grid, rb = (int64_t)(b + 1) * out_ / grid;
    const int64_t n = (int64_t)s->row_ptr[rb] - s->row_ptr[ra];
    if (n > max_cta) max_cta = n;
  }
  const size_t side_ent_off = align_up((size_t)4 * RG * KW * ((size_t)class_rows + 1), 16);
  const size_t side_stride = align_up(side_ent_off + 4 * (size_t)max_cta, 16);
  if (side_stride > (size_t)INT32_MAX) return fail(STAGQ_EINVAL, "side record too large per CTA");
  const size_t side_bytes = (size_t)grid * side_stride;
  // The same record cut for the single-vector kernel: one CTA per SM, rows in order.
  const int grid1 = gemv1_grid(s->out, prop.multiProcessorCount);
  const int rows_cap1 = (int)((out_ + grid1 - 1) / grid1);
  int64_t max_cta1 = 0;
  for (int b = 0; b < grid1; ++b) {
    const int64_t ra = (int64_t)b * out_ / grid1, rb = (int64_t)(b + 1) * out_ / grid1;
    const int64_t n = (int64_t)s->row_ptr[rb] - s->row_ptr[ra];
    if (n > max_cta1) max_cta1 = n;
  }
  const size_t side1_ent_off = align_up((size_t)4 * ((size_t)rows_cap1 + 1), 16);
  const size_t side1_stride = align_up(side1_ent_off + 4 * (size_t)max_cta1, 16);
  if (side1_stride > (size_t)INT32_MAX) return fail(STAGQ_EINVAL, "side record too large per CTA");
  const size_t side1_bytes = (size_t)grid1 * side1_stride;
  size_t off = 0;
  const size_t o_base = off; off = align_up(off + base_bytes, 256);
  size_t o_plane[STAGQ_MAX_PLANES] = {};
  for (int k = 0; k < np; ++k) { o_plane[k] = off; off = align_up(off + plane_bytes, 256); }
  const size_t o_pair = off; off = align_up(off + pair_bytes, 256);
  const size_t o_side = off; off = align_up(off + side_bytes, 256);
  const size_t o_side1 = off; off = align_up(off + side1_bytes, 256);
  const size_t o_tab = off; off = align_up(off + tab_bytes, 256);
  const size_t o_dlo = off; off = align_up(off + dlo_bytes, 256);
  const size_t o_status = off; off = align_up(off + 4, 256);
  const size_t total = off;

  stagq_matrix* h = new (std::nothrow) stagq_matrix();
  if (!h) return fail(STAGQ_ENOMEM, "host allocation failed");
  h->device = device;
  e = cudaMalloc(&h->d_mem, total);
  if (e != cudaSuccess) {
    delete h;
    cudaGetLastError();
    return fail(STAGQ_ENOMEM, std::string("cudaMalloc of stream failed: ") + cudaGetErrorString(e));
  }
  h->d_bytes = total;
  uint8_t* d = static_cast<uint8_t*>(h->d_mem);

  std::vector<float2> tabs;
  std::vector<float> dlo;
  build_tables(members, nmem, tabs, dlo);
  std::vector<uint8_t> side(side_bytes, 0);
  {
    for (int b = 0; b < grid; ++b) {
      const int64_t ra = (int64_t)b * out_ / grid, rb = (int64_t)(b + 1) * out_ / grid, n = rb - ra;
      uint8_t* blk = &side[(size_t)b * side_stride];
      int32_t* offs = reinterpret_cast<int32_t*>(blk);
      uint32_t* ent = reinterpret_cast<uint32_t*>(blk + side_ent_off);
      int32_t pos = 0;
      for (int rg = 0; rg < RG; ++rg) {
        const int64_t nm = n > rg ? (n - rg + RG - 1) / RG : 0;
        for (int kw = 0; kw < KW; ++kw) {
          int32_t* o = offs + ((size_t)rg * KW + kw) * ((size_t)class_rows + 1);
          for (int64_t m = 0; m < nm; ++m) {
            const int64_t r = ra + rg + (int64_t)RG * m;
            o[m] = pos;
            int64_t e = s->row_ptr[r];
            const int64_t e1 = s->row_ptr[r + 1];
            // columns increase within a row; the entry keeps the post-grid flag (bit 15)
            while (e < e1 && (s->col[e] & kColMask) < (int64_t)kw * kSliceWeights) ++e;
            for (; e < e1 && (s->col[e] & kColMask) < (int64_t)(kw + 1) * kSliceWeights; ++e)
              ent[pos++] = (uint32_t)s->col[e] | ((uint32_t)s->val[e] << 16);
          }
          o[nm] = pos;
        }
      }
    }
  }
  std::vector<uint8_t> side1(side1_bytes, 0);
  for (int b = 0; b < grid1; ++b) {
    const int64_t ra = (int64_t)b * out_ / grid1, rb = (int64_t)(b + 1) * out_ / grid1, n = rb - ra;
    uint8_t* blk = &side1[(size_t)b * side1_stride];
    int32_t* offs = reinterpret_cast<int32_t*>(blk);
    uint32_t* ent = reinterpret_cast<uint32_t*>(blk + side1_ent_off);
    int32_t pos = 0;
    for (int64_t r = 0; r < n; ++r) {
      offs[r] = pos;
      for (int64_t e = s->row_ptr[ra + r]; e < s->row_ptr[ra + r + 1]; ++e)
        ent[pos++] = (uint32_t)(s->col[e] & kColMask) | (uint32_t)(s->col[e] & STAGQ_SIDE_POST) |
                     ((uint32_t)s->val[e] << 16);
    }
    offs[n] = pos;
  }
  std::vector<uint8_t> pairs(pair_bytes, 0);
  for (int64_t r = 0; r < out_; ++r) std::memcpy(&pairs[(size_t)r * pair_stride], s->pair_idx + (size_t)r * pair_row, pair_row);

  struct Copy { size_t off; const void* src; size_t n; };
  std::vector<Copy> copies = {{o_base, s->planes, base_bytes}};
  for (int k = 0; k < np; ++k) copies.push_back({o_plane[k], s->planes + base_bytes + (size_t)k * plane_bytes, plane_bytes});
  copies.push_back({o_pair, pairs.data(), pair_bytes});
  copies.push_back({o_side, side.data(), side_bytes});
  copies.push_back({o_side1, side1.data(), side1_bytes});
  copies.push_back({o_tab, tabs.data(), tab_bytes});
  copies.push_back({o_dlo, dlo.data(), dlo_bytes});
  for (const Copy& c : copies) {
    e = cudaMemcpy(d + c.off, c.src, c.n, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaFree(h->d_mem);
      delete h;
      return cuda_fail(e, "cudaMemcpy of stream");
    }
  }
  e = cudaMemset(d + o_status, 0, 4);
  int smem_limit = 0, smem_sm = 0, smem_reserved = 0;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_limit, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock, device);
  if (e != cudaSuccess) {
    cudaFree(h->d_mem);
    delete h;
    return cuda_fail(e, "cudaDeviceGetAttribute");
  }
  DeviceMatrix& m = h->dm;
  m.out = s->out; m.in = s->in; m.group = s->group; m.n_planes = np; m.nnz = s->nnz;
  m.base = d + o_base;
  for (int k = 0; k < 4; ++k) m.plane[k] = k < np ? d + o_plane[k] : nullptr;
  m.pair = d + o_pair;
  m.pair_stride = (int32_t)pair_stride;
  m.smem_limit = smem_limit;
  m.side = d + o_side;
  m.side_stride = (int32_t)side_stride;
  m.side_ent_off = (int32_t)side_ent_off;
  m.side_grid = grid;
  m.side1 = d + o_side1;
  m.side1_stride = (int32_t)side1_stride;
  m.side1_ent_off = (int32_t)side1_ent_off;
  m.side1_grid = grid1;
  m.side1_max = (int32_t)max_cta1;
  m.tables = reinterpret_cast<const float2*>(d + o_tab);
  m.dlo = reinterpret_cast<const float*>(d + o_dlo);
  m.has_post = has_post;
  m.nmem = nmem;
  for (int j = 0, r = 0; j < kMaxStack; ++j) {  // first row of each member; absent members never start
    m.mem_row[j] = j < nmem ? r : INT32_MAX;
    if (j < nmem) r += members[j]->out;
  }
  m.status = reinterpret_cast<uint32_t*>(d + o_status);
  m.num_sms = prop.multiProcessorCount;
  m.smem_pair_budget = smem_sm / 2 - smem_reserved;
  if (m.smem_pair_budget > smem_limit) m.smem_pair_budget = smem_limit;
  for (int b = 2; b <= 2 + np; ++b)
    for (int nb = 1; nb <= STAGQ_MAX_BATCH; ++nb) h->plan_ok[b][nb] = make_plan(m, b, nb, &h->plan[b][nb]);
  // The single-vector kernel serves every launch it can plan (n = 1, and
  // n = 2..4 with groups of 64 or more): one CTA per SM that has the SM to
  // itself. A chain of launches of one shape of CTA stays evenly placed (see
  // make_plan1); on the Llama-3.1-8B layer chain this measured 24 % faster
  // than giving the general kernel (whose CTAs share an SM) the matrices of up
  // to 2^24 weights, and at n = 4 it takes 28 % less time than the general
  // kernel.
  for (int b = 2; b <= 2 + np; ++b) {
    for (int nb = 1; nb <= STAGQ_MAX_BATCH; ++nb) h->plan1_ok[b][nb] = make_plan1(m, b, nb, &h->plan1[b][nb]);
    h->prefer1[b] = true;
  }
  if (!h->plan_ok[2][1]) {
    cudaFree(h->d_mem);
    delete h;
    return fail(STAGQ_EINVAL, "shape cannot be planned on this device");
  }
  *out = h;
  return STAGQ_OK;
}

}  // namespace

extern "C" int stagq_load(const stagq_host_stream* s, int device, stagq_handle* out) {
  if (!out) return fail(STAGQ_EINVAL, "stagq_load: null output handle");
  *out = nullptr;
  int st = validate_stream(s);
  if (st) return st;
  const stagq_host_stream* members[1] = {s};
  return load_impl(s, members, 1, device, out);
}

extern "C" int stagq_load_stack(const stagq_host_stream* const* members, int count, int device, stagq_handle* out) {
  if (!out) return fail(STAGQ_EINVAL, "stagq_load_stack: null output handle");
  *out = nullptr;
  if (!members || count < 1 || count > STAGQ_MAX_STACK) return fail(STAGQ_EINVAL, "count outside 1..STAGQ_MAX_STACK");
  int64_t out_total = 0, nnz = 0;
  for (int j = 0; j < count; ++j) {
    int st = validate_stream(members[j]);
    if (st) return st;
    const stagq_host_stream* m = members[j];
    if (m->in != members[0]->in || m->group != members[0]->group || m->n_planes != members[0]->n_planes)
      return fail(STAGQ_EINVAL, "stacked members must share in, group and n_planes");
    out_total += m->out;
    nnz += m->nnz;
  }
  const int64_t in = members[0]->in;
  const int np = members[0]->n_planes;
  int st = check_shape(out_total, in, members[0]->group, np);
  if (st) return st;
  // The stacked stream: every plane region holds the members' rows in order
  // (each plane is row-major), then the pair bytes and the side record
  // (row pointers shifted by the entries of the members before).
  HostStreamBuffers buf;
  try {
    buf.planes.resize((size_t)stagq_stream_plane_bytes((int32_t)out_total, (int32_t)in, np));
    buf.pair_idx.resize((size_t)(out_total * (in / members[0]->group)));
    buf.row_ptr.resize((size_t)out_total + 1);
    buf.col.resize((size_t)nnz);
    buf.val.resize((size_t)nnz);
  } catch (...) {
    return fail(STAGQ_ENOMEM, "host allocation for the stacked stream failed");
  }
  int64_t r0 = 0, e0 = 0;
  const int64_t ngr = in / members[0]->group;
  buf.row_ptr[0] = 0;
  for (int j = 0; j < count; ++j) {
    const stagq_host_stream* m = members[j];
    const int64_t rows = m->out;
    std::memcpy(&buf.planes[(size_t)(r0 * in / 4)], m->planes, (size_t)(rows * in / 4));
    for (int k = 3; k < 3 + np; ++k)
      std::memcpy(&buf.planes[(size_t)(plane_region_offset(out_total, in, k) + r0 * in / 8)],
                  m->planes + plane_region_offset(rows, in, k), (size_t)(rows * in / 8));
    std::memcpy(&buf.pair_idx[(size_t)(r0 * ngr)], m->pair_idx, (size_t)(rows * ngr));
    for (int64_t r = 0; r < rows; ++r) buf.row_ptr[(size_t)(r0 + r + 1)] = (int32_t)(e0 + m->row_ptr[r + 1]);
    if (m->nnz) {
      std::memcpy(&buf.col[(size_t)e0], m->col, (size_t)m->nnz * 2);
      std::memcpy(&buf.val[(size_t)e0], m->val, (size_t)m->nnz * 2);
    }
    r0 += rows;
    e0 += m->nnz;
  }
  stagq_host_stream& v = buf.view;
  v.out = (int32_t)out_total; v.in = (int32_t)in; v.group = members[0]->group; v.n_planes = np; v.nnz = nnz;
  std::memcpy(v.codebook_log2s, members[0]->codebook_log2s, 32);      // per member: see build_tables
  std::memcpy(v.codebook_lo_over_s, members[0]->codebook_lo_over_s, 32);
  v.planes = buf.planes.data(); v.pair_idx = buf.pair_idx.data(); v.row_ptr = buf.row_ptr.data();
  v.col = buf.col.data(); v.val = buf.val.data();
  return load_impl(&v, members, count, device, out);
}

extern "C" int stagq_load_file(const char* path, int device, stagq_handle* out) {
  HostStreamBuffers buf;
  int st = read_stream_file(path, &buf);
  if (st) return st;
  return stagq_load(&buf.view, device, out);
}

namespace {

// y = W_hat^(bits) (x .* in_scale) for n vectors; in_scale null = no scale.
int gemv_impl(stagq_handle h, int bits, const void* x, int n, const float* in_scale, void* y, uint32_t flags,
              void* cuda_stream) {
  int st = check_handle_bits(h, bits);
  if (st) return st;
  if (!x || !y) return fail(STAGQ_EINVAL, "null x or y");
  if (n < 1 || n > STAGQ_MAX_BATCH) return fail(STAGQ_EINVAL, "n outside 1..STAGQ_MAX_BATCH");
  if (reinterpret_cast<uintptr_t>(x) % 16) return fail(STAGQ_EINVAL, "x must be 16-byte aligned");
  if (in_scale && reinterpret_cast<uintptr_t>(in_scale) % 16) return fail(STAGQ_EINVAL, "in_scale must be 16-byte aligned");
  if (flags & ~(STAGQ_Y_F32 | STAGQ_KERNEL_GENERAL | STAGQ_KERNEL_SINGLE)) return fail(STAGQ_EINVAL, "unknown flags");
  const bool force_general = flags & STAGQ_KERNEL_GENERAL, force_single = flags & STAGQ_KERNEL_SINGLE;
  if (force_general && force_single) return fail(STAGQ_EINVAL, "both kernels forced");
  if (force_single && !h->plan1_ok[bits][n])
    return fail(STAGQ_EINVAL, "the single-vector kernel cannot plan this shape and vector count");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  const int yf32 = (flags & STAGQ_Y_F32) ? 1 : 0;
  const size_t ysz = yf32 ? 4 : 2;
  if (force_single || (!force_general && h->plan1_ok[bits][n] && h->prefer1[bits])) {
    cudaError_t e = launch_gemv1(h->dm, h->plan1[bits][n], bits, x, in_scale, y, yf32, stream);
    if (e != cudaSuccess) return cuda_fail(e, "GEMV launch");
    return STAGQ_OK;
  }
  if (h->plan_ok[bits][n]) {  // one launch: the weights are read once for all n vectors
    cudaError_t e = launch_gemv(h->dm, h->plan[bits][n], bits, x, in_scale, y, yf32, stream);
    if (e != cudaSuccess) return cuda_fail(e, "GEMV launch");
    return STAGQ_OK;
  }
  if (!h->plan_ok[bits][1]) return fail(STAGQ_EINVAL, "no launch plan for this precision");
  for (int j = 0; j < n; ++j) {  // shapes whose n-vector plan does not fit: one launch per vector
    const void* xj = static_cast<const uint8_t*>(x) + (size_t)j * h->dm.in * 2;
    void* yj = static_cast<uint8_t*>(y) + (size_t)j * h->dm.out * ysz;
    cudaError_t e = launch_gemv(h->dm, h->plan[bits][1], bits, xj, in_scale, yj, yf32, stream);
    if (e != cudaSuccess) return cuda_fail(e, "GEMV launch");
  }
  return STAGQ_OK;
}

}  // namespace

extern "C" int stagq_gemv_ex(stagq_handle h, int bits, const void* x, int n, void* y, uint32_t flags,
                             void* cuda_stream) {
  return gemv_impl(h, bits, x, n, nullptr, y, flags, cuda_stream);
}

extern "C" int stagq_gemv_scaled(stagq_handle h, int bits, const void* x, int n, const float* in_scale, void* y,
                                 uint32_t flags, void* cuda_stream) {
  if (!in_scale) return fail(STAGQ_EINVAL, "null in_scale");
  return gemv_impl(h, bits, x, n, in_scale, y, flags, cuda_stream);
}

extern "C" int stagq_gemv(stagq_handle h, int bits, const void* x, void* y, void* cuda_stream) {
  return stagq_gemv_ex(h, bits, x, 1, y, 0u, cuda_stream);
}

extern "C" int stagq_gemv_n(stagq_handle h, int bits, const void* x, int n, void* y, void* cuda_stream) {
  return stagq_gemv_ex(h, bits, x, n, y, 0u, cuda_stream);
}

extern "C" int stagq_gemv_host(stagq_handle h, int bits, const void* x_host, int n, void* y_host,
                               void* cuda_stream) {
  int st = check_handle_bits(h, bits);
  if (st) return st;
  if (!x_host || !y_host) return fail(STAGQ_EINVAL, "null x or y");
  if (n < 1 || n > STAGQ_MAX_BATCH) return fail(STAGQ_EINVAL, "n outside 1..STAGQ_MAX_BATCH");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");
  const size_t xb = (size_t)n * h->dm.in * 2, yb = (size_t)n * h->dm.out * 2;
  const size_t need = align_up(xb, 256) + yb;
  if (h->stage_bytes < need) {
    if (h->d_stage) cudaFree(h->d_stage);
    h->d_stage = nullptr;
    h->stage_bytes = 0;
    cudaError_t e = cudaMalloc(&h->d_stage, need);
    if (e != cudaSuccess) { cudaGetLastError(); return fail(STAGQ_ENOMEM, "staging allocation failed"); }
    h->stage_bytes = need;
  }
  uint8_t* dx = static_cast<uint8_t*>(h->d_stage);
  uint8_t* dy = dx + align_up(xb, 256);
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = cudaMemcpyAsync(dx, x_host, xb, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, "copy of x");
  st = stagq_gemv_ex(h, bits, dx, n, dy, 0u, cuda_stream);
  if (st) return st;
  e = cudaMemcpyAsync(y_host, dy, yb, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return cuda_fail(e, "copy of y");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return STAGQ_OK;
}

namespace {
// Device staging of stagq_gemv_host_many: one growing buffer per device.
struct ManyStage {
  std::mutex mu;
  void* ptr[64] = {};
  size_t bytes[64] = {};
};
ManyStage& many_stage() {
  static ManyStage s;
  return s;
}
}  // namespace

extern "C" int stagq_gemv_host_many(int count, const stagq_handle* hs, const int* bits, const void* const* x_hosts,
                                    const int* ns, void* const* y_hosts, void* cuda_stream) {
  if (count < 1 || count > STAGQ_MAX_MANY) return fail(STAGQ_EINVAL, "count outside 1..STAGQ_MAX_MANY");
  if (!hs || !bits || !x_hosts || !ns || !y_hosts) return fail(STAGQ_EINVAL, "null array");
  size_t need = 0;
  for (int i = 0; i < count; ++i) {
    int st = check_handle_bits(hs[i], bits[i]);
    if (st) return st;
    if (!x_hosts[i] || !y_hosts[i]) return fail(STAGQ_EINVAL, "null x or y");
    if (ns[i] < 1 || ns[i] > STAGQ_MAX_BATCH) return fail(STAGQ_EINVAL, "n outside 1..STAGQ_MAX_BATCH");
    if (hs[i]->device != hs[0]->device) return fail(STAGQ_EINVAL, "handles on different devices");
    need += align_up((size_t)ns[i] * hs[i]->dm.in * 2, 256) + align_up((size_t)ns[i] * hs[i]->dm.out * 2, 256);
  }
  const int dev = hs[0]->device;
  if (dev < 0 || dev >= 64) return fail(STAGQ_EINVAL, "device index outside 0..63");
  DeviceGuard guard(dev);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");
  ManyStage& ms = many_stage();
  std::lock_guard<std::mutex> lock(ms.mu);
  if (ms.bytes[dev] < need) {
    if (ms.ptr[dev]) cudaFree(ms.ptr[dev]);
    ms.ptr[dev] = nullptr;
    ms.bytes[dev] = 0;
    cudaError_t e = cudaMalloc(&ms.ptr[dev], need);
    if (e != cudaSuccess) { cudaGetLastError(); return fail(STAGQ_ENOMEM, "staging allocation failed"); }
    ms.bytes[dev] = need;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  // x regions first, then y regions, each on 256 bytes
  uint8_t* base = static_cast<uint8_t*>(ms.ptr[dev]);
  size_t off = 0;
  for (int i = 0; i < count; ++i) {
    const size_t xb = (size_t)ns[i] * hs[i]->dm.in * 2;
    cudaError_t e = cudaMemcpyAsync(base + off, x_hosts[i], xb, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(e, "copy of x");
    off += align_up(xb, 256);
  }
  const size_t y0 = off;
  off = 0;
  size_t yoff = y0;
  for (int i = 0; i < count; ++i) {
    const size_t xb = (size_t)ns[i] * hs[i]->dm.in * 2, yb = (size_t)ns[i] * hs[i]->dm.out * 2;
    int st = stagq_gemv_ex(hs[i], bits[i], base + off, ns[i], base + yoff, 0u, cuda_stream);
    if (st) return st;
    off += align_up(xb, 256);
    yoff += align_up(yb, 256);
  }
  yoff = y0;
  for (int i = 0; i < count; ++i) {
    const size_t yb = (size_t)ns[i] * hs[i]->dm.out * 2;
    cudaError_t e = cudaMemcpyAsync(y_hosts[i], base + yoff, yb, cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return cuda_fail(e, "copy of y");
    yoff += align_up(yb, 256);
  }
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return STAGQ_OK;
}

extern "C" int stagq_decode_levels(stagq_handle h, int bits, uint8_t* u_dev, void* cuda_stream) {
  int st = check_handle_bits(h, bits);
  if (st) return st;
  if (!u_dev) return fail(STAGQ_EINVAL, "null output");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");
  cudaError_t e = launch_decode_levels(h->dm, bits, u_dev, static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return STAGQ_OK;
}

extern "C" int64_t stagq_bytes(stagq_handle h, int bits, int n) {
  if (!h || bits < 2 || bits > 2 + h->dm.n_planes || n < 1) return -1;
  const int64_t out = h->dm.out, in = h->dm.in;
  return out * in * bits / 8 + out * in / h->dm.group + 4 * h->dm.nnz + 4 * (out + 1) + 2 * (int64_t)n * in +
         2 * (int64_t)n * out;
}

extern "C" int stagq_check(stagq_handle h) {
  if (!h) return fail(STAGQ_EINVAL, "null handle");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "work on the handle's device failed");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending CUDA error");
  uint32_t word = 0;
  e = cudaMemcpy(&word, h->dm.status, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word) {
    e = cudaMemset(h->dm.status, 0, 4);
    if (e != cudaSuccess) return cuda_fail(e, "status reset");
    return fail(STAGQ_ETIMEOUT, "a GEMV kernel gave up waiting for its copies (status " + std::to_string(word) + ")");
  }
  return STAGQ_OK;
}

extern "C" int stagq_debug_stall(stagq_handle h, uint32_t stall_ns) {
  if (!h) return fail(STAGQ_EINVAL, "null handle");
  h->dm.debug_stall_ns = stall_ns;
  return STAGQ_OK;
}

extern "C" int stagq_debug_side_record(stagq_handle h, stagq_side_layout_t* layout, void* cut_host, int64_t cut_bytes,
                                       void* cut1_host, int64_t cut1_bytes) {
  if (!h || !layout) return fail(STAGQ_EINVAL, "null argument");
  const DeviceMatrix& m = h->dm;
  const int KW = k_slices(m.in), RG = row_groups(KW);
  const int rows_cap = (m.out + m.side_grid - 1) / m.side_grid;
  layout->grid = m.side_grid;
  layout->stride = m.side_stride;
  layout->ent_off = m.side_ent_off;
  layout->row_groups = RG;
  layout->k_slices = KW;
  layout->class_rows = (rows_cap + RG - 1) / RG;
  layout->grid1 = m.side1_grid;
  layout->stride1 = m.side1_stride;
  layout->ent_off1 = m.side1_ent_off;
  const int64_t need = (int64_t)m.side_grid * m.side_stride, need1 = (int64_t)m.side1_grid * m.side1_stride;
  if ((cut_host && cut_bytes < need) || (cut1_host && cut1_bytes < need1))
    return fail(STAGQ_EINVAL, "host buffer smaller than the cut");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");
  cudaError_t e = cudaSuccess;
  if (cut_host) e = cudaMemcpy(cut_host, m.side, (size_t)need, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && cut1_host) e = cudaMemcpy(cut1_host, m.side1, (size_t)need1, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "copy of the side record");
  return STAGQ_OK;
}

extern "C" int stagq_info(stagq_handle h, stagq_info_t* info) {
  if (!h || !info) return fail(STAGQ_EINVAL, "null argument");
  info->out = h->dm.out; info->in = h->dm.in; info->group = h->dm.group; info->n_planes = h->dm.n_planes;
  info->nnz = h->dm.nnz; info->device = h->device;
  info->device_bytes = (int64_t)(h->d_bytes + h->stage_bytes);
  return STAGQ_OK;
}

extern "C" void stagq_free(stagq_handle h) {
  if (!h) return;
  DeviceGuard guard(h->device);
  if (h->d_mem) cudaFree(h->d_mem);
  if (h->d_stage) cudaFree(h->d_stage);
  delete h;
}

// ---------------------------------------------------------------------------
// Host-buffer GEMV that allocates no device memory.
//
// stagq_gemv_host stages x and y in a device buffer that the handle allocates
// with cudaMalloc on first use. Some callers must not allocate at that point:
// code that runs under a fixed device-memory budget owned by another
// allocator, or in a phase where any new allocation is forbidden. This
// variant stages through kNoAllocStageBytes of statically reserved device
// memory instead (x at offset 0, y at kNoAllocXBytes). Every GPU that loads
// this library holds the array until the process exits.
namespace stagq {
namespace {

constexpr size_t kNoAllocXBytes = (size_t)STAGQ_MAX_BATCH * STAGQ_MAX_IN * 2;       // 256 KiB: any x
constexpr size_t kNoAllocStageBytes = (size_t)STAGQ_NOALLOC_STAGE_BYTES;            // x and y together

static __device__ __align__(256) uint8_t g_noalloc_stage[kNoAllocStageBytes];

// Device address of g_noalloc_stage on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the handle's device current -- on every call, not cached: a device reset
// (cudaDeviceReset) rebuilds the context and the array may then sit at a new
// address. The lookup allocates nothing and costs far less than the call's
// synchronous copies.
int noalloc_stage(uint8_t** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_stage);
  if (e != cudaSuccess || !p) return cuda_fail(e == cudaSuccess ? cudaErrorInvalidSymbol : e, "cudaGetSymbolAddress");
  *out = static_cast<uint8_t*>(p);
  return STAGQ_OK;
}

}  // namespace
}  // namespace stagq

extern "C" int stagq_gemv_host_noalloc(stagq_handle h, int bits, const void* x_host, int n, void* y_host,
                                       void* cuda_stream) {
  int st = check_handle_bits(h, bits);
  if (st) return st;
  if (!x_host || !y_host) return fail(STAGQ_EINVAL, "null x or y");
  if (n < 1 || n > STAGQ_MAX_BATCH) return fail(STAGQ_EINVAL, "n outside 1..STAGQ_MAX_BATCH");
  const size_t xb = (size_t)n * h->dm.in * 2, yb = (size_t)n * h->dm.out * 2;
  if (xb > kNoAllocXBytes || yb > kNoAllocStageBytes - kNoAllocXBytes)
    return fail(STAGQ_EINVAL, "n * out * 2 exceeds the static staging area (STAGQ_NOALLOC_STAGE_BYTES - 256 KiB)");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(STAGQ_ECUDA, "cudaSetDevice failed");
  uint8_t* stage = nullptr;
  st = noalloc_stage(&stage);
  if (st) return st;
  uint8_t* dx = stage;
  uint8_t* dy = stage + kNoAllocXBytes;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  // x is overwritten in full and the kernel writes every element of y, so
  // nothing left in the array by an earlier call is read.
  cudaError_t e = cudaMemcpyAsync(dx, x_host, xb, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, "copy of x");
  st = stagq_gemv_ex(h, bits, dx, n, dy, 0u, cuda_stream);
  if (st) return st;
  e = cudaMemcpyAsync(y_host, dy, yb, cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return cuda_fail(e, "copy of y");
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return STAGQ_OK;
}
