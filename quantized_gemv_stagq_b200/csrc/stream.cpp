// Plane-major packer, host re-read of packed levels, stream validation and
// the on-disk stream file (host only).
#include <sys/types.h>

#include <cstdio>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

#include "host_common.hpp"
#include "layout.cuh"
#include "stream.hpp"

namespace stagq {

static thread_local std::string g_last_error;
void set_error(const std::string& msg) { g_last_error = msg; }
const char* last_error() { return g_last_error.c_str(); }

int check_shape(int64_t out, int64_t in, int64_t group, int n_planes) {
  if (out <= 0 || in <= 0) return fail(STAGQ_EINVAL, "shape must be positive");
  if (in % STAGQ_IN_MULTIPLE) return fail(STAGQ_EINVAL, "in must be a multiple of 128");
  if (in > STAGQ_MAX_IN) return fail(STAGQ_EINVAL, "in exceeds STAGQ_MAX_IN");
  if (group < STAGQ_MIN_GROUP || in % group || (group & (group - 1)) != 0)
    return fail(STAGQ_EINVAL, "group must be a power of two >= 16 that divides in");
  if (n_planes < 0 || n_planes > STAGQ_MAX_PLANES) return fail(STAGQ_EINVAL, "n_planes out of range");
  if (out > (int64_t)1 << 30) return fail(STAGQ_EINVAL, "out too large");
  return STAGQ_OK;
}

int validate_stream(const stagq_host_stream* s) {
  if (!s) return fail(STAGQ_EINVAL, "null stream");
  int st = check_shape(s->out, s->in, s->group, s->n_planes);
  if (st) return st;
  if (!s->planes || !s->pair_idx || !s->row_ptr) return fail(STAGQ_EINVAL, "null stream array");
  if (s->nnz < 0 || s->nnz > (int64_t)s->out * s->in) return fail(STAGQ_EFORMAT, "nnz out of range");
  if (s->nnz > 0 && (!s->col || !s->val)) return fail(STAGQ_EINVAL, "null side-record array");
  if (s->row_ptr[0] != 0) return fail(STAGQ_EFORMAT, "row_ptr[0] != 0");
  for (int64_t r = 0; r < s->out; ++r) {
    if (s->row_ptr[r + 1] < s->row_ptr[r]) return fail(STAGQ_EFORMAT, "row_ptr not monotone");
    if (s->row_ptr[r + 1] - s->row_ptr[r] > s->in) return fail(STAGQ_EFORMAT, "row holds more entries than columns");
  }
  if (s->row_ptr[s->out] != s->nnz) return fail(STAGQ_EFORMAT, "row_ptr[out] != nnz");
  constexpr uint16_t kCol = 0x7FFF;  // bit 15: post-grid flag (STAGQ_SIDE_POST)
  for (int64_t e = 0; e < s->nnz; ++e)
    if ((s->col[e] & kCol) >= s->in) return fail(STAGQ_EFORMAT, "side-record column >= in");
  for (int64_t r = 0; r < s->out; ++r)
    for (int64_t e = (int64_t)s->row_ptr[r] + 1; e < s->row_ptr[r + 1]; ++e)
      if ((s->col[e] & kCol) <= (s->col[e - 1] & kCol))
        return fail(STAGQ_EFORMAT, "side-record columns not increasing in a row");
  // Digits under the side record (Section 3.6: the planes skip held-out
  // positions). The GEMV corrects a held-out position by x_c (v - lo_M) or
  // x_c (r + lo - lo_M), which is exact only if the main stream decodes lo_M
  // there (a pre-grid entry: q = 0 and zero planes) or lo_M + s q (a
  // post-grid entry: zero planes). Checked at the stream's full depth N.
  const int N = 2 + s->n_planes;
  const int64_t out = s->out, in = s->in;
  for (int64_t r = 0; r < out; ++r) {
    for (int64_t e = s->row_ptr[r]; e < s->row_ptr[r + 1]; ++e) {
      const int64_t c = s->col[e] & kCol, chunk = c / kChunk;
      uint32_t base[4];
      uint32_t pw[STAGQ_MAX_PLANES][2] = {};
      std::memcpy(base, s->planes + base_chunk_offset(r, in, chunk), 16);
      for (int k = 3; k <= N; ++k)
        std::memcpy(pw[k - 3], s->planes + plane_region_offset(out, in, k) + plane_chunk_offset(r, in, chunk), 8);
      const int u = chunk_level(base, pw, N, (int)(c % kChunk));
      const bool post = (s->col[e] & STAGQ_SIDE_POST) != 0;
      if (post ? (u & ((1 << (N - 2)) - 1)) != 0 : u != 0)
        return fail(STAGQ_EFORMAT, post ? "nonzero plane digit under a post-grid side-record entry"
                                        : "nonzero digit under a pre-grid side-record entry");
    }
  }
  return STAGQ_OK;
}

}  // namespace stagq

using namespace stagq;

extern "C" const char* stagq_last_error(void) { return stagq::last_error(); }

extern "C" const char* stagq_strerror(int status) {
  switch (status) {
    case STAGQ_OK: return "ok";
    case STAGQ_EINVAL: return "invalid argument";
    case STAGQ_EFORMAT: return "malformed stream";
    case STAGQ_ENOMEM: return "out of memory";
    case STAGQ_ECUDA: return "CUDA error";
    case STAGQ_EIO: return "I/O error";
    case STAGQ_ENODEV: return "no usable sm_100 device";
    case STAGQ_ETIMEOUT: return "kernel gave up waiting for its copies";
    default: return "unknown status";
  }
}

extern "C" int64_t stagq_stream_plane_bytes(int32_t out, int32_t in, int32_t n_planes) {
  return (int64_t)out * in / 4 + (int64_t)n_planes * ((int64_t)out * in / 8);
}

extern "C" int stagq_pack(const stagq_fields* f, uint8_t* planes_out) {
  if (!f || !planes_out || !f->q) return fail(STAGQ_EINVAL, "stagq_pack: null argument");
  int st = check_shape(f->out, f->in, f->group, f->n_planes);
  if (st) return st;
  if (f->n_planes && !f->planes) return fail(STAGQ_EINVAL, "stagq_pack: null planes");
  const int64_t out = f->out, in = f->in, total = out * in, nchunk = in / kChunk;
  const int np = f->n_planes;
  std::memset(planes_out, 0, (size_t)stagq_stream_plane_bytes(f->out, f->in, np));
  for (int64_t r = 0; r < out; ++r) {
    for (int64_t c = 0; c < nchunk; ++c) {
      uint32_t base[4] = {0, 0, 0, 0};
      uint32_t pw[STAGQ_MAX_PLANES][2] = {};
      for (int t = 0; t < kChunk; ++t) {
        const int64_t idx = r * in + c * kChunk + t;
        const ChunkPos p = chunk_pos(t);
        const uint32_t q = f->q[idx];
        if (q > 3) return fail(STAGQ_EINVAL, "stagq_pack: base digit > 3");
        base[p.i] |= q << base_bit(p);
        for (int k = 3; k < 3 + np; ++k) {
          const uint32_t b = f->planes[(int64_t)(k - 3) * total + idx];
          if (b > 1) return fail(STAGQ_EINVAL, "stagq_pack: plane digit > 1");
          const int bit = k == 3 ? plane3_bit(p) : k == 4 ? plane4_bit(p) : plane56_bit(p);
          pw[k - 3][p.i >> 1] |= b << bit;
        }
      }
      std::memcpy(planes_out + base_chunk_offset(r, in, c), base, 16);
      for (int k = 3; k < 3 + np; ++k)
        std::memcpy(planes_out + plane_region_offset(out, in, k) + plane_chunk_offset(r, in, c), pw[k - 3], 8);
    }
  }
  return STAGQ_OK;
}

extern "C" int stagq_unpack_levels_host(const stagq_host_stream* s, int bits, uint8_t* u_out) {
  if (!s || !u_out || !s->planes) return fail(STAGQ_EINVAL, "stagq_unpack_levels_host: null argument");
  int st = check_shape(s->out, s->in, s->group, s->n_planes);
  if (st) return st;
  if (bits < 2 || bits > 2 + s->n_planes) return fail(STAGQ_EINVAL, "bits out of range");
  const int64_t out = s->out, in = s->in, nchunk = in / kChunk;
  for (int64_t r = 0; r < out; ++r) {
    for (int64_t c = 0; c < nchunk; ++c) {
      uint32_t base[4];
      uint32_t pw[STAGQ_MAX_PLANES][2] = {};
      std::memcpy(base, s->planes + base_chunk_offset(r, in, c), 16);
      for (int k = 3; k <= bits; ++k)
        std::memcpy(pw[k - 3], s->planes + plane_region_offset(out, in, k) + plane_chunk_offset(r, in, c), 8);
      for (int t = 0; t < kChunk; ++t)
        u_out[r * in + c * kChunk + t] = (uint8_t)chunk_level(base, pw, bits, t);
    }
  }
  return STAGQ_OK;
}

// ---------------------------------------------------------------- files
namespace {
constexpr char kMagic[8] = {'S', 'T', 'A', 'G', 'Q', 'S', '1', '\0'};
struct FileHeader {
  char magic[8];
  int32_t out, in, group, n_planes;
  int64_t nnz;
  uint16_t cb_log2s[16], cb_lo_over_s[16];
};
}  // namespace

extern "C" int stagq_save(const stagq_host_stream* s, const char* path) {
  int st = validate_stream(s);
  if (st) return st;
  if (!path) return fail(STAGQ_EINVAL, "stagq_save: null path");
  FILE* fp = std::fopen(path, "wb");
  if (!fp) return fail(STAGQ_EIO, std::string("cannot open ") + path);
  FileHeader h;
  std::memcpy(h.magic, kMagic, 8);
  h.out = s->out; h.in = s->in; h.group = s->group; h.n_planes = s->n_planes; h.nnz = s->nnz;
  std::memcpy(h.cb_log2s, s->codebook_log2s, 32);
  std::memcpy(h.cb_lo_over_s, s->codebook_lo_over_s, 32);
  const int64_t pb = stagq_stream_plane_bytes(s->out, s->in, s->n_planes);
  const int64_t ngr = (int64_t)s->out * (s->in / s->group);
  bool ok = std::fwrite(&h, sizeof h, 1, fp) == 1 &&
            std::fwrite(s->planes, 1, pb, fp) == (size_t)pb &&
            std::fwrite(s->pair_idx, 1, ngr, fp) == (size_t)ngr &&
            std::fwrite(s->row_ptr, 4, s->out + 1, fp) == (size_t)(s->out + 1) &&
            (s->nnz == 0 || (std::fwrite(s->col, 2, s->nnz, fp) == (size_t)s->nnz &&
                             std::fwrite(s->val, 2, s->nnz, fp) == (size_t)s->nnz));
  ok = (std::fclose(fp) == 0) && ok;
  return ok ? STAGQ_OK : fail(STAGQ_EIO, "short write");
}

namespace stagq {
int read_stream_file(const char* path, HostStreamBuffers* buf) {
  if (!path || !buf) return fail(STAGQ_EINVAL, "null argument");
  FILE* fp = std::fopen(path, "rb");
  if (!fp) return fail(STAGQ_EIO, std::string("cannot open ") + path);
  FileHeader h;
  if (std::fread(&h, sizeof h, 1, fp) != 1 || std::memcmp(h.magic, kMagic, 8) != 0) {
    std::fclose(fp);
    return fail(STAGQ_EFORMAT, "not a StagQ stream file");
  }
  int st = check_shape(h.out, h.in, h.group, h.n_planes);
  if (st || h.nnz < 0 || h.nnz > (int64_t)h.out * h.in) {
    std::fclose(fp);
    return st ? st : fail(STAGQ_EFORMAT, "bad nnz in header");
  }
  const int64_t pb = stagq_stream_plane_bytes(h.out, h.in, h.n_planes);
  const int64_t ngr = (int64_t)h.out * (h.in / h.group);
  // The file must hold exactly what its header declares: checked before any
  // allocation, so a corrupt or hostile header cannot ask for terabytes.
  const int64_t expect = (int64_t)sizeof h + pb + ngr + 4 * ((int64_t)h.out + 1) + 4 * h.nnz;
  if (fseeko(fp, 0, SEEK_END) != 0 || ftello(fp) != (off_t)expect || fseeko(fp, (off_t)sizeof h, SEEK_SET) != 0) {
    std::fclose(fp);
    return fail(STAGQ_EFORMAT, "stream file size does not match its header");
  }
  try {
    buf->planes.resize(pb);
    buf->pair_idx.resize(ngr);
    buf->row_ptr.resize(h.out + 1);
    buf->col.resize(h.nnz);
    buf->val.resize(h.nnz);
  } catch (...) {
    std::fclose(fp);
    return fail(STAGQ_ENOMEM, "host allocation for stream file failed");
  }
  bool ok = std::fread(buf->planes.data(), 1, pb, fp) == (size_t)pb &&
            std::fread(buf->pair_idx.data(), 1, ngr, fp) == (size_t)ngr &&
            std::fread(buf->row_ptr.data(), 4, h.out + 1, fp) == (size_t)(h.out + 1) &&
            (h.nnz == 0 || (std::fread(buf->col.data(), 2, h.nnz, fp) == (size_t)h.nnz &&
                            std::fread(buf->val.data(), 2, h.nnz, fp) == (size_t)h.nnz));
  std::fclose(fp);
  if (!ok) return fail(STAGQ_EFORMAT, "truncated stream file");
  stagq_host_stream& s = buf->view;
  s.out = h.out; s.in = h.in; s.group = h.group; s.n_planes = h.n_planes; s.nnz = h.nnz;
  std::memcpy(s.codebook_log2s, h.cb_log2s, 32);
  std::memcpy(s.codebook_lo_over_s, h.cb_lo_over_s, 32);
  s.planes = buf->planes.data();
  s.pair_idx = buf->pair_idx.data();
  s.row_ptr = buf->row_ptr.data();
  s.col = buf->col.data();
  s.val = buf->val.data();
  return validate_stream(&s);
}
}  // namespace stagq
