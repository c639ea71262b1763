// StagQ encoder for synthetic fp16 matrices (host, multithreaded).
//
// Follows the encoder of the StagQ paper (arXiv 2610.05977), Sections 3.1-3.6
// and Appendices B and E, with the readings used for synthetic workloads:
//   1. side record = the largest-|w| entries (global density), ties to the
//      smaller flat index; the recorded value P is the fp16 weight (Eq. 4);
//   2. held-out entries are clipped to the next value inward for the pair fit
//      (Section 3.1): the group's largest retained value for w >= 0, its
//      smallest for w < 0;
//   3. initial pair (Appendix B): four symmetric levels, outer ones 6 % in
//      from the group's ends; groups with no retained entry or zero range
//      stay out of the codebook fit (the latter are always searched, the
//      former take pair 0 and zero digits);
//   4. uniform fp16 codebooks over the initial pairs' log2(s) and lo/s
//      (Appendix E);
//   5. per-group pair: argmin of Eq. (5)-(6) with unit channel weights, or
//      the labelled "fast" rule (nearest codebook entry per coordinate);
//   6. base by nearest rounding (half up), 7. planes = sign of the residual
//      with sign(0) = +1 and half-steps s / 2^(k-1) (Eq. 7); held-out
//      positions keep zero digits.
// Every floating-point step is fp64 and sums run in index order, so the
// fields are reproducible bit for bit.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <functional>
#include <thread>
#include <vector>

#include "host_common.hpp"

namespace stagq {
namespace {

constexpr double kEdgeFraction = 0.06;  // Appendix B
constexpr double kFloorLambda = 4.0;    // Section 3.1
constexpr double kDegenerateStep = 0.000000059604644775390625;  // 2^-24

void parallel_for(int64_t n, int n_threads, const std::function<void(int64_t, int64_t)>& fn) {
  if (n <= 0) return;
  int T = n_threads > 0 ? n_threads : (int)std::thread::hardware_concurrency();
  if (T < 1) T = 1;
  if (T > n) T = (int)n;
  if (T == 1) {
    fn(0, n);
    return;
  }
  std::vector<std::thread> th;
  th.reserve(T);
  for (int t = 0; t < T; ++t) {
    const int64_t a = n * t / T, b = n * (t + 1) / T;
    th.emplace_back([&, a, b] { fn(a, b); });
  }
  for (auto& x : th) x.join();
}

// Greedy digits of one value under (lo, s): base by nearest rounding, then
// the sign planes. recon[M-2] receives W^(M), M = 2..N.
inline int digits(double w, double lo, double s, int N, uint8_t* bits, double* recon) {
  double qf = std::floor((w - lo) / s + 0.5);
  qf = qf < 0.0 ? 0.0 : (qf > 3.0 ? 3.0 : qf);
  double r = lo + s * qf;
  recon[0] = r;
  for (int k = 3; k <= N; ++k) {
    const int b = (w - r) >= 0.0 ? 1 : 0;
    r = r + (2.0 * b - 1.0) * (s / std::ldexp(1.0, k - 1));
    if (bits) bits[k - 3] = (uint8_t)b;
    recon[k - 2] = r;
  }
  return (int)qf;
}

}  // namespace
}  // namespace stagq

using namespace stagq;

extern "C" int64_t stagq_side_record_count(int32_t out, int32_t in, double density) {
  return (int64_t)std::floor(density * (double)out * (double)in + 0.5);
}

extern "C" int stagq_encode(const uint16_t* w, double density, int32_t pair_mode, int32_t n_threads,
                            stagq_fields* f) {
  if (!w || !f) return fail(STAGQ_EINVAL, "stagq_encode: null argument");
  const int64_t out = f->out, in = f->in, g = f->group;
  const int n_planes = f->n_planes;
  if (out <= 0 || in <= 0 || g <= 0 || in % g) return fail(STAGQ_EINVAL, "stagq_encode: bad shape or group");
  if (in > STAGQ_MAX_IN) return fail(STAGQ_EINVAL, "stagq_encode: in exceeds STAGQ_MAX_IN");
  if (n_planes < 0 || n_planes > STAGQ_MAX_PLANES) return fail(STAGQ_EINVAL, "stagq_encode: n_planes out of range");
  if (!(density >= 0.0 && density <= 1.0)) return fail(STAGQ_EINVAL, "stagq_encode: density outside [0,1]");
  if (pair_mode != STAGQ_PAIR_SEARCH && pair_mode != STAGQ_PAIR_FAST)
    return fail(STAGQ_EINVAL, "stagq_encode: unknown pair mode");
  const int64_t nnz = stagq_side_record_count((int32_t)out, (int32_t)in, density);
  if (f->nnz != nnz) return fail(STAGQ_EINVAL, "stagq_encode: f->nnz must equal stagq_side_record_count");
  if (!f->q || (n_planes && !f->planes) || !f->pair_idx || !f->row_ptr || (nnz && (!f->col || !f->val)))
    return fail(STAGQ_EINVAL, "stagq_encode: null field buffer");

  const int N = 2 + n_planes;
  const int64_t total = out * in, ng = in / g, ngroups = out * ng;

  // 1. side record: top-|w| by the magnitude bits (monotone in |w|), ties to the smaller index.
  std::vector<uint8_t> held(total, 0);
  if (nnz >= total) {
    std::fill(held.begin(), held.end(), 1);
  } else if (nnz > 0) {
    std::vector<int64_t> hist(32768, 0);
    for (int64_t i = 0; i < total; ++i) hist[w[i] & 0x7FFF]++;
    int64_t acc = 0;
    int thr = 32767;
    for (; thr >= 0; --thr) {
      if (acc + hist[thr] >= nnz) break;
      acc += hist[thr];
    }
    int64_t need_tied = nnz - acc;  // entries with magnitude == thr to take, lowest index first
    for (int64_t i = 0; i < total; ++i) {
      const int m = w[i] & 0x7FFF;
      if (m > thr) held[i] = 1;
      else if (m == thr && need_tied > 0) { held[i] = 1; --need_tied; }
    }
  }

  // 2-3. clipped groups and initial pairs.
  std::vector<double> lo0(ngroups), s0(ngroups);
  std::vector<uint8_t> empty(ngroups, 0), flat(ngroups, 0);
  parallel_for(ngroups, n_threads, [&](int64_t a, int64_t b) {
    for (int64_t G = a; G < b; ++G) {
      const int64_t base = (G / ng) * in + (G % ng) * g;
      double mx = -INFINITY, mn = INFINITY;
      bool any = false;
      for (int64_t c = 0; c < g; ++c) {
        if (held[base + c]) continue;
        const double v = half_to_double(w[base + c]);
        mx = std::max(mx, v);
        mn = std::min(mn, v);
        any = true;
      }
      if (!any) { empty[G] = 1; mx = mn = 0.0; }
      // clipped values lie inside [mn, mx], so the clipped range is [mn, mx].
      const double R = mx - mn;
      const double l = mn + kEdgeFraction * R;
      const double top = mx - kEdgeFraction * R;
      lo0[G] = l;
      s0[G] = R > 0.0 ? (top - l) / 3.0 : kDegenerateStep;
      flat[G] = R > 0.0 ? 0 : 1;
    }
  });

  // 4. uniform codebooks over the groups with retained entries and a nonzero range.
  double lmin = INFINITY, lmax = -INFINITY, rmin = INFINITY, rmax = -INFINITY;
  bool any_group = false;
  for (int64_t G = 0; G < ngroups; ++G) {
    if (empty[G] || flat[G]) continue;
    const double L = std::log2(s0[G]);
    const double r = lo0[G] / s0[G];
    lmin = std::min(lmin, L); lmax = std::max(lmax, L);
    rmin = std::min(rmin, r); rmax = std::max(rmax, r);
    any_group = true;
  }
  for (int i = 0; i < 16; ++i) {
    f->codebook_log2s[i] = any_group ? double_to_half(lmin + (double)i * (lmax - lmin) / 15.0) : 0;
    f->codebook_lo_over_s[i] = any_group ? double_to_half(rmin + (double)i * (rmax - rmin) / 15.0) : 0;
  }
  double cbs[16], cbr[16], tab_lo[256], tab_s[256];
  for (int i = 0; i < 16; ++i) {
    cbs[i] = half_to_double(f->codebook_log2s[i]);
    cbr[i] = half_to_double(f->codebook_lo_over_s[i]);
  }
  for (int p = 0; p < 256; ++p) {
    tab_s[p] = std::exp2(cbs[p >> 4]);
    tab_lo[p] = cbr[p & 15] * tab_s[p];
  }
  double reach_sum = 0.0;
  for (int k = 3; k <= N; ++k) reach_sum += std::ldexp(1.0, -(k - 1));

  // 5-7. pair per group, then the digits.
  parallel_for(ngroups, n_threads, [&](int64_t a, int64_t b) {
    std::vector<double> V(g), rec((size_t)g * (N - 1));
    std::vector<uint8_t> bits(N > 2 ? N - 2 : 1);
    double recon_one[8];
    for (int64_t G = a; G < b; ++G) {
      const int64_t row = G / ng, base = row * in + (G % ng) * g;
      int pair = 0;
      if (!empty[G]) {
        // clipped group values
        double mx = -INFINITY, mn = INFINITY;
        for (int64_t c = 0; c < g; ++c)
          if (!held[base + c]) { const double v = half_to_double(w[base + c]); mx = std::max(mx, v); mn = std::min(mn, v); }
        for (int64_t c = 0; c < g; ++c) {
          const double v = half_to_double(w[base + c]);
          V[c] = held[base + c] ? (v >= 0.0 ? mx : mn) : v;
        }
        if (pair_mode == STAGQ_PAIR_FAST && !flat[G]) {
          const double L = std::log2(s0[G]), r = lo0[G] / s0[G];
          int ba = 0, bb = 0;
          for (int i = 1; i < 16; ++i) {
            if (std::fabs(cbs[i] - L) < std::fabs(cbs[ba] - L)) ba = i;
            if (std::fabs(cbr[i] - r) < std::fabs(cbr[bb] - r)) bb = i;
          }
          pair = ba * 16 + bb;
        } else {
          double best = INFINITY;
          for (int p = 0; p < 256; ++p) {
            const double lo = tab_lo[p], s = tab_s[p];
            for (int64_t c = 0; c < g; ++c) {
              digits(V[c], lo, s, N, nullptr, recon_one);
              for (int M = 2; M <= N; ++M) rec[(size_t)(M - 2) * g + c] = recon_one[M - 2];
            }
            double first = 0.0;
            for (int M = 2; M <= N; ++M) {
              double sm = 0.0;
              for (int64_t c = 0; c < g; ++c) {
                const double e = V[c] - rec[(size_t)(M - 2) * g + c];
                sm = sm + e * e;
              }
              first = first + sm;
            }
            first = first / (double)(N - 1);
            const double rho = s * reach_sum;
            double fl = 0.0;
            for (int64_t c = 0; c < g; ++c) {
              double e = std::fabs(V[c] - rec[c]) - rho;
              e = e > 0.0 ? e : 0.0;
              fl = fl + e * e;
            }
            const double D = first + kFloorLambda * fl;
            if (D < best) { best = D; pair = p; }
          }
        }
      }
      f->pair_idx[G] = (uint8_t)pair;
      const double lo = tab_lo[pair], s = tab_s[pair];
      for (int64_t c = 0; c < g; ++c) {
        const int64_t idx = base + c;
        if (held[idx]) {
          f->q[idx] = 0;
          for (int k = 0; k < n_planes; ++k) f->planes[(int64_t)k * total + idx] = 0;
          continue;
        }
        const int q = digits(half_to_double(w[idx]), lo, s, N, bits.data(), recon_one);
        f->q[idx] = (uint8_t)q;
        for (int k = 0; k < n_planes; ++k) f->planes[(int64_t)k * total + idx] = bits[k];
      }
    }
  });

  // side record, row-major CSR
  int64_t e = 0;
  for (int64_t r = 0; r < out; ++r) {
    f->row_ptr[r] = (int32_t)e;
    for (int64_t c = 0; c < in; ++c) {
      if (!held[r * in + c]) continue;
      f->col[e] = (uint16_t)c;
      f->val[e] = w[r * in + c];
      ++e;
    }
  }
  f->row_ptr[out] = (int32_t)e;
  return STAGQ_OK;
}
