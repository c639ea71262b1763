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
//   4. fp16 codebooks over the initial pairs' log2(s) and lo/s (Appendix
//      E): uniform placement, or (STAGQ_CODEBOOK_RULES) the best of the nine
//      combinations of uniform, Lloyd and anchored-Lloyd placement by the
//      first term of Eq. 5, kept unless the deepest precision's error exceeds
//      a tenth of the two-bit error;
//   5. per-group pair: argmin of Eq. (5)-(6) with unit channel weights, or
//      the labelled "fast" rule (nearest codebook entry per coordinate);
//   6. base by nearest rounding (half up), 7. planes = sign of the residual
//      with sign(0) = +1 and half-steps s / 2^(k-1) (Eq. 7); held-out
//      positions keep zero digits.
// stagq_encode_guarded replaces step 1 by the paper's pre-grid ratio guard
// (Section 3.5: a group's largest-|w| entry when it exceeds T times the
// second largest) and adds the post-grid guard (Appendix E: per row, the
// position with the largest two-bit error (w - (lo + s q))^2; its base digit
// stays, its planes are zero, and it records the fp16 residual; the
// reconstruction there is lo + s q + residual, Eq. 4). The post-grid entry's
// column carries STAGQ_SIDE_POST.
// Every floating-point step is fp64 and sums run in index order, so the
// fields are reproducible bit for bit.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <functional>
#include <string>
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

// A codebook: fp64 values of its fp16 points, and the fp16 bits.
struct Book {
  double cb[16];
  uint16_t h[16];
};
constexpr int kRuleUniform = 0, kRuleLloyd = 1, kRuleAnchored = 2;
constexpr int kLloydMaxSteps = 100;        // Appendix E, Lloyd's rule: at most this many assignment steps
constexpr double kFallbackRatio = 0.1;      // Appendix E: deepest-precision error vs two-bit error

// Uniform placement (Appendix E): v_min + i (v_max - v_min) / 15; Lloyd's rule
// from there (each point the mean of its nearest values, summed in index
// order, ties to the lower point, empty points stay, at most 100 steps, until
// no assignment changes); anchored: points 0 and 15 stay at the range ends.
// No values: all zeros.
Book codebook_by_rule(const std::vector<double>& v, int rule) {
  Book b{};
  if (v.empty()) return b;
  double vmin = INFINITY, vmax = -INFINITY;
  for (double x : v) { vmin = std::min(vmin, x); vmax = std::max(vmax, x); }
  double c[16];
  for (int i = 0; i < 16; ++i) c[i] = vmin + (double)i * (vmax - vmin) / 15.0;
  if (rule != kRuleUniform) {
    std::vector<int> assign(v.size(), -1), a(v.size());
    for (int step = 0; step < kLloydMaxSteps; ++step) {
      for (size_t j = 0; j < v.size(); ++j) {
        int bi = 0;
        for (int i = 1; i < 16; ++i)
          if (std::fabs(v[j] - c[i]) < std::fabs(v[j] - c[bi])) bi = i;
        a[j] = bi;
      }
      if (step > 0 && a == assign) break;
      assign = a;
      for (int i = 0; i < 16; ++i) {
        if (rule == kRuleAnchored && (i == 0 || i == 15)) continue;
        double sm = 0.0;
        int64_t n = 0;
        for (size_t j = 0; j < v.size(); ++j)
          if (a[j] == i) { sm = sm + v[j]; ++n; }
        if (n) c[i] = sm / (double)n;
      }
    }
  }
  for (int i = 0; i < 16; ++i) {
    b.h[i] = double_to_half(c[i]);
    b.cb[i] = half_to_double(b.h[i]);
  }
  return b;
}

// The 256 (lo, s) of a codebook pair (Section 3.1), fp64 from the fp16 points.
struct PairTable {
  double lo[256], s[256], cbs[16], cbr[16];
};
PairTable make_pair_table(const Book& bs, const Book& br) {
  PairTable T;
  for (int i = 0; i < 16; ++i) { T.cbs[i] = bs.cb[i]; T.cbr[i] = br.cb[i]; }
  for (int p = 0; p < 256; ++p) {
    T.s[p] = std::exp2(T.cbs[p >> 4]);
    T.lo[p] = T.cbr[p & 15] * T.s[p];
  }
  return T;
}

// Eq. (5)-(6) of one group under (lo, s): (first term / (N-1), floor term sum).
std::pair<double, double> pair_terms(const double* V, int64_t g, int N, double lo, double s, double reach_sum,
                                     double* rec) {
  double recon_one[8];
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
  return {first, fl};
}

// Pair of one (non-empty) group: the Eq. (5) argmin (ties to the smaller
// index), or the labelled fast rule for groups with a nonzero range.
int choose_pair(const double* V, int64_t g, int N, const PairTable& T, int pair_mode, bool flat, double lo0, double s0,
                double reach_sum, double* rec) {
  if (pair_mode == STAGQ_PAIR_FAST && !flat) {
    const double L = std::log2(s0), r = lo0 / s0;
    int ba = 0, bb = 0;
    for (int i = 1; i < 16; ++i) {
      if (std::fabs(T.cbs[i] - L) < std::fabs(T.cbs[ba] - L)) ba = i;
      if (std::fabs(T.cbr[i] - r) < std::fabs(T.cbr[bb] - r)) bb = i;
    }
    return ba * 16 + bb;
  }
  double best = INFINITY;
  int pair = 0;
  for (int p = 0; p < 256; ++p) {
    const std::pair<double, double> t = pair_terms(V, g, N, T.lo[p], T.s[p], reach_sum, rec);
    const double D = t.first + kFloorLambda * t.second;
    if (D < best) { best = D; pair = p; }
  }
  return pair;
}

}  // namespace
}  // namespace stagq

using namespace stagq;

extern "C" int64_t stagq_side_record_count(int32_t out, int32_t in, double density) {
  return (int64_t)std::floor(density * (double)out * (double)in + 0.5);
}

namespace {

// Steps 2-7 (and the post-grid guard) for a given pre-grid hold-out set;
// writes at most `cap` side-record entries and sets f->nnz.
int encode_with(const uint16_t* w, const std::vector<uint8_t>& held, bool post_guard, int32_t pair_mode,
                int32_t n_threads, int64_t cap, stagq_fields* f);

int check_encode_args(const uint16_t* w, stagq_fields* f, int32_t pair_mode, const char* who) {
  if (!w || !f) return fail(STAGQ_EINVAL, std::string(who) + ": null argument");
  const int64_t out = f->out, in = f->in, g = f->group;
  if (out <= 0 || in <= 0 || g <= 0 || in % g) return fail(STAGQ_EINVAL, std::string(who) + ": bad shape or group");
  if (in > STAGQ_MAX_IN) return fail(STAGQ_EINVAL, std::string(who) + ": in exceeds STAGQ_MAX_IN");
  if (f->n_planes < 0 || f->n_planes > STAGQ_MAX_PLANES)
    return fail(STAGQ_EINVAL, std::string(who) + ": n_planes out of range");
  const int32_t pm = pair_mode & ~(int32_t)STAGQ_CODEBOOK_RULES;
  if (pm != STAGQ_PAIR_SEARCH && pm != STAGQ_PAIR_FAST)
    return fail(STAGQ_EINVAL, std::string(who) + ": unknown pair mode");
  if (!f->q || (f->n_planes && !f->planes) || !f->pair_idx || !f->row_ptr)
    return fail(STAGQ_EINVAL, std::string(who) + ": null field buffer");
  return STAGQ_OK;
}

}  // namespace

extern "C" int64_t stagq_guard_capacity(int32_t out, int32_t in, int32_t group) {
  if (out <= 0 || in <= 0 || group <= 0) return 0;
  return (int64_t)out * (in / group) + out;
}

extern "C" int stagq_encode_guarded(const uint16_t* w, double ratio_T, int32_t post_guard, int32_t pair_mode,
                                    int32_t n_threads, stagq_fields* f) {
  int st = check_encode_args(w, f, pair_mode, "stagq_encode_guarded");
  if (st) return st;
  if (!(ratio_T >= 1.0)) return fail(STAGQ_EINVAL, "stagq_encode_guarded: ratio_T must be >= 1");
  const int64_t out = f->out, in = f->in, g = f->group, ng = in / g;
  const int64_t cap = f->nnz;
  if (cap < stagq_guard_capacity((int32_t)out, (int32_t)in, (int32_t)g))
    return fail(STAGQ_EINVAL, "stagq_encode_guarded: f->nnz must be at least stagq_guard_capacity");
  if (cap && (!f->col || !f->val)) return fail(STAGQ_EINVAL, "stagq_encode_guarded: null field buffer");
  // pre-grid ratio guard: per group the first largest |w| (fp16 magnitude
  // bits order like |w|), held out when |w1| > T |w2|, w2 the largest of the rest.
  std::vector<uint8_t> held(out * in, 0);
  parallel_for(out * ng, n_threads, [&](int64_t a, int64_t b) {
    for (int64_t G = a; G < b; ++G) {
      const int64_t base = (G / ng) * in + (G % ng) * g;
      int64_t j1 = 0;
      for (int64_t c = 1; c < g; ++c)
        if ((w[base + c] & 0x7FFF) > (w[base + j1] & 0x7FFF)) j1 = c;
      double a2 = 0.0;
      for (int64_t c = 0; c < g; ++c)
        if (c != j1) a2 = std::max(a2, half_to_double(w[base + c] & 0x7FFF));
      const double a1 = half_to_double(w[base + j1] & 0x7FFF);
      if (a1 > ratio_T * a2) held[base + j1] = 1;
    }
  });
  return encode_with(w, held, post_guard != 0, pair_mode, n_threads, cap, f);
}

extern "C" int stagq_encode(const uint16_t* w, double density, int32_t pair_mode, int32_t n_threads,
                            stagq_fields* f) {
  int st = check_encode_args(w, f, pair_mode, "stagq_encode");
  if (st) return st;
  if (!(density >= 0.0 && density <= 1.0)) return fail(STAGQ_EINVAL, "stagq_encode: density outside [0,1]");
  const int64_t out = f->out, in = f->in;
  const int64_t nnz = stagq_side_record_count((int32_t)out, (int32_t)in, density);
  if (f->nnz != nnz) return fail(STAGQ_EINVAL, "stagq_encode: f->nnz must equal stagq_side_record_count");
  if (nnz && (!f->col || !f->val)) return fail(STAGQ_EINVAL, "stagq_encode: null field buffer");
  const int64_t total = out * in;

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
  return encode_with(w, held, false, pair_mode, n_threads, nnz, f);
}

namespace {

int encode_with(const uint16_t* w, const std::vector<uint8_t>& held, bool post_guard, int32_t pair_mode_flags,
                int32_t n_threads, int64_t cap, stagq_fields* f) {
  const bool codebook_rules = (pair_mode_flags & STAGQ_CODEBOOK_RULES) != 0;
  const int32_t pair_mode = pair_mode_flags & ~(int32_t)STAGQ_CODEBOOK_RULES;
  const int64_t out = f->out, in = f->in, g = f->group;
  const int n_planes = f->n_planes;
  const int N = 2 + n_planes;
  const int64_t total = out * in, ng = in / g, ngroups = out * ng;

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

  // clipped group values for the pair fit
  auto clipped = [&](int64_t G, double* V) {
    const int64_t base = (G / ng) * in + (G % ng) * g;
    double mx = -INFINITY, mn = INFINITY;
    for (int64_t c = 0; c < g; ++c)
      if (!held[base + c]) { const double v = half_to_double(w[base + c]); mx = std::max(mx, v); mn = std::min(mn, v); }
    for (int64_t c = 0; c < g; ++c) {
      const double v = half_to_double(w[base + c]);
      V[c] = held[base + c] ? (v >= 0.0 ? mx : mn) : v;
    }
  };
  double reach_sum = 0.0;
  for (int k = 3; k <= N; ++k) reach_sum += std::ldexp(1.0, -(k - 1));

  // 4. codebooks over the initial pairs of the groups with retained entries
  // and a nonzero range (group order): uniform placement, or with
  // STAGQ_CODEBOOK_RULES Appendix E's choice among uniform, Lloyd and
  // anchored-Lloyd placement for each codebook and its fallback.
  std::vector<double> vls, vrl;
  for (int64_t G = 0; G < ngroups; ++G) {
    if (empty[G] || flat[G]) continue;
    vls.push_back(std::log2(s0[G]));
    vrl.push_back(lo0[G] / s0[G]);
  }
  Book chosen_s = codebook_by_rule(vls, kRuleUniform), chosen_r = codebook_by_rule(vrl, kRuleUniform);
  if (codebook_rules) {
    Book bs[3], br[3];
    for (int r = 0; r < 3; ++r) { bs[r] = codebook_by_rule(vls, r); br[r] = codebook_by_rule(vrl, r); }
    std::vector<double> gmin(ngroups);
    double best = INFINITY;
    int best_s = 0, best_r = 0;
    for (int rs = 0; rs < 3; ++rs) {
      for (int rr = 0; rr < 3; ++rr) {
        const PairTable T = make_pair_table(bs[rs], br[rr]);
        parallel_for(ngroups, n_threads, [&](int64_t a, int64_t b) {
          std::vector<double> V(g), rec((size_t)g * (N - 1));
          for (int64_t G = a; G < b; ++G) {
            if (empty[G]) { gmin[G] = 0.0; continue; }
            clipped(G, V.data());
            double m = INFINITY;
            for (int p = 0; p < 256; ++p) m = std::min(m, pair_terms(V.data(), g, N, T.lo[p], T.s[p], reach_sum, rec.data()).first);
            gmin[G] = m;
          }
        });
        double tot = 0.0;
        for (int64_t G = 0; G < ngroups; ++G) tot = tot + gmin[G];
        if (tot < best) { best = tot; best_s = rs; best_r = rr; }
      }
    }
    // fallback: the deepest precision's error against the two-bit error under
    // the chosen codebooks and the final pair choice
    const PairTable T = make_pair_table(bs[best_s], br[best_r]);
    std::vector<double> e2g(ngroups, 0.0), eNg(ngroups, 0.0);
    parallel_for(ngroups, n_threads, [&](int64_t a, int64_t b) {
      std::vector<double> V(g), rec((size_t)g * (N - 1));
      double recon_one[8];
      for (int64_t G = a; G < b; ++G) {
        if (empty[G]) continue;
        clipped(G, V.data());
        const int pair = choose_pair(V.data(), g, N, T, pair_mode, flat[G], lo0[G], s0[G], reach_sum, rec.data());
        double e2 = 0.0, eN = 0.0;
        for (int64_t c = 0; c < g; ++c) {
          digits(V[c], T.lo[pair], T.s[pair], N, nullptr, recon_one);
          const double d2 = V[c] - recon_one[0], dN = V[c] - recon_one[N - 2];
          e2 = e2 + d2 * d2;
          eN = eN + dN * dN;
        }
        e2g[G] = e2;
        eNg[G] = eN;
      }
    });
    double e2 = 0.0, eN = 0.0;
    for (int64_t G = 0; G < ngroups; ++G) { e2 = e2 + e2g[G]; eN = eN + eNg[G]; }
    if (!(eN > kFallbackRatio * e2)) { chosen_s = bs[best_s]; chosen_r = br[best_r]; }
  }
  for (int i = 0; i < 16; ++i) {
    f->codebook_log2s[i] = chosen_s.h[i];
    f->codebook_lo_over_s[i] = chosen_r.h[i];
  }
  const PairTable T = make_pair_table(chosen_s, chosen_r);

  // 5-7. pair per group, then the digits.
  parallel_for(ngroups, n_threads, [&](int64_t a, int64_t b) {
    std::vector<double> V(g), rec((size_t)g * (N - 1));
    std::vector<uint8_t> bits(N > 2 ? N - 2 : 1);
    double recon_one[8];
    for (int64_t G = a; G < b; ++G) {
      const int64_t row = G / ng, base = row * in + (G % ng) * g;
      int pair = 0;
      if (!empty[G]) {
        clipped(G, V.data());
        pair = choose_pair(V.data(), g, N, T, pair_mode, flat[G], lo0[G], s0[G], reach_sum, rec.data());
      }
      f->pair_idx[G] = (uint8_t)pair;
      const double lo = T.lo[pair], s = T.s[pair];
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

  // post-grid guard: per row, the first position (not held out) with the
  // largest (w - (lo + s q))^2; keep q, zero its planes, record the residual.
  std::vector<int64_t> post_col(out, -1);
  std::vector<uint16_t> post_val(out, 0);
  if (post_guard) {
    parallel_for(out, n_threads, [&](int64_t a, int64_t b) {
      for (int64_t r = a; r < b; ++r) {
        double best = -1.0, best_r2 = 0.0;
        int64_t bc = -1;
        for (int64_t c = 0; c < in; ++c) {
          const int64_t idx = r * in + c;
          if (held[idx]) continue;
          const int p = f->pair_idx[r * ng + c / g];
          const double r2 = T.lo[p] + T.s[p] * (double)f->q[idx];
          const double d = half_to_double(w[idx]) - r2;
          const double e = d * d;
          if (e > best) { best = e; bc = c; best_r2 = r2; }
        }
        if (bc < 0) continue;
        post_col[r] = bc;
        post_val[r] = double_to_half(half_to_double(w[r * in + bc]) - best_r2);
        for (int k = 0; k < n_planes; ++k) f->planes[(int64_t)k * total + r * in + bc] = 0;
      }
    });
  }

  // side record, row-major CSR
  int64_t e = 0;
  for (int64_t r = 0; r < out; ++r) {
    f->row_ptr[r] = (int32_t)e;
    for (int64_t c = 0; c < in; ++c) {
      const bool pre = held[r * in + c] != 0, post = post_col[r] == c;
      if (!pre && !post) continue;
      if (e >= cap) return fail(STAGQ_EINVAL, "encoder: side record exceeds f->nnz");
      f->col[e] = (uint16_t)(post ? (c | STAGQ_SIDE_POST) : c);
      f->val[e] = post ? post_val[r] : w[r * in + c];
      ++e;
    }
  }
  f->row_ptr[out] = (int32_t)e;
  f->nnz = e;
  return STAGQ_OK;
}

}  // namespace
