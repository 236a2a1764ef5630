// CPU oracle for the score -> select -> compact path.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
// calls this file; only the tests, the package's smoke check and the bench's
// CPU-baseline leg do.  It shares no code with the CUDA path: it has its own
// bf16 decoding, band pairing, frequencies, fold, scores, selection and
// compaction, written as plainly as possible in fp64.
//
// Source: the web page "The future-offset average in TriAttention can be
// precomputed" (hozhoke.com).  Section names below are that page's:
//   "The score TriAttention computes"              cosine form of S_trig
//   "The same score, read as arrows in the plane"  complex (phasor) form
//   "The averaging step - the one we improve"      offset average, its
//        factorisation, the folded form with W_f and the polar form with mu'_f
// The real 2x2 per-band map is the page's closing remark of that section (the
// weight folds into the real cosine/sine coefficients as a fixed 2x2 map).
//
// Keep-highest selection: same page, opening section (the cache keeps the
// highest-scoring keys); the budget B is TriAttention's KV budget (README of
// WeianMao/triattention, default 2048).
//
// Readings where the page is silent (each one listed in the design notes):
//   * band pairing: half split (f, f + d/2) by default, interleaved (2f, 2f+1)
//     as an option; the page only says that the rotation turns two
//     coordinates at a time;
//   * the kept distance Delta is one scalar per pruning event (delta0);
//   * mean over the schedule D taken as a multiset (duplicates count);
//   * order: score descending, then index ascending; NaN ranks lowest and
//     -0 equals +0; kept indices are returned ascending;
//   * paged compaction is an in-place hole fill (see orc_holefill).
//
// Parity status: every function here is pinned by a CPU test against a
// closed form, a textbook special case, an invariant or brute force.

#include <algorithm>
#include <cmath>
#include <complex>
#include <cstdint>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

using cplx = std::complex<double>;

namespace {

// bf16 is the top half of an IEEE binary32: widen exactly.
double bf16_value(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Which two coordinates of a d-vector form rotary band f.
void band_coords(int d, int pairing, int f, int* re, int* im) {
  if (pairing == 0) {          // half split (rotate_half convention)
    *re = f;
    *im = f + d / 2;
  } else {                     // interleaved pairs
    *re = 2 * f;
    *im = 2 * f + 1;
  }
}

// omega_f = theta^(-2f/d)   ("The score TriAttention computes")
std::vector<double> frequencies(double theta, int d) {
  std::vector<double> w(d / 2);
  for (int f = 0; f < d / 2; ++f) w[f] = std::pow(theta, -2.0 * f / d);
  return w;
}

// W_f = (1/|D|) sum_{delta in D} e^{i omega_f delta}   (folded form)
std::vector<cplx> offset_weights(const std::vector<double>& omega, const double* D, int nD) {
  std::vector<cplx> W(omega.size());
  for (size_t f = 0; f < omega.size(); ++f) {
    cplx acc(0.0, 0.0);
    for (int t = 0; t < nD; ++t) acc += std::polar(1.0, omega[f] * D[t]);
    W[f] = acc / static_cast<double>(nD);
  }
  return W;
}

// Band f of a vector as a complex number.
cplx band_of_keys(const uint16_t* k, int d, int pairing, int f) {
  int re, im;
  band_coords(d, pairing, f, &re, &im);
  return cplx(bf16_value(k[re]), bf16_value(k[im]));
}

cplx band_of_center(const float* q, int d, int pairing, int f) {
  int re, im;
  band_coords(d, pairing, f, &re, &im);
  return cplx(static_cast<double>(q[re]), static_cast<double>(q[im]));
}

// Run fn(i) for i in [0, n) over nthreads std::threads (contiguous ranges).
void parallel_for(int64_t n, int nthreads, const std::function<void(int64_t)>& fn) {
  if (nthreads <= 1 || n < 2) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  int t = static_cast<int>(std::min<int64_t>(nthreads, n));
  std::vector<std::thread> pool;
  int64_t chunk = (n + t - 1) / t;
  for (int k = 0; k < t; ++k) {
    int64_t lo = k * chunk, hi = std::min(n, lo + chunk);
    if (lo >= hi) break;
    pool.emplace_back([lo, hi, &fn] {
      for (int64_t i = lo; i < hi; ++i) fn(i);
    });
  }
  for (auto& th : pool) th.join();
}

// Strict "ranks above" for the selection order: larger score first, NaN last,
// equal scores (with -0 == +0) by lower index.
template <typename T>
bool ranks_above(T si, int64_t i, T sj, int64_t j) {
  bool ni = std::isnan(si), nj = std::isnan(sj);
  if (ni || nj) {
    if (ni && nj) return i < j;
    return nj;                 // a number ranks above NaN
  }
  if (si != sj) return si > sj;
  return i < j;
}

template <typename T>
int64_t select_top(const T* s, int64_t n, int64_t B, int32_t* kept) {
  std::vector<int64_t> order(n);
  for (int64_t i = 0; i < n; ++i) order[i] = i;
  std::sort(order.begin(), order.end(),
            [s](int64_t a, int64_t b) { return ranks_above(s[a], a, s[b], b); });
  int64_t m = std::min(n, B);
  std::vector<int64_t> top(order.begin(), order.begin() + m);
  std::sort(top.begin(), top.end());
  for (int64_t j = 0; j < m; ++j) kept[j] = static_cast<int32_t>(top[j]);
  return m;
}

}  // namespace

extern "C" {

// omega_f for f = 0..d/2-1.
void orc_frequencies(double theta, int d, double* omega_out) {
  std::vector<double> w = frequencies(theta, d);
  for (int f = 0; f < d / 2; ++f) omega_out[f] = w[f];
}

// W_f for f = 0..d/2-1 (real and imaginary parts).
void orc_offset_weights(double theta, int d, const double* D, int nD, double* W_re, double* W_im) {
  std::vector<cplx> W = offset_weights(frequencies(theta, d), D, nD);
  for (int f = 0; f < d / 2; ++f) {
    W_re[f] = W[f].real();
    W_im[f] = W[f].imag();
  }
}

// O-i, the cosine form, averaged literally over the schedule:
//   s = (1/|D|) sum_delta sum_f |q_f| |k_f| cos(omega_f (delta0 + delta) + phi_f),
//   phi_f = arg q_f - arg k_f.
// ("The score TriAttention computes", averaged as in "The averaging step").
// A band whose query or key part is zero contributes 0.
void orc_score_cosine(const uint16_t* keys, int64_t n, int d, const float* qc, double theta,
                      const double* D, int nD, double delta0, int pairing, int nthreads,
                      double* out) {
  std::vector<double> omega = frequencies(theta, d);
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    double total = 0.0;
    for (int t = 0; t < nD; ++t) {
      double s = 0.0;
      for (int f = 0; f < d / 2; ++f) {
        cplx q = band_of_center(qc, d, pairing, f);
        cplx kf = band_of_keys(k, d, pairing, f);
        double nq = std::hypot(q.real(), q.imag());
        double nk = std::hypot(kf.real(), kf.imag());
        if (nq == 0.0 || nk == 0.0) continue;
        double phi = std::atan2(q.imag(), q.real()) - std::atan2(kf.imag(), kf.real());
        s += nq * nk * std::cos(omega[f] * (delta0 + D[t]) + phi);
      }
      total += s;
    }
    out[i] = total / nD;
  });
}

// O-ii, the complex form, averaged literally over the schedule:
//   s = (1/|D|) sum_delta Re sum_f q_f conj(k_f) e^{i omega_f (delta0 + delta)}.
// The rotation e^{i omega_f (delta0+delta)} does not involve the key, so it is
// tabulated once per call ([|D|][F]), as the upstream table of cosines is.
void orc_score_literal(const uint16_t* keys, int64_t n, int d, const float* qc, double theta,
                       const double* D, int nD, double delta0, int pairing, int nthreads,
                       double* out) {
  const int F = d / 2;
  std::vector<double> omega = frequencies(theta, d);
  std::vector<cplx> rot(static_cast<size_t>(nD) * F);
  for (int t = 0; t < nD; ++t)
    for (int f = 0; f < F; ++f) rot[static_cast<size_t>(t) * F + f] = std::polar(1.0, omega[f] * (delta0 + D[t]));
  std::vector<cplx> q(F);
  for (int f = 0; f < F; ++f) q[f] = band_of_center(qc, d, pairing, f);
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    std::vector<cplx> qk(F);
    for (int f = 0; f < F; ++f) qk[f] = q[f] * std::conj(band_of_keys(k, d, pairing, f));
    double total = 0.0;
    for (int t = 0; t < nD; ++t) {
      cplx s(0.0, 0.0);
      for (int f = 0; f < F; ++f) s += qk[f] * rot[static_cast<size_t>(t) * F + f];
      total += s.real();
    }
    out[i] = total / nD;
  });
}

// Per-key distances (pre-RoPE cache): key i sits at position pos[i], the
// query at position t, so its distance is t - pos[i]; the offset average is
//   s_i = (1/|D|) sum_delta Re sum_f q_f conj(k_f) e^{i omega_f (t - pos[i] + delta)},
// evaluated literally ("The averaging step - the one we improve", with the
// distance carried per key).
void orc_score_at_positions(const uint16_t* keys, int64_t n, int d, const float* qc, double theta,
                            const double* D, int nD, const int64_t* pos, int64_t t, int pairing,
                            int nthreads, double* out) {
  const int F = d / 2;
  std::vector<double> omega = frequencies(theta, d);
  std::vector<cplx> q(F);
  for (int f = 0; f < F; ++f) q[f] = band_of_center(qc, d, pairing, f);
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    const double dist = static_cast<double>(t - pos[i]);
    double total = 0.0;
    for (int u = 0; u < nD; ++u) {
      cplx s(0.0, 0.0);
      for (int f = 0; f < F; ++f)
        s += q[f] * std::conj(band_of_keys(k, d, pairing, f)) * std::polar(1.0, omega[f] * (dist + D[u]));
      total += s.real();
    }
    out[i] = total / nD;
  });
}

// The max-over-offsets variant (same page, "What it saves, and what it does
// not": a maximum over the offsets instead of the mean; not linear, so the
// fold does not apply):
//   s = max_{delta in D} Re sum_f q_f conj(k_f) e^{i omega_f (delta0 + delta)},
// each offset's score evaluated literally.
void orc_score_max_literal(const uint16_t* keys, int64_t n, int d, const float* qc, double theta,
                           const double* D, int nD, double delta0, int pairing, int nthreads,
                           double* out) {
  const int F = d / 2;
  std::vector<double> omega = frequencies(theta, d);
  std::vector<cplx> q(F);
  for (int f = 0; f < F; ++f) q[f] = band_of_center(qc, d, pairing, f);
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    double best = -INFINITY;
    for (int t = 0; t < nD; ++t) {
      cplx s(0.0, 0.0);
      for (int f = 0; f < F; ++f)
        s += q[f] * std::conj(band_of_keys(k, d, pairing, f)) * std::polar(1.0, omega[f] * (delta0 + D[t]));
      best = std::max(best, s.real());
    }
    out[i] = best;
  });
}

// O-iii, the folded complex form:
//   s = Re sum_f q_f conj(k_f) e^{i omega_f delta0} W_f.
void orc_score_folded(const uint16_t* keys, int64_t n, int d, const float* qc, double theta,
                      const double* D, int nD, double delta0, int pairing, int nthreads,
                      double* out) {
  const int F = d / 2;
  std::vector<double> omega = frequencies(theta, d);
  std::vector<cplx> W = offset_weights(omega, D, nD);
  std::vector<cplx> q(F);
  for (int f = 0; f < F; ++f) q[f] = band_of_center(qc, d, pairing, f);
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    cplx s(0.0, 0.0);
    for (int f = 0; f < F; ++f)
      s += q[f] * std::conj(band_of_keys(k, d, pairing, f)) * std::polar(1.0, omega[f] * delta0) * W[f];
    out[i] = s.real();
  });
}

// O-iv, the folded polar form with the offset-averaged center mu'_f = q_f W_f:
//   s = sum_f |mu'_f| |k_f| cos(omega_f delta0 + arg mu'_f - arg k_f).
void orc_score_polar(const uint16_t* keys, int64_t n, int d, const float* qc, double theta,
                     const double* D, int nD, double delta0, int pairing, int nthreads,
                     double* out) {
  const int F = d / 2;
  std::vector<double> omega = frequencies(theta, d);
  std::vector<cplx> W = offset_weights(omega, D, nD);
  std::vector<cplx> mu(F);
  for (int f = 0; f < F; ++f) mu[f] = band_of_center(qc, d, pairing, f) * W[f];
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    double s = 0.0;
    for (int f = 0; f < F; ++f) {
      cplx kf = band_of_keys(k, d, pairing, f);
      double nm = std::abs(mu[f]), nk = std::abs(kf);
      if (nm == 0.0 || nk == 0.0) continue;
      s += nm * nk * std::cos(omega[f] * delta0 + std::arg(mu[f]) - std::arg(kf));
    }
    out[i] = s;
  });
}

// The real per-band 2x2 map: for each center, the real weight vector w (length
// d) with  s = sum_j w[j] k[j].  Per band,
//   [w_re; w_im] = R(omega_f delta0) * [[W_re, -W_im], [W_im, W_re]] * [q_re; q_im]
// where R(a) = [[cos a, -sin a], [sin a, cos a]], written with real matrices
// (not complex numbers), so that it checks the complex forms independently.
void orc_fold_w(const float* qc, int n_centers, int d, double theta, const double* D, int nD,
                double delta0, int pairing, double* w_out) {
  const int F = d / 2;
  std::vector<double> omega = frequencies(theta, d);
  std::vector<double> Wre(F), Wim(F);
  for (int f = 0; f < F; ++f) {
    double c = 0.0, s = 0.0;
    for (int t = 0; t < nD; ++t) {
      c += std::cos(omega[f] * D[t]);
      s += std::sin(omega[f] * D[t]);
    }
    Wre[f] = c / nD;
    Wim[f] = s / nD;
  }
  for (int u = 0; u < n_centers; ++u) {
    const float* q = qc + static_cast<int64_t>(u) * d;
    double* w = w_out + static_cast<int64_t>(u) * d;
    for (int f = 0; f < F; ++f) {
      int re, im;
      band_coords(d, pairing, f, &re, &im);
      double qr = q[re], qi = q[im];
      // M = [[Wre, -Wim], [Wim, Wre]]
      double m0 = Wre[f] * qr - Wim[f] * qi;
      double m1 = Wim[f] * qr + Wre[f] * qi;
      double ca = std::cos(omega[f] * delta0), sa = std::sin(omega[f] * delta0);
      w[re] = ca * m0 - sa * m1;
      w[im] = sa * m0 + ca * m1;
    }
  }
}

// O-v, the real dot product with the fp64 weight vector of orc_fold_w.
void orc_score_realdot(const uint16_t* keys, int64_t n, int d, const double* w, int nthreads,
                       double* out) {
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    double s = 0.0;
    for (int j = 0; j < d; ++j) s += w[j] * bf16_value(k[j]);
    out[i] = s;
  });
}

// sum_j |w[j] k[j]|: the scale of the rounding error of a dot product.
void orc_abs_dot(const uint16_t* keys, int64_t n, int d, const double* w, int nthreads,
                 double* out) {
  parallel_for(n, nthreads, [&](int64_t i) {
    const uint16_t* k = keys + i * d;
    double s = 0.0;
    for (int j = 0; j < d; ++j) s += std::fabs(w[j] * bf16_value(k[j]));
    out[i] = s;
  });
}

// Top-min(B, n) keys under (score descending, index ascending), NaN lowest,
// returned as ascending indices.  Returns the number kept.
int64_t orc_select_f64(const double* s, int64_t n, int64_t B, int32_t* kept) {
  return select_top(s, n, B, kept);
}

int64_t orc_select_f32(const float* s, int64_t n, int64_t B, int32_t* kept) {
  return select_top(s, n, B, kept);
}

// Out-of-place compaction: out[j] = rows[kept[j]] for j < count (rows of d
// bf16 values, copied bit for bit).
void orc_gather_rows(const uint16_t* rows, int d, const int32_t* kept, int64_t count,
                     uint16_t* out) {
  for (int64_t j = 0; j < count; ++j)
    std::memcpy(out + j * d, rows + static_cast<int64_t>(kept[j]) * d, sizeof(uint16_t) * d);
}

// In-place hole fill of one unit's logical rows [n][d] after keeping the
// ascending index list kept[0..count).  Survivors with index < B stay where
// they are; the evicted positions below B ("holes"), in ascending order,
// receive the survivors with index >= B, in ascending order.  Rows at or past
// min(B, n) are left as they were.  Returns the number of rows moved.
int64_t orc_holefill(uint16_t* rows, int64_t n, int d, const int32_t* kept, int64_t count,
                     int64_t B) {
  if (n <= B) return 0;
  std::vector<char> stays(B, 0);
  std::vector<int64_t> movers;
  for (int64_t j = 0; j < count; ++j) {
    if (kept[j] < B) stays[kept[j]] = 1;
    else movers.push_back(kept[j]);
  }
  std::vector<int64_t> holes;
  for (int64_t p = 0; p < B; ++p)
    if (!stays[p]) holes.push_back(p);
  size_t m = std::min(holes.size(), movers.size());
  for (size_t j = 0; j < m; ++j)
    std::memcpy(rows + holes[j] * d, rows + movers[j] * d, sizeof(uint16_t) * d);
  return static_cast<int64_t>(m);
}

}  // extern "C"
