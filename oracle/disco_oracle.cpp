// CPU oracle for the spherical DISCO convolution.  TEST INFRASTRUCTURE ONLY:
// only the tests, the smoke check and the benchmark's CPU-baseline leg may
// load this library.  It shares no code with the CUDA product path.
//
// Everything is fp64 and written the slow, obvious way, following the
// definition on the page "torch_harmonics.DiscreteContinuousConvS2"
// (forward equation and the description of Psi right below it):
//
//   g^{co}(theta'_j, lambda'_q) = sum_ci sum_k w_k^{co,ci}
//                                 sum_{i,p} Psi_{k,j,(i,p)} f^{ci}(theta_i, lambda'_q + lambda_p)
//
// Psi holds the basis functions evaluated at the input grid points, rotated
// so that the output point sits at the north pole, times the quadrature
// weights; equispaced longitudes make Psi independent of the output
// longitude (p-shift symmetry).  The pages leave the basis formulas, the
// quadrature rule, the rotation convention, the normalisation and the
// backward formulas open; the readings taken here are:
//   * grids: lambda_p = 2*pi*p/nlon; by default theta_i = pi*i/(nlat-1)
//     (poles included) with Clenshaw-Curtis weights in cos(theta) (Waldvogel's
//     closed form); the other latitude grids the constructor names
//     (grid_in / grid_out) arrive as colatitude and weight arrays computed
//     by the Python side of the oracle; point weight w_i * 2*pi/nlon_in
//     (total 4*pi);
//   * distance r and bearing alpha (east of local north) of an input point
//     seen from the output point: haversine for r, atan2 for alpha;
//   * basis "piecewise linear": radial hats at r_k = k*theta_c/(n_r-1); the
//     anisotropic form merges the r=0 hat and multiplies the outer radial
//     hats by n_alpha azimuthal hats, K = 1 + (n_r-1)*n_alpha;
//   * tie rules (tau = 1e-10): a point is inside iff r <= theta_c + tau, an
//     entry is kept iff phi_k > tau.  Exact ties (points on the cutoff circle
//     or on a hat end point) land within rounding (~1e-16) of theta_c or 0,
//     far below tau; a computed r - theta_c or phi inside the band
//     [tau/10, 10*tau] around a threshold is reported as an error rather
//     than guessed, so two implementations that round differently by less
//     than 1e-11 always take the same decisions;
//   * "nodal" normalisation: every (k, j) row of Psi sums to one;
//   * output longitude q reads input longitude (q*s + p) mod nlon_in,
//     s = nlon_in / nlon_out;
//   * groups: output channel o reads input channels of group o/(C_out/G).
// Backward (not printed on the pages): dx is the exact adjoint of the
// forward map, dw and dbias are its derivatives with respect to w and bias.
//
// Parity status: the absolute Psi values are parity unpinned against the
// pages (they print no worked values); they are pinned by the mathematics
// (exact quadrature of polynomials, row sums, brute force without the
// p-shift, adjoint and Euler identities) in the test suite.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

const double kPi = 3.14159265358979323846;
const double kTau = 1e-10;       // tie threshold
const double kGapLo = 1e-11;     // no computed value may fall in [kGapLo, kGapHi]
const double kGapHi = 1e-9;      // around a threshold

struct Spec {
  int nlat_in, nlon_in, nlat_out, nlon_out, n_r, n_alpha;
  double theta_cutoff;
  const double* th_in;   // input colatitudes, or NULL for the equiangular grid
  const double* w_in;    // their quadrature weights on cos(theta) (with th_in)
  const double* th_out;  // output colatitudes, or NULL for the equiangular grid
};

struct Entry {
  int k, j, i, p;
  double val;
};

struct Psi {
  Spec s;
  int K;
  std::vector<Entry> e;          // sorted by (j, k, i, p)
  std::vector<long long> row;    // offsets of (j, k) rows: row[j*K + k] .. row[j*K + k + 1]
};

int num_basis(const Spec& s) { return s.n_alpha == 1 ? s.n_r : 1 + (s.n_r - 1) * s.n_alpha; }

// Clenshaw-Curtis weights on t = cos(theta), theta_i = pi*i/n, n = nlat-1.
void cc_weights(int nlat, double* w) {
  const int n = nlat - 1;
  for (int i = 0; i <= n; ++i) {
    const double th = kPi * i / n;
    double sum = 0.0;
    for (int m = 1; m <= n / 2; ++m) {
      const double b = (2 * m == n) ? 1.0 : 2.0;
      sum += b * std::cos(2.0 * m * th) / (4.0 * m * m - 1.0);
    }
    const double c = (i == 0 || i == n) ? 1.0 : 2.0;
    w[i] = c / n * (1.0 - sum);
  }
}

// Great-circle distance (haversine) and bearing east of local north of the
// point (th_in, dlam) seen from (th_out, 0); colatitudes.
void geodesic(double th_out, double th_in, double dlam, double* r, double* alpha) {
  const double a = std::sin(0.5 * (th_in - th_out));
  const double b = std::sin(0.5 * dlam);
  double h = a * a + std::sin(th_in) * std::sin(th_out) * b * b;
  h = std::min(1.0, std::max(0.0, h));
  *r = 2.0 * std::asin(std::sqrt(h));
  const double A = std::sin(th_in) * std::sin(dlam);
  const double B = std::sin(th_out) * std::cos(th_in) - std::cos(th_out) * std::sin(th_in) * std::cos(dlam);
  *alpha = std::atan2(A, B);
}

double hat(double r, double center, double width) {
  return std::max(0.0, 1.0 - std::fabs(r - center) / width);
}

// Value of basis function k at (r, alpha); zero outside the cutoff.
double basis(const Spec& s, int k, double r, double alpha) {
  const double tc = s.theta_cutoff;
  if (r > tc + kTau) return 0.0;
  const double d = tc / (s.n_r - 1);
  if (s.n_alpha == 1) return hat(r, k * d, d);
  if (k == 0) return hat(r, 0.0, d);
  const int kr = 1 + (k - 1) / s.n_alpha;
  const int l = (k - 1) % s.n_alpha;
  const double h = 2.0 * kPi / s.n_alpha;
  const double da = std::remainder(alpha - l * h, 2.0 * kPi);
  return hat(r, kr * d, d) * std::max(0.0, 1.0 - std::fabs(da) / h);
}

int validate(const Spec& s) {
  if (s.nlat_in < 2 || s.nlat_out < 2 || s.nlon_in < 1 || s.nlon_out < 1) return 1;
  if (s.nlon_in % s.nlon_out) return 2;
  if (s.n_r < 2 || s.n_alpha < 1) return 1;
  if (!(s.theta_cutoff > 0.0)) return 1;
  return 0;
}

// Dense Psi row j: psi[(k*nlat_in + i)*nlon_in + p], normalised.
// Returns 0, or -1 for a value inside a gap band, -2 for a row of zero mass.
int dense_row(const Spec& s, int j, double* psi) {
  const int K = num_basis(s);
  const double th_out = s.th_out ? s.th_out[j] : kPi * j / (s.nlat_out - 1);
  std::vector<double> w(s.nlat_in);
  if (s.th_in) {
    for (int i = 0; i < s.nlat_in; ++i) w[i] = s.w_in[i];
  } else {
    cc_weights(s.nlat_in, w.data());
  }
  const double tc = s.theta_cutoff;
  int status = 0;
  for (int i = 0; i < s.nlat_in; ++i) {
    const double th_in = s.th_in ? s.th_in[i] : kPi * i / (s.nlat_in - 1);
    const double qw = w[i] * 2.0 * kPi / s.nlon_in;
    for (int p = 0; p < s.nlon_in; ++p) {
      double r, alpha;
      geodesic(th_out, th_in, 2.0 * kPi * p / s.nlon_in, &r, &alpha);
      if (r - tc >= kGapLo && r - tc <= kGapHi) status = -1;
      for (int k = 0; k < K; ++k) {
        const double v = basis(s, k, r, alpha);
        if (v >= kGapLo && v <= kGapHi) status = -1;
        psi[((size_t)k * s.nlat_in + i) * s.nlon_in + p] = v > kTau ? v * qw : 0.0;
      }
    }
  }
  const size_t n = (size_t)s.nlat_in * s.nlon_in;
  for (int k = 0; k < K; ++k) {
    double sum = 0.0;
    for (size_t t = 0; t < n; ++t) sum += psi[k * n + t];
    if (sum == 0.0) { status = status ? status : -2; continue; }
    for (size_t t = 0; t < n; ++t) psi[k * n + t] /= sum;
  }
  return status;
}

int group_of(int ch, int C, int G) { return ch / (C / G); }

}  // namespace

extern "C" {

struct orc_spec {
  int nlat_in, nlon_in, nlat_out, nlon_out, n_r, n_alpha;
  double theta_cutoff;
  const double* th_in;
  const double* w_in;
  const double* th_out;
};

static Spec to_spec(const orc_spec* o) {
  return Spec{o->nlat_in, o->nlon_in, o->nlat_out, o->nlon_out, o->n_r, o->n_alpha, o->theta_cutoff,
              o->th_in, o->w_in, o->th_out};
}

int orc_num_basis(const orc_spec* o) { return num_basis(to_spec(o)); }

void orc_cc_weights(int nlat, double* w) { cc_weights(nlat, w); }

void orc_geodesic(double th_out, double th_in, double dlam, double* r, double* alpha) {
  geodesic(th_out, th_in, dlam, r, alpha);
}

double orc_basis(const orc_spec* o, int k, double r, double alpha) { return basis(to_spec(o), k, r, alpha); }

int orc_psi_dense_row(const orc_spec* o, int j, double* psi) {
  const Spec s = to_spec(o);
  if (int v = validate(s)) return v;
  return dense_row(s, j, psi);
}

// Builds the sparse Psi (every (i,p) evaluated, exact zeros dropped).
// Returns an opaque handle, or NULL with *status set.
void* orc_psi_build(const orc_spec* o, int* status) {
  const Spec s = to_spec(o);
  *status = validate(s);
  if (*status) return nullptr;
  const int K = num_basis(s);
  std::vector<std::vector<Entry>> rows(s.nlat_out);
  int bad = 0;
#pragma omp parallel
  {
    std::vector<double> psi((size_t)K * s.nlat_in * s.nlon_in);
#pragma omp for schedule(dynamic) reduction(min : bad)
    for (int j = 0; j < s.nlat_out; ++j) {
      const int st = dense_row(s, j, psi.data());
      if (st) bad = std::min(bad, st);
      for (int k = 0; k < K; ++k)
        for (int i = 0; i < s.nlat_in; ++i)
          for (int p = 0; p < s.nlon_in; ++p) {
            const double v = psi[((size_t)k * s.nlat_in + i) * s.nlon_in + p];
            if (v != 0.0) rows[j].push_back(Entry{k, j, i, p, v});
          }
    }
  }
  if (bad) { *status = bad; return nullptr; }
  Psi* h = new Psi;
  h->s = s;
  h->s.th_in = h->s.w_in = h->s.th_out = nullptr;  // the caller's arrays are not kept
  h->K = K;
  h->row.assign((size_t)s.nlat_out * K + 1, 0);
  for (int j = 0; j < s.nlat_out; ++j)
    for (const Entry& e : rows[j]) {
      h->e.push_back(e);
      h->row[(size_t)j * K + e.k + 1]++;
    }
  for (size_t t = 1; t < h->row.size(); ++t) h->row[t] += h->row[t - 1];
  return h;
}

void orc_psi_free(void* h) { delete static_cast<Psi*>(h); }

long long orc_psi_nnz(const void* h) { return (long long)static_cast<const Psi*>(h)->e.size(); }

void orc_psi_export(const void* hv, int* k, int* j, int* i, int* p, double* val) {
  const Psi* h = static_cast<const Psi*>(hv);
  for (size_t t = 0; t < h->e.size(); ++t) {
    k[t] = h->e[t].k; j[t] = h->e[t].j; i[t] = h->e[t].i; p[t] = h->e[t].p; val[t] = h->e[t].val;
  }
}

// y[b,c,k,j,q] = sum_{(i,p)} Psi[k,j,(i,p)] x[b,c,i,(q*s+p) mod nlon_in]
void orc_contract(const void* hv, int B, int C, const double* x, double* y) {
  const Psi* h = static_cast<const Psi*>(hv);
  const Spec& s = h->s;
  const int K = h->K, sft = s.nlon_in / s.nlon_out;
  const size_t xin = (size_t)s.nlat_in * s.nlon_in, yout = (size_t)s.nlat_out * s.nlon_out;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int bc = 0; bc < B * C; ++bc)
    for (int j = 0; j < s.nlat_out; ++j) {
      const double* xb = x + (size_t)bc * xin;
      for (int k = 0; k < K; ++k) {
        double* yr = y + ((size_t)bc * K + k) * yout + (size_t)j * s.nlon_out;
        const long long e0 = h->row[(size_t)j * K + k], e1 = h->row[(size_t)j * K + k + 1];
        for (int q = 0; q < s.nlon_out; ++q) {
          double acc = 0.0;
          for (long long t = e0; t < e1; ++t) {
            const Entry& e = h->e[t];
            acc += e.val * xb[(size_t)e.i * s.nlon_in + (q * sft + e.p) % s.nlon_in];
          }
          yr[q] = acc;
        }
      }
    }
}

// out[b,o,j,q] = sum_{c in group(o), k} w[o, c', k] y[b,c,k,j,q] + bias[o]
void orc_mix(const void* hv, int B, int C_in, int C_out, int G, const double* y, const double* w,
             const double* bias, double* out) {
  const Psi* h = static_cast<const Psi*>(hv);
  const int K = h->K, cg = C_in / G;
  const size_t n = (size_t)h->s.nlat_out * h->s.nlon_out;
#pragma omp parallel for collapse(2)
  for (int b = 0; b < B; ++b)
    for (int o = 0; o < C_out; ++o) {
      const int g = group_of(o, C_out, G);
      double* ob = out + ((size_t)b * C_out + o) * n;
      for (size_t t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int c = 0; c < cg; ++c)
          for (int k = 0; k < K; ++k)
            acc += w[((size_t)o * cg + c) * K + k] * y[(((size_t)b * C_in + g * cg + c) * K + k) * n + t];
        ob[t] = acc + (bias ? bias[o] : 0.0);
      }
    }
}

namespace {

// y planes of one input channel plane bc: yk[k][j][q] (the contraction of one channel).
void contract_plane(const Psi* h, const double* xb, double* yk) {
  const Spec& s = h->s;
  const int K = h->K, sft = s.nlon_in / s.nlon_out;
  const size_t yout = (size_t)s.nlat_out * s.nlon_out;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < s.nlat_out; ++j) {
      double* yr = yk + (size_t)k * yout + (size_t)j * s.nlon_out;
      const long long e0 = h->row[(size_t)j * K + k], e1 = h->row[(size_t)j * K + k + 1];
      for (int q = 0; q < s.nlon_out; ++q) {
        double acc = 0.0;
        for (long long t = e0; t < e1; ++t) {
          const Entry& e = h->e[t];
          acc += e.val * xb[(size_t)e.i * s.nlon_in + (q * sft + e.p) % s.nlon_in];
        }
        yr[q] = acc;
      }
    }
}

}  // namespace

// Full forward: y (optional) and out.  Channels are taken one plane at a
// time (y of one channel, then its share of every output of its group), so
// memory stays at one K-expanded plane; the sum over (c, k) runs in a fixed
// order, the same for every output point.
void orc_forward(const void* hv, int B, int C_in, int C_out, int G, const double* x, const double* w,
                 const double* bias, double* y_opt, double* out) {
  const Psi* h = static_cast<const Psi*>(hv);
  const Spec& s = h->s;
  const int K = h->K, cg = C_in / G, og = C_out / G;
  const size_t nin = (size_t)s.nlat_in * s.nlon_in, n = (size_t)s.nlat_out * s.nlon_out;
  std::vector<double> yk((size_t)K * n);
  std::fill(out, out + (size_t)B * C_out * n, 0.0);
  for (int b = 0; b < B; ++b)
    for (int c = 0; c < C_in; ++c) {
      contract_plane(h, x + ((size_t)b * C_in + c) * nin, yk.data());
      if (y_opt) std::copy(yk.begin(), yk.end(), y_opt + ((size_t)b * C_in + c) * K * n);
      const int g = group_of(c, C_in, G), cl = c - g * cg;
#pragma omp parallel for
      for (int ol = 0; ol < og; ++ol) {
        const int o = g * og + ol;
        double* ob = out + ((size_t)b * C_out + o) * n;
        for (int k = 0; k < K; ++k) {
          const double wv = w[((size_t)o * cg + cl) * K + k];
          const double* yr = yk.data() + (size_t)k * n;
          for (size_t t = 0; t < n; ++t) ob[t] += wv * yr[t];
        }
      }
    }
  if (bias)
    for (int b = 0; b < B; ++b)
      for (int o = 0; o < C_out; ++o) {
        double* ob = out + ((size_t)b * C_out + o) * n;
        for (size_t t = 0; t < n; ++t) ob[t] += bias[o];
      }
}

// dx = adjoint of the forward map (without bias) applied to dout.
void orc_backward_input(const void* hv, int B, int C_in, int C_out, int G, const double* dout,
                        const double* w, double* dx) {
  const Psi* h = static_cast<const Psi*>(hv);
  const Spec& s = h->s;
  const int K = h->K, cg = C_in / G, og = C_out / G, sft = s.nlon_in / s.nlon_out;
  const size_t nout = (size_t)s.nlat_out * s.nlon_out, nin = (size_t)s.nlat_in * s.nlon_in;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int c = 0; c < C_in; ++c) {
      const int g = group_of(c, C_in, G), cl = c - g * cg;
      // dy[k, j, q] = sum_{o in group} w[o, c', k] dout[b, o, j, q]
      std::vector<double> dy((size_t)K * nout, 0.0);
      for (int ol = 0; ol < og; ++ol) {
        const int o = g * og + ol;
        const double* db = dout + ((size_t)b * C_out + o) * nout;
        for (int k = 0; k < K; ++k) {
          const double wv = w[((size_t)o * cg + cl) * K + k];
          for (size_t t = 0; t < nout; ++t) dy[k * nout + t] += wv * db[t];
        }
      }
      // transpose of the contraction: scatter every Psi entry back
      double* dxb = dx + ((size_t)b * C_in + c) * nin;
      std::fill(dxb, dxb + nin, 0.0);
      for (const Entry& e : h->e) {
        const double* dyr = dy.data() + (size_t)e.k * nout + (size_t)e.j * s.nlon_out;
        double* dxr = dxb + (size_t)e.i * s.nlon_in;
        for (int q = 0; q < s.nlon_out; ++q) dxr[(q * sft + e.p) % s.nlon_in] += e.val * dyr[q];
      }
    }
}

// dw[o, c', k] = sum_{b,j,q} dout[b,o,j,q] y[b,c,k,j,q];  dbias[o] = sum dout[b,o,:,:]
// y is recomputed one channel plane at a time from x.
void orc_backward_weight(const void* hv, int B, int C_in, int C_out, int G, const double* dout,
                         const double* x, double* dw, double* dbias) {
  const Psi* h = static_cast<const Psi*>(hv);
  const Spec& s = h->s;
  const int K = h->K, cg = C_in / G, og = C_out / G;
  const size_t nin = (size_t)s.nlat_in * s.nlon_in, nout = (size_t)s.nlat_out * s.nlon_out;
  std::vector<double> yk((size_t)K * nout);
  std::fill(dw, dw + (size_t)C_out * cg * K, 0.0);
  for (int b = 0; b < B; ++b)
    for (int c = 0; c < C_in; ++c) {
      contract_plane(h, x + ((size_t)b * C_in + c) * nin, yk.data());
      const int g = group_of(c, C_in, G), cl = c - g * cg;
#pragma omp parallel for
      for (int ol = 0; ol < og; ++ol) {
        const int o = g * og + ol;
        const double* db = dout + ((size_t)b * C_out + o) * nout;
        for (int k = 0; k < K; ++k) {
          const double* yr = yk.data() + (size_t)k * nout;
          double acc = 0.0;
          for (size_t t = 0; t < nout; ++t) acc += db[t] * yr[t];
          dw[((size_t)o * cg + cl) * K + k] += acc;
        }
      }
    }
  if (dbias)
    for (int o = 0; o < C_out; ++o) {
      double acc = 0.0;
      for (int b = 0; b < B; ++b) {
        const double* db = dout + ((size_t)b * C_out + o) * nout;
        for (size_t t = 0; t < nout; ++t) acc += db[t];
      }
      dbias[o] = acc;
    }
}

// y at sampled points, summing densely over every input point (i,p) of the
// dense Psi row (zeros included).  Samples are (b, c, k, j, q) tuples.
int orc_contract_dense_samples(const orc_spec* o, int B, int C, const double* x, int n, const int* sb,
                               const int* sc, const int* sk, const int* sj, const int* sq, double* out) {
  const Spec s = to_spec(o);
  if (int v = validate(s)) return v;
  (void)B;
  const int K = num_basis(s), sft = s.nlon_in / s.nlon_out;
  const size_t nin = (size_t)s.nlat_in * s.nlon_in;
  std::vector<int> order(n);
  for (int t = 0; t < n; ++t) order[t] = t;
  std::sort(order.begin(), order.end(), [&](int a, int b) { return sj[a] < sj[b]; });
  std::vector<double> psi((size_t)K * nin);
  int cur = -1, status = 0;
  for (int t : order) {
    if (sj[t] != cur) {
      cur = sj[t];
      const int st = dense_row(s, cur, psi.data());
      if (st) status = st;
    }
    const double* xb = x + ((size_t)sb[t] * C + sc[t]) * nin;
    double acc = 0.0;
    for (int i = 0; i < s.nlat_in; ++i)
      for (int p = 0; p < s.nlon_in; ++p)
        acc += psi[((size_t)sk[t] * s.nlat_in + i) * s.nlon_in + p] *
               xb[(size_t)i * s.nlon_in + (sq[t] * sft + p) % s.nlon_in];
    out[t] = acc;
  }
  return status;
}

// Thread count of the OpenMP loops (n >= 1); used to time the oracle on one core and on all.
void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
