// Psi builder and gather plans for libdisco (host C++).
//
// Psi follows the definition on the page "torch_harmonics.DiscreteContinuousConvS2":
// basis values at input grid points rotated so that the output point sits at
// the north pole, times quadrature weights; one row per output latitude j
// (p-shift symmetry).  The page leaves the formulas open; this builder takes
// these readings:
//   * longitudes lambda_p = 2*pi*p/nlon; latitude grids (the grid_in / grid_out choices
//     "equiangular", "legendre-gauss", "lobatto", "equiangular-trapezoidal", which the page
//     names but does not define) read as the textbook rules on t = cos(theta):
//       - equiangular: theta_i = pi*i/(nlat-1), poles included, Clenshaw-Curtis weights
//         computed from the Chebyshev coefficients of the interpolant;
//       - legendre-gauss: the nlat Gauss-Legendre nodes and weights (no poles);
//       - lobatto: the nlat Gauss-Lobatto-Legendre nodes (poles included) and weights;
//       - equiangular-trapezoidal: equiangular nodes, trapezoidal weights in t;
//     nodes run north to south; point weight w_i * 2*pi / nlon_in;
//   * the input point is rotated with R_y(-theta'_j) (output point (theta'_j, 0)
//     to the pole); distance r = atan2(|(x', y')|, z'), bearing east of local
//     north alpha = atan2(y', -x');
//   * piecewise-linear basis: radial hats of width theta_c/(n_r-1) at
//     r_k = k*theta_c/(n_r-1); anisotropic: merged r = 0 hat, then for every
//     outer ring n_alpha azimuthal hats of width 2*pi/n_alpha centred at
//     2*pi*l/n_alpha, index k = 1 + (k_r-1)*n_alpha + l;
//   * inside iff r <= theta_c + 1e-10, kept iff phi > 1e-10; a computed
//     r - theta_c or phi in [1e-11, 1e-9] is a geometry error (a decision
//     too close to call);
//   * nodal normalisation: every (k, j) row sums to one.
// Only input rows with |theta_i - theta'_j| <= theta_c (plus a margin) are
// visited: the great-circle distance is never below the colatitude gap.

#include "psi_builder.h"

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <numeric>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace disco {
namespace {

constexpr double kPiD = 3.141592653589793238462643383279502884;
constexpr double kTie = 1e-10;
constexpr double kBandLo = 1e-11;
constexpr double kBandHi = 1e-9;

std::vector<double> clenshaw_curtis(int nlat) {
  const int n = nlat - 1;
  std::vector<double> w(nlat);
  for (int i = 0; i <= n; ++i) {
    const double th = kPiD * i / n;
    double acc = 0.0;
    for (int m = 0; m <= n; m += 2) {
      double t = 2.0 * std::cos(m * th) / (1.0 - double(m) * double(m));
      if (m == 0 || m == n) t *= 0.5;
      acc += t;
    }
    w[i] = 2.0 / n * ((i == 0 || i == n) ? 0.5 : 1.0) * acc;
  }
  return w;
}

// Legendre polynomial P_n(t) and its derivative, by the three-term recurrence.
void legendre(int n, double t, double* pn, double* dpn) {
  double p0 = 1.0, p1 = t;
  if (n == 0) {
    *pn = 1.0;
    *dpn = 0.0;
    return;
  }
  for (int m = 2; m <= n; ++m) {
    const double p2 = ((2.0 * m - 1.0) * t * p1 - (m - 1.0) * p0) / m;
    p0 = p1;
    p1 = p2;
  }
  *pn = p1;
  // (1 - t^2) P_n' = n (P_{n-1} - t P_n); never evaluated at t = +-1 here
  *dpn = n * (p0 - t * p1) / (1.0 - t * t);
}

}  // namespace

bool latitude_grid(int grid, int nlat, std::vector<double>& theta, std::vector<double>& weight) {
  if (nlat < 2) return false;
  theta.assign(nlat, 0.0);
  weight.assign(nlat, 0.0);
  switch (grid) {
    case 0:  // equiangular, Clenshaw-Curtis
    case 3: {  // equiangular, trapezoidal in t
      for (int i = 0; i < nlat; ++i) theta[i] = kPiD * i / (nlat - 1);
      if (grid == 0) {
        weight = clenshaw_curtis(nlat);
      } else {
        for (int i = 0; i < nlat; ++i) {
          const double lo = std::cos(theta[std::max(i - 1, 0)]), hi = std::cos(theta[std::min(i + 1, nlat - 1)]);
          weight[i] = 0.5 * (lo - hi);
        }
      }
      return true;
    }
    case 1: {  // Gauss-Legendre: roots of P_n, Newton from cos(pi (i + 3/4) / (n + 1/2))
      const int n = nlat;
      for (int i = 0; i < n; ++i) {
        double t = std::cos(kPiD * (i + 0.75) / (n + 0.5)), pn = 0.0, dpn = 1.0;
        for (int it = 0; it < 100; ++it) {
          legendre(n, t, &pn, &dpn);
          const double dt = pn / dpn;
          t -= dt;
          if (std::fabs(dt) < 1e-16) break;
        }
        legendre(n, t, &pn, &dpn);
        theta[i] = std::acos(t);
        weight[i] = 2.0 / ((1.0 - t * t) * dpn * dpn);
      }
      return true;
    }
    case 2: {  // Gauss-Lobatto-Legendre: +-1 and the roots of P'_{n-1}
      const int m = nlat - 1;
      const double end = 2.0 / (m * (m + 1.0));
      theta[0] = 0.0;
      theta[m] = kPiD;
      weight[0] = weight[m] = end;
      for (int i = 1; i < m; ++i) {
        // Newton on P'_m, with P''_m from Legendre's equation, starting at the Chebyshev-Lobatto point
        double t = std::cos(kPiD * i / m), pm = 0.0, dpm = 1.0;
        for (int it = 0; it < 100; ++it) {
          legendre(m, t, &pm, &dpm);
          const double d2 = (2.0 * t * dpm - m * (m + 1.0) * pm) / (1.0 - t * t);
          const double dt = dpm / d2;
          t -= dt;
          if (std::fabs(dt) < 1e-16) break;
        }
        legendre(m, t, &pm, &dpm);
        theta[i] = std::acos(t);
        weight[i] = end / (pm * pm);
      }
      return true;
    }
    default:
      return false;
  }
}

namespace {

inline double radial_hat(double r, int kr, double width) {
  return std::max(0.0, 1.0 - std::fabs(r - kr * width) / width);
}

void basis_all(const Geometry& g, double r, double alpha, double* phi) {
  const double width = g.theta_cutoff / (g.n_r - 1);
  if (g.n_alpha == 1) {
    for (int k = 0; k < g.n_r; ++k) phi[k] = radial_hat(r, k, width);
    return;
  }
  phi[0] = radial_hat(r, 0, width);
  const double h = 2.0 * kPiD / g.n_alpha;
  for (int kr = 1; kr < g.n_r; ++kr) {
    const double rad = radial_hat(r, kr, width);
    for (int l = 0; l < g.n_alpha; ++l) {
      double da = alpha - l * h;
      da -= 2.0 * kPiD * std::nearbyint(da / (2.0 * kPiD));
      phi[1 + (kr - 1) * g.n_alpha + l] = rad * std::max(0.0, 1.0 - std::fabs(da) / h);
    }
  }
}

int pos_mod(int a, int n) {
  const int r = a % n;
  return r < 0 ? r + n : r;
}

// Smallest circular interval [start, start + span) holding every p of a sorted list.
void circular_interval(const std::vector<int>& ps, int n, int* start, int* span) {
  const int m = (int)ps.size();
  int best_gap = ps[0] + n - ps[m - 1] - 1;  // the wrap-around gap
  int best_after = 0;
  for (int t = 0; t + 1 < m; ++t) {
    const int gap = ps[t + 1] - ps[t] - 1;
    if (gap > best_gap) { best_gap = gap; best_after = t + 1; }
  }
  const int s0 = ps[best_after];
  const int last = ps[(best_after + m - 1) % m];
  *span = pos_mod(last - s0, n) + 1;
  *start = (s0 > n / 2) ? s0 - n : s0;
}

}  // namespace

int build_psi_entries(const Geometry& g, std::vector<PsiEntry>& out, std::string& msg, int j_begin, int j_end) {
  if (j_end < 0) j_end = g.nlat_out;
  if (j_begin < 0 || j_begin >= j_end || j_end > g.nlat_out) {
    msg = "output row range out of bounds";
    return 1;
  }
  const int n_rows = j_end - j_begin;
  const int K = g.K;
  const double tc = g.theta_cutoff;
  std::vector<double> th_in, qw, th_out, unused;
  if (!latitude_grid(g.grid_in, g.nlat_in, th_in, qw) || !latitude_grid(g.grid_out, g.nlat_out, th_out, unused)) {
    msg = "unknown latitude grid";
    return 2;
  }
  std::vector<double> cl(g.nlon_in), sl(g.nlon_in);
  for (int p = 0; p < g.nlon_in; ++p) {
    cl[p] = std::cos(2.0 * kPiD * p / g.nlon_in);
    sl[p] = std::sin(2.0 * kPiD * p / g.nlon_in);
  }
  std::vector<std::vector<PsiEntry>> rows(n_rows);
  std::vector<int> bad(n_rows, 0);
#pragma omp parallel for schedule(dynamic)
  for (int jr = 0; jr < n_rows; ++jr) {
    const int j = j_begin + jr;
    const double tho = th_out[j];
    const double ct = std::cos(tho), st = std::sin(tho);
    std::vector<double> phi(K);
    std::vector<PsiEntry>& row = rows[jr];
    for (int i = 0; i < g.nlat_in; ++i) {
      const double thi = th_in[i];
      if (std::fabs(thi - tho) > tc + 1e-9) continue;
      const double si = std::sin(thi), ci = std::cos(thi);
      const double wq = qw[i] * 2.0 * kPiD / g.nlon_in;
      for (int p = 0; p < g.nlon_in; ++p) {
        const double vx = si * cl[p], vy = si * sl[p], vz = ci;
        const double xr = vx * ct - vz * st;
        const double yr = vy;
        const double zr = vx * st + vz * ct;
        const double r = std::atan2(std::hypot(xr, yr), zr);
        if (r - tc >= kBandLo && r - tc <= kBandHi) bad[jr] = 1;
        if (r > tc + kTie) continue;
        basis_all(g, r, std::atan2(yr, -xr), phi.data());
        for (int k = 0; k < K; ++k) {
          if (phi[k] >= kBandLo && phi[k] <= kBandHi) bad[jr] = 1;
          if (phi[k] > kTie) row.push_back(PsiEntry{k, j, i, p, phi[k] * wq});
        }
      }
    }
    std::vector<double> mass(K, 0.0);
    for (const PsiEntry& e : row) mass[e.k] += e.v;
    for (int k = 0; k < K; ++k)
      if (!(mass[k] > 0.0)) bad[jr] = bad[jr] ? bad[jr] : 2;
    for (PsiEntry& e : row) e.v /= mass[e.k];
    std::sort(row.begin(), row.end(), [](const PsiEntry& a, const PsiEntry& b) {
      if (a.k != b.k) return a.k < b.k;
      if (a.i != b.i) return a.i < b.i;
      return a.p < b.p;
    });
  }
  for (int jr = 0; jr < n_rows; ++jr) {
    const int j = j_begin + jr;
    if (bad[jr] == 1) {
      msg = "Psi row " + std::to_string(j) +
            ": a distance or basis value lies within [1e-11, 1e-9] of a threshold (tie too close to call)";
      return 6;
    }
    if (bad[jr] == 2) {
      msg = "Psi row " + std::to_string(j) + ": a basis function has no support on the input grid";
      return 6;
    }
  }
  out.clear();
  size_t total = 0;
  for (auto& r : rows) total += r.size();
  out.reserve(total);
  for (auto& r : rows) out.insert(out.end(), r.begin(), r.end());
  return 0;
}

namespace {

void order_rows(GatherPlan& P) {
  for (const RowPlan& rp : P.rows) {
    P.max_src = std::max(P.max_src, rp.src_end - rp.src_begin);
    P.max_ring = std::max(P.max_ring, rp.ring_end - rp.ring_begin);
  }
  std::stable_sort(P.rows.begin(), P.rows.end(),
                   [](const RowPlan& a, const RowPlan& b) { return a.cost > b.cost; });
}

// Appends chunks over a dense table tab[nk][span] (column t has an entry when has[t]).
void emit_chunks(GatherPlan& P, const std::vector<double>& tab, const std::vector<char>& has, int span,
                 int nk, int src_rel, float* cost) {
  int t = 0;
  while (t < span) {
    if (!has[t]) { ++t; continue; }
    const int t0 = t;
    int last = t0;
    for (int u = t0; u < std::min(span, t0 + kChunkW); ++u)
      if (has[u]) last = u;
    const int w = last - t0 + 1;
    Chunk c;
    c.src = src_rel;
    c.t0 = t0;
    c.voff = (int)P.vals.size();
    int kmask = 0;
    for (int k = 0; k < nk; ++k)
      for (int u = 0; u < kChunkW; ++u) {
        const double v = (u < w) ? tab[(size_t)k * span + t0 + u] : 0.0;
        if (v != 0.0) kmask |= 1 << k;
        P.vals.push_back((float)v);
      }
    c.wk = w | (kmask << 8);
    *cost += (float)(__builtin_popcount(kmask) * w);
    P.chunks.push_back(c);
    t = t0 + w;
  }
}

// True when `vals` covers all n longitudes of a circle with one value (to 1e-12 relative).
bool constant_ring(const std::vector<double>& vals, int n, double* mean) {
  if ((int)vals.size() != n) return false;
  double s = 0.0, lo = vals[0], hi = vals[0];
  for (double v : vals) {
    s += v;
    lo = std::min(lo, v);
    hi = std::max(hi, v);
  }
  *mean = s / n;
  return hi - lo <= 1e-12 * std::fabs(*mean);
}

}  // namespace

int stage_elems(const GatherPlan& P, const RowPlan& r, int qb) {
  int n = 0;
  for (int s = r.src_begin; s < r.src_end; ++s) n += staged_words(staged_len(P.src[s].span, qb, P.step));
  return n;
}

GatherPlan make_forward_plan(const Geometry& g, const std::vector<PsiEntry>& e) {
  GatherPlan P;
  P.nk = g.K;
  P.step = g.stride;
  P.residues = 1;
  size_t a = 0;
  for (int j = 0; j < g.nlat_out; ++j) {
    size_t b = a;
    while (b < e.size() && e[b].j == j) ++b;
    // entries of row j, regrouped by input row i
    std::vector<const PsiEntry*> rowe;
    for (size_t t = a; t < b; ++t) rowe.push_back(&e[t]);
    std::stable_sort(rowe.begin(), rowe.end(), [](const PsiEntry* x, const PsiEntry* y) { return x->i < y->i; });
    RowPlan rp{};
    rp.row = j;
    rp.src_begin = (int)P.src.size();
    rp.chunk_start[0] = (int)P.chunks.size();
    rp.ring_begin = (int)P.rings.size();
    float cost = 0.0f, staged = 0.0f;
    size_t u = 0;
    while (u < rowe.size()) {
      const int i = rowe[u]->i;
      size_t v = u;
      while (v < rowe.size() && rowe[v]->i == i) ++v;
      // full circles of one constant value become ring terms
      std::vector<char> is_ring(g.K, 0);
      for (int k = 0; k < g.K; ++k) {
        std::vector<double> vk;
        for (size_t t = u; t < v; ++t)
          if (rowe[t]->k == k) vk.push_back(rowe[t]->v);
        double mean;
        if (constant_ring(vk, g.nlon_in, &mean)) {
          is_ring[k] = 1;
          P.rings.push_back(Ring{i, k, (float)mean, 0});
          cost += 0.01f * g.nlon_in / std::max(1, g.nlon_out);
        }
      }
      std::vector<const PsiEntry*> keep;
      for (size_t t = u; t < v; ++t)
        if (!is_ring[rowe[t]->k]) keep.push_back(rowe[t]);
      if (keep.empty()) {
        u = v;
        continue;
      }
      std::vector<int> ps;
      for (const PsiEntry* e : keep) ps.push_back(e->p);
      std::sort(ps.begin(), ps.end());
      ps.erase(std::unique(ps.begin(), ps.end()), ps.end());
      int d0, span;
      circular_interval(ps, g.nlon_in, &d0, &span);
      // stage from a multiple of kAlign so that staging moves 16-byte vectors
      const int lead = pos_mod(d0, kAlign);
      const int a0 = d0 - lead;
      span += lead;
      P.src.push_back(SrcRow{i, a0, span, 0});
      staged += (float)(span + 128 * g.stride);
      std::vector<double> tab((size_t)g.K * span, 0.0);
      std::vector<char> has(span, 0);
      for (const PsiEntry* e : keep) {
        const int col = lead + pos_mod(e->p - d0, g.nlon_in);
        tab[(size_t)e->k * span + col] = e->v;
        has[col] = 1;
      }
      emit_chunks(P, tab, has, span, g.K, (int)P.src.size() - 1 - rp.src_begin, &cost);
      u = v;
    }
    rp.src_end = (int)P.src.size();
    rp.chunk_end[0] = (int)P.chunks.size();
    rp.ring_end = (int)P.rings.size();
    for (int rho = 1; rho < kMaxStride; ++rho) rp.chunk_start[rho] = rp.chunk_end[rho] = rp.chunk_end[0];
    rp.cost = cost + 0.02f * staged;
    P.rows.push_back(rp);
    a = b;
  }
  order_rows(P);
  return P;
}

GatherPlan make_band_plan(int n_rows, const GatherPlan& one, int nb_max, int max_chunks) {
  GatherPlan P;
  P.nk = one.nk;
  P.step = one.step;
  P.residues = one.residues;
  std::vector<int> by_row(n_rows, -1);
  for (size_t t = 0; t < one.rows.size(); ++t) by_row[one.rows[t].row] = (int)t;
  auto light = [&](const RowPlan& r) {
    if (r.ring_end > r.ring_begin) return false;
    if (r.chunk_end[kMaxStride - 1] - r.chunk_start[0] > max_chunks) return false;
    for (int s = r.src_begin; s < r.src_end; ++s)
      if (one.src[s].span > 64) return false;
    return true;
  };
  int j = 0;
  while (j < n_rows) {
    std::vector<int> members{by_row[j]};
    if (light(one.rows[by_row[j]]))
      while ((int)members.size() < nb_max && j + (int)members.size() < n_rows &&
             light(one.rows[by_row[j + members.size()]]))
        members.push_back(by_row[j + members.size()]);
    j += (int)members.size();
    // union of the members' source intervals, per source row
    std::vector<SrcRow> band_src;
    for (int m : members) {
      const RowPlan& r = one.rows[m];
      for (int s = r.src_begin; s < r.src_end; ++s) {
        const SrcRow& sr = one.src[s];
        auto it = std::find_if(band_src.begin(), band_src.end(), [&](const SrcRow& b) { return b.row == sr.row; });
        if (it == band_src.end()) {
          band_src.push_back(sr);
        } else {
          const int lo = std::min(it->start, sr.start);
          const int hi = std::max(it->start + it->span, sr.start + sr.span);
          it->start = lo;
          it->span = hi - lo;
        }
      }
    }
    std::sort(band_src.begin(), band_src.end(), [](const SrcRow& a, const SrcRow& b) { return a.row < b.row; });
    BandPlan bp{(int)P.rows.size(), 0, 0.0f, 0};
    const int src_begin = (int)P.src.size();
    P.src.insert(P.src.end(), band_src.begin(), band_src.end());
    float cost = 0.0f;
    for (int m : members) {
      const RowPlan& r = one.rows[m];
      RowPlan nr = r;
      nr.src_begin = src_begin;
      nr.src_end = (int)P.src.size();
      for (int rho = 0; rho < kMaxStride; ++rho) {
        nr.chunk_start[rho] = (int)P.chunks.size();
        for (int c = r.chunk_start[rho]; c < r.chunk_end[rho]; ++c) {
          Chunk ch = one.chunks[c];
          const SrcRow& own = one.src[r.src_begin + ch.src];
          const int bi = (int)(std::find_if(band_src.begin(), band_src.end(),
                                            [&](const SrcRow& b) { return b.row == own.row; }) -
                               band_src.begin());
          ch.t0 += own.start - band_src[bi].start;
          ch.src = bi;
          const int nv = one.nk * kChunkW;
          const int voff = (int)P.vals.size();
          P.vals.insert(P.vals.end(), one.vals.begin() + ch.voff, one.vals.begin() + ch.voff + nv);
          ch.voff = voff;
          P.chunks.push_back(ch);
        }
        nr.chunk_end[rho] = (int)P.chunks.size();
      }
      nr.ring_begin = (int)P.rings.size();
      for (int t = r.ring_begin; t < r.ring_end; ++t) P.rings.push_back(one.rings[t]);
      nr.ring_end = (int)P.rings.size();
      cost += r.cost;
      P.rows.push_back(nr);
    }
    bp.rp_end = (int)P.rows.size();
    bp.cost = cost;
    P.bands.push_back(bp);
  }
  for (const RowPlan& rp : P.rows) {
    P.max_src = std::max(P.max_src, rp.src_end - rp.src_begin);
    P.max_ring = std::max(P.max_ring, rp.ring_end - rp.ring_begin);
  }
  std::stable_sort(P.bands.begin(), P.bands.end(),
                   [](const BandPlan& a, const BandPlan& b) { return a.cost > b.cost; });
  return P;
}

void split_bands(GatherPlan& P, int qb, int light_words) {
  auto heavy = [&](const BandPlan& b) { return stage_elems(P, P.rows[b.rp_begin], qb) > light_words; };
  std::stable_partition(P.bands.begin(), P.bands.end(), heavy);
  P.n_heavy = 0;
  for (const BandPlan& b : P.bands) P.n_heavy += heavy(b) ? 1 : 0;
}

GatherPlan make_adjoint_plan(const Geometry& g, const std::vector<PsiEntry>& e) {
  GatherPlan P;
  const int s = g.stride;
  P.nk = 1;
  P.step = 1;
  P.residues = s;
  std::vector<std::vector<const PsiEntry*>> by_i(g.nlat_in);
  for (const PsiEntry& x : e) by_i[x.i].push_back(&x);
  for (int i = 0; i < g.nlat_in; ++i) {
    auto& ent = by_i[i];
    std::stable_sort(ent.begin(), ent.end(), [](const PsiEntry* x, const PsiEntry* y) {
      if (x->j != y->j) return x->j < y->j;
      return x->k < y->k;
    });
    RowPlan rp{};
    rp.row = i;
    rp.src_begin = (int)P.src.size();
    rp.ring_begin = (int)P.rings.size();
    float cost = 0.0f, staged = 0.0f;
    struct Pending { int rho; std::vector<double> tab; std::vector<char> has; int span; int src_rel; };
    std::vector<Pending> pend;
    size_t u = 0;
    while (u < ent.size()) {
      const int j = ent[u]->j;
      size_t v = u;
      while (v < ent.size() && ent[v]->j == j) ++v;
      // the same circular interval of the (j, i) pair as in the forward plan
      std::vector<int> ps;
      for (size_t t = u; t < v; ++t) ps.push_back(ent[t]->p);
      std::sort(ps.begin(), ps.end());
      ps.erase(std::unique(ps.begin(), ps.end()), ps.end());
      int d0, span;
      circular_interval(ps, g.nlon_in, &d0, &span);
      size_t w0 = u;
      while (w0 < v) {
        const int k = ent[w0]->k;
        size_t w1 = w0;
        while (w1 < v && ent[w1]->k == k) ++w1;
        {
          // a constant full circle: every dx[l] takes v * (sum of the dy row)
          std::vector<double> vk;
          for (size_t t = w0; t < w1; ++t) vk.push_back(ent[t]->v);
          double mean;
          if (constant_ring(vk, g.nlon_in, &mean)) {
            P.rings.push_back(Ring{k * g.nlat_out + j, 0, (float)mean, 0});
            cost += 0.01f * g.nlon_out;
            w0 = w1;
            continue;
          }
        }
        // dx[l = s*m + rho] takes dy[m + e] with e = (rho - d)/s, d the signed offset, rho = d mod s
        int emin = 1 << 30, emax = -(1 << 30);
        for (size_t t = w0; t < w1; ++t) {
          const int d = d0 + pos_mod(ent[t]->p - d0, g.nlon_in);
          const int ev = (pos_mod(d, s) - d) / s;
          emin = std::min(emin, ev);
          emax = std::max(emax, ev);
        }
        const int lead = pos_mod(emin, kAlign);
        emin -= lead;
        const int espan = emax - emin + 1;
        P.src.push_back(SrcRow{k * g.nlat_out + j, emin, espan, 0});
        staged += (float)(espan + 128);
        const int src_rel = (int)P.src.size() - 1 - rp.src_begin;
        for (int rho = 0; rho < s; ++rho) {
          Pending pd{rho, std::vector<double>(espan, 0.0), std::vector<char>(espan, 0), espan, src_rel};
          bool any = false;
          for (size_t t = w0; t < w1; ++t) {
            const int d = d0 + pos_mod(ent[t]->p - d0, g.nlon_in);
            if (pos_mod(d, s) != rho) continue;
            const int col = (rho - d) / s - emin;
            pd.tab[col] = ent[t]->v;
            pd.has[col] = 1;
            any = true;
          }
          if (any) pend.push_back(std::move(pd));
        }
        w0 = w1;
      }
      u = v;
    }
    for (int rho = 0; rho < kMaxStride; ++rho) {
      rp.chunk_start[rho] = (int)P.chunks.size();
      for (const Pending& pd : pend)
        if (pd.rho == rho) emit_chunks(P, pd.tab, pd.has, pd.span, 1, pd.src_rel, &cost);
      rp.chunk_end[rho] = (int)P.chunks.size();
    }
    rp.src_end = (int)P.src.size();
    rp.ring_end = (int)P.rings.size();
    rp.cost = cost + 0.02f * staged;
    P.rows.push_back(rp);
  }
  order_rows(P);
  return P;
}

}  // namespace disco
