// Host construction of the Toeplitz plan used by the tensor-core contraction.
//
// The forward contraction of the page "torch_harmonics.DiscreteContinuousConvS2" (the sum over
// input points of Psi_k times the signal, with Psi stored once for output longitude 0 and
// shifted along the longitude for the others) is, for one output row j and one input row i, a
// 1-D correlation along the longitude ring:
//     y[c, k, j, q] += sum_p Psi_k(j, i, p) * x[c, i, (q + p) mod nlon].
// Written for 8 consecutive outputs q = q0 + u (u < 8) and a window of input longitudes
// q0 + lon_off + p' (p' < 16*nk), the coefficient of x at p' for output u is
// Psi_k(lon_off + p' - u): a banded Toeplitz matrix that does not depend on q0.  This file
// builds that matrix once per (j, i), in bf16 (hi part, and the bf16 rounding of the remainder
// as the lo part), cut into slabs of at most kTzSlabK K-steps of 16 longitudes.  The two parts
// sit side by side in the MMA's N dimension when 2*K*8 <= 128 columns, else in two blocks that
// two MMAs accumulate into the same columns (tensor memory holds more outputs that way).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <numeric>
#include <climits>
#include <cstdint>
#include <map>

#include "psi_builder.h"

namespace disco {
namespace {

uint16_t bf16_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16);  // inf / nan kept
  u += 0x7FFFu + ((u >> 16) & 1u);                                     // round to nearest even
  return (uint16_t)(u >> 16);
}

float bf16_value(uint16_t h) {
  const uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

}  // namespace

namespace {

// One term of a correlation along the ring: out[.., k, out_row, q] += v * src[.., src_row, q + off].
struct Term {
  int out_row, src_row, k, off;
  double v;
};

ToeplitzPlan build(int n_out_rows, int nlon, int K, std::vector<Term>& terms) {
  ToeplitzPlan P;
  P.K = K;
  P.parts = 16 * K <= 128 ? 1 : 2;
  P.N = P.parts == 1 ? 16 * K : (8 * K + 15) / 16 * 16;
  const int n = nlon, N = P.N;
  // offsets centred in (-n/2, n/2] so that an arc around offset 0 is one contiguous range
  for (Term& t : terms) {
    t.off = ((t.off % n) + n) % n;
    if (t.off > n / 2) t.off -= n;
  }
  std::sort(terms.begin(), terms.end(), [](const Term& a, const Term& b) {
    if (a.out_row != b.out_row) return a.out_row < b.out_row;
    if (a.src_row != b.src_row) return a.src_row < b.src_row;
    return a.off < b.off;
  });
  P.row_begin.assign(n_out_rows + 1, 0);
  std::vector<long long> row_steps(n_out_rows, 0);
  std::vector<double> dense;
  size_t a = 0;
  int row = 0;
  while (a < terms.size()) {
    const int j = terms[a].out_row, i = terms[a].src_row;
    size_t b = a;
    while (b < terms.size() && terms[b].out_row == j && terms[b].src_row == i) ++b;
    while (row <= j) P.row_begin[row++] = (int)P.slabs.size();
    const int pmin = terms[a].off, pmax = terms[b - 1].off;
    const int s = pmax - pmin + 1;
    dense.assign((size_t)K * s, 0.0);
    for (size_t t = a; t < b; ++t) dense[(size_t)terms[t].k * s + (terms[t].off - pmin)] += terms[t].v;
    const int delta = ((pmin % 8) + 8) % 8;
    const int p0 = pmin - delta;
    const int ks = (delta + s + 7 + 15) / 16;  // K-steps of 16 longitudes
    for (int c = 0; c * kTzSlabK < ks; ++c) {
      TzSlab sl;
      sl.i = i;
      sl.lon_off = p0 + 16 * kTzSlabK * c;
      sl.nk = std::min(kTzSlabK, ks - kTzSlabK * c);
      sl.boff = (int)(P.b.size() / 8);
      for (int part = 0; part < P.parts; ++part)
        for (int o = 0; o < 2 * sl.nk; ++o)
          for (int col = 0; col < N; ++col) {
            const int u = col % 8;
            const int k = P.parts == 1 ? (col / 8) % K : col / 8;
            const int h = P.parts == 1 ? col / (8 * K) : part;
            for (int el = 0; el < 8; ++el) {
              const int off = sl.lon_off + 8 * o + el - u;  // offset of this (p', u)
              double v = 0.0;
              if (k < K && h < 2 && off >= pmin && off <= pmax) v = dense[(size_t)k * s + (off - pmin)];
              const uint16_t hi = bf16_bits((float)v);
              P.b.push_back(h == 0 ? hi : bf16_bits((float)(v - (double)bf16_value(hi))));
            }
          }
      P.slabs.push_back(sl);
      P.ksteps += sl.nk;
      row_steps[j] += sl.nk;
    }
    a = b;
  }
  while (row <= n_out_rows) P.row_begin[row++] = (int)P.slabs.size();
  P.order.resize(n_out_rows);
  std::iota(P.order.begin(), P.order.end(), 0);
  std::stable_sort(P.order.begin(), P.order.end(),
                   [&](int x, int y) { return row_steps[x] > row_steps[y]; });
  for (int r : P.order) {
    P.slots.push_back(r);
    P.slots.push_back(P.row_begin[r]);
    P.slots.push_back(P.row_begin[r + 1]);
    P.slots.push_back(0);
  }
  return P;
}

}  // namespace

ToeplitzPlan make_toeplitz_plan(const Geometry& g, const std::vector<PsiEntry>& e) {
  std::vector<Term> t;
  t.reserve(e.size());
  for (const PsiEntry& x : e) t.push_back(Term{x.j, x.i, x.k, x.p, x.v});
  return build(g.nlat_out, g.nlon_in, g.K, t);
}

ToeplitzPlan make_adjoint_toeplitz_plan(const Geometry& g, const std::vector<PsiEntry>& e) {
  std::vector<Term> t;
  t.reserve(e.size());
  for (const PsiEntry& x : e) t.push_back(Term{x.i, x.k * g.nlat_out + x.j, 0, -x.p, x.v});
  return build(g.nlat_in, g.nlon_in, 1, t);
}

}  // namespace disco
