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

ToeplitzPlan make_toeplitz_plan(const Geometry& g, const std::vector<PsiEntry>& e) {
  ToeplitzPlan P;
  P.K = g.K;
  P.parts = 16 * g.K <= 128 ? 1 : 2;
  P.N = P.parts == 1 ? 16 * g.K : (8 * g.K + 15) / 16 * 16;
  const int n = g.nlon_in, K = g.K, N = P.N;
  // entries grouped by (j, i); offsets centred in (-n/2, n/2] so that an arc around offset 0
  // is one contiguous range
  auto centred = [n](int p) { return p > n / 2 ? p - n : p; };
  std::vector<size_t> idx(e.size());
  std::iota(idx.begin(), idx.end(), 0);
  std::sort(idx.begin(), idx.end(), [&](size_t a, size_t b) {
    if (e[a].j != e[b].j) return e[a].j < e[b].j;
    if (e[a].i != e[b].i) return e[a].i < e[b].i;
    return centred(e[a].p) < centred(e[b].p);
  });
  P.row_begin.assign(g.nlat_out + 1, 0);
  std::vector<long long> row_steps(g.nlat_out, 0);
  std::vector<double> dense;
  size_t a = 0;
  int row = 0;
  while (a < idx.size()) {
    const int j = e[idx[a]].j, i = e[idx[a]].i;
    size_t b = a;
    while (b < idx.size() && e[idx[b]].j == j && e[idx[b]].i == i) ++b;
    while (row <= j) P.row_begin[row++] = (int)P.slabs.size();
    int pmin = centred(e[idx[a]].p), pmax = centred(e[idx[b - 1]].p);
    const int s = pmax - pmin + 1;
    dense.assign((size_t)K * s, 0.0);
    for (size_t t = a; t < b; ++t) dense[(size_t)e[idx[t]].k * s + (centred(e[idx[t]].p) - pmin)] += e[idx[t]].v;
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
              const int off = sl.lon_off + 8 * o + el - u;  // Psi offset of this (p', u)
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
  while (row <= g.nlat_out) P.row_begin[row++] = (int)P.slabs.size();
  P.order.resize(g.nlat_out);
  std::iota(P.order.begin(), P.order.end(), 0);
  std::stable_sort(P.order.begin(), P.order.end(),
                   [&](int x, int y) { return row_steps[x] > row_steps[y]; });
  return P;
}

}  // namespace disco
