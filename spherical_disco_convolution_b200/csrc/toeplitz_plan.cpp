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

PackedPlan make_packed_plan(const Geometry& g, const std::vector<PsiEntry>& e, bool adjoint, int T, int NR,
                            int strip_rows, int ksmax) {
  PackedPlan P;
  const int K = adjoint ? 1 : g.K, n = g.nlon_in;
  const int n_out = adjoint ? g.nlat_in : g.nlat_out;
  P.K = K;
  P.Nr = 16 * K;
  P.NR = NR;
  P.T = T;
  const int max_rows = 256 / P.Nr;
  // terms of the correlation, offsets centred in (-n/2, n/2]
  std::vector<Term> terms;
  terms.reserve(e.size());
  for (const PsiEntry& x : e)
    terms.push_back(adjoint ? Term{x.i, x.k * g.nlat_out + x.j, 0, -x.p, x.v} : Term{x.j, x.i, x.k, x.p, x.v});
  for (Term& t : terms) {
    t.off = ((t.off % n) + n) % n;
    if (t.off > n / 2) t.off -= n;
  }
  std::sort(terms.begin(), terms.end(), [](const Term& a, const Term& b) {
    if (a.out_row != b.out_row) return a.out_row < b.out_row;
    if (a.src_row != b.src_row) return a.src_row < b.src_row;
    return a.off < b.off;
  });
  // pairs (o, s): offset range and term range
  struct Pair {
    int o, s, pmin, pmax;
    size_t t0, t1;
  };
  std::vector<Pair> pairs;
  std::vector<int> row_first(n_out + 1, 0);
  for (size_t a = 0; a < terms.size();) {
    size_t b = a;
    while (b < terms.size() && terms[b].out_row == terms[a].out_row && terms[b].src_row == terms[a].src_row) ++b;
    pairs.push_back(Pair{terms[a].out_row, terms[a].src_row, terms[a].off, terms[b - 1].off, a, b});
    a = b;
  }
  {
    int r = 0;
    for (size_t q = 0; q < pairs.size(); ++q)
      while (r <= pairs[q].o) row_first[r++] = (int)q;
    while (r <= n_out) row_first[r++] = (int)pairs.size();
  }
  auto ks_of = [](int pmin, int pmax) {
    const int ls = 8 * (int)std::floor(pmin / 8.0);
    return (pmax - ls + 8 + 15) / 16;
  };
  std::vector<char> regular(n_out, 0);
  for (int o = 0; o < n_out; ++o) {
    bool ok = row_first[o + 1] > row_first[o];  // a row without terms is left to the per-pair plan
    for (int q = row_first[o]; q < row_first[o + 1] && ok; ++q) ok = ks_of(pairs[q].pmin, pairs[q].pmax) <= ksmax;
    regular[o] = ok;
  }
  // the order of source rows within a strip follows their output rows; for the adjoint the
  // source rows k*nlat_out + j of one j are adjacent
  auto src_key = [&](int s) { return adjoint ? (long long)(s % g.nlat_out) * K + s / g.nlat_out : (long long)s; };
  auto build_strip = [&](int o0, int o1) -> bool {
    struct Ent {
      int s, o_a, o_b;
      long long key;
    };
    std::map<int, std::pair<int, int>> range;  // s -> [o_a, o_b]
    for (int o = o0; o < o1; ++o)
      for (int q = row_first[o]; q < row_first[o + 1]; ++q) {
        auto it = range.find(pairs[q].s);
        if (it == range.end()) range[pairs[q].s] = {o, o};
        else it->second.second = std::max(it->second.second, o);
      }
    std::vector<Ent> ents;
    for (auto& kv : range) ents.push_back(Ent{kv.first, kv.second.first, kv.second.second, src_key(kv.first)});
    std::sort(ents.begin(), ents.end(), [](const Ent& a, const Ent& b) {
      if (a.o_a != b.o_a) return a.o_a < b.o_a;
      if (a.o_b != b.o_b) return a.o_b < b.o_b;
      return a.key < b.key;
    });
    const int ne = (int)ents.size();
    std::vector<int> start(o1 - o0, -1), done(o1 - o0, -1);
    for (int x = 0; x < ne; ++x) {
      if (ents[x].o_b - ents[x].o_a + 1 > max_rows) return false;
      for (int o = ents[x].o_a; o <= ents[x].o_b; ++o) {
        if (start[o - o0] < 0) start[o - o0] = x;
        done[o - o0] = x;
      }
    }
    for (int x = 0; x < ne; ++x) {  // rows live at entry x must fit the slots
      int lo = INT32_MAX, hi = -1;
      for (int o = o0; o < o1; ++o)
        if (start[o - o0] <= x && x <= done[o - o0]) {
          lo = std::min(lo, o);
          hi = std::max(hi, o);
        }
      if (hi >= 0 && hi - lo + 1 > NR) return false;
    }
    // emit
    const int e_begin = (int)P.entries.size();
    std::vector<double> dense;
    for (int x = 0; x < ne; ++x) {
      const Ent& en = ents[x];
      const int nrow = en.o_b - en.o_a + 1;
      int pmin = INT32_MAX, pmax = INT32_MIN;
      for (int o = en.o_a; o <= en.o_b; ++o)
        for (int q = row_first[o]; q < row_first[o + 1]; ++q)
          if (pairs[q].s == en.s) {
            pmin = std::min(pmin, pairs[q].pmin);
            pmax = std::max(pmax, pairs[q].pmax);
          }
      const int ls = 8 * (int)std::floor(pmin / 8.0);
      const int ks = (pmax - ls + 8 + 15) / 16;
      if (ks > ksmax) {
        P.entries.resize(e_begin);
        return false;
      }
      PackedEntry pe;
      pe.s = en.s;
      pe.lon_start = ls;
      pe.ks = ks;
      pe.boff = (int)(P.b.size() / 8);
      pe.o_a = en.o_a - o0;
      pe.n_rows = nrow;
      pe.new_mask = 0;
      for (int r = 0; r < nrow; ++r)
        if (start[en.o_a + r - o0] == x) pe.new_mask |= 1 << r;
      pe.done_begin = (int)P.done.size();
      for (int o = o0; o < o1; ++o)
        if (done[o - o0] == x) P.done.push_back(o - o0);
      pe.done_end = (int)P.done.size();
      pe.done_base = pe.done_end > pe.done_begin ? P.done[pe.done_begin] : 0;
      pe.done_mask = 0;
      for (int d = pe.done_begin; d < pe.done_end; ++d) {
        if (P.done[d] - pe.done_base >= 16) {  // completed rows span more than 16
          P.entries.resize(e_begin);
          return false;
        }
        pe.done_mask |= 1 << (P.done[d] - pe.done_base);
      }
      // block [2ks octets][nrow*Nr][8]: column r*Nr + (h*K + k)*8 + u
      const int W = 16 * ks, NC = nrow * P.Nr;
      dense.assign((size_t)nrow * K * W, 0.0);  // [r][k][p'] value at offset ls + p' (before the u shift)
      for (int r = 0; r < nrow; ++r) {
        const int o = en.o_a + r;
        for (int q = row_first[o]; q < row_first[o + 1]; ++q)
          if (pairs[q].s == en.s)
            for (size_t t = pairs[q].t0; t < pairs[q].t1; ++t)
              dense[((size_t)r * K + terms[t].k) * W + (terms[t].off - ls)] += terms[t].v;
      }
      for (int oc = 0; oc < 2 * ks; ++oc)
        for (int col = 0; col < NC; ++col) {
          const int r = col / P.Nr, c = col % P.Nr, u = c % 8, k = (c / 8) % K, h = c / (8 * K);
          for (int el = 0; el < 8; ++el) {
            const int pp = 8 * oc + el - u;  // offset - ls of this (p', u)
            const double v = (pp >= 0 && pp < W) ? dense[((size_t)r * K + k) * W + pp] : 0.0;
            const uint16_t hi = bf16_bits((float)v);
            P.b.push_back(h == 0 ? hi : bf16_bits((float)(v - (double)bf16_value(hi))));
          }
        }
      if (pe.o_a >= 32768 || nrow >= 256 || ks >= 256) {
        P.entries.resize(e_begin);
        return false;
      }
      P.entries.push_back(pe);
    }
    P.strips.push_back(e_begin);
    P.strips.push_back((int)P.entries.size());
    P.strips.push_back(o0);
    P.strips.push_back(o1 - o0);
    return true;
  };
  int o = 0;
  while (o < n_out) {
    if (!regular[o]) {
      P.rest.push_back(o++);
      continue;
    }
    int o1 = o;
    while (o1 < n_out && regular[o1] && o1 - o < strip_rows) ++o1;
    const size_t done0 = P.done.size(), b0 = P.b.size();
    if (!build_strip(o, o1)) {
      P.done.resize(done0);
      P.b.resize(b0);
      for (int r = o; r < o1; ++r) P.rest.push_back(r);
    }
    o = o1;
  }
  P.mmas_per_group = 0;
  for (const PackedEntry& pe : P.entries) {
    P.mmas_per_group += pe.ks;
    const int rec[8] = {pe.s, pe.lon_start, pe.ks | pe.n_rows << 8 | pe.o_a << 16, pe.boff, pe.new_mask,
                        pe.done_base | pe.done_mask << 16, 0, 0};
    P.dev.insert(P.dev.end(), rec, rec + 8);
  }
  return P;
}

}  // namespace disco
