// Host construction of the ring plan of the strip-staged tensor-core contraction.
//
// The forward contraction of the page "torch_harmonics.DiscreteContinuousConvS2" (class
// description: Psi is stored for output longitude 0 and shifted along the longitude for the
// others) is, for an output row r and a source row s, the correlation
//     out[.., k, r, q] += sum_off v_k(off) src[.., s, q + off]
// along the longitude ring.  For 16 consecutive outputs q0 + u and a window of 16*ks source
// longitudes starting at q0 + 8*lo it is a product with the banded Toeplitz block
//     B[p', (k, u)] = v_k(8*lo + p' - u)                      (bf16, one rounding of Psi)
// which is the same for every q0.  Block b of a tile (outputs q0 + 16b ..) reads the window
// shifted by two octets per block.  This file groups those products into the script that the
// kernel replays for every tile (see RingPlan in psi_builder.h).
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "psi_builder.h"

namespace disco {
namespace {

uint16_t to_bf16(double v) {
  const float f = (float)v;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);  // round to nearest even (finite values only)
  return (uint16_t)(u >> 16);
}

int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }

struct Pair {
  int r, s;        // output row, source row
  int pmin, pmax;  // offsets reached
  int lo, ks, M;   // first octet of block 0's window, K-steps, octet pairs for nb blocks
  size_t t0, t1;   // terms
  int boff;        // B offset (16-byte units)
};

}  // namespace

namespace {

bool build_ring(int n_out, int n_src, int n, int K, std::vector<RingTerm> terms, const std::vector<int>& mo,
                const std::vector<int>& ms, const RingParams& prm, bool allow_share, RingPlan& P, std::string& msg);

}  // namespace

bool make_ring_plan(int n_out, int n_src, int n, int K, std::vector<RingTerm> terms, const std::vector<int>& mo,
                    const std::vector<int>& ms, const RingParams& prm, RingPlan& P, std::string& msg) {
  // sources shared by the rows of a strip when the ring has room for them, else every
  // (row, source) pair loads its own window
  if (build_ring(n_out, n_src, n, K, terms, mo, ms, prm, true, P, msg)) return true;
  const std::string first = msg;
  if (build_ring(n_out, n_src, n, K, std::move(terms), mo, ms, prm, false, P, msg)) return true;
  msg = first + "; without shared sources: " + msg;
  return false;
}

namespace {

bool build_ring(int n_out, int n_src, int n, int K, std::vector<RingTerm> terms, const std::vector<int>& mo,
                const std::vector<int>& ms, const RingParams& prm, bool allow_share, RingPlan& P, std::string& msg) {
  P = RingPlan{};
  const bool mirror = !mo.empty();
  P.K = K;
  P.N = 16 * K;
  P.mirror = mirror ? 1 : 0;
  P.nb = prm.nb;
  P.wmax = prm.wmax;
  P.ns = prm.ns;
  P.nrb = prm.nrb;
  P.bk = prm.bk;
  P.nbs = prm.nbs;
  P.src_order = prm.src_order;
  const int nb = prm.nb, N = P.N;
  if (n % 8 || nb < 1 || prm.wmax < 2 || prm.wmax % 2 || prm.ns < 2 || prm.ns > 15 || prm.nrb < 1 || prm.nrb > 8 || nb > 8 ||
      prm.bk < 1 || prm.nbs < 1 || n_out >= 0xFFFF || n_src >= 0xFFFF || prm.max_rows > 64) {
    msg = "ring plan: unsupported parameters";
    return false;
  }
  if (mirror && ((int)mo.size() != n_out || (int)ms.size() != n_src)) {
    msg = "ring plan: mirror maps of the wrong size";
    return false;
  }
  // offsets centred in (-n/2, n/2] so that an arc around offset 0 is one contiguous range
  for (RingTerm& t : terms) {
    t.off = ((t.off % n) + n) % n;
    if (t.off > n / 2) t.off -= n;
  }
  std::sort(terms.begin(), terms.end(), [](const RingTerm& a, const RingTerm& b) {
    if (a.out_row != b.out_row) return a.out_row < b.out_row;
    if (a.src_row != b.src_row) return a.src_row < b.src_row;
    if (a.off != b.off) return a.off < b.off;
    return a.k < b.k;
  });
  std::vector<size_t> row_t(n_out + 1, 0);
  {
    size_t t = 0;
    for (int r = 0; r <= n_out; ++r) {
      while (t < terms.size() && terms[t].out_row < r) ++t;
      row_t[r] = t;
    }
  }
  // mirror mode: the terms of the mirror row of r are those of r with mirrored sources
  if (mirror) {
    for (int r = 0; r < n_out; ++r) {
      const int rb = mo[r];
      if (rb < 0 || rb >= n_out || mo[rb] != r) {
        msg = "ring plan: the output mirror map is not an involution";
        return false;
      }
      if (rb <= r) continue;
      std::vector<RingTerm> mapped(terms.begin() + row_t[r], terms.begin() + row_t[r + 1]);
      for (RingTerm& t : mapped) t.src_row = ms[t.src_row];
      std::sort(mapped.begin(), mapped.end(), [](const RingTerm& a, const RingTerm& b) {
        if (a.src_row != b.src_row) return a.src_row < b.src_row;
        if (a.off != b.off) return a.off < b.off;
        return a.k < b.k;
      });
      const size_t nr = row_t[rb + 1] - row_t[rb];
      if (nr != mapped.size()) {
        msg = "ring plan: Psi is not mirror-symmetric (entry counts differ)";
        return false;
      }
      for (size_t q = 0; q < nr; ++q) {
        const RingTerm& a = mapped[q];
        const RingTerm& b = terms[row_t[rb] + q];
        // values to 1e-12 absolute (entries are at most 1): the two rows are computed from
        // their own rotations, and small hat values near their end points carry relative
        // differences far above the absolute ones
        if (a.src_row != b.src_row || a.off != b.off || a.k != b.k ||
            std::fabs(a.v - b.v) > 1e-12 * std::max(1.0, std::max(std::fabs(a.v), std::fabs(b.v)))) {
          msg = "ring plan: Psi is not mirror-symmetric";
          return false;
        }
      }
    }
  }
  // output rows of the plan: every row, or the canonical row of each mirror pair
  std::vector<int> out_rows;
  for (int r = 0; r < n_out; ++r)
    if (!mirror || r <= mo[r]) out_rows.push_back(r);
  // pairs and their Toeplitz blocks
  std::vector<Pair> pairs;
  std::vector<int> row_pair(n_out + 1, 0);  // pairs of out_rows[x]: [row_pair[x], row_pair[x + 1])
  std::vector<double> dense;
  for (size_t x = 0; x < out_rows.size(); ++x) {
    const int r = out_rows[x];
    row_pair[x] = (int)pairs.size();
    for (size_t a = row_t[r]; a < row_t[r + 1];) {
      size_t b = a;
      while (b < row_t[r + 1] && terms[b].src_row == terms[a].src_row) ++b;
      Pair pr;
      pr.r = r;
      pr.s = terms[a].src_row;
      pr.pmin = terms[a].off;
      pr.pmax = terms[b - 1].off;
      pr.lo = floor_div(pr.pmin, 8);
      const int hi = floor_div(15 + pr.pmax, 8);
      pr.ks = (hi - pr.lo + 2) / 2;
      pr.M = nb + pr.ks - 1;
      pr.t0 = a;
      pr.t1 = b;
      if (pr.ks > 255) {
        msg = "ring plan: a window wider than 255 K-steps";
        return false;
      }
      pr.boff = (int)(P.b.size() / 8);
      const int span = pr.pmax - pr.pmin + 1;
      dense.assign((size_t)K * span, 0.0);
      for (size_t t = a; t < b; ++t) dense[(size_t)terms[t].k * span + (terms[t].off - pr.pmin)] += terms[t].v;
      // [ks][2 octets][N = 16K columns][8 longitudes], column k*16 + u
      for (int kk = 0; kk < pr.ks; ++kk)
        for (int oc = 0; oc < 2; ++oc)
          for (int col = 0; col < N; ++col) {
            const int k = col / 16, u = col % 16;
            for (int el = 0; el < 8; ++el) {
              const int off = 8 * pr.lo + 16 * kk + 8 * oc + el - u;
              const double v = (off >= pr.pmin && off <= pr.pmax) ? dense[(size_t)k * span + (off - pr.pmin)] : 0.0;
              P.b.push_back(to_bf16(v));
            }
          }
      pairs.push_back(pr);
      a = b;
    }
  }
  row_pair[out_rows.size()] = (int)pairs.size();
  // a source is shared (one load per strip) when the union of its windows fits a slot
  std::vector<int> s_lo(n_src, INT_MAX), s_hi(n_src, INT_MIN);
  for (const Pair& pr : pairs) {
    s_lo[pr.s] = std::min(s_lo[pr.s], pr.lo);
    s_hi[pr.s] = std::max(s_hi[pr.s], pr.lo + 2 * pr.M);
  }
  std::vector<char> shared(n_src, 0);
  for (int s = 0; s < n_src; ++s) shared[s] = allow_share && s_hi[s] > s_lo[s] && s_hi[s] - s_lo[s] <= prm.wmax;
  // strips: consecutive plan rows, balanced by MMA count
  std::vector<long long> cost(out_rows.size(), 0);
  long long total = 0;
  for (size_t x = 0; x < out_rows.size(); ++x) {
    for (int q = row_pair[x]; q < row_pair[x + 1]; ++q) cost[x] += (long long)nb * pairs[q].ks;
    total += cost[x];
  }
  const long long target = std::max(1LL, total / std::max(1, prm.target_strips));
  struct StripRec {
    int x0, x1;
    long long cost;
  };
  std::vector<StripRec> srec;
  for (size_t x = 0; x < out_rows.size();) {
    size_t y = x;
    long long c = 0;
    while (y < out_rows.size() && (y == x || (c < target && (int)(y - x) < prm.max_rows))) c += cost[y++];
    srec.push_back(StripRec{(int)x, (int)y, c});
    x = y;
  }
  std::stable_sort(srec.begin(), srec.end(), [](const StripRec& a, const StripRec& b) { return a.cost > b.cost; });
  // script of one strip
  const int Mc = prm.wmax / 2;  // octet pairs per chunk of a long window
  for (const StripRec& st : srec) {
    struct Load {
      int s, o0, n_oct, first, last, slot;
    };
    struct Item {
      int load, row, a_off, ks, kb0, nkb, boff, flags;
    };
    std::vector<Load> loads;
    std::vector<Item> items;
    std::map<int, int> shared_load;  // source -> load index
    auto emit = [&](int L, int row, const Pair& pr, int a_off, int k0, int k1) {
      for (int kb = k0; kb < k1; kb += prm.bk) {
        Item it;
        it.load = L;
        it.row = row;
        it.a_off = a_off;
        it.ks = pr.ks;
        it.kb0 = kb;
        it.nkb = std::min(prm.bk, k1 - kb);
        it.boff = pr.boff + kb * (2 * N);  // one K-step: 2 octets x N columns x 16 bytes
        it.flags = 0;
        items.push_back(it);
        loads[L].last = (int)items.size() - 1;
      }
    };
    auto pair_items = [&](int row, const Pair& pr) {
      if (shared[pr.s]) {
        auto f = shared_load.find(pr.s);
        int L;
        if (f == shared_load.end()) {
          L = (int)loads.size();
          loads.push_back(Load{pr.s, s_lo[pr.s], s_hi[pr.s] - s_lo[pr.s], (int)items.size(), -1, -1});
          shared_load[pr.s] = L;
        } else {
          L = f->second;
        }
        emit(L, row, pr, pr.lo - s_lo[pr.s], 0, pr.ks);
      } else {
        for (int m0 = 0; m0 < pr.M; m0 += Mc) {
          const int m1 = std::min(pr.M, m0 + Mc);
          const int L = (int)loads.size();
          loads.push_back(Load{pr.s, pr.lo + 2 * m0, 2 * (m1 - m0), (int)items.size(), -1, -1});
          emit(L, row, pr, -2 * m0, std::max(0, m0 - nb + 1), std::min(pr.ks, m1));
        }
      }
    };
    const int nrows = st.x1 - st.x0;
    std::vector<int> row_first(nrows, -1), row_last(nrows, -1);
    if (!prm.src_order) {
      for (int x = st.x0; x < st.x1; ++x)
        for (int q = row_pair[x]; q < row_pair[x + 1]; ++q) pair_items(x - st.x0, pairs[q]);
    } else {
      // grouped by source: every pair of the strip's rows, ordered by source row
      std::vector<std::pair<int, int>> ord;  // (source key, pair)
      for (int x = st.x0; x < st.x1; ++x)
        for (int q = row_pair[x]; q < row_pair[x + 1]; ++q)
          ord.push_back({prm.src_key.empty() ? pairs[q].s : prm.src_key[pairs[q].s], q});
      std::stable_sort(ord.begin(), ord.end());
      for (auto& sp : ord) {
        const Pair& pr = pairs[sp.second];
        int x = 0;
        while (out_rows[st.x0 + x] != pr.r) ++x;
        pair_items(x, pr);
      }
    }
    for (size_t t = 0; t < items.size(); ++t) {
      const int rw = items[t].row;
      if (row_first[rw] < 0) row_first[rw] = (int)t;
      row_last[rw] = (int)t;
    }
    // ring slots: a load may take a slot once the slot's previous load has had its last use
    {
      std::vector<int> slot_free_after(prm.ns, -1);  // last item of the slot's current load
      for (Load& l : loads) {
        int best = -1;
        for (int q = 0; q < prm.ns; ++q)
          if (slot_free_after[q] < l.first && (best < 0 || slot_free_after[q] < slot_free_after[best])) best = q;
        if (best < 0) {
          msg = "ring plan: more loads live at once than ring slots";
          return false;
        }
        l.slot = best;
        slot_free_after[best] = l.last;
      }
    }
    // accumulator row buffers, in the order rows start
    std::vector<int> row_order;
    for (int rw = 0; rw < nrows; ++rw)
      if (row_first[rw] >= 0) row_order.push_back(rw);
    std::stable_sort(row_order.begin(), row_order.end(), [&](int a, int b) { return row_first[a] < row_first[b]; });
    std::vector<int> rbuf(nrows, 0);
    {
      std::vector<int> buf_free_after(prm.nrb, -1);
      for (int rw : row_order) {
        int best = -1;
        for (int q = 0; q < prm.nrb; ++q)
          if (buf_free_after[q] < row_first[rw] && (best < 0 || buf_free_after[q] < buf_free_after[best])) best = q;
        if (best < 0) {
          msg = "ring plan: more rows live at once than accumulator buffers";
          return false;
        }
        rbuf[rw] = best;
        buf_free_after[best] = row_last[rw];
      }
    }
    // The epilogue drains rows in start order, and a buffer's next row may start only after the
    // buffer was drained: every row that starts before it must then be complete.  Rows are
    // drained in start order, so require row_last of every earlier-starting row < row_first.
    for (size_t a = 0; a < row_order.size(); ++a)
      for (size_t b = a + 1; b < row_order.size(); ++b)
        if (rbuf[row_order[b]] == rbuf[row_order[a]]) {
          for (size_t c = 0; c <= a; ++c)
            if (row_last[row_order[c]] > row_first[row_order[b]]) {
              msg = "ring plan: a row buffer would be reused before the rows started earlier are complete";
              return false;
            }
          break;
        }
    for (size_t t = 0; t < items.size(); ++t) {
      Item& it = items[t];
      if (loads[it.load].last == (int)t) it.flags |= kItemLast;
      if (row_last[it.row] == (int)t) it.flags |= kItemRowEnd;
      if (row_first[it.row] == (int)t) it.flags |= kItemRowStart;
    }
    // emit
    const int item0 = (int)(P.items.size() / 4), load0 = (int)(P.loads.size() / 2), row0 = (int)(P.rows.size() / 2);
    for (const Load& l : loads) {
      if (l.o0 < -32768 || l.o0 > 32767 || l.n_oct > 255) {
        msg = "ring plan: load out of range";
        return false;
      }
      P.loads.push_back(l.s | (mirror ? ms[l.s] : 0xFFFF) << 16);
      P.loads.push_back((l.o0 & 0xFFFF) | l.n_oct << 16 | l.slot << 24);
      P.load_octets += l.n_oct;
    }
    for (const Item& it : items) {
      if (it.a_off < -32768 || it.a_off > 32767 || it.nkb > 255 || it.kb0 > 255 || it.load > 0xFFFF) {
        msg = "ring plan: item out of range";
        return false;
      }
      P.items.push_back(it.load | it.row << 16);
      P.items.push_back((it.a_off & 0xFFFF) | it.ks << 16 | it.flags << 24);
      P.items.push_back(it.kb0 | it.nkb << 8 | loads[it.load].n_oct << 16 | rbuf[it.row] << 24 |
                        loads[it.load].slot << 28);
      P.items.push_back(it.boff);
      // MMAs: (block, K-step) pairs inside the load
      for (int b = 0; b < nb; ++b)
        for (int k = it.kb0; k < it.kb0 + it.nkb && k < it.ks; ++k) {
          const int o = it.a_off + 2 * b + 2 * k;
          if (o >= 0 && o + 2 <= loads[it.load].n_oct) ++P.mmas;
        }
    }
    // rows in start order, rows without entries after them (they need no accumulator)
    for (int rw : row_order) {
      const int r = out_rows[st.x0 + rw];
      const int rb = mirror ? mo[r] : 0xFFFF;
      P.rows.push_back(r | rb << 16);
      P.rows.push_back(rbuf[rw] << 8);
    }
    for (int rw = 0; rw < nrows; ++rw)
      if (row_first[rw] < 0) {
        const int r = out_rows[st.x0 + rw];
        P.rows.push_back(r | (mirror ? mo[r] : 0xFFFF) << 16);
        P.rows.push_back(kRowEmpty);
      }
    // the items' row field is strip-relative in start order
    std::vector<int> pos(nrows, -1);
    for (size_t a = 0; a < row_order.size(); ++a) pos[row_order[a]] = (int)a;
    for (size_t t = 0; t < items.size(); ++t) {
      int& w0 = P.items[4 * (item0 + t)];
      w0 = (w0 & 0xFFFF) | pos[items[t].row] << 16;
    }
    const int rec[8] = {item0, (int)(P.items.size() / 4), load0, (int)(P.loads.size() / 2), row0,
                        (int)(P.rows.size() / 2), (int)std::min<long long>(st.cost, INT_MAX), 0};
    P.strips.insert(P.strips.end(), rec, rec + 8);
  }
  return true;
}

}  // namespace
}  // namespace disco
