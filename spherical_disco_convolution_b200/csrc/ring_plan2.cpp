// Host construction of the tile-script plan of the TMA-staged strip contraction.
//
// The forward contraction of the page "torch_harmonics.DiscreteContinuousConvS2" (class
// description: Psi is stored for output longitude 0 and shifted along the longitude for the
// others) is, for an output row r and a source row s, the correlation
//     out[.., k, r, q] += sum_off v_k(off) src[.., s, q + off]
// along the longitude ring.  For 16 consecutive outputs q0 + u and a window of 16*ks source
// longitudes starting at q0 + 8*lo it is a product with the banded Toeplitz block
//     B[p', (k, u)] = v_k(8*lo + p' - u)                      (bf16, one rounding of Psi)
// which is the same for every q0.  Block b of a tile (outputs q0 + 16b ..) reads the window
// shifted by two octets per block.
//
// This file writes, for every (strip of output rows, tile of 16*nb longitudes), the script the
// kernel replays: the source-row windows to stage (TMA boxes of 64 longitudes x 64 planes), the
// Toeplitz K-steps to copy, the MMAs of each of the four issuers with their shared-memory
// addresses, and the waits and commits between them.  A window that crosses the longitude seam
// is split into pieces at the seam; each piece is staged at its own shift (the TMA fills zeros
// outside [0, nlon)), and a K-step is applied to every piece it touches, so that every source
// longitude is counted exactly once.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <queue>
#include <string>
#include <utility>
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

constexpr int kWinMax = 15;  // octets of a staged window: two chunks of 8, the second at +7

struct Pair {
  int r, s;        // output row, source row
  int pmin, pmax;  // offsets reached
  int lo, ks, M;   // first octet of block 0's window, K-steps, octet pairs for nb blocks
  long long boff;  // B offset of K-step 0 (16-byte units)
};

bool build_tiles(int n_out, int n_src, int n, int K, std::vector<RingTerm> terms, const std::vector<int>& mo,
                 const std::vector<int>& ms, const TileParams& prm, bool allow_share, TilePlan& P, std::string& msg);

}  // namespace

bool make_tile_plan(int n_out, int n_src, int n, int K, std::vector<RingTerm> terms, const std::vector<int>& mo,
                    const std::vector<int>& ms, const TileParams& prm, TilePlan& P, std::string& msg) {
  // sources shared by the rows of a strip when the ring has room for them, else every
  // (row, source) pair loads its own window
  if (build_tiles(n_out, n_src, n, K, terms, mo, ms, prm, true, P, msg)) return true;
  const std::string first = msg;
  if (build_tiles(n_out, n_src, n, K, std::move(terms), mo, ms, prm, false, P, msg)) return true;
  msg = first + "; without shared sources: " + msg;
  return false;
}

namespace {

bool build_tiles(int n_out, int n_src, int n, int K, std::vector<RingTerm> terms, const std::vector<int>& mo,
                 const std::vector<int>& ms, const TileParams& prm, bool allow_share, TilePlan& P, std::string& msg) {
  P = TilePlan{};
  const bool mirror = !mo.empty();
  const int nb = prm.nb, N = 16 * K;
  const int kstep_bytes = 2 * N * 16;  // one Toeplitz K-step: 2 octets x N columns x 16 bytes
  P.K = K;
  P.N = N;
  P.mirror = mirror ? 1 : 0;
  P.nb = nb;
  P.ns = prm.ns;
  P.nrb = prm.nrb;
  P.nbs = prm.nbs;
  P.bslot_bytes = prm.bslot_bytes;
  P.src_order = prm.src_order;
  P.n_ctas = prm.n_ctas;
  if (n % 8 || nb != 4 || prm.ns < 2 || prm.ns > 8 || prm.nrb < 1 || prm.nrb > 8 || prm.nrb * nb * N > 512 ||
      prm.nbs < 1 || prm.nbs > 8 || prm.bslot_bytes % 16 || prm.bslot_bytes > 16384 || prm.bslot_bytes < kMetaBytes + kstep_bytes ||
      prm.n_ctas < 1 || n_out >= 0xFFFF || n_src >= 0xFFFF || prm.max_rows > 64) {
    msg = "tile plan: unsupported parameters";
    return false;
  }
  if (mirror && ((int)mo.size() != n_out || (int)ms.size() != n_src)) {
    msg = "tile plan: mirror maps of the wrong size";
    return false;
  }
  const int R = n / 8;  // octets around the ring
  // K-steps of one item: the room a B slot has after its batch record
  const int bk = (prm.bslot_bytes - kMetaBytes) / kstep_bytes;
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
        msg = "tile plan: the output mirror map is not an involution";
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
        msg = "tile plan: Psi is not mirror-symmetric (entry counts differ)";
        return false;
      }
      for (size_t q = 0; q < nr; ++q) {
        const RingTerm& a = mapped[q];
        const RingTerm& b = terms[row_t[rb] + q];
        // values to 1e-12 absolute (entries are at most 1): the two rows are computed from their
        // own rotations, and small hat values near their end points differ in relative terms
        if (a.src_row != b.src_row || a.off != b.off || a.k != b.k ||
            std::fabs(a.v - b.v) > 1e-12 * std::max(1.0, std::max(std::fabs(a.v), std::fabs(b.v)))) {
          msg = "tile plan: Psi is not mirror-symmetric";
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
  std::vector<int> row_pair(out_rows.size() + 1, 0);
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
      pr.boff = (long long)(P.b.size() / 8);
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
  if (P.b.size() / 8 > (size_t)INT_MAX) {
    msg = "tile plan: Toeplitz blocks too large";
    return false;
  }
  // a source is shared (one window per strip) when the union of its windows fits two chunks
  std::vector<int> s_lo(n_src, INT_MAX), s_hi(n_src, INT_MIN);
  for (const Pair& pr : pairs) {
    s_lo[pr.s] = std::min(s_lo[pr.s], pr.lo);
    s_hi[pr.s] = std::max(s_hi[pr.s], pr.lo + 2 * pr.M);
  }
  std::vector<char> shared(n_src, 0);
  for (int s = 0; s < n_src; ++s) shared[s] = s_hi[s] > s_lo[s] && s_hi[s] - s_lo[s] <= kWinMax;
  // strips: consecutive plan rows, balanced by MMA count
  std::vector<long long> cost(out_rows.size(), 0);
  long long total = 0;
  for (size_t x = 0; x < out_rows.size(); ++x) {
    for (int q = row_pair[x]; q < row_pair[x + 1]; ++q) cost[x] += (long long)nb * pairs[q].ks;
    total += cost[x];
  }
  const long long target = std::max(1LL, total / std::max(1, prm.target_strips));
  std::vector<std::pair<int, int>> strips;
  for (size_t x = 0; x < out_rows.size();) {
    size_t y = x;
    long long c = 0;
    while (y < out_rows.size() && (y == x || (c < target && (int)(y - x) < prm.max_rows))) c += cost[y++];
    strips.push_back({(int)x, (int)y});
    x = y;
  }
  P.n_strips = (int)strips.size();
  P.n_qt = (n + 16 * nb - 1) / (16 * nb);
  std::vector<long long> script_cost;
  // ---------------------------------------------------------------- one script per (strip, tile)
  for (const auto& st : strips) {
    const int nrows = st.second - st.first;
    // (row, pair) in the order the items are issued
    std::vector<std::pair<int, int>> order;
    if (!prm.src_order) {
      for (int x = st.first; x < st.second; ++x)
        for (int q = row_pair[x]; q < row_pair[x + 1]; ++q) order.push_back({x - st.first, q});
    } else {
      std::vector<std::pair<int, std::pair<int, int>>> ord;  // (source key, (row, pair))
      for (int x = st.first; x < st.second; ++x)
        for (int q = row_pair[x]; q < row_pair[x + 1]; ++q)
          ord.push_back({prm.src_key.empty() ? pairs[q].s : prm.src_key[pairs[q].s], {x - st.first, q}});
      std::stable_sort(ord.begin(), ord.end(),
                       [](const auto& a, const auto& b) { return a.first < b.first; });
      for (auto& o : ord) order.push_back(o.second);
    }
    // one script: with shared sources when the ring has room for them in this tile, else with
    // every (row, source) pair's own windows; a failed attempt leaves the plan as it was
    auto build_script = [&](int qt, bool share) -> bool {
      const int q8 = qt * 2 * nb;                                       // first output octet
      const int nbv = std::min(nb, (n - 16 * nb * qt + 15) / 16);       // blocks inside the ring
      // physical loads: (source, shifted origin) -> index; origin = absolute octet of chunk 0
      struct Load {
        int s, origin, first = -1, last = -1, slot = -1, mask = 0;
      };
      std::vector<Load> loads;
      std::map<std::pair<int, int>, int> load_of;  // (logical load id, piece shift) -> load
      struct Mma {
        int b, k, o;  // block, K-step, octet relative to the load
      };
      struct Item {
        int row, pair, load, kb0, kb1;  // K-steps [kb0, kb1)
        std::vector<Mma> mmas;
        int batch = -1, dst = 0;
      };
      std::vector<Item> items;
      int logical = 0;
      std::map<int, int> shared_logical;  // source -> logical load id (shared windows)
      for (const auto& rp : order) {
        const Pair& pr = pairs[rp.second];
        // logical loads of this pair: (id, absolute origin, octets, octet of K-step position 0)
        struct LL {
          int id, A, len, obase;
        };
        std::vector<LL> lls;
        if (share && shared[pr.s]) {
          auto f = shared_logical.find(pr.s);
          int id;
          if (f == shared_logical.end()) {
            id = logical++;
            shared_logical[pr.s] = id;
          } else {
            id = f->second;
          }
          lls.push_back(LL{id, q8 + s_lo[pr.s], s_hi[pr.s] - s_lo[pr.s], pr.lo - s_lo[pr.s]});
        } else {
          for (int m = 0; 14 * m < 2 * pr.M - 1; ++m) {
            const int len = std::min(kWinMax, 2 * pr.M - 14 * m);
            lls.push_back(LL{logical++, q8 + pr.lo + 14 * m, len, -14 * m});
          }
        }
        for (const LL& ll : lls) {
          // MMAs of this window, by the piece (seam shift) each touches
          std::map<int, std::vector<Mma>> by_piece;
          for (int b = 0; b < nbv; ++b)
            for (int k = 0; k < pr.ks; ++k) {
              const int o = ll.obase + 2 * (b + k);
              if (o < 0 || o + 2 > ll.len) continue;
              const int p1 = floor_div(ll.A + o, R), p2 = floor_div(ll.A + o + 1, R);
              by_piece[p1].push_back(Mma{b, k, o});
              if (p2 != p1) by_piece[p2].push_back(Mma{b, k, o});
            }
          for (auto& bp : by_piece) {
            const auto key = std::make_pair(ll.id, bp.first);
            auto f = load_of.find(key);
            int L;
            if (f == load_of.end()) {
              L = (int)loads.size();
              Load ld;
              ld.s = pr.s;
              ld.origin = ll.A - bp.first * R;
              loads.push_back(ld);
              load_of[key] = L;
            } else {
              L = f->second;
            }
            // items of at most bk K-steps
            int kmin = INT_MAX, kmax = INT_MIN;
            for (const Mma& mm : bp.second) {
              kmin = std::min(kmin, mm.k);
              kmax = std::max(kmax, mm.k);
              loads[L].mask |= 1 << (mm.o / 7);
            }
            for (int k0 = kmin; k0 <= kmax; k0 += bk) {
              Item it;
              it.row = rp.first;
              it.pair = rp.second;
              it.load = L;
              it.kb0 = k0;
              it.kb1 = std::min(kmax + 1, k0 + bk);
              for (const Mma& mm : bp.second)
                if (mm.k >= it.kb0 && mm.k < it.kb1) it.mmas.push_back(mm);
              if (!it.mmas.empty()) items.push_back(std::move(it));
            }
          }
        }
      }
      for (size_t t = 0; t < items.size(); ++t) {
        Load& l = loads[items[t].load];
        if (l.first < 0) l.first = (int)t;
        l.last = (int)t;
      }
      // B batches: consecutive items whose K-steps fit one B slot.  The issuers commit once per
      // batch; a ring slot, a finished row and a B slot are all released by the completion of a
      // batch (the batch that holds their last use).
      // A batch also ends before an item that would make more windows or rows live in it (used
      // in it, or before and after it) than there are ring slots or row buffers.
      std::vector<int> rfirst(nrows, -1), rlast(nrows, -1);
      for (size_t t = 0; t < items.size(); ++t) {
        if (rfirst[items[t].row] < 0) rfirst[items[t].row] = (int)t;
        rlast[items[t].row] = (int)t;
      }
      int nbatch = 0, fill = 0;
      {
        std::vector<char> lin(loads.size(), 0), rin(nrows, 0);
        int nl = 0, nr = 0, n_new_l = 0, n_new_r = 0, n_words = 0, n_items = 0;
        auto open_batch = [&](size_t t0) {
          // windows and rows used before t0 and again at or after it stay live
          std::fill(lin.begin(), lin.end(), 0);
          std::fill(rin.begin(), rin.end(), 0);
          nl = nr = 0;
          for (size_t L = 0; L < loads.size(); ++L)
            if (loads[L].first >= 0 && loads[L].first < (int)t0 && loads[L].last >= (int)t0) lin[L] = 1, ++nl;
          for (int rw = 0; rw < nrows; ++rw)
            if (rfirst[rw] >= 0 && rfirst[rw] < (int)t0 && rlast[rw] >= (int)t0) rin[rw] = 1, ++nr;
          ++nbatch;
          fill = 0;
          n_new_l = n_new_r = n_words = n_items = 0;
        };
        const int b_cap = prm.bslot_bytes - kMetaBytes;
        for (size_t t = 0; t < items.size(); ++t) {
          const int bytes = (items[t].kb1 - items[t].kb0) * kstep_bytes;
          const int L = items[t].load, rw = items[t].row;
          const bool new_l = loads[L].first == (int)t, new_r = rfirst[rw] == (int)t;
          const int words = (int)items[t].mmas.size();
          const bool full = fill + bytes > b_cap || nl + (lin[L] ? 0 : 1) > prm.ns ||
                            nr + (rin[rw] ? 0 : 1) > prm.nrb || n_new_l + new_l > kMaxLoadStarts ||
                            n_new_r + new_r > kMaxRowStarts || 4 + n_words + words > kMaxMetaWords ||
                            n_items + 1 > 31;
          if (t == 0 || full) {
            open_batch(t);
            if (nl + (lin[L] ? 0 : 1) > prm.ns || nr + (rin[rw] ? 0 : 1) > prm.nrb) {
              msg = "tile plan: more windows or rows live across a batch boundary than slots or buffers";
              return false;
            }
          }
          if (!lin[L]) lin[L] = 1, ++nl;
          if (!rin[rw]) rin[rw] = 1, ++nr;
          n_new_l += new_l;
          n_new_r += new_r;
          n_words += words;
          ++n_items;
          if (4 + n_words > kMaxMetaWords) {
            msg = "tile plan: an item with more MMAs than a batch holds";
            return false;
          }
          if (fill + bytes > b_cap) {
            msg = "tile plan: an item with more K-steps than a B slot holds";
            return false;
          }
          items[t].batch = nbatch - 1;
          items[t].dst = kMetaBytes + fill;
          fill += bytes;
        }
      }
      std::vector<int> batch_bytes(nbatch, 0), batch_first(nbatch, -1), batch_last(nbatch, -1);
      for (size_t t = 0; t < items.size(); ++t) {
        const int bt = items[t].batch;
        batch_bytes[bt] += (items[t].kb1 - items[t].kb0) * kstep_bytes;
        if (batch_first[bt] < 0) batch_first[bt] = (int)t;
        batch_last[bt] = (int)t;
      }
      auto bat = [&](int t) { return items[t].batch; };
      // loads in the order of first use; a slot takes a load once the batch of its previous
      // load's last use precedes the batch of the new load's first use
      std::vector<int> lorder;
      for (size_t L = 0; L < loads.size(); ++L)
        if (loads[L].first >= 0) lorder.push_back((int)L);
      std::stable_sort(lorder.begin(), lorder.end(), [&](int a, int b) { return loads[a].first < loads[b].first; });
      {
        std::vector<int> slot_free_after(prm.ns, -1);
        for (int L : lorder) {
          int best = -1;
          for (int q = 0; q < prm.ns; ++q)
            if (slot_free_after[q] < bat(loads[L].first) && (best < 0 || slot_free_after[q] < slot_free_after[best]))
              best = q;
          if (best < 0) {
            msg = "tile plan: more windows live at once than ring slots";
            return false;
          }
          loads[L].slot = best;
          slot_free_after[best] = bat(loads[L].last);
        }
      }
      // rows: first and last item, accumulator buffers in start order
      std::vector<int> row_first(nrows, -1), row_last(nrows, -1);
      for (size_t t = 0; t < items.size(); ++t) {
        const int rw = items[t].row;
        if (row_first[rw] < 0) row_first[rw] = (int)t;
        row_last[rw] = (int)t;
      }
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
            if (buf_free_after[q] < bat(row_first[rw]) && (best < 0 || buf_free_after[q] < buf_free_after[best]))
              best = q;
          if (best < 0) {
            msg = "tile plan: more rows live at once than accumulator buffers";
            return false;
          }
          rbuf[rw] = best;
          buf_free_after[best] = bat(row_last[rw]);
        }
      }
      // the epilogue drains rows in start order: a buffer's next row may start only after every
      // row started before the buffer's previous row is complete, in an earlier batch
      for (size_t a = 0; a < row_order.size(); ++a)
        for (size_t b = a + 1; b < row_order.size(); ++b)
          if (rbuf[row_order[b]] == rbuf[row_order[a]]) {
            for (size_t c = 0; c <= a; ++c)
              if (bat(row_last[row_order[c]]) >= bat(row_first[row_order[b]])) {
                msg = "tile plan: a row buffer would be reused before the rows started earlier are complete";
                return false;
              }
            break;
          }
      // every block inside the ring of every row with items gets at least one MMA (the first one
      // clears the accumulator)
      {
        std::vector<int> seen(nrows, 0);
        for (const Item& it : items)
          for (const Mma& mm : it.mmas) seen[it.row] |= 1 << mm.b;
        for (int rw : row_order)
          if (seen[rw] != (1 << nbv) - 1) {
            msg = "tile plan: a block of a row has no product";
            return false;
          }
      }
      // ------------------------------------------------------------ emit the script
      int rec[kTileInts] = {};
      rec[0] = (int)(P.loads.size() / 4);
      std::vector<int> lpos(loads.size(), -1);
      for (int L : lorder) {
        const Load& l = loads[L];
        lpos[L] = (int)(P.loads.size() / 4) - rec[0];
        const int sbar = mirror ? ms[l.s] : 0xFFFF;
        P.loads.push_back(l.s | sbar << 16);
        P.loads.push_back(l.slot | l.mask << 8);
        P.loads.push_back(8 * l.origin);
        P.loads.push_back(bat(l.last) | bat(l.first) << 16);
        P.boxes += 2 * __builtin_popcount(l.mask);
      }
      rec[1] = (int)(P.loads.size() / 4);
      rec[2] = (int)(P.copies.size() / 4);  // (copies are written with the batch records below)
      // rows: start order, then the rows without entries
      rec[4] = (int)(P.rows.size() / 2);
      for (int rw : row_order) {
        const int r = out_rows[st.first + rw];
        P.rows.push_back(r | (mirror ? mo[r] : 0xFFFF) << 16);
        P.rows.push_back(rbuf[rw] << 8 | bat(row_last[rw]) << 12);
      }
      for (int rw = 0; rw < nrows; ++rw)
        if (row_first[rw] < 0) {
          const int r = out_rows[st.first + rw];
          P.rows.push_back(r | (mirror ? mo[r] : 0xFFFF) << 16);
          P.rows.push_back(kRowEmpty);
        }
      rec[5] = (int)(P.rows.size() / 2);
      // batch records: a header, each issuer's MMA words, then the items' Toeplitz K-steps;
      // the copies of a batch bring the record and the K-steps into its B slot
      int mma_max = 0;
      rec[6] = (int)P.cmds.size();
      {
        std::vector<int> n_mma(nb, 0);
        std::vector<std::vector<int>> started(nb, std::vector<int>(nrows, 0));
        size_t t = 0;
        for (int bt = 0; bt < nbatch; ++bt) {
          const size_t t0 = t;
          while (t < items.size() && items[t].batch == bt) ++t;
          if (t0 == t || t - t0 > 31 || nbatch > 0xFFFF) {
            msg = "tile plan: an empty batch, more than 31 items in a batch or too many batches";
            return false;
          }
          std::vector<std::vector<uint32_t>> lists(nb);
          uint32_t lstarts = 0, rstarts = 0;
          int nls = 0, nrs = 0;
          for (size_t u = t0; u < t; ++u) {
            const Item& it = items[u];
            const Load& l = loads[it.load];
            const int rb = rbuf[it.row];
            if (l.first == (int)u) lstarts |= (uint32_t)l.slot << (3 + 4 * nls++);
            if (row_first[it.row] == (int)u) rstarts |= (uint32_t)rb << (3 + 3 * nrs++);
            for (const Mma& mm : it.mmas) {
              const int c = mm.o / 7, pos = mm.o - 7 * c;
              const uint32_t a16 = (uint32_t)(l.slot * kSlotBytes + c * kChunkBytes + pos * 16) >> 4;
              const uint32_t b16 = (uint32_t)(it.dst + (mm.k - it.kb0) * kstep_bytes) >> 4;
              if (a16 >= (1u << 14) || b16 >= (1u << 10)) {
                msg = "tile plan: operand address out of range";
                return false;
              }
              const uint32_t acc = started[mm.b][it.row] ? 1u : 0u;
              started[mm.b][it.row] = 1;
              lists[mm.b].push_back(a16 | b16 << 14 | (uint32_t)rb << 24 | acc << 27);
            }
          }
          // header: MMA counts; word offsets of the lists of issuers 1..3; ring slots whose loads
          // are first used here; row buffers whose rows start here
          uint32_t cnt = 0, offs = 0;
          int off = 4;
          for (int iw = 0; iw < nb; ++iw) {
            if (lists[iw].size() > 255) {
              msg = "tile plan: more than 255 MMAs of one issuer in a batch";
              return false;
            }
            cnt |= (uint32_t)lists[iw].size() << (8 * iw);
            if (iw > 0) offs |= (uint32_t)off << (10 * (iw - 1));
            off += (int)lists[iw].size();
            n_mma[iw] += (int)lists[iw].size();
          }
          const size_t m0 = P.cmds.size();
          P.cmds.push_back(cnt);
          P.cmds.push_back(offs);
          P.cmds.push_back((uint32_t)nls | lstarts);
          P.cmds.push_back((uint32_t)nrs | rstarts);
          for (int iw = 0; iw < nb; ++iw) P.cmds.insert(P.cmds.end(), lists[iw].begin(), lists[iw].end());
          while ((P.cmds.size() - m0) % 4) P.cmds.push_back(0u);
          const int meta_bytes = (int)(P.cmds.size() - m0) * 4;
          if (meta_bytes > kMetaBytes || m0 / 4 > (size_t)INT_MAX) {
            msg = "tile plan: batch record too large";
            return false;
          }
          const int total = meta_bytes + batch_bytes[bt];
          P.copies.push_back((int)(m0 / 4));
          P.copies.push_back(meta_bytes);
          P.copies.push_back(0);
          P.copies.push_back(kCopyBatchStart | kCopyMeta | total << 8 | (int)(1 + t - t0) << 24);
          for (size_t u = t0; u < t; ++u) {
            const Item& it = items[u];
            const Pair& pr = pairs[it.pair];
            const int bytes = (it.kb1 - it.kb0) * kstep_bytes;
            const long long boff = pr.boff + (long long)it.kb0 * (2 * N);
            if (boff > INT_MAX) {
              msg = "tile plan: B offset out of range";
              return false;
            }
            P.copies.push_back((int)boff);
            P.copies.push_back(bytes);
            P.copies.push_back(it.dst);
            P.copies.push_back(u + 1 == t ? kCopyBatchEnd : 0);
            P.copies_bytes += bytes;
          }
        }
        for (int iw = 0; iw < nb; ++iw) {
          mma_max = std::max(mma_max, n_mma[iw]);
          P.mmas += n_mma[iw];
        }
      }
      rec[7] = (int)P.cmds.size();
      rec[3] = (int)(P.copies.size() / 4);
      P.items += (long long)items.size();
      // cost in cycles: the busiest issuer (about 190 cycles per MMA and 60 per item) against the
      // staging (about 24 bytes per cycle) and the epilogue (about 1500 cycles per row)
      long long boxes = 0;
      for (const Load& l : loads) boxes += 2 * __builtin_popcount(l.mask);
      const long long c_mma = 190LL * mma_max + 60LL * (long long)items.size();
      const long long c_x = boxes * 8192 / 24;
      const long long c_y = 1500LL * nrows;
      const long long c = std::max(c_mma, std::max(c_x, c_y)) + 2000;
      rec[11] = nbatch;
      rec[12] = (int)std::min<long long>(c, INT_MAX);
      P.tiles.insert(P.tiles.end(), rec, rec + kTileInts);
      script_cost.push_back(c);
      if (P.cmds.size() > (size_t)INT_MAX / 2 || P.loads.size() > (size_t)INT_MAX / 2) {
        msg = "tile plan: too large";
        return false;
      }
      return true;
    };
    for (int qt = 0; qt < P.n_qt; ++qt) {
      const size_t n_loads = P.loads.size(), n_copies = P.copies.size(), n_rows = P.rows.size(), n_cmds = P.cmds.size();
      const long long mmas = P.mmas, boxes = P.boxes, cbytes = P.copies_bytes, nitems = P.items;
      if (build_script(qt, allow_share)) continue;
      P.loads.resize(n_loads);
      P.copies.resize(n_copies);
      P.rows.resize(n_rows);
      P.cmds.resize(n_cmds);
      P.mmas = mmas;
      P.boxes = boxes;
      P.copies_bytes = cbytes;
      P.items = nitems;
      if (!allow_share || !build_script(qt, false)) return false;
    }
  }
  // scripts to CTAs: longest first, each to the least loaded CTA
  {
    const int S = (int)script_cost.size();
    std::vector<int> idx(S);
    for (int i = 0; i < S; ++i) idx[i] = i;
    std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return script_cost[a] > script_cost[b]; });
    const int C = std::max(1, std::min(prm.n_ctas, S));
    P.n_ctas = C;
    std::priority_queue<std::pair<long long, int>, std::vector<std::pair<long long, int>>, std::greater<>> pq;
    for (int c = 0; c < C; ++c) pq.push({0, c});
    std::vector<std::vector<int>> lists(C);
    for (int i : idx) {
      auto top = pq.top();
      pq.pop();
      lists[top.second].push_back(i);
      pq.push({top.first + script_cost[i], top.second});
    }
    P.cta_tiles.assign(C + 1, 0);
    for (int c = 0; c < C; ++c) P.cta_tiles[c + 1] = P.cta_tiles[c] + (int)lists[c].size();
    for (int c = 0; c < C; ++c)
      for (int i : lists[c]) P.cta_tiles.push_back(i);
  }
  return true;
}

}  // namespace
}  // namespace disco
