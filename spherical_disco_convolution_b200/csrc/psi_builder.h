// Host-side Psi builder and plan construction for libdisco.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "plan.h"

namespace disco {

struct Geometry {
  int nlat_in, nlon_in, nlat_out, nlon_out;
  int n_r, n_alpha;
  double theta_cutoff;
  int K;        // number of basis functions
  int stride;   // nlon_in / nlon_out
  int grid_in = 0, grid_out = 0;  // latitude grids (DISCO_GRID_* codes)
};

// Colatitudes theta[0..nlat) (north to south) of a latitude grid, and its quadrature weights
// on t = cos(theta) (they sum to 2).  grid: 0 equiangular (Clenshaw-Curtis), 1 Legendre-Gauss,
// 2 Lobatto (Gauss-Lobatto-Legendre), 3 equiangular with trapezoidal weights.  Returns false
// for an unknown grid or too few points.
bool latitude_grid(int grid, int nlat, std::vector<double>& theta, std::vector<double>& weight);

struct PsiEntry {
  int k, j, i, p;   // basis, output row, input row, longitude offset in [0, nlon_in)
  double v;
};

// Status codes mirror disco_status (0 ok, 1 invalid, 2 unsupported, 6 geometry).  Builds the
// rows j in [j_begin, j_end) (j_end < 0: to the last row); entries keep their global indices.
int build_psi_entries(const Geometry& g, std::vector<PsiEntry>& out, std::string& msg, int j_begin = 0,
                      int j_end = -1);

struct GatherPlan {
  std::vector<RowPlan> rows;   // ordered heaviest first
  std::vector<SrcRow> src;
  std::vector<Chunk> chunks;
  std::vector<float> vals;
  std::vector<Ring> rings;
  std::vector<BandPlan> bands;  // banded plans only: heavy bands first, then light ones
  int n_heavy = 0;              // bands whose staging exceeds the light budget
  int nk = 1;          // value sets per chunk (K for the forward, 1 for the adjoint)
  int step = 1;        // source positions advance by `step` per output (forward: s; adjoint: 1)
  int residues = 1;    // output residue classes (adjoint: s)
  int max_src = 0;     // most source rows of any output row
  int max_ring = 0;    // most ring terms of any output row
};

// Elements staged per channel for output row `r` and a block of qb outputs.
int stage_elems(const GatherPlan& P, const RowPlan& r, int qb);

// Forward gather plan: output rows j, sources x rows i, K accumulators.
GatherPlan make_forward_plan(const Geometry& g, const std::vector<PsiEntry>& e);

// Banded plan: consecutive light output rows (no ring terms, spans <= 64, at most max_chunks
// chunks) are grouped into bands of up to nb_max rows that share their staged source rows;
// other rows form bands of one.  Works on the forward plan (rows j) and the adjoint plan
// (rows i, one chunk list per residue class).
GatherPlan make_band_plan(int n_rows, const GatherPlan& single, int nb_max, int max_chunks);

// Orders a banded plan's bands as [heavy ..., light ...] where a band is heavy when one channel
// pair's staging for a block of qb outputs exceeds light_words; sets n_heavy.
void split_bands(GatherPlan& P, int qb, int light_words);

// Toeplitz plan of the tensor-core contraction (stride 1).  For output row j and source row i,
// y[c, k, j, q] gets sum_p Psi_k(j, i, p) x[c, i, q + p]: the same correlation for every q, so
// one expanded block B[p', (h, k, u)] = Psi_k(lon_off + p' - u) serves every group of 8 outputs
// whose window starts lon_off longitudes after it.
struct ToeplitzPlan {
  int K = 0;
  int N = 0;                         // MMA columns
  int parts = 1;                     // 1: hi and lo parts side by side in N (N = 16K); 2: one
                                     // block per part, two MMAs into one accumulator (N = 8K
                                     // rounded up to 16), for K above 8
  std::vector<TzSlab> slabs;         // grouped by output row
  std::vector<int> row_begin;        // slabs of row j: [row_begin[j], row_begin[j + 1])
  std::vector<int> order;            // output rows, most K-steps first
  std::vector<int> slots;            // per position in `order`: {row, first slab, end slab, 0}
  std::vector<uint16_t> b;           // expanded Psi blocks, bf16 bits
  long long ksteps = 0;              // sum of nk over all slabs
};

// Forward plan: output rows j, source rows i of x, K basis functions, offsets p.
ToeplitzPlan make_toeplitz_plan(const Geometry& g, const std::vector<PsiEntry>& e);

// Adjoint plan (input gradient, stride 1): output rows i of dx, source rows k*nlat_out + j of dy
// (one basis function), offsets -p:  dx[c, i, l] = sum_{k,j} sum_p Psi_k(j, i, p) dy[c, k, j, l - p].
ToeplitzPlan make_adjoint_toeplitz_plan(const Geometry& g, const std::vector<PsiEntry>& e);

// Ring plan of the strip-staged tensor-core contraction (contract_ring.cu).
//
// The correlation of an output row r with a source row s (p-shift symmetry, page
// "torch_harmonics.DiscreteContinuousConvS2", class description) is, for 16 consecutive
// outputs, a product with a banded Toeplitz block: B[p', (k, u)] = Psi_k(8*lo + p' - u) for a
// window of 16*ks source longitudes starting 8*lo after the first output (lo = floor(pmin/8)).
// A tile covers nb such blocks of 16 outputs of a strip of consecutive output rows.  The plan is
// a script replayed for every tile: `loads` put source-row windows (octets of 8 longitudes)
// into a ring of shared-memory slots, `items` apply one Toeplitz block (a range of its K-steps)
// to one loaded window for every block of the tile.  A source whose windows for all the rows of
// a strip fit one slot is loaded once and shared by every row that reaches it; a longer window
// is loaded in chunks, each used by one row.  M rows 0..63 of an MMA are 64 planes of the row,
// rows 64..127 either the mirror row (mirror = 1: the north-south mirror of the output row and
// of each source row, whose Psi blocks are the same) or the next 64 planes (mirror = 0).
struct RingPlan {
  int K = 0, N = 0;       // basis functions per term, MMA columns (16 outputs per function)
  int mirror = 0;
  int nb = 0;             // blocks of 16 outputs per tile
  int wmax = 0;           // octets per ring slot
  int ns = 0;             // ring slots
  int nrb = 0;            // accumulator row buffers (tensor memory)
  int bk = 0;             // Toeplitz K-steps per B slot
  int nbs = 0;            // B slots
  int src_order = 0;      // 0: items grouped by output row; 1: grouped by source
  std::vector<int> strips;  // 8 ints per strip, heaviest first: item0, item1, load0, load1, row0, row1, cost, 0
  std::vector<int> loads;   // 2 ints per load (see below)
  std::vector<int> items;   // 4 ints per item (see ring_item_*)
  std::vector<int> rows;    // 2 ints per row, in accumulator order: r | rbar << 16, flags (kRowEmpty)
  std::vector<uint16_t> b;  // Toeplitz blocks (bf16 bits), per (row, source) pair ks K-steps of [2][N][8]
  long long mmas = 0;       // MMAs of one tile column (all strips, one q-tile, one plane tile)
  long long load_octets = 0;  // octets loaded per tile column
};
// (flags kRowEmpty, kItemLast, kItemRowEnd, kItemRowStart: plan.h)
// load ints:  [0] source row | mirror source row << 16 (0xFFFF: none); [1] first octet (signed
//             16 bits, relative to q0/8) | octets << 16 | ring slot << 24
// item ints:  [0] load (strip-relative) | row (strip-relative) << 16; [1] a_off (signed 16 bits:
//             octet of the pair's window start relative to the load's first octet) | ks << 16 |
//             flags << 24; [2] kb0 | nkb << 8 | octets of the load << 16 | row buffer << 24 |
//             ring slot << 28; [3] B
//             offset of K-step kb0 in 16-byte units.  Block b, K-step k (kb0 <= k < kb0 + nkb,
//             k < ks) reads octets a_off + 2b + 2k and the next one of the load, when both lie
//             inside it; every (block, K-step) of a pair is covered by exactly one item.
// row ints:   [0] r | rbar << 16 (rbar = r: self-mirror row, 0xFFFF: no mirror row);
//             [1] flags | row buffer << 8

struct RingTerm {
  int out_row, src_row, k, off;
  double v;
};
struct RingParams {
  int nb, wmax, ns, nrb, bk, nbs;
  int src_order;
  int target_strips, max_rows;
  std::vector<int> src_key;  // order of sources when items are grouped by source (empty: row index)
};
// Builds the ring plan from terms out[.., k, out_row, q] += v * src[.., src_row, q + off].
// mirror_out / mirror_src: the mirror row of each output / source row (empty: no mirror mode).
// Returns false (msg set) when the terms are not mirror-symmetric in mirror mode or when an
// invariant of the ring protocol cannot be met.
bool make_ring_plan(int n_out_rows, int n_src_rows, int nlon, int K, std::vector<RingTerm> terms,
                    const std::vector<int>& mirror_out, const std::vector<int>& mirror_src, const RingParams& prm,
                    RingPlan& P, std::string& msg);

// Tile-script plan of the TMA-staged strip contraction (contract_ring2.cu).  Same products as
// RingPlan (Toeplitz blocks of the p-shift symmetry, strips of output rows, nb blocks of 16
// outputs per tile), with one script per (strip, longitude tile) so that every index, shared-
// memory address and seam crossing is fixed on the host:
//   * a load is a source-row window staged by TMA as up to two chunks of 8 octets (64 longitudes,
//     128-byte swizzled rows of 64 planes, 16 KB with both M groups); chunk c starts 7c octets
//     after the window, so every K-step (two octets) lies inside one chunk.  A window that
//     crosses the longitude seam is split into pieces, each staged at its own shift with zeros
//     outside [0, nlon) (the TMA fill), and a K-step that straddles the seam is applied to both;
//   * B copies move each batch's record and its items' Toeplitz K-steps into a B slot (one
//     barrier each); the record lists, for each of the four MMA issuers (issuer b owns block b),
//     its MMAs with absolute operand addresses, and the loads and rows that start in the batch;
//   * the completion of a batch (one commit per issuer) releases its B slot and every ring slot
//     and finished row whose last use it holds.
struct TileParams {
  int nb = 4, ns = 5, nrb = 2, nbs = 3, bslot_bytes = 12288;
  int src_order = 0;
  int target_strips = 24, max_rows = 64;
  int n_ctas = 148;
  std::vector<int> src_key;
};
struct TilePlan {
  int K = 0, N = 0, mirror = 0, nb = 0, ns = 0, nrb = 0, nbs = 0, bslot_bytes = 0, src_order = 0;
  int n_strips = 0, n_qt = 0, n_ctas = 0;
  std::vector<int> tiles;     // kTileInts per script (strip-major, then longitude tile)
  std::vector<int> loads;     // 4 ints: s | sbar << 16; slot | chunk mask << 8; x0 (longitude of chunk 0); 0
  std::vector<int> copies;    // 4 ints: B offset (16-byte units); bytes; offset in the B slot; flags | batch bytes << 8
  std::vector<uint32_t> cmds; // batch records (header and the issuers' MMA words, kMetaBytes in plan.h)
  std::vector<int> rows;      // 2 ints: r | rbar << 16; flags | row buffer << 8 (start order, empty rows last)
  std::vector<int> cta_tiles; // n_ctas + 1 offsets, then the scripts of each CTA
  std::vector<uint16_t> b;    // Toeplitz blocks, per (row, source) pair ks K-steps of [2][N][8]
  long long mmas = 0, boxes = 0, copies_bytes = 0, items = 0;  // totals over all scripts
};
bool make_tile_plan(int n_out_rows, int n_src_rows, int nlon, int K, std::vector<RingTerm> terms,
                    const std::vector<int>& mirror_out, const std::vector<int>& mirror_src, const TileParams& prm,
                    TilePlan& P, std::string& msg);

// Adjoint gather plan: output rows i of dx, sources rows (k, j) of dy, one accumulator,
// output longitude l = stride*m + rho.
GatherPlan make_adjoint_plan(const Geometry& g, const std::vector<PsiEntry>& e);

}  // namespace disco
