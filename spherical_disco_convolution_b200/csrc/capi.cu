// C ABI of libdisco: argument checks, workspace layout and kernel dispatch.
// See include/disco.h for the contract of every entry point.
#include <cuda_runtime.h>
#include <cstdlib>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "../../include/disco.h"
#include "gather_common.cuh"
#include "kernels.h"
#include "psi_builder.h"

namespace disco {
namespace {
std::atomic<unsigned long long> g_launches{0};
}
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace disco

namespace {

thread_local std::string g_last_error;

disco_status fail(disco_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

disco_status cuda_fail(cudaError_t e, const char* where) {
  return fail(DISCO_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

struct DevPlan {
  disco::RowPlan* rows = nullptr;
  disco::SrcRow* srcs = nullptr;
  disco::Chunk* chunks = nullptr;
  float* vals = nullptr;
  disco::Ring* rings = nullptr;
  disco::BandPlan* bands = nullptr;
  int n_rows = 0;
  int n_bands = 0;
};

template <typename T>
cudaError_t upload(const std::vector<T>& v, T** dst) {
  *dst = nullptr;
  if (v.empty()) return cudaSuccess;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(dst), v.size() * sizeof(T));
  if (e != cudaSuccess) return e;
  return cudaMemcpy(*dst, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice);
}

cudaError_t upload_plan(const disco::GatherPlan& P, DevPlan* d) {
  d->n_rows = (int)P.rows.size();
  d->n_bands = (int)P.bands.size();
  cudaError_t e;
  if ((e = upload(P.bands, &d->bands)) != cudaSuccess) return e;
  if ((e = upload(P.rows, &d->rows)) != cudaSuccess) return e;
  if ((e = upload(P.src, &d->srcs)) != cudaSuccess) return e;
  if ((e = upload(P.chunks, &d->chunks)) != cudaSuccess) return e;
  if ((e = upload(P.rings, &d->rings)) != cudaSuccess) return e;
  return upload(P.vals, &d->vals);
}

void free_plan(DevPlan* d) {
  cudaFree(d->rows);
  cudaFree(d->srcs);
  cudaFree(d->chunks);
  cudaFree(d->vals);
  cudaFree(d->rings);
  cudaFree(d->bands);
  *d = DevPlan{};
}

constexpr int kChannelsPerCta = 16;
constexpr int kStageFloats = 12288;          // 48 KB of staging for the unfused gathers
constexpr size_t kSmemLimit = 227 * 1024;    // dynamic shared memory per CTA on sm_100
constexpr size_t kFusedTileBytes = 160 * 1024;

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace

// Device copy of the Toeplitz plan of the tensor-core contraction.
struct DevTz {
  disco::TzSlab* slabs = nullptr;
  int* row_begin = nullptr;
  int* slots = nullptr;
  uint16_t* b = nullptr;
};

cudaError_t upload_tz(const disco::ToeplitzPlan& P, DevTz* d) {
  cudaError_t e;
  if ((e = upload(P.slabs, &d->slabs)) != cudaSuccess) return e;
  if ((e = upload(P.row_begin, &d->row_begin)) != cudaSuccess) return e;
  if ((e = upload(P.slots, &d->slots)) != cudaSuccess) return e;
  return upload(P.b, &d->b);
}

void free_tz(DevTz* d) {
  cudaFree(d->slabs);
  cudaFree(d->row_begin);
  cudaFree(d->slots);
  cudaFree(d->b);
  *d = DevTz{};
}

// Device copy of a ring plan (strip-staged tensor-core contraction).
struct DevRing {
  int* strips = nullptr;
  int* loads = nullptr;
  int* items = nullptr;
  int* rows = nullptr;
  uint16_t* b = nullptr;
  int n_strips = 0;
  bool ok = false;
};

cudaError_t upload_ring(const disco::RingPlan& P, DevRing* d) {
  cudaError_t e;
  if ((e = upload(P.strips, &d->strips)) != cudaSuccess) return e;
  if ((e = upload(P.loads, &d->loads)) != cudaSuccess) return e;
  if ((e = upload(P.items, &d->items)) != cudaSuccess) return e;
  if ((e = upload(P.rows, &d->rows)) != cudaSuccess) return e;
  if ((e = upload(P.b, &d->b)) != cudaSuccess) return e;
  d->n_strips = (int)(P.strips.size() / 8);
  d->ok = true;
  return cudaSuccess;
}

void free_ring(DevRing* d) {
  cudaFree(d->strips);
  cudaFree(d->loads);
  cudaFree(d->items);
  cudaFree(d->rows);
  cudaFree(d->b);
  *d = DevRing{};
}

// Device copy of a tile-script plan (TMA-staged strip contraction).
struct DevTile {
  int* tiles = nullptr;
  int* loads = nullptr;
  int* copies = nullptr;
  uint32_t* cmds = nullptr;
  int* rows = nullptr;
  int* cta_tiles = nullptr;
  uint16_t* b = nullptr;
  bool ok = false;
};

cudaError_t upload_tile(const disco::TilePlan& P, DevTile* d) {
  cudaError_t e;
  if ((e = upload(P.tiles, &d->tiles)) != cudaSuccess) return e;
  if ((e = upload(P.loads, &d->loads)) != cudaSuccess) return e;
  if ((e = upload(P.copies, &d->copies)) != cudaSuccess) return e;
  {
    // the issuers read their streams four words at a time with three groups ahead
    std::vector<uint32_t> padded(P.cmds);
    padded.resize(P.cmds.size() + 64, 0u);
    if ((e = upload(padded, &d->cmds)) != cudaSuccess) return e;
  }
  if ((e = upload(P.rows, &d->rows)) != cudaSuccess) return e;
  if ((e = upload(P.cta_tiles, &d->cta_tiles)) != cudaSuccess) return e;
  if ((e = upload(P.b, &d->b)) != cudaSuccess) return e;
  d->ok = true;
  return cudaSuccess;
}

void free_tile(DevTile* d) {
  cudaFree(d->tiles);
  cudaFree(d->loads);
  cudaFree(d->copies);
  cudaFree(d->cmds);
  cudaFree(d->rows);
  cudaFree(d->cta_tiles);
  cudaFree(d->b);
  *d = DevTile{};
}

struct disco_psi {
  disco::Geometry g;
  int device = -1;
  cudaStream_t side = nullptr;        // heavy-row launches run here, forked from the caller's stream
  cudaEvent_t fork = nullptr, join = nullptr;
  std::vector<disco::PsiEntry> entries;
  disco::GatherPlan fwd, adj, fwdb, adjb;
  DevPlan dfwd, dadj, dfwdb, dadjb;
  bool tz_ok = false;                 // tensor-core contraction available (bf16 signals)
  disco::ToeplitzPlan tz, tza;        // forward (x -> y) and adjoint (dy -> dx) Toeplitz plans
  DevTz dtz, dtza;
  // ring plans of the strip-staged kernel: [0] forward with mirror rows, [1] forward with plane
  // pairs, [2] adjoint with mirror rows, [3] adjoint with plane pairs (empty when not built)
  disco::RingPlan ring[4];
  bool ring_built[4] = {false, false, false, false};
  std::string ring_msg[4];            // why a ring plan was not built
  DevRing dring[4];
  // tile-script plans of the TMA-staged strip kernel, same four kinds as the ring plans
  disco::TilePlan tile[4];
  bool tile_built[4] = {false, false, false, false};
  std::string tile_msg[4];
  DevTile dtile[4];
  // the forward plan of the fused variant (mirror rows; fewer B slots: the mix weights take room)
  disco::TilePlan tile_fused;
  bool tile_fused_built = false;
  DevTile dtile_fused;
  // the input gradient with dy mixed in: the transposed contraction of dout with the K basis
  // functions kept (z[o, k, i, q] = sum_{j, p} Psi_k(j, i, p) dout[o, j, q - p]), then
  // dx[c] = sum_{o, k} W[o, c, k] z[o, k] in the epilogue
  disco::TilePlan tile_fused_adj;
  bool tile_fused_adj_built = false;
  DevTile dtile_fused_adj;
  // rows without entries (handles of a band of input latitudes): output rows of the forward and
  // input rows of the adjoint, zeroed after each contraction into them
  std::vector<int> empty_out, empty_in;
  int* d_empty_out = nullptr;
  int* d_empty_in = nullptr;
};

namespace {

// Block of outputs per CTA: at most `cap` (a multiple of kTaskR), balanced over the row.
void block_shape(int n, int cap, int* qb, int* nblk) {
  int nb = (n + cap - 1) / cap;
  const int per = (n + nb - 1) / nb;
  *qb = (per + disco::kTaskR - 1) / disco::kTaskR * disco::kTaskR;
  *nblk = (n + *qb - 1) / *qb;
}

int max_stage(const disco::GatherPlan& P, int qb) {
  int m = 0;
  for (const disco::RowPlan& r : P.rows) m = std::max(m, disco::stage_elems(P, r, qb));
  return m;
}

constexpr int kChunkCacheMax = 96;
constexpr int kLightStage = 6656;  // float2 words of staging per CTA for the light bands

int max_stage_bands(const disco::GatherPlan& P, int b0, int b1, int qb) {
  int m = 1;
  for (int b = b0; b < b1; ++b) m = std::max(m, disco::stage_elems(P, P.rows[P.bands[b].rp_begin], qb));
  return m;
}

// Dynamic shared memory of a gather CTA (layout in gather_common.cuh) plus `extra` floats.
size_t gather_bytes(int cache, int nk, int stage_floats, size_t extra = 0) {
  return 4 * (disco::gather_smem_floats(cache, nk, stage_floats) + extra);
}

// Chunks per row kept in shared memory: enough for the typical row, bounded.
int chunk_cache(const disco::GatherPlan& P) {
  std::vector<int> n;
  for (const disco::RowPlan& r : P.rows) n.push_back(r.chunk_end[disco::kMaxStride - 1] - r.chunk_start[0]);
  if (n.empty()) return 0;
  std::sort(n.begin(), n.end());
  return std::min(kChunkCacheMax, n[n.size() * 9 / 10]);
}

disco::GatherArgs gather_args(const DevPlan& d, int BC, int qb, int nblk, int n_src, int n_src_rows, int n_out,
                              int n_out_rows, int budget, int cache, bool bf16) {
  disco::GatherArgs a;
  a.rows = d.rows;
  a.srcs = d.srcs;
  a.chunks = d.chunks;
  a.vals = d.vals;
  a.rings = d.rings;
  a.bands = d.bands;
  a.n_bands = d.n_bands;
  a.band0 = 0;
  a.n_rows = d.n_rows;
  a.BC = BC;
  a.cb = kChannelsPerCta;
  a.qb = qb;
  a.nblk = nblk;
  a.n_src = n_src;
  a.n_src_rows = n_src_rows;
  a.n_out = n_out;
  a.n_out_rows = n_out_rows;
  a.stage_budget = budget;
  a.chunk_cache = cache;
  a.vec_stage = (n_src % (bf16 ? 8 : 4)) == 0;
  return a;
}

disco_status check_common(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype) {
  if (!psi) return fail(DISCO_ERR_INVALID_ARG, "psi is NULL");
  if (psi->device < 0) return fail(DISCO_ERR_INVALID_ARG, "psi was built host-only (device < 0)");
  if (B <= 0 || C_in <= 0 || C_out <= 0 || groups <= 0)
    return fail(DISCO_ERR_INVALID_ARG, "B, C_in, C_out and groups must be positive");
  if (C_in % groups || C_out % groups)
    return fail(DISCO_ERR_INVALID_ARG, "groups must divide both C_in and C_out");
  if (dtype != DISCO_F32 && dtype != DISCO_BF16) return fail(DISCO_ERR_INVALID_ARG, "unknown dtype");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != psi->device) return fail(DISCO_ERR_INVALID_ARG, "current device differs from the device of psi");
  return DISCO_OK;
}

struct WsLayout {
  size_t wt = 0, dy = 0, ybuf = 0, part = 0, bpart = 0, total = 0;
  int nchunk = 0, nc = 0;
  bool tc = false;  // weight gradient on tensor cores
};

// Weight einsum (and its transpose): tensor cores for bf16 when TMA can address the rows.
cudaError_t launch_mix(bool bf16, const disco::MixArgs& m, cudaStream_t st) {
  if (bf16 && disco::mix_tc_supported(m.Mg, m.Rg, m.N)) return disco::launch_mix_tc(m, st);
  return disco::launch_mix_simt(bf16, m, st);
}

// Scratch of an operation on K kernel indices and n_out output points per plane.
WsLayout layout_kn(int K, size_t n_out, int op, int B, int C_in, int C_out, int groups, disco_dtype dtype) {
  WsLayout L;
  const size_t es = dtype == DISCO_BF16 ? 2 : 4;
  const size_t y_elems = (size_t)B * C_in * K * n_out;
  if (op == DISCO_OP_EINSUM_ADJOINT) {
    L.wt = 0;
    L.total = align256((size_t)C_out * (C_in / groups) * K * es);
  } else if (op == DISCO_OP_BWD_INPUT) {
    L.wt = 0;
    L.dy = align256((size_t)C_out * (C_in / groups) * K * es);
    L.total = L.dy + align256(y_elems * es);
  } else if (op == DISCO_OP_BWD_WEIGHT || op == DISCO_OP_BWD_WEIGHT_RECOMPUTE) {
    const int N = (int)n_out;
    L.tc = dtype == DISCO_BF16 && disco::dw_tc_supported(C_out / groups, (C_in / groups) * K, N);
    if (L.tc) {
      // one CTA per (split, batch, group), about one per SM of a B200 (148): the splits cover the
      // positions in multiples of the 64-element stage
      const int want = std::max(1, (148 + B * groups / 2) / (B * groups));
      L.nc = (int)((((long)N + want - 1) / want + 63) / 64 * 64);
    } else {
      L.nc = 4096;
    }
    L.nchunk = (N + L.nc - 1) / L.nc;
    const size_t nsplit = (size_t)B * L.nchunk;
    size_t off = 0;
    if (op == DISCO_OP_BWD_WEIGHT_RECOMPUTE) {
      L.ybuf = 0;
      off = align256(y_elems * es);
    }
    L.part = off;
    off += align256(nsplit * (size_t)C_out * (C_in / groups) * K * sizeof(float));
    L.bpart = off;
    off += align256(nsplit * (size_t)C_out * sizeof(float));
    L.total = off;
  }
  return L;
}

WsLayout layout(const disco_psi* psi, int op, int B, int C_in, int C_out, int groups, disco_dtype dtype) {
  return layout_kn(psi->g.K, (size_t)psi->g.nlat_out * psi->g.nlon_out, op, B, C_in, C_out, groups, dtype);
}

}  // namespace

namespace {

// Shape of the ring plan for a layer: blocks per tile, ring slots and their size, accumulator
// row buffers and B slots, chosen so that shared memory (x ring + B slots + two y staging
// blocks) and tensor memory (row buffers x blocks x 16K columns) fit.  K is the number of basis
// functions per term (1 for the adjoint).  False when the kernel has no such shape.
bool ring_params(int K, bool adjoint, disco::RingParams* p) {
  p->src_order = adjoint ? 1 : 0;
  p->target_strips = 24;
  p->max_rows = 64;
  // {nb, wmax, ns, nrb, bk, nbs, src_order, target strips, most rows per strip}
  if (adjoint && K == 1) {
    *p = disco::RingParams{4, 12, 8, 6, 4, 8, 1, 24, 64, {}};
    return true;
  }
  if (!adjoint && K == 3) {
    *p = disco::RingParams{4, 12, 6, 2, 4, 4, 0, 24, 64, {}};
    return true;
  }
  if (!adjoint && K == 5) {
    *p = disco::RingParams{4, 8, 5, 1, 4, 4, 0, 24, 64, {}};
    return true;
  }
  return false;
}

// Ring plans of the strip-staged kernel for a bf16 stride-1 layer: forward and adjoint, each
// with mirror rows (north-south mirror pairs share their Toeplitz blocks: mirror-symmetric
// latitude grids and an isotropic basis; checked entry by entry) and with plane pairs.  A plan
// that cannot be built is left out; the per-pair kernel serves that case.
void build_ring_plans(disco_psi* h) {
  const disco::Geometry& g = h->g;
  const int J = g.nlat_out, I = g.nlat_in, K = g.K;
  std::vector<disco::RingTerm> fwd, adj;
  fwd.reserve(h->entries.size());
  adj.reserve(h->entries.size());
  for (const disco::PsiEntry& e : h->entries) {
    fwd.push_back(disco::RingTerm{e.j, e.i, e.k, e.p, e.v});
    adj.push_back(disco::RingTerm{e.i, e.k * J + e.j, 0, -e.p, e.v});
  }
  std::vector<int> mo_f(J), ms_f(I), mo_a(I), ms_a((size_t)K * J), key_a((size_t)K * J);
  for (int j = 0; j < J; ++j) mo_f[j] = J - 1 - j;
  for (int i = 0; i < I; ++i) ms_f[i] = mo_a[i] = I - 1 - i;
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < J; ++j) {
      ms_a[(size_t)k * J + j] = k * J + (J - 1 - j);
      key_a[(size_t)k * J + j] = j * K + k;  // sources of one output row j adjacent, basis function inside
    }
  const std::vector<int> none;
  for (int which = 0; which < 4; ++which) {
    const bool adjoint = which >= 2, mirror = (which & 1) == 0;
    disco::RingParams prm;
    if (!ring_params(adjoint ? 1 : K, adjoint, &prm)) {
      h->ring_msg[which] = "the strip-staged kernel has no shape for this number of basis functions";
      continue;
    }
    if (adjoint) prm.src_key = key_a;
    std::string msg;
    h->ring_built[which] =
        adjoint ? disco::make_ring_plan(I, K * J, g.nlon_in, 1, adj, mirror ? mo_a : none, mirror ? ms_a : none, prm,
                                        h->ring[which], msg)
                : disco::make_ring_plan(J, I, g.nlon_in, K, fwd, mirror ? mo_f : none, mirror ? ms_f : none, prm,
                                        h->ring[which], msg);
    if (!h->ring_built[which]) {
      h->ring[which] = disco::RingPlan{};
      h->ring_msg[which] = msg;
    }
  }
}

// Shape of the tile-script plan: five ring slots of two chunks (160 KB), four B slots (1 KB of
// batch record and about 9 KB of Toeplitz K-steps each), the row
// buffers that tensor memory holds (512 columns / (4 blocks x 16K)), and the y staging of the
// epilogue (16 KB) within 227 KB of shared memory.
bool tile_params(int K, bool adjoint, int n_ctas, disco::TileParams* p) {
  if (!(K == 1 || K == 3 || K == 5)) return false;
  p->nb = 4;
  p->ns = 5;
  p->nrb = std::min(8, 512 / (4 * 16 * K));
  p->nbs = 4;
  const int kstep = 2 * 16 * K * 16;
  p->bslot_bytes = disco::kMetaBytes + (9216 / kstep) * kstep;  // the batch record, then the K-steps
  p->src_order = adjoint ? 1 : 0;
  p->target_strips = 24;
  p->max_rows = 64;
  p->n_ctas = n_ctas;
  return true;
}

// The fused variant keeps the mix weights (K x 8 KB) and the y staging of every kernel index
// (K x 16 KB) in shared memory and the mix accumulators (128 columns) in tensor memory: four ring
// slots, three B slots of 1 KB of record and four K-steps, and the row buffers that the
// remaining 384 columns hold.
bool tile_params_fused(int K, int n_ctas, disco::TileParams* p) {
  if (!(K == 1 || K == 3)) return false;
  p->nb = 4;
  p->ns = 4;  // the y staging of every kernel index (K x 16 KB) takes one slot's room
  p->nrb = std::min(8, 384 / (4 * 16 * K));
  p->nbs = 3;
  p->bslot_bytes = disco::kMetaBytes + 4 * (2 * 16 * K * 16);
  p->src_order = 0;
  p->target_strips = 24;
  p->max_rows = 64;
  p->n_ctas = n_ctas;
  return true;
}

void build_tile_plans(disco_psi* h, int n_ctas) {
  const disco::Geometry& g = h->g;
  const int J = g.nlat_out, I = g.nlat_in, K = g.K;
  std::vector<disco::RingTerm> fwd, adj;
  fwd.reserve(h->entries.size());
  adj.reserve(h->entries.size());
  for (const disco::PsiEntry& e : h->entries) {
    fwd.push_back(disco::RingTerm{e.j, e.i, e.k, e.p, e.v});
    adj.push_back(disco::RingTerm{e.i, e.k * J + e.j, 0, -e.p, e.v});
  }
  std::vector<int> mo_f(J), ms_f(I), mo_a(I), ms_a((size_t)K * J), key_a((size_t)K * J);
  for (int j = 0; j < J; ++j) mo_f[j] = J - 1 - j;
  for (int i = 0; i < I; ++i) ms_f[i] = mo_a[i] = I - 1 - i;
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < J; ++j) {
      ms_a[(size_t)k * J + j] = k * J + (J - 1 - j);
      key_a[(size_t)k * J + j] = j * K + k;
    }
  const std::vector<int> none;
  for (int which = 0; which < 4; ++which) {
    const bool adjoint = which >= 2, mirror = (which & 1) == 0;
    disco::TileParams prm;
    if (!tile_params(adjoint ? 1 : K, adjoint, n_ctas, &prm) || g.nlon_in < 64) {
      h->tile_msg[which] = "the TMA-staged strip kernel has no shape for this layer";
      continue;
    }
    if (adjoint) prm.src_key = key_a;
    std::string msg;
    h->tile_built[which] =
        adjoint ? disco::make_tile_plan(I, K * J, g.nlon_in, 1, adj, mirror ? mo_a : none, mirror ? ms_a : none, prm,
                                        h->tile[which], msg)
                : disco::make_tile_plan(J, I, g.nlon_in, K, fwd, mirror ? mo_f : none, mirror ? ms_f : none, prm,
                                        h->tile[which], msg);
    if (!h->tile_built[which]) {
      h->tile[which] = disco::TilePlan{};
      h->tile_msg[which] = msg;
    }
  }
  disco::TileParams pf;
  if (tile_params_fused(K, n_ctas, &pf) && g.nlon_in >= 64) {
    std::string msg;
    h->tile_fused_built = disco::make_tile_plan(J, I, g.nlon_in, K, fwd, mo_f, ms_f, pf, h->tile_fused, msg);
    if (!h->tile_fused_built) h->tile_fused = disco::TilePlan{};
    std::vector<disco::RingTerm> adjk;
    adjk.reserve(h->entries.size());
    for (const disco::PsiEntry& e : h->entries) adjk.push_back(disco::RingTerm{e.i, e.j, e.k, -e.p, e.v});
    h->tile_fused_adj_built =
        disco::make_tile_plan(I, J, g.nlon_in, K, std::move(adjk), mo_a, mo_f, pf, h->tile_fused_adj, msg);
    if (!h->tile_fused_adj_built) h->tile_fused_adj = disco::TilePlan{};
  }
}

// Tile-script plan for a call with BC planes (mirror rows up to 64 planes, plane pairs above);
// -1 when the layer has none.  DISCO_RING2=0 turns the kernel off, DISCO_RING2_ADJ=0 keeps the
// adjoint on the other kernels.
int tile_choice(const disco_psi* psi, int BC, bool adjoint) {
  const char* off = std::getenv("DISCO_RING2");
  if (off && off[0] == '0') return -1;
  if (adjoint) {
    const char* a = std::getenv("DISCO_RING2_ADJ");
    if (a && a[0] == '0') return -1;
  }
  const int base = adjoint ? 2 : 0;
  if (BC <= 64) return psi->dtile[base].ok ? base : -1;
  return psi->dtile[base + 1].ok ? base + 1 : -1;
}

disco::Ring2Launch tile_launch(const disco_psi* psi, int which, int BC, int n_src_rows, int n_out_rows) {
  const disco::TilePlan& P = psi->tile[which];
  const DevTile& d = psi->dtile[which];
  disco::Ring2Launch L{d.tiles, d.loads, d.copies, d.cmds, d.rows, d.cta_tiles, d.b, P.n_ctas, P.n_qt, P.K, P.nb,
                       P.ns, P.nrb, P.nbs, P.bslot_bytes, P.mirror, BC, n_src_rows, n_out_rows, psi->g.nlon_in};
  return L;
}

// Ring plan for a call with BC planes: mirror rows for at most 64 planes, plane pairs above 64;
// -1 when the layer has none (the per-pair kernel runs).  The adjoint plans are built for
// inspection only: on one B200 the strip-staged adjoint measured slower than the per-pair one
// (721x1440: 0.85 against 0.72 ms; 361x720 with 512 planes: 4.92 against 4.68 ms), so the
// device copies are not made and the adjoint keeps the per-pair kernel.
int ring_choice(const disco_psi* psi, int BC, bool adjoint) {
  if (adjoint) return -1;
  const int base = 0;
  if (BC <= 64) return psi->dring[base].ok ? base : -1;
  return psi->dring[base + 1].ok ? base + 1 : -1;
}

disco::RingLaunch ring_launch(const disco_psi* psi, int which, int BC, int n_src_rows, int n_out_rows) {
  const disco::RingPlan& P = psi->ring[which];
  const DevRing& d = psi->dring[which];
  disco::RingLaunch L{d.strips, d.loads, d.items, d.rows, d.b, d.n_strips, P.K, P.nb, P.wmax, P.ns, P.nrb,
                      P.bk, P.nbs, P.mirror, BC, n_src_rows, n_out_rows, psi->g.nlon_in};
  return L;
}

// Runs a banded gather as two launches so that the few bands with long staged rows do not set
// the shared-memory size (and so the occupancy) of all the others: heavy bands run on the
// plan's side stream, forked from and joined back to the caller's stream; light bands run on
// the caller's stream with a small staging area.
template <typename Launch>
disco_status run_banded(const disco_psi* psi, const disco::GatherPlan& P, disco::GatherArgs a, int nk,
                        cudaStream_t st, Launch launch, const char* what) {
  const int nb = (int)P.bands.size(), nh = P.n_heavy;
  if (nh > 0) {
    disco::GatherArgs h = a;
    h.band0 = 0;
    h.n_bands = nh;
    h.stage_budget = max_stage_bands(P, 0, nh, a.qb);
    if (disco::gather2_bytes(a.chunk_cache, nk, h.stage_budget) > kSmemLimit)
      return fail(DISCO_ERR_UNSUPPORTED, "a Psi row needs more staging than shared memory holds");
    cudaError_t e = cudaEventRecord(psi->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(psi->side, psi->fork, 0);
    if (e == cudaSuccess) e = launch(h, psi->side);
    if (e == cudaSuccess) e = cudaEventRecord(psi->join, psi->side);
    if (e != cudaSuccess) return cuda_fail(e, what);
  }
  if (nb > nh) {
    disco::GatherArgs l = a;
    l.band0 = nh;
    l.n_bands = nb - nh;
    // a staging area larger than the longest light row lets a CTA stage more channel
    // pairs per round, so fewer rounds (and barriers) per block of outputs
    l.stage_budget = std::max(kLightStage, max_stage_bands(P, nh, nb, a.qb));
    cudaError_t e = launch(l, st);
    if (e != cudaSuccess) return cuda_fail(e, what);
  }
  if (nh > 0) {
    cudaError_t e = cudaStreamWaitEvent(st, psi->join, 0);
    if (e != cudaSuccess) return cuda_fail(e, what);
  }
  return DISCO_OK;
}

// Forward contraction x -> y with the best gather form for the layer.
disco_status launch_contract_core(const disco_psi* psi, int BC, disco_dtype dtype, const void* x, void* y,
                             cudaStream_t st, const char* what) {
  const disco::Geometry& g = psi->g;
  if (dtype == DISCO_BF16 && psi->tz_ok && !(reinterpret_cast<uintptr_t>(x) & 15) &&
      !(reinterpret_cast<uintptr_t>(y) & 15)) {
    const int wt = tile_choice(psi, BC, false);
    if (wt >= 0) {
      // TMA-staged strip kernel over the tile scripts
      cudaError_t e = disco::launch_contract_ring2(tile_launch(psi, wt, BC, g.nlat_in, g.nlat_out), x, y, st);
      if (e != cudaSuccess) return cuda_fail(e, what);
      return DISCO_OK;
    }
    const int which = ring_choice(psi, BC, false);
    if (which >= 0) {
      // strip-staged kernel: each source row loaded once per tile for all the rows it reaches
      cudaError_t e = disco::launch_contract_ring(ring_launch(psi, which, BC, g.nlat_in, g.nlat_out), x, y, st);
      if (e != cudaSuccess) return cuda_fail(e, what);
      return DISCO_OK;
    }
    // Toeplitz blocks of Psi on tensor cores, one (output row, source row) pair at a time
    disco::TzLaunch L{psi->dtz.slabs, psi->dtz.row_begin, psi->dtz.slots, psi->dtz.b, psi->tz.K, psi->tz.parts,
                      psi->tz.N, BC, g.nlat_in, g.nlat_out, g.nlon_in};
    cudaError_t e = disco::launch_contract_tc(L, x, y, st);
    if (e != cudaSuccess) return cuda_fail(e, what);
    return DISCO_OK;
  }
  int qb, nblk;
  block_shape(g.nlon_out, 128, &qb, &nblk);
  const int need = max_stage(psi->fwd, qb);
  if (g.K == 3) {
    // banded paired gather: a band's chunks are cached together
    const bool bf16 = dtype == DISCO_BF16;
    disco::GatherArgs a = gather_args(psi->dfwdb, BC, qb, nblk, g.nlon_in, g.nlat_in, g.nlon_out, g.nlat_out, 0, 64,
                                      bf16);
    return run_banded(psi, psi->fwdb, a, g.K, st,
                      [&](const disco::GatherArgs& la, cudaStream_t ls) {
                        return disco::launch_fwd_gather2_band(bf16, g.K, g.stride, la, x, y, ls);
                      },
                      what);
  }
  const int budget = std::max(kStageFloats, need);
  if (gather_bytes(chunk_cache(psi->fwd), g.K, budget) > kSmemLimit)
    return fail(DISCO_ERR_UNSUPPORTED, "a Psi row needs more staging than shared memory holds");
  disco::GatherArgs a = gather_args(psi->dfwd, BC, qb, nblk, g.nlon_in, g.nlat_in, g.nlon_out, g.nlat_out, budget,
                                    chunk_cache(psi->fwd), dtype == DISCO_BF16);
  cudaError_t e = disco::launch_fwd_gather(dtype == DISCO_BF16, g.K, g.stride, a, x, y, st);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return DISCO_OK;
}

// dy = w^T dout (the transposed weight einsum): w transposed into `wt`, then the channel mix.
// dy = W^T dout on N points per plane (the transposed weight einsum)
disco_status launch_dy_kn(int K, int N, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                          const void* dout, const void* w, void* wt, void* dy, cudaStream_t st) {
  const bool bf16 = dtype == DISCO_BF16;
  const int Cg = C_in / groups, Og = C_out / groups;
  cudaError_t e = disco::launch_transpose_weight(bf16, w, wt, groups, Og, Cg, K, st);
  if (e != cudaSuccess) return cuda_fail(e, "weight transpose launch");
  disco::MixArgs m{dout, wt, nullptr, dy, B, groups, Cg * K, Og, N};
  e = launch_mix(bf16, m, st);
  if (e != cudaSuccess) return cuda_fail(e, "transposed einsum launch");
  return DISCO_OK;
}

disco_status launch_dy(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                       const void* dout, const void* w, void* wt, void* dy, cudaStream_t st) {
  const disco::Geometry& g = psi->g;
  return launch_dy_kn(g.K, g.nlat_out * g.nlon_out, B, C_in, C_out, groups, dtype, dout, w, wt, dy, st);
}

// dw (and dbias when non-NULL) from dout and y on N points per plane, with the split-K partial
// sums in the scratch that L describes
disco_status launch_dw_kn(int K, int N, const WsLayout& L, int B, int C_in, int C_out, int groups,
                          disco_dtype dtype, const void* dout, const void* y, char* ws, void* dw, void* dbias,
                          cudaStream_t st) {
  const bool bf16 = dtype == DISCO_BF16;
  const int Og = C_out / groups, Rg = (C_in / groups) * K;
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* bpart = dbias ? reinterpret_cast<float*>(ws + L.bpart) : nullptr;
  disco::DwArgs d{dout, y, part, bpart, B, groups, Og, Rg, N, L.nc, L.nchunk};
  cudaError_t e = L.tc ? disco::launch_dw_tc(d, st) : disco::launch_dw_partial_simt(bf16, d, st);
  if (e != cudaSuccess) return cuda_fail(e, "weight-gradient launch");
  e = disco::launch_dw_reduce(bf16, part, bpart, dw, dbias, B * L.nchunk, groups, Og, Rg, st);
  if (e != cudaSuccess) return cuda_fail(e, "weight-gradient reduce launch");
  return DISCO_OK;
}

// dx from dy: the adjoint contraction with the best kernel for the layer.
disco_status launch_adjoint_core(const disco_psi* psi, int BC, disco_dtype dtype, const void* dy, void* dx,
                            cudaStream_t st) {
  const disco::Geometry& g = psi->g;
  const bool bf16 = dtype == DISCO_BF16;
  if (bf16 && psi->tz_ok && !(reinterpret_cast<uintptr_t>(dx) & 15) && !(reinterpret_cast<uintptr_t>(dy) & 15)) {
    const int wt = tile_choice(psi, BC, true);
    if (wt >= 0) {
      cudaError_t e =
          disco::launch_contract_ring2(tile_launch(psi, wt, BC, g.K * g.nlat_out, g.nlat_in), dy, dx, st);
      if (e != cudaSuccess) return cuda_fail(e, "adjoint contraction launch");
      return DISCO_OK;
    }
    const int which = ring_choice(psi, BC, true);
    if (which >= 0) {
      cudaError_t e =
          disco::launch_contract_ring(ring_launch(psi, which, BC, g.K * g.nlat_out, g.nlat_in), dy, dx, st);
      if (e != cudaSuccess) return cuda_fail(e, "adjoint contraction launch");
      return DISCO_OK;
    }
    // Toeplitz blocks of the reversed Psi on tensor cores: dy rows (k, j) are the source rows
    const disco::ToeplitzPlan& P = psi->tza;
    disco::TzLaunch T{psi->dtza.slabs, psi->dtza.row_begin, psi->dtza.slots, psi->dtza.b, P.K, P.parts, P.N,
                      BC, g.K * g.nlat_out, g.nlat_in, g.nlon_in};
    cudaError_t e = disco::launch_contract_tc(T, dy, dx, st);
    if (e != cudaSuccess) return cuda_fail(e, "adjoint contraction launch");
    return DISCO_OK;
  }
  int qb, nblk;
  block_shape(g.nlon_out, 128, &qb, &nblk);
  if (g.K == 3) {
    // paired, banded adjoint gather (few basis functions: the staged dy rows of a band
    // fit with room for several channel pairs)
    disco::GatherArgs a = gather_args(psi->dadjb, BC, qb, nblk, g.nlon_out, g.K * g.nlat_out, g.nlon_in,
                                      g.nlat_in, 0, 96, bf16);
    return run_banded(psi, psi->adjb, a, 1, st,
                      [&](const disco::GatherArgs& la, cudaStream_t ls) {
                        return disco::launch_adj_gather2_band(bf16, g.stride, la, dy, dx, ls);
                      },
                      "adjoint contraction launch");
  }
  const int need = max_stage(psi->adj, qb);
  const int budget = std::max(kStageFloats, need);
  if (gather_bytes(chunk_cache(psi->adj), 1, budget) > kSmemLimit)
    return fail(DISCO_ERR_UNSUPPORTED, "a Psi column needs more staging than shared memory holds");
  disco::GatherArgs a = gather_args(psi->dadj, BC, qb, nblk, g.nlon_out, g.K * g.nlat_out, g.nlon_in, g.nlat_in,
                                    budget, chunk_cache(psi->adj), bf16);
  cudaError_t e = disco::launch_adj_gather(bf16, g.stride, a, dy, dx, st);
  if (e != cudaSuccess) return cuda_fail(e, "adjoint contraction launch");
  return DISCO_OK;
}

// The contractions with the rows that have no entries (handles of a band of input latitudes)
// set to zero afterwards, whatever kernel ran.
disco_status launch_contract(const disco_psi* psi, int BC, disco_dtype dtype, const void* x, void* y,
                             cudaStream_t st, const char* what) {
  disco_status s = launch_contract_core(psi, BC, dtype, x, y, st, what);
  if (s || psi->empty_out.empty()) return s;
  const disco::Geometry& g = psi->g;
  cudaError_t e = disco::launch_zero_rows(y, dtype == DISCO_BF16 ? 2 : 4, psi->d_empty_out, (int)psi->empty_out.size(),
                                          BC * g.K, g.nlat_out, g.nlon_out, st);
  return e == cudaSuccess ? DISCO_OK : cuda_fail(e, what);
}

disco_status launch_adjoint(const disco_psi* psi, int BC, disco_dtype dtype, const void* dy, void* dx,
                            cudaStream_t st) {
  disco_status s = launch_adjoint_core(psi, BC, dtype, dy, dx, st);
  if (s || psi->empty_in.empty()) return s;
  const disco::Geometry& g = psi->g;
  cudaError_t e = disco::launch_zero_rows(dx, dtype == DISCO_BF16 ? 2 : 4, psi->d_empty_in, (int)psi->empty_in.size(),
                                          BC, g.nlat_in, g.nlon_in, st);
  return e == cudaSuccess ? DISCO_OK : cuda_fail(e, "adjoint contraction");
}

}  // namespace

extern "C" {


const char* disco_last_error(void) { return g_last_error.c_str(); }

unsigned long long disco_launch_count(void) { return disco::g_launches.load(); }

disco_status disco_wait_selftest(unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return fail(DISCO_ERR_INVALID_ARG, "limit_us must be in [1, 1000000]");
  const cudaError_t e = disco::launch_wait_selftest(limit_us, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
  return DISCO_OK;
}

disco_status disco_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronisation");
  if (disco::take_mix_tc_status() | disco::take_fused_tc_status() | disco::take_contract_tc_status() |
      disco::take_contract_ring_status() | disco::take_contract_ring2_status())
    return fail(DISCO_ERR_TIMEOUT, "a bounded device-side wait expired");
  return DISCO_OK;
}

namespace {

// Psi of the output rows [j_begin, j_end) (j_end < 0: all rows).  A band (not all rows) is
// re-indexed to a layer of its own: output rows j - j_begin, input rows i - i_begin over the
// input rows [i_begin, i_end) that its entries reach.
disco_status psi_build_rows(const disco_spec_t* spec, int j_begin, int j_end, int device, disco_psi** out,
                            int* i_begin, int* i_end, int in_begin = -1, int in_end = -1) {
  if (!out) return fail(DISCO_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!spec) return fail(DISCO_ERR_INVALID_ARG, "spec is NULL");
  if (spec->grid_in < DISCO_GRID_EQUIANGULAR || spec->grid_in > DISCO_GRID_EQUIANGULAR_TRAPEZOIDAL ||
      spec->grid_out < DISCO_GRID_EQUIANGULAR || spec->grid_out > DISCO_GRID_EQUIANGULAR_TRAPEZOIDAL)
    return fail(DISCO_ERR_UNSUPPORTED, "unknown latitude grid");
  if (spec->basis_type != DISCO_BASIS_PIECEWISE_LINEAR)
    return fail(DISCO_ERR_UNSUPPORTED, "only the piecewise-linear basis is supported");
  if (spec->basis_norm_mode != DISCO_NORM_NODAL)
    return fail(DISCO_ERR_UNSUPPORTED, "only nodal basis normalisation is supported");
  if (spec->nlat_in < 2 || spec->nlat_out < 2 || spec->nlon_in < 1 || spec->nlon_out < 1)
    return fail(DISCO_ERR_INVALID_ARG, "grids need nlat >= 2 and nlon >= 1");
  if (!(spec->theta_cutoff > 0.0)) return fail(DISCO_ERR_INVALID_ARG, "theta_cutoff must be > 0");
  if (spec->kernel_shape[0] < 2 || spec->kernel_shape[1] < 1)
    return fail(DISCO_ERR_INVALID_ARG, "kernel_shape needs n_r >= 2 and n_alpha >= 1");
  if (spec->nlon_in % spec->nlon_out)
    return fail(DISCO_ERR_UNSUPPORTED, "nlon_in must be a multiple of nlon_out (p-shift symmetry)");
  disco::Geometry g;
  g.nlat_in = spec->nlat_in;
  g.nlon_in = spec->nlon_in;
  g.nlat_out = spec->nlat_out;
  g.nlon_out = spec->nlon_out;
  g.n_r = spec->kernel_shape[0];
  g.n_alpha = spec->kernel_shape[1];
  g.theta_cutoff = spec->theta_cutoff;
  g.K = g.n_alpha == 1 ? g.n_r : 1 + (g.n_r - 1) * g.n_alpha;
  g.stride = g.nlon_in / g.nlon_out;
  g.grid_in = spec->grid_in;
  g.grid_out = spec->grid_out;
  if (g.K > disco::kMaxK) return fail(DISCO_ERR_UNSUPPORTED, "more basis functions than the kernels support");
  if (g.stride > disco::kMaxStride) return fail(DISCO_ERR_UNSUPPORTED, "nlon_in / nlon_out above 4");
  disco_psi* h = new (std::nothrow) disco_psi;
  if (!h) return fail(DISCO_ERR_ALLOC, "host allocation failed");
  std::string msg;
  const int st = disco::build_psi_entries(g, h->entries, msg, j_begin, j_end);
  if (st) {
    delete h;
    return fail(static_cast<disco_status>(st), msg);
  }
  if (j_end < 0) j_end = g.nlat_out;
  int ib = 0, ie = g.nlat_in;
  if (in_begin >= 0) {
    // a band of input latitudes: its entries of every output row, input rows re-indexed
    std::vector<disco::PsiEntry> keep;
    keep.reserve(h->entries.size());
    for (const disco::PsiEntry& en : h->entries)
      if (en.i >= in_begin && en.i < in_end) {
        disco::PsiEntry e2 = en;
        e2.i -= in_begin;
        keep.push_back(e2);
      }
    h->entries.swap(keep);
    g.nlat_in = in_end - in_begin;
    ib = in_begin;
    ie = in_end;
    std::vector<char> has_out(g.nlat_out, 0), has_in(g.nlat_in, 0);
    for (const disco::PsiEntry& en : h->entries) {
      has_out[en.j] = 1;
      has_in[en.i] = 1;
    }
    for (int j = 0; j < g.nlat_out; ++j)
      if (!has_out[j]) h->empty_out.push_back(j);
    for (int i = 0; i < g.nlat_in; ++i)
      if (!has_in[i]) h->empty_in.push_back(i);
  } else if (j_begin != 0 || j_end != g.nlat_out) {
    ib = g.nlat_in;
    ie = 0;
    for (const disco::PsiEntry& en : h->entries) {
      ib = std::min(ib, en.i);
      ie = std::max(ie, en.i + 1);
    }
    for (disco::PsiEntry& en : h->entries) {
      en.j -= j_begin;
      en.i -= ib;
    }
    g.nlat_out = j_end - j_begin;
    g.nlat_in = ie - ib;
  }
  if (i_begin) *i_begin = ib;
  if (i_end) *i_end = ie;
  h->g = g;
  h->fwd = disco::make_forward_plan(g, h->entries);
  h->adj = disco::make_adjoint_plan(g, h->entries);
  h->fwdb = disco::make_band_plan(g.nlat_out, h->fwd, 4, 24);
  h->adjb = disco::make_band_plan(g.nlat_in, h->adj, 4, 48);
  disco::split_bands(h->fwdb, 128, kLightStage);
  disco::split_bands(h->adjb, 128, kLightStage);
  if (h->fwd.max_src > disco::kMaxSrc || h->adj.max_src > disco::kMaxSrc || h->fwd.max_ring > disco::kMaxRing ||
      h->adj.max_ring > disco::kMaxRing || h->fwdb.max_src > disco::kMaxSrc || h->adjb.max_src > disco::kMaxSrc) {
    delete h;
    return fail(DISCO_ERR_UNSUPPORTED, "an output row reaches more source rows than the kernels support");
  }
  h->device = device;
  if (device < 0 && disco::toeplitz_geometry(g.K, g.stride, g.nlon_in, g.nlon_out)) {
    // host-only handle: the Toeplitz plans are built for inspection (disco_toeplitz_export)
    h->tz = disco::make_toeplitz_plan(g, h->entries);
    h->tza = disco::make_adjoint_toeplitz_plan(g, h->entries);
    build_ring_plans(h);
    build_tile_plans(h, 148);
  }
  if (device >= 0) {
    int prev = -1;
    cudaGetDevice(&prev);
    cudaError_t e = cudaSetDevice(device);
    if (e == cudaSuccess) e = upload_plan(h->fwd, &h->dfwd);
    if (e == cudaSuccess) e = upload_plan(h->adj, &h->dadj);
    if (e == cudaSuccess) e = upload_plan(h->fwdb, &h->dfwdb);
    if (e == cudaSuccess) e = upload_plan(h->adjb, &h->dadjb);
    if (e == cudaSuccess && !h->empty_out.empty()) e = upload(h->empty_out, &h->d_empty_out);
    if (e == cudaSuccess && !h->empty_in.empty()) e = upload(h->empty_in, &h->d_empty_in);
    // tensor-core contraction for bf16 signals (DISCO_SIMT_CONTRACT=1 keeps the gather kernels)
    const char* simt = std::getenv("DISCO_SIMT_CONTRACT");
    if (e == cudaSuccess && !(simt && simt[0] == '1') &&
        disco::contract_tc_supported(g.K, g.stride, g.nlon_in, g.nlon_out)) {
      h->tz = disco::make_toeplitz_plan(g, h->entries);
      h->tza = disco::make_adjoint_toeplitz_plan(g, h->entries);
      e = upload_tz(h->tz, &h->dtz);
      if (e == cudaSuccess) e = upload_tz(h->tza, &h->dtza);
      h->tz_ok = e == cudaSuccess;
      // strip-staged kernel (DISCO_RING=0 keeps the per-pair kernels)
      const char* rg = std::getenv("DISCO_RING");
      if (e == cudaSuccess && !(rg && rg[0] == '0')) {
        build_ring_plans(h);
        for (int w = 0; w < 2 && e == cudaSuccess; ++w)
          if (h->ring_built[w] && disco::ring_kernel_k(h->ring[w].K)) e = upload_ring(h->ring[w], &h->dring[w]);
        int sms = 148;
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
        if (e == cudaSuccess) build_tile_plans(h, sms);
        for (int w = 0; w < 4 && e == cudaSuccess; ++w)
          if (h->tile_built[w] && disco::ring2_kernel_k(h->tile[w].K)) e = upload_tile(h->tile[w], &h->dtile[w]);
        if (e == cudaSuccess && h->tile_fused_built) e = upload_tile(h->tile_fused, &h->dtile_fused);
        if (e == cudaSuccess && h->tile_fused_adj_built) e = upload_tile(h->tile_fused_adj, &h->dtile_fused_adj);
      }
    }
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->join, cudaEventDisableTiming);
    if (prev >= 0) cudaSetDevice(prev);
    if (e != cudaSuccess) {
      free_plan(&h->dfwd);
      free_plan(&h->dadj);
      free_plan(&h->dfwdb);
      free_plan(&h->dadjb);
      free_tz(&h->dtz);
      free_tz(&h->dtza);
      for (int w = 0; w < 4; ++w) free_ring(&h->dring[w]);
      for (int w = 0; w < 4; ++w) free_tile(&h->dtile[w]);
      free_tile(&h->dtile_fused);
      free_tile(&h->dtile_fused_adj);
      cudaFree(h->d_empty_out);
      cudaFree(h->d_empty_in);
      delete h;
      return fail(DISCO_ERR_ALLOC, std::string("Psi upload failed: ") + cudaGetErrorString(e));
    }
  }
  *out = h;
  return DISCO_OK;
}

}  // namespace

disco_status disco_psi_build(const disco_spec_t* spec, int device, disco_psi** out) {
  return psi_build_rows(spec, 0, -1, device, out, nullptr, nullptr);
}

disco_status disco_psi_build_band(const disco_spec_t* spec, int j_begin, int j_end, int device, disco_psi** out,
                                  int* i_begin, int* i_end) {
  if (!spec) return fail(DISCO_ERR_INVALID_ARG, "spec is NULL");
  if (!i_begin || !i_end) return fail(DISCO_ERR_INVALID_ARG, "i_begin / i_end is NULL");
  if (j_begin < 0 || j_end <= j_begin || j_end > spec->nlat_out)
    return fail(DISCO_ERR_INVALID_ARG, "need 0 <= j_begin < j_end <= nlat_out");
  return psi_build_rows(spec, j_begin, j_end, device, out, i_begin, i_end);
}

disco_status disco_psi_build_inputs(const disco_spec_t* spec, int i_begin, int i_end, int device, disco_psi** out) {
  if (!spec) return fail(DISCO_ERR_INVALID_ARG, "spec is NULL");
  if (i_begin < 0 || i_end <= i_begin || i_end > spec->nlat_in)
    return fail(DISCO_ERR_INVALID_ARG, "need 0 <= i_begin < i_end <= nlat_in");
  return psi_build_rows(spec, 0, -1, device, out, nullptr, nullptr, i_begin, i_end);
}

disco_status disco_psi_destroy(disco_psi* psi) {
  if (!psi) return DISCO_OK;
  if (psi->device >= 0) {
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(psi->device);
    cudaDeviceSynchronize();
    free_plan(&psi->dfwd);
    free_plan(&psi->dadj);
    free_plan(&psi->dfwdb);
    free_plan(&psi->dadjb);
    free_tz(&psi->dtz);
    free_tz(&psi->dtza);
    for (int w = 0; w < 4; ++w) free_ring(&psi->dring[w]);
    for (int w = 0; w < 4; ++w) free_tile(&psi->dtile[w]);
    free_tile(&psi->dtile_fused);
    free_tile(&psi->dtile_fused_adj);
    cudaFree(psi->d_empty_out);
    cudaFree(psi->d_empty_in);
    if (psi->side) cudaStreamDestroy(psi->side);
    if (psi->fork) cudaEventDestroy(psi->fork);
    if (psi->join) cudaEventDestroy(psi->join);
    if (prev >= 0) cudaSetDevice(prev);
  }
  delete psi;
  return DISCO_OK;
}

disco_status disco_psi_info(const disco_psi* psi, int* K, long long* nnz) {
  if (!psi) return fail(DISCO_ERR_INVALID_ARG, "psi is NULL");
  if (K) *K = psi->g.K;
  if (nnz) *nnz = (long long)psi->entries.size();
  return DISCO_OK;
}

disco_status disco_psi_export(const disco_psi* psi, int* k, int* j, int* i, int* p, double* val) {
  if (!psi || !k || !j || !i || !p || !val) return fail(DISCO_ERR_INVALID_ARG, "NULL argument");
  for (size_t t = 0; t < psi->entries.size(); ++t) {
    const disco::PsiEntry& e = psi->entries[t];
    k[t] = e.k;
    j[t] = e.j;
    i[t] = e.i;
    p[t] = e.p;
    val[t] = e.v;
  }
  return DISCO_OK;
}

disco_status disco_plan_info(const disco_psi* psi, int which, int* dims) {
  if (!psi || !dims || which < 0 || which > 3) return fail(DISCO_ERR_INVALID_ARG, "bad plan query");
  const disco::GatherPlan& P = which == 0 ? psi->fwd : which == 1 ? psi->adj : which == 2 ? psi->fwdb : psi->adjb;
  dims[0] = (int)P.rows.size();
  dims[1] = (int)P.src.size();
  dims[2] = (int)P.chunks.size();
  dims[3] = (int)P.vals.size();
  dims[4] = P.nk;
  dims[5] = P.step;
  dims[6] = P.residues;
  dims[7] = (int)(sizeof(disco::RowPlan) / sizeof(int));
  dims[8] = (int)P.rings.size();
  return DISCO_OK;
}

disco_status disco_plan_export(const disco_psi* psi, int which, int* rows, int* srcs, int* chunks, float* vals,
                               int* rings) {
  if (!psi || !rows || !srcs || !chunks || !vals || !rings || which < 0 || which > 3)
    return fail(DISCO_ERR_INVALID_ARG, "bad plan export");
  const disco::GatherPlan& P = which == 0 ? psi->fwd : which == 1 ? psi->adj : which == 2 ? psi->fwdb : psi->adjb;
  std::memcpy(rings, P.rings.data(), P.rings.size() * sizeof(disco::Ring));
  std::memcpy(rows, P.rows.data(), P.rows.size() * sizeof(disco::RowPlan));
  std::memcpy(srcs, P.src.data(), P.src.size() * sizeof(disco::SrcRow));
  std::memcpy(chunks, P.chunks.data(), P.chunks.size() * sizeof(disco::Chunk));
  std::memcpy(vals, P.vals.data(), P.vals.size() * sizeof(float));
  return DISCO_OK;
}

disco_status disco_toeplitz_info(const disco_psi* psi, int which, int* dims) {
  if (!psi || !dims || which < 0 || which > 1) return fail(DISCO_ERR_INVALID_ARG, "bad Toeplitz plan query");
  const disco::ToeplitzPlan& P = which == 0 ? psi->tz : psi->tza;
  if (P.slots.empty()) return fail(DISCO_ERR_UNSUPPORTED, "no Toeplitz plan for this layer");
  dims[0] = P.K;
  dims[1] = P.parts;
  dims[2] = P.N;
  dims[3] = (int)P.slabs.size();
  dims[4] = (int)(P.slots.size() / 4);
  dims[5] = (int)P.b.size();
  dims[6] = disco::kTzSlabK;
  dims[7] = (int)P.ksteps;
  return DISCO_OK;
}

disco_status disco_toeplitz_export(const disco_psi* psi, int which, int* slabs, int* slots, unsigned short* b) {
  if (!psi || !slabs || !slots || !b || which < 0 || which > 1)
    return fail(DISCO_ERR_INVALID_ARG, "bad Toeplitz plan export");
  const disco::ToeplitzPlan& P = which == 0 ? psi->tz : psi->tza;
  if (P.slots.empty()) return fail(DISCO_ERR_UNSUPPORTED, "no Toeplitz plan for this layer");
  std::memcpy(slabs, P.slabs.data(), P.slabs.size() * sizeof(disco::TzSlab));
  std::memcpy(slots, P.slots.data(), P.slots.size() * sizeof(int));
  std::memcpy(b, P.b.data(), P.b.size() * sizeof(uint16_t));
  return DISCO_OK;
}

disco_status disco_ring_info(const disco_psi* psi, int which, int* dims) {
  if (!psi || !dims || which < 0 || which > 3) return fail(DISCO_ERR_INVALID_ARG, "bad ring plan query");
  if (!psi->ring_built[which])
    return fail(DISCO_ERR_UNSUPPORTED, "no ring plan of this kind for this layer: " + psi->ring_msg[which]);
  const disco::RingPlan& P = psi->ring[which];
  const int v[16] = {P.K, P.N, P.mirror, P.nb, P.wmax, P.ns, P.nrb, P.bk, P.nbs, P.src_order,
                     (int)(P.strips.size() / 8), (int)(P.loads.size() / 2), (int)(P.items.size() / 4),
                     (int)(P.rows.size() / 2), (int)P.b.size(), (int)std::min<long long>(P.mmas, INT32_MAX)};
  std::memcpy(dims, v, sizeof(v));
  return DISCO_OK;
}

disco_status disco_tile_info(const disco_psi* psi, int which, int* dims) {
  if (!psi || !dims || which < 0 || which > 3) return fail(DISCO_ERR_INVALID_ARG, "bad tile plan query");
  if (!psi->tile_built[which])
    return fail(DISCO_ERR_UNSUPPORTED, "no tile plan of this kind for this layer: " + psi->tile_msg[which]);
  const disco::TilePlan& P = psi->tile[which];
  auto c = [](long long v) { return (int)std::min<long long>(v, INT32_MAX); };
  const int v[20] = {P.K, P.N, P.mirror, P.nb, P.ns, P.nrb, P.nbs, P.bslot_bytes, P.src_order, P.n_strips, P.n_qt,
                     P.n_ctas, c((long long)P.loads.size() / 4), c((long long)P.copies.size() / 4), c((long long)P.cmds.size()),
                     c((long long)P.rows.size() / 2), c((long long)P.b.size()), c(P.mmas), c(P.boxes),
                     c((long long)P.cta_tiles.size())};
  std::memcpy(dims, v, sizeof(v));
  return DISCO_OK;
}
disco_status disco_tile_export(const disco_psi* psi, int which, int* tiles, int* loads, int* copies, unsigned int* cmds,
                               int* rows, int* cta_tiles, unsigned short* b) {
  if (!psi || !tiles || !loads || !copies || !cmds || !rows || !cta_tiles || !b || which < 0 || which > 3)
    return fail(DISCO_ERR_INVALID_ARG, "bad tile plan export");
  if (!psi->tile_built[which]) return fail(DISCO_ERR_UNSUPPORTED, "no tile plan of this kind for this layer");
  const disco::TilePlan& P = psi->tile[which];
  std::memcpy(tiles, P.tiles.data(), P.tiles.size() * sizeof(int));
  std::memcpy(loads, P.loads.data(), P.loads.size() * sizeof(int));
  std::memcpy(copies, P.copies.data(), P.copies.size() * sizeof(int));
  std::memcpy(cmds, P.cmds.data(), P.cmds.size() * sizeof(uint32_t));
  std::memcpy(rows, P.rows.data(), P.rows.size() * sizeof(int));
  std::memcpy(cta_tiles, P.cta_tiles.data(), P.cta_tiles.size() * sizeof(int));
  std::memcpy(b, P.b.data(), P.b.size() * sizeof(uint16_t));
  return DISCO_OK;
}
disco_status disco_ring_export(const disco_psi* psi, int which, int* strips, int* loads, int* items, int* rows,
                               unsigned short* b) {
  if (!psi || !strips || !loads || !items || !rows || !b || which < 0 || which > 3)
    return fail(DISCO_ERR_INVALID_ARG, "bad ring plan export");
  if (!psi->ring_built[which]) return fail(DISCO_ERR_UNSUPPORTED, "no ring plan of this kind for this layer");
  const disco::RingPlan& P = psi->ring[which];
  std::memcpy(strips, P.strips.data(), P.strips.size() * sizeof(int));
  std::memcpy(loads, P.loads.data(), P.loads.size() * sizeof(int));
  std::memcpy(items, P.items.data(), P.items.size() * sizeof(int));
  std::memcpy(rows, P.rows.data(), P.rows.size() * sizeof(int));
  std::memcpy(b, P.b.data(), P.b.size() * sizeof(uint16_t));
  return DISCO_OK;
}

disco_status disco_workspace_size(const disco_psi* psi, int op, int B, int C_in, int C_out, int groups,
                                  disco_dtype dtype, size_t* bytes) {
  if (!psi || !bytes) return fail(DISCO_ERR_INVALID_ARG, "NULL argument");
  if (B <= 0 || C_in <= 0 || C_out <= 0 || groups <= 0 || C_in % groups || C_out % groups)
    return fail(DISCO_ERR_INVALID_ARG, "bad sizes");
  if (op < DISCO_OP_FWD || op > DISCO_OP_EINSUM_ADJOINT) return fail(DISCO_ERR_INVALID_ARG, "unknown op");
  *bytes = layout(psi, op, B, C_in, C_out, groups, dtype).total;
  return DISCO_OK;
}


disco_status disco_contract(const disco_psi* psi, int B, int C, disco_dtype dtype, const void* x, void* y,
                            void* stream) {
  disco_status s = check_common(psi, B, C, C, 1, dtype);
  if (s) return s;
  if (!x || !y) return fail(DISCO_ERR_INVALID_ARG, "x and y must be non-NULL");
  if (!disco::gather_supports(psi->g.K, psi->g.stride)) return fail(DISCO_ERR_UNSUPPORTED, "K or stride not compiled");
  return launch_contract(psi, B * C, dtype, x, y, static_cast<cudaStream_t>(stream), "contraction launch");
}

disco_status disco_einsum(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                          const void* y, const void* w, const void* bias, void* out, void* stream) {
  disco_status s = check_common(psi, B, C_in, C_out, groups, dtype);
  if (s) return s;
  if (!y || !w || !out) return fail(DISCO_ERR_INVALID_ARG, "y, w and out must be non-NULL");
  const disco::Geometry& g = psi->g;
  disco::MixArgs m{y, w, bias, out, B, groups, C_out / groups, (C_in / groups) * g.K, g.nlat_out * g.nlon_out};
  cudaError_t e = launch_mix(dtype == DISCO_BF16, m, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "einsum launch");
  return DISCO_OK;
}

disco_status disco_fwd(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                       const void* x, const void* w, const void* bias, void* y, void* out, void* workspace,
                       size_t ws_bytes, void* stream) {
  (void)workspace;
  (void)ws_bytes;
  disco_status s = check_common(psi, B, C_in, C_out, groups, dtype);
  if (s) return s;
  if (!x || !w || !y || !out) return fail(DISCO_ERR_INVALID_ARG, "x, w, y and out must be non-NULL");
  s = disco_contract(psi, B, C_in, dtype, x, y, stream);
  if (s) return s;
  return disco_einsum(psi, B, C_in, C_out, groups, dtype, y, w, bias, out, stream);
}

static disco_status fwd_fused_core(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                                   const void* x, const void* w, const void* bias, void* out, cudaStream_t st);

disco_status disco_fwd_fused(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                             const void* x, const void* w, const void* bias, void* out, void* workspace,
                             size_t ws_bytes, void* stream) {
  (void)workspace;
  (void)ws_bytes;
  disco_status s = check_common(psi, B, C_in, C_out, groups, dtype);
  if (s) return s;
  if (!x || !w || !out) return fail(DISCO_ERR_INVALID_ARG, "x, w and out must be non-NULL");
  const disco::Geometry& g = psi->g;
  if (!disco::gather_supports(g.K, g.stride)) return fail(DISCO_ERR_UNSUPPORTED, "K or stride not compiled");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = fwd_fused_core(psi, B, C_in, C_out, groups, dtype, x, w, bias, out, st);
  if (s || psi->empty_out.empty()) return s;
  // output rows without entries (a band of input latitudes): out = bias there, whatever the
  // kernel left in them
  cudaError_t e = disco::launch_fill_rows(dtype == DISCO_BF16, out, psi->d_empty_out, (int)psi->empty_out.size(),
                                          B * C_out, g.nlat_out, g.nlon_out, bias, C_out, st);
  return e == cudaSuccess ? DISCO_OK : cuda_fail(e, "fused forward row fill");
}

static disco_status fwd_fused_core(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                                   const void* x, const void* w, const void* bias, void* out, cudaStream_t st) {
  const disco::Geometry& g = psi->g;
  const bool bf16 = dtype == DISCO_BF16;
  const int Cg = C_in / groups;
  const char* rf = std::getenv("DISCO_RING2_FUSED");
  const char* r2 = std::getenv("DISCO_RING2");
  if (bf16 && psi->dtile_fused.ok && !(rf && rf[0] == '0') && !(r2 && r2[0] == '0') && C_in == 64 && groups == 1 &&
      C_out <= 64 && !(reinterpret_cast<uintptr_t>(x) & 15) && !(reinterpret_cast<uintptr_t>(out) & 15) &&
      !(reinterpret_cast<uintptr_t>(w) & 1) && !(reinterpret_cast<uintptr_t>(bias) & 1)) {
    // TMA-staged strip contraction with the channel mix on tensor cores in its epilogue
    const disco::TilePlan& P = psi->tile_fused;
    const DevTile& d = psi->dtile_fused;
    disco::Ring2Launch L{d.tiles, d.loads, d.copies, d.cmds, d.rows, d.cta_tiles, d.b, P.n_ctas, P.n_qt, P.K, P.nb,
                         P.ns, P.nrb, P.nbs, P.bslot_bytes, P.mirror, B * C_in, g.nlat_in, g.nlat_out, g.nlon_in};
    disco::Ring2Fused F{x, w, bias, out, C_in, C_out};
    cudaError_t e = disco::launch_fused_ring2(L, F, st);
    if (e != cudaSuccess) return cuda_fail(e, "fused strip-contraction launch");
    return DISCO_OK;
  }
  if (bf16 && psi->tz_ok && disco::fused_tz_supported(g.K, C_in, C_out, groups) &&
      !(reinterpret_cast<uintptr_t>(x) & 15) && !(reinterpret_cast<uintptr_t>(w) & 15)) {
    // Toeplitz contraction and channel mix, both on tensor cores, y tile in shared memory
    const disco::ToeplitzPlan& P = psi->tz;
    disco::TzLaunch L{psi->dtz.slabs, psi->dtz.row_begin, psi->dtz.slots, psi->dtz.b, P.K, P.parts, P.N,
                      B * C_in, g.nlat_in, g.nlat_out, g.nlon_in};
    disco::TzFused F{x, w, bias, out, C_in, C_out, groups};
    cudaError_t e = disco::launch_fused_tz(L, F, st);
    if (e != cudaSuccess) return cuda_fail(e, "fused tensor-core launch");
    return DISCO_OK;
  }
  if (bf16) {
    // gather into an on-chip y tile, tensor-core mix: blocks of exactly 128 outputs
    const int qb = 128, nblk = (g.nlon_out + qb - 1) / qb;
    const int need = max_stage(psi->fwd, qb);
    const int cache = std::min(chunk_cache(psi->fwd), 48);
    for (int budget : {std::max(need, 12288), std::max(need, 8192), need}) {
      int pass_ch, a_sbo, w_chunks;
      size_t smem;
      if (!disco::fused_tc_plan(C_in, C_out, groups, g.K, cache, budget, &pass_ch, &a_sbo, &w_chunks, &smem)) continue;
      disco::GatherArgs a = gather_args(psi->dfwd, B * C_in, qb, nblk, g.nlon_in, g.nlat_in, g.nlon_out, g.nlat_out,
                                        budget, cache, true);
      cudaError_t e = disco::launch_fused_tc(g.K, g.stride, a, x, w, bias, out, B, C_in, C_out, groups, pass_ch,
                                             a_sbo, w_chunks, st);
      if (e != cudaSuccess) return cuda_fail(e, "fused tensor-core launch");
      return DISCO_OK;
    }
  }
  const size_t per_q = (size_t)Cg * g.K * 4;
  int cap = (int)std::min<size_t>(128, kFusedTileBytes / per_q) / disco::kTaskR * disco::kTaskR;
  if (cap < disco::kTaskR) return fail(DISCO_ERR_UNSUPPORTED, "C_in/groups * K too large for the fused tile");
  int qb, nblk;
  block_shape(g.nlon_out, cap, &qb, &nblk);
  const int need = max_stage(psi->fwd, qb);
  const int ytile = Cg * g.K * qb;
  const int cache = chunk_cache(psi->fwd);
  const long room = (long)(kSmemLimit - gather_bytes(cache, g.K, 0, ytile)) / 4;
  int budget = std::max(need, (int)std::min<long>(16384, room));
  if (gather_bytes(cache, g.K, budget, ytile) > kSmemLimit)
    return fail(DISCO_ERR_UNSUPPORTED, "fused tile and staging exceed shared memory");
  disco::FusedArgs f;
  f.g = gather_args(psi->dfwd, B * C_in, qb, nblk, g.nlon_in, g.nlat_in, g.nlon_out, g.nlat_out, budget, cache, bf16);
  f.x = x;
  f.w = w;
  f.bias = bias;
  f.out = out;
  f.B = B;
  f.C_in = C_in;
  f.C_out = C_out;
  f.G = groups;
  f.K = g.K;
  f.ytile_floats = ytile;
  cudaError_t e = disco::launch_fused_simt(bf16, g.K, g.stride, f, st);
  if (e != cudaSuccess) return cuda_fail(e, "fused launch");
  return DISCO_OK;
}

disco_status disco_bwd_input(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                             const void* dout, const void* w, void* dx, void* workspace, size_t ws_bytes,
                             void* stream) {
  disco_status s = check_common(psi, B, C_in, C_out, groups, dtype);
  if (s) return s;
  if (!dout || !w || !dx) return fail(DISCO_ERR_INVALID_ARG, "dout, w and dx must be non-NULL");
  if (!disco::gather_supports(psi->g.K, psi->g.stride)) return fail(DISCO_ERR_UNSUPPORTED, "K or stride not compiled");
  const WsLayout L = layout(psi, DISCO_OP_BWD_INPUT, B, C_in, C_out, groups, dtype);
  if (!workspace || ws_bytes < L.total) return fail(DISCO_ERR_INVALID_ARG, "workspace missing or too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const char* rf = std::getenv("DISCO_RING2_FUSED");
  const char* r2 = std::getenv("DISCO_RING2");
  if (dtype == DISCO_BF16 && psi->dtile_fused_adj.ok && !(rf && rf[0] == '0') && !(r2 && r2[0] == '0') &&
      C_out == 64 && groups == 1 && C_in <= 64 && !(reinterpret_cast<uintptr_t>(dout) & 15) &&
      !(reinterpret_cast<uintptr_t>(dx) & 15) && !(reinterpret_cast<uintptr_t>(w) & 1)) {
    // one launch: the transposed contraction of dout with the K basis functions kept, and the
    // mix with W^T in the epilogue (no dy in memory)
    const disco::Geometry& g = psi->g;
    const disco::TilePlan& P = psi->tile_fused_adj;
    const DevTile& d = psi->dtile_fused_adj;
    disco::Ring2Launch R{d.tiles, d.loads, d.copies, d.cmds, d.rows, d.cta_tiles, d.b, P.n_ctas, P.n_qt, P.K, P.nb,
                         P.ns, P.nrb, P.nbs, P.bslot_bytes, P.mirror, B * C_out, g.nlat_out, g.nlat_in, g.nlon_in};
    disco::Ring2Fused F{dout, w, nullptr, dx, C_out, C_in, 1};
    cudaError_t e = disco::launch_fused_ring2(R, F, st);
    if (e == cudaSuccess && !psi->empty_in.empty())  // input rows no entry reaches: dx = 0 there
      e = disco::launch_zero_rows(dx, 2, psi->d_empty_in, (int)psi->empty_in.size(), B * C_in, g.nlat_in, g.nlon_in,
                                  st);
    if (e != cudaSuccess) return cuda_fail(e, "fused input-gradient launch");
    return DISCO_OK;
  }
  char* ws = static_cast<char*>(workspace);
  void* dy = ws + L.dy;
  s = launch_dy(psi, B, C_in, C_out, groups, dtype, dout, w, ws + L.wt, dy, st);
  if (s) return s;
  return launch_adjoint(psi, B * C_in, dtype, dy, dx, st);
}

disco_status disco_einsum_adjoint(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                                  const void* dout, const void* w, void* dy, void* workspace, size_t ws_bytes,
                                  void* stream) {
  disco_status s = check_common(psi, B, C_in, C_out, groups, dtype);
  if (s) return s;
  if (!dout || !w || !dy) return fail(DISCO_ERR_INVALID_ARG, "dout, w and dy must be non-NULL");
  const WsLayout L = layout(psi, DISCO_OP_EINSUM_ADJOINT, B, C_in, C_out, groups, dtype);
  if (!workspace || ws_bytes < L.total) return fail(DISCO_ERR_INVALID_ARG, "workspace missing or too small");
  return launch_dy(psi, B, C_in, C_out, groups, dtype, dout, w, static_cast<char*>(workspace) + L.wt, dy,
                   static_cast<cudaStream_t>(stream));
}

disco_status disco_contract_adjoint(const disco_psi* psi, int B, int C, disco_dtype dtype, const void* dy, void* dx,
                                    void* stream) {
  disco_status s = check_common(psi, B, C, C, 1, dtype);
  if (s) return s;
  if (!dy || !dx) return fail(DISCO_ERR_INVALID_ARG, "dy and dx must be non-NULL");
  if (!disco::gather_supports(psi->g.K, psi->g.stride)) return fail(DISCO_ERR_UNSUPPORTED, "K or stride not compiled");
  return launch_adjoint(psi, B * C, dtype, dy, dx, static_cast<cudaStream_t>(stream));
}

disco_status disco_bwd_weight(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                              const void* dout, const void* y, const void* x, void* dw, void* dbias, void* workspace,
                              size_t ws_bytes, void* stream) {
  disco_status s = check_common(psi, B, C_in, C_out, groups, dtype);
  if (s) return s;
  if (!dout || !dw || (!y && !x)) return fail(DISCO_ERR_INVALID_ARG, "dout, dw and one of y/x must be non-NULL");
  const disco::Geometry& g = psi->g;
  if (!disco::gather_supports(g.K, g.stride)) return fail(DISCO_ERR_UNSUPPORTED, "K or stride not compiled");
  const int op = y ? DISCO_OP_BWD_WEIGHT : DISCO_OP_BWD_WEIGHT_RECOMPUTE;
  const WsLayout L = layout(psi, op, B, C_in, C_out, groups, dtype);
  if (!workspace || ws_bytes < L.total) return fail(DISCO_ERR_INVALID_ARG, "workspace missing or too small");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const void* yv = y;
  if (!y) {
    s = launch_contract(psi, B * C_in, dtype, x, ws + L.ybuf, st, "recompute contraction launch");
    if (s) return s;
    yv = ws + L.ybuf;
  }
  return launch_dw_kn(g.K, g.nlat_out * g.nlon_out, L, B, C_in, C_out, groups, dtype, dout, yv, ws, dw, dbias, st);
}

// ------------------------------------------------------------------ the weight einsum on a set of points
// The three channel-mixing steps on K kernel indices and npts points per (b, channel) plane, with
// no Psi handle: the points may be any slice of the output grid that is contiguous in every
// plane (the longitudes an azimuth rank owns, after the transpose back).

static disco_status check_mix(int B, int C_in, int C_out, int groups, int K, long long npts, disco_dtype dtype) {
  if (B <= 0 || C_in <= 0 || C_out <= 0 || groups <= 0 || K <= 0 || npts <= 0)
    return fail(DISCO_ERR_INVALID_ARG, "B, C_in, C_out, groups, K and npts must be positive");
  if (C_in % groups || C_out % groups) return fail(DISCO_ERR_INVALID_ARG, "groups must divide both C_in and C_out");
  if (npts > (long long)INT32_MAX) return fail(DISCO_ERR_INVALID_ARG, "npts exceeds 2^31 - 1");
  if ((long long)(C_in / groups) * K > (long long)INT32_MAX) return fail(DISCO_ERR_INVALID_ARG, "C_in/groups * K too large");
  if (dtype != DISCO_F32 && dtype != DISCO_BF16) return fail(DISCO_ERR_INVALID_ARG, "unknown dtype");
  return DISCO_OK;
}

disco_status disco_mix_workspace_size(int op, int B, int C_in, int C_out, int groups, int K, long long npts,
                                      disco_dtype dtype, size_t* bytes) {
  if (!bytes) return fail(DISCO_ERR_INVALID_ARG, "NULL argument");
  disco_status s = check_mix(B, C_in, C_out, groups, K, npts, dtype);
  if (s) return s;
  if (op != DISCO_OP_EINSUM_ADJOINT && op != DISCO_OP_BWD_WEIGHT)
    return fail(DISCO_ERR_INVALID_ARG, "op is DISCO_OP_EINSUM_ADJOINT or DISCO_OP_BWD_WEIGHT");
  *bytes = layout_kn(K, (size_t)npts, op, B, C_in, C_out, groups, dtype).total;
  return DISCO_OK;
}

disco_status disco_mix(int B, int C_in, int C_out, int groups, int K, long long npts, disco_dtype dtype,
                       const void* y, const void* w, const void* bias, void* out, void* stream) {
  disco_status s = check_mix(B, C_in, C_out, groups, K, npts, dtype);
  if (s) return s;
  if (!y || !w || !out) return fail(DISCO_ERR_INVALID_ARG, "y, w and out must be non-NULL");
  disco::MixArgs m{y, w, bias, out, B, groups, C_out / groups, (C_in / groups) * K, (int)npts};
  cudaError_t e = launch_mix(dtype == DISCO_BF16, m, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "einsum launch");
  return DISCO_OK;
}

disco_status disco_mix_adjoint(int B, int C_in, int C_out, int groups, int K, long long npts, disco_dtype dtype,
                               const void* dout, const void* w, void* dy, void* workspace, size_t ws_bytes,
                               void* stream) {
  disco_status s = check_mix(B, C_in, C_out, groups, K, npts, dtype);
  if (s) return s;
  if (!dout || !w || !dy) return fail(DISCO_ERR_INVALID_ARG, "dout, w and dy must be non-NULL");
  const WsLayout L = layout_kn(K, (size_t)npts, DISCO_OP_EINSUM_ADJOINT, B, C_in, C_out, groups, dtype);
  if (!workspace || ws_bytes < L.total) return fail(DISCO_ERR_INVALID_ARG, "workspace missing or too small");
  return launch_dy_kn(K, (int)npts, B, C_in, C_out, groups, dtype, dout, w, static_cast<char*>(workspace) + L.wt,
                      dy, static_cast<cudaStream_t>(stream));
}

disco_status disco_mix_weight(int B, int C_in, int C_out, int groups, int K, long long npts, disco_dtype dtype,
                              const void* dout, const void* y, void* dw, void* dbias, void* workspace, size_t ws_bytes,
                              void* stream) {
  disco_status s = check_mix(B, C_in, C_out, groups, K, npts, dtype);
  if (s) return s;
  if (!dout || !y || !dw) return fail(DISCO_ERR_INVALID_ARG, "dout, y and dw must be non-NULL");
  const WsLayout L = layout_kn(K, (size_t)npts, DISCO_OP_BWD_WEIGHT, B, C_in, C_out, groups, dtype);
  if (!workspace || ws_bytes < L.total) return fail(DISCO_ERR_INVALID_ARG, "workspace missing or too small");
  return launch_dw_kn(K, (int)npts, L, B, C_in, C_out, groups, dtype, dout, y, static_cast<char*>(workspace), dw,
                      dbias, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Weight gradient without any device allocation.
//
// The split-K partial sums of disco_bwd_weight normally live in a workspace
// that the caller allocates.  This variant keeps them in a fixed array that is
// part of the library image instead, for callers that may not allocate device
// memory at all.  The array is reached from host code only through the device
// address that cudaGetSymbolAddress returns (the host-side name of a
// __device__ array is not a device address).

static constexpr size_t kNoAllocScratchFloats = size_t(1) << 21;  // 8 MiB of fp32
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

namespace {

std::mutex g_noalloc_mu;
constexpr int kNoAllocMaxDevices = 64;
// Per device: the context the address was looked up in, and the address.  A device reset (or any
// other change of the current context on that device) reloads the library's module, so the
// address is looked up again whenever the current context differs from the recorded one.
struct NoAllocEntry {
  void* ctx;
  float* addr;
};
NoAllocEntry g_noalloc[kNoAllocMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);

// cuCtxGetCurrent through the runtime's driver entry point (no link against libcuda); NULL when
// the driver does not provide it, in which case the address is looked up on every call.
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  return fn;
}

// Device address of the scratch array on the current device `dev`.
disco_status noalloc_scratch(int dev, float** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(DISCO_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  void* ctx = nullptr;
  const CtxGetCurrentFn get = ctx_get_current_fn();
  const bool known = get && get(&ctx) == 0 && ctx != nullptr;
  if (!known || !g_noalloc[dev].addr || g_noalloc[dev].ctx != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
    g_noalloc[dev] = NoAllocEntry{known ? ctx : nullptr, static_cast<float*>(p)};
  }
  *out = g_noalloc[dev].addr;
  return DISCO_OK;
}

}  // namespace

extern "C" disco_status disco_bwd_weight_noalloc(const disco_psi* psi, int B, int C_in, int C_out, int groups,
                                                 disco_dtype dtype, const void* dout, const void* y, void* dw,
                                                 void* dbias, void* stream) {
  disco_status s = check_common(psi, B, C_in, C_out, groups, dtype);
  if (s) return s;
  if (!dout || !y || !dw) return fail(DISCO_ERR_INVALID_ARG, "dout, y and dw must be non-NULL");
  const disco::Geometry& g = psi->g;
  const int Og = C_out / groups, Rg = (C_in / groups) * g.K, N = g.nlat_out * g.nlon_out;
  // one split needs C_out*Rg partial weights plus C_out partial biases; every batch needs a split
  const size_t per_split = (size_t)C_out * Rg + (size_t)C_out;
  const size_t max_splits = kNoAllocScratchFloats / per_split;
  if (max_splits < (size_t)B)
    return fail(DISCO_ERR_UNSUPPORTED,
                "B * (C_out * (C_in/groups) * K + C_out) floats exceed the 8 MiB static scratch of "
                "disco_bwd_weight_noalloc; use disco_bwd_weight with a workspace");
  int nchunk = std::min<long>((N + 4095) / 4096, (long)(max_splits / B));
  nchunk = std::max(nchunk, 1);
  const int nc = (N + nchunk - 1) / nchunk;
  nchunk = (N + nc - 1) / nc;
  int dev = -1;
  const cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) return cuda_fail(de, "cudaGetDevice");
  float* scratch = nullptr;
  s = noalloc_scratch(dev, &scratch);
  if (s) return s;
  const size_t nsplit = (size_t)B * nchunk;
  // The partial kernel writes every (split, o, r) entry and every (split, o) bias entry that the
  // reduction reads, so nothing left by an earlier call is used and nothing needs clearing.
  float* part = scratch;
  float* bpart = dbias ? scratch + nsplit * (size_t)C_out * Rg : nullptr;
  const bool bf16 = dtype == DISCO_BF16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  disco::DwArgs d{dout, y, part, bpart, B, groups, Og, Rg, N, nc, nchunk};
  cudaError_t e = disco::launch_dw_partial_simt(bf16, d, st);
  if (e != cudaSuccess) return cuda_fail(e, "weight-gradient launch");
  e = disco::launch_dw_reduce(bf16, part, bpart, dw, dbias, (int)nsplit, groups, Og, Rg, st);
  if (e != cudaSuccess) return cuda_fail(e, "weight-gradient reduce launch");
  return DISCO_OK;
}
