// Tensor-core (tcgen05) form of the sparse contraction x -> y for bf16 signals, stride 1, and of
// the fused forward (contraction and channel mix with y kept on chip).
//
// The contraction of the page "torch_harmonics.DiscreteContinuousConvS2",
//     y[c, k, j, q] = sum_i sum_p Psi_k(j, i, p) x[c, i, (q + p) mod nlon],
// is, for every pair of an output row j and an input row i, a correlation along the longitude
// ring with the same coefficients for every output longitude q.  For 8 consecutive outputs and a
// window of input longitudes that correlation is a product with a banded Toeplitz block B of Psi
// (built once on the host, bf16 hi + lo parts: toeplitz_plan.cpp), so
//     D[(channel, shift), (h, k, u)] += sum_{p'} X[channel, window + 8*shift + p'] B[p', (h, k, u)]
// is one tcgen05 MMA per 16 window longitudes with
//   * A = X staged in shared memory as [octet][64 channels][8 longitudes] (one TMA box of 8
//     longitudes x 64 channels per octet, so a window may wrap around the ring), read K-major
//     without swizzle: core matrices of 8 channels x 8 longitudes, M rows 64..127 are the same
//     64 channels one octet (8 longitudes) later, so one M = 128 tile covers 16 outputs;
//   * B = the Toeplitz slab, [octet][N][8] bf16, copied by one bulk copy per slab;
//   * D = fp32 in tensor memory, T groups of 16 outputs per tile, two tiles in flight (double
//     buffer); the hi and lo parts of Psi either sit side by side in N (N = 16K, summed in the
//     epilogue) or are two MMAs into the same columns (N = 8K rounded up to 16, K > 8).
//
// Persistent CTAs, 10 warps.  Four producer warps (0, 7, 8, 9) fill a ring of stages, each
// holding as many (source row, window slab) pairs of one tile as fit: the x windows by 16-byte
// cp.async copies (lanes cover 4 octets x 8 channels, so global reads are 64-byte runs and
// shared writes 128-byte rows; each warp copies 2 of the 8 channel groups, since one warp alone
// cannot issue copies fast enough), each Psi slab by one bulk copy, and a table of slab offsets
// for the MMA issuers.  Each lane's copies arrive on the stage's barrier by themselves when they
// land (cp.async.mbarrier.arrive.noinc), so no producer waits for its own copies; the MMA
// issuers order them before their tensor-core reads with a generic-to-async proxy fence after
// the barrier wait.  Lane 0 of warps 1 and 6 issues the MMAs (even and odd groups of 16
// outputs); warps 2..5 read the accumulator of the previous tile back (each warp its TMEM lane
// quadrant) into a [64 channels][K][16T] bf16 tile in shared memory that one TMA store writes
// to y.  Every wait is bounded (tc_common.cuh): on expiry the kernel records the timeout and
// stops.
//
// Fused forward (FUSED): a tile is 128 outputs of one output row for the 64 input channels of
// one (batch, group), contracted as two halves of 64 outputs.  The epilogue warps round each
// half's accumulator to bf16 into a y tile Y[q][c*K + k] in shared memory (MN-major, no
// swizzle), then the MMA issuer runs the channel mix D2[q][o] = sum_r Y[q][r] w[g*Og + o][r]
// with w staged by TMA (K-major, 128-byte swizzle), and the epilogue adds the bias and stores
// out.  y is never written to global memory.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace disco {
namespace {

constexpr int kCT = 64;                       // channels per tile
constexpr uint32_t kOctBytes = kCT * 16;      // one staged octet: 64 channels x 8 bf16
constexpr int kProducers = 4;  // copy warps: 0 and 7..6+kProducers-1
constexpr int kThreads = 32 * (6 + kProducers);  // producer, MMA issuer, four epilogue warps, MMA issuer, producers
constexpr uint32_t kTmemCols = 512;
constexpr int kStages = 4;                    // most stages (barriers are laid out for this many)
constexpr int kMaxSlabs = 24;                 // slab table entries per stage
constexpr int kBars = 2 * kStages + 8;        // full/empty per stage, tfull/tempty x2, yfull, d2full, d2empty, w

struct TzArgs {
  const int4* slabs;  // TzSlab records
  const int4* slots;  // {row, first slab, end slab, 0} per row position
  const uint8_t* bglob;
  const __nv_bfloat16* x;
  int BC;
  int n_lat_in, n_lon, n_lat_out;
  int n_seg, n_ctile, n_tiles;
  uint32_t stage_bytes;
  int n_stages;        // stages of this launch (at most kStages)
  uint32_t r0_bytes;   // output staging tile (contraction) or y tile (fused)
  uint32_t w_bytes;    // fused: staged w of one group
  // fused forward
  __nv_bfloat16* out;
  const __nv_bfloat16* bias;
  int C_in, C_out, G, Og;
  uint32_t a_sbo;      // bytes between 8-output blocks of the y tile
  int w_chunks;        // 64-wide chunks of r = c*K + k
};

// Columns of the MMA for K basis functions with the hi/lo parts of Psi inside N (PARTS = 1) or
// in two MMAs (PARTS = 2), and groups of 16 outputs per contraction tile: two accumulator
// buffers in 512 tensor-memory columns and at most 8 groups (the output box is at most 128
// longitudes); the fused forward contracts halves of 4 groups (64 outputs).
template <int K, int PARTS, bool FUSED>
struct TzShape {
  static constexpr int N = PARTS == 1 ? 16 * K : (8 * K + 15) / 16 * 16;
  static constexpr int T = FUSED ? 4 : ((256 / N) < 8 ? 256 / N : 8);
  // fused: two contraction halves of 64 outputs (y tile of 128 rows) for K <= 5; one half
  // for larger K, whose 128-row y tile would not fit shared memory (the mix then runs on
  // M = 128 with its upper 64 rows discarded)
  static constexpr int NH = FUSED ? (K <= 5 ? 2 : 1) : 1;
  static constexpr int QT = 16 * T * NH;                 // outputs per tile
  static constexpr int NB = FUSED ? (2 * T * N + 64 <= 512 ? 2 : 1) : 2;  // accumulator buffers
};

struct Tile {
  int j, q0, ct, s_begin, s_end;
};

__device__ __forceinline__ Tile decode(const TzArgs& a, int tile, int QT) {
  Tile t;
  t.ct = tile % a.n_ctile;
  const int r = tile / a.n_ctile;
  t.q0 = (r % a.n_seg) * QT;
  const int4 sl = a.slots[r / a.n_seg];  // one load: no dependent chain
  t.j = sl.x;
  t.s_begin = sl.y;
  t.s_end = sl.z;
  return t;
}

// Stage table: word 0 = slab count | first << 8 | last << 9 (first / last stage of its
// contraction tile); then per slab {nk | x offset << 8, B offset}, offsets in 16-byte units
// from the stage base.
constexpr int kFirst = 1 << 8, kLast = 1 << 9;
constexpr int kMetaWords = 1 + 2 * kMaxSlabs;

template <int K, int PARTS, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1) contract_tc_kernel(const __grid_constant__ CUtensorMap ymap,
                                                                  const __grid_constant__ CUtensorMap wmap,
                                                                  TzArgs a) {
  using Sh = TzShape<K, PARTS, FUSED>;
  constexpr int N = Sh::N, T = Sh::T, NH = Sh::NH, QT = Sh::QT, NB = Sh::NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sR0 = smem;                 // output staging tile / y tile
  uint8_t* sW = smem + a.r0_bytes;     // fused: w of the current group
  uint8_t* sS = sW + a.w_bytes;        // n_stages stages of stage_bytes
  const int S = a.n_stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(sS + (size_t)S * a.stage_bytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;  // [2] contraction accumulator ready for the epilogue
  uint64_t* tempty = tfull + 2;       // [2] contraction accumulator drained by the epilogue
  uint64_t* yfull = tempty + 2;       // fused: y tile written
  uint64_t* d2full = yfull + 1;       // fused: mix accumulator ready
  uint64_t* d2empty = d2full + 1;     // fused: mix accumulator drained
  uint64_t* wbar = d2empty + 1;       // fused: w staged
  int* meta = reinterpret_cast<int*>(full + kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + kStages * kMetaWords);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ring = a.n_lon / 8;
  constexpr uint32_t TN = (uint32_t)(T * N);
  constexpr uint32_t bk = (uint32_t)N * 16;  // bytes per octet of a Psi block

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 32 * kProducers + 1);  // every producer lane's copy completions + the closing arrival
      tc::mbar_init(&empty[s], 2);  // both MMA issuers commit
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 2);
      tc::mbar_init(&tempty[b], 4);
    }
    tc::mbar_init(yfull, 1);
    tc::mbar_init(d2full, 1);
    tc::mbar_init(d2empty, 4);
    tc::mbar_init(wbar, 1);
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp >= 7) {
    // ---------------------------------------------------------------- producer warps
    // kProducers warps run the same stage packing (so they agree on every stage and offset)
    // and each copies its share of the 8 channel groups; the first also writes the stage
    // tables, issues the bulk copies and closes the stages.
    constexpr int CG = 8 / kProducers;
    const int pw = warp == 0 ? 0 : warp - 6;
    const size_t chan = (size_t)a.n_lat_in * a.n_lon;
    const int csub = lane >> 2, osub = lane & 3;  // channel within 8, octet within 4
    uint32_t n = 0;                               // stages opened so far
    bool ok = true;
    int st = 0, cnt = 0;
    uint32_t used = 0;                            // bytes of the open stage
    // opens stage n: waits until the MMAs of its previous use are done
    auto open = [&]() -> bool {
      st = (int)(n % S);
      cnt = 0;
      used = 0;
      if (n >= (uint32_t)S) {
        int good = 1;
        if (lane == 0) good = tc::mbar_wait(&empty[st], ((n / S) & 1) ^ 1);
        if (!__shfl_sync(0xffffffffu, good, 0)) return false;
        __syncwarp();  // order every lane's copies after lane 0's wait
      }
      return true;
    };
    // closes stage n: every lane's copies arrive on its barrier when they have landed
    auto close = [&](int flags) {
      if (lane == 0 && pw == 0) {
        meta[st * kMetaWords] = cnt | flags;
        tc::mbar_arrive(&full[st]);
      }
      tc::cp_async_arrive_noinc(&full[st]);
      ++n;
    };
    int tile = blockIdx.x;
    Tile t, t1;
    if (tile < a.n_tiles) t = decode(a, tile, QT);
    if (tile + (int)gridDim.x < a.n_tiles) t1 = decode(a, tile + gridDim.x, QT);
    int4 mine = make_int4(0, 0, 0, 0);
    if (tile < a.n_tiles && t.s_begin + lane < t.s_end) mine = a.slabs[t.s_begin + lane];
    for (; tile < a.n_tiles && ok; tile += gridDim.x) {
      // prefetch: the tile after next is decoded and the next tile's slabs are loaded while this
      // tile's copies are issued
      const int tile1 = tile + gridDim.x, tile2 = tile1 + gridDim.x;
      // this lane's channels ct*64 + 8*cg + csub: base pointer and which of them exist
      const __nv_bfloat16* xl = a.x + (size_t)(t.ct * kCT + csub) * chan;
      uint32_t cmask = 0;
#pragma unroll
      for (int cg = 0; cg < 8; ++cg) cmask |= (t.ct * kCT + 8 * cg + csub < a.BC ? 1u : 0u) << cg;
      Tile t2;
      if (tile2 < a.n_tiles) t2 = decode(a, tile2, QT);
      int4 mine1 = make_int4(0, 0, 0, 0);
      if (tile1 < a.n_tiles && t1.s_begin + lane < t1.s_end) mine1 = a.slabs[t1.s_begin + lane];
      const int nsl = max(t.s_end - t.s_begin, 1);  // a row without slabs still passes one stage
      const int4 mine0 = mine;
      for (int h = 0; h < NH && ok; ++h) {
        const int q0 = t.q0 + 16 * T * h;
        mine = mine0;
        if (!(ok = open())) break;
        bool first = true;
        for (int r = 0; r < nsl; ++r) {
          if (r > 0 && (r & 31) == 0) {
            mine = make_int4(0, 0, 0, 0);
            if (t.s_begin + r + lane < t.s_end) mine = a.slabs[t.s_begin + r + lane];
          }
          const int q = r & 31;
          const int si = __shfl_sync(0xffffffffu, mine.x, q);
          const int lon_off = __shfl_sync(0xffffffffu, mine.y, q);
          const int nk = __shfl_sync(0xffffffffu, mine.z, q);
          const int boff = __shfl_sync(0xffffffffu, mine.w, q);
          const int n_oct = nk ? 2 * T + 2 * nk - 1 : 0;
          const uint32_t xbytes = (uint32_t)n_oct * kOctBytes;
          const uint32_t bbytes = (uint32_t)(PARTS * 2 * nk) * bk;
          if (cnt > 0 && (used + xbytes + bbytes > a.stage_bytes || cnt == kMaxSlabs)) {
            close(first ? kFirst : 0);
            first = false;
            if (!(ok = open())) break;
          }
          uint8_t* base = sS + (size_t)st * a.stage_bytes;
          if (lane == 0 && pw == 0) {
            meta[st * kMetaWords + 1 + 2 * cnt] = nk | (int)(used >> 4) << 8;
            meta[st * kMetaWords + 2 + 2 * cnt] = (int)((used + xbytes) >> 4);
            if (nk) {
              tc::mbar_expect_tx(&full[st], bbytes);
              tc::bulk_load(base + used + xbytes, a.bglob + (size_t)boff * 16, bbytes, &full[st]);
            }
          }
          if (nk) {
            int o0 = ((q0 + lon_off) / 8) % ring;  // q0 + lon_off is a multiple of 8
            if (o0 < 0) o0 += ring;
            const __nv_bfloat16* xrow = xl + (size_t)si * a.n_lon;
            uint8_t* dst = base + used + csub * 16;
            int oo = o0 + osub;
            for (int o = osub; o < n_oct; o += 4, oo += 4) {
              while (oo >= ring) oo -= ring;
              const __nv_bfloat16* src = xrow + oo * 8;
              uint8_t* d = dst + o * kOctBytes;
#pragma unroll
              for (int cg = pw * CG; cg < pw * CG + CG; ++cg) {
                const bool v = (cmask >> cg) & 1u;
                tc::cp_async16(d + cg * 128, v ? src + (size_t)cg * 8 * chan : a.x, v ? 16u : 0u);
              }
            }
          }
          used += xbytes + bbytes;
          ++cnt;
        }
        if (!ok) break;
        close((first ? kFirst : 0) | kLast);
      }
      t = t1;
      t1 = t2;
      mine = mine1;
    }
    // no copy may still be in flight when the CTA exits
    tc::cp_async_wait_all();
  } else if (warp == 1 || warp == 6) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuers
      // two threads issue the contraction's MMAs, the even and the odd groups of 16 outputs
      // (disjoint accumulator columns), which halves each one's issue overhead; the first
      // also runs the fused mode's channel mix
      const int gsel = warp == 1 ? 0 : 1;
      constexpr uint32_t idesc = tc::idesc_bf16(128, N, false, false);
      // descriptors differ only in their 14-bit start-address field (address >> 4, below
      // 256 KB, so adding to it never carries into the other fields)
      const uint64_t a_fix = tc::desc_noswz(0, kOctBytes, 128);
      const uint64_t b_fix = tc::desc_noswz(0, bk, 128);
      const uint32_t a_step = (2 * kOctBytes) >> 4;  // one K-step (16 longitudes) of A
      const uint32_t b_step = (2 * bk) >> 4;         // one K-step of B
      uint32_t n = 0;
      int sc = 0;      // contraction tiles (halves) so far
      int items = 0;   // tiles so far
      int wg = -1;     // group whose w is staged
      int wloads = 0;  // w stagings so far (phase of wbar)
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x, ++items) {
        for (int h = 0; h < NH && ok; ++h, ++sc) {
          const int buf = sc % NB, use = sc / NB;
          if (sc >= NB && !tc::mbar_wait(&tempty[buf], (use & 1) ^ 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t d0 = tmem + (uint32_t)buf * TN;
          while (true) {
            const int st = (int)(n % S);
            if (!tc::mbar_wait(&full[st], (n / S) & 1)) {
              ok = false;
              break;
            }
            tc::fence_after_sync();
            tc::fence_proxy_async();  // the stage's cp.async data (generic proxy) before the MMA reads
            const volatile int* m = meta + st * kMetaWords;
            const int hdr = m[0];
            const uint32_t sbase4 = tc::smem_u32(sS + (size_t)st * a.stage_bytes) >> 4;
            for (int sl = 0; sl < (hdr & 0xFF); ++sl) {
              const int e0 = m[1 + 2 * sl], e1 = m[2 + 2 * sl];
              const int nk = e0 & 0xFF;
              if (nk == 0) continue;  // the empty stage of a row without slabs
              // the first MMA of each group of outputs in a tile starts the accumulator
              const uint32_t acc0 = ((hdr & kFirst) && sl == 0) ? 0u : 1u;
#pragma unroll
              for (int part = 0; part < PARTS; ++part) {
                const uint64_t bd0 = b_fix | (uint64_t)(sbase4 + (uint32_t)e1 + (uint32_t)(part * nk) * b_step);
                for (int g = gsel; g < T; g += 2) {
                  uint64_t ad = a_fix | (uint64_t)(sbase4 + (uint32_t)(e0 >> 8) + (uint32_t)g * a_step);
                  uint64_t bd = bd0;
                  const uint32_t d = d0 + (uint32_t)(g * N);
                  tc::mma_bf16(d, ad, bd, idesc, part == 0 ? acc0 : 1u);
                  for (int kk = 1; kk < nk; ++kk) {
                    ad += a_step;
                    bd += b_step;
                    tc::mma_bf16(d, ad, bd, idesc, 1u);
                  }
                }
              }
            }
            tc::mma_commit(&empty[st]);
            ++n;
            if (hdr & kLast) break;
          }
          if (!ok) break;
          tc::mma_commit(&tfull[buf]);
        }
        if (FUSED && ok && gsel == 0) {
          // ------------------------------------------------ channel mix of the tile
          const int ct = tile % a.n_ctile, g = ct % a.G;
          if (g != wg) {  // stage w of this group (after the previous mix has read the old one)
            if (items > 0 && !tc::mbar_wait(d2full, (items - 1) & 1)) {
              ok = false;
              break;
            }
            tc::mbar_arrive_expect_tx(wbar, (uint32_t)a.w_bytes);
            for (int c = 0; c < a.w_chunks; ++c)
              tc::tma_load_2d(sW + (size_t)c * a.Og * 128, &wmap, wbar, c * 64, g * a.Og);
            if (!tc::mbar_wait(wbar, wloads & 1)) {
              ok = false;
              break;
            }
            ++wloads;
            wg = g;
          }
          ok = ok && tc::mbar_wait(yfull, items & 1);
          if (items > 0) ok = ok && tc::mbar_wait(d2empty, (items - 1) & 1);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t idesc2 = tc::idesc_bf16(128, a.Og, true, false);
          const uint32_t d2 = tmem + (uint32_t)NB * TN;
          const uint32_t y0 = tc::smem_u32(sR0), w0 = tc::smem_u32(sW);
          for (int ks = 0; ks < 4 * K; ++ks) {  // r = c*K + k < 64K, 16 per step
            const int rg = 16 * ks;
            const uint64_t ad = tc::desc_noswz(y0 + (uint32_t)ks * 256, 128, a.a_sbo);
            const uint64_t bd = tc::desc_sw128(w0 + (uint32_t)((rg / 64) * a.Og * 128 + (rg % 64) * 2), 16, 1024);
            tc::mma_bf16(d2, ad, bd, idesc2, ks > 0 ? 1u : 0u);
          }
          tc::mma_commit(d2full);
        }
      }
    }
  } else if (!FUSED) {
    // ---------------------------------------------------------------- epilogue warps (y)
    // TMEM lane quadrant (warp % 4); row m = channel (m % 64) at shift m / 64
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    const int half = m >> 6;
    const bool issuer = warp == 2 && lane == 0;
    uint8_t* myrow = sR0 + (size_t)(m & 63) * K * QT * 2;
    if (warp == 2) tc::prefetch_map(&ymap);
    int tcount = 0;
    Tile t;
    if (blockIdx.x < a.n_tiles) t = decode(a, blockIdx.x, QT);
    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++tcount) {
      Tile tn;  // the next tile's record is fetched while this one is drained
      if (tile + (int)gridDim.x < a.n_tiles) tn = decode(a, tile + gridDim.x, QT);
      const int buf = tcount & 1, use = tcount >> 1;
      const bool ok = tc::mbar_wait(&tfull[buf], use & 1);
      tc::fence_after_sync();
      // the staging tile is free once the previous store has read it; the four warps leave
      // together when a wait expired
      if (issuer) tc::bulk_wait_read0();
      if (!tc::named_bar_and(1, 128, ok)) break;
      const bool has = t.s_end > t.s_begin;
      const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * TN;
#pragma unroll 1
      for (int g = 0; g < T; ++g) {
        uint32_t r[N];
        if (has) {
          tc::tmem_ld_chunks<N / 16>(tb + (uint32_t)(g * N), r);
        } else {
#pragma unroll
          for (int i = 0; i < N; ++i) r[i] = 0u;
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
          uint4 v;
          uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v0 = __uint_as_float(r[8 * k + 2 * e]), v1 = __uint_as_float(r[8 * k + 2 * e + 1]);
            if (PARTS == 1) {  // add the lo part's columns
              v0 += __uint_as_float(r[8 * K + 8 * k + 2 * e]);
              v1 += __uint_as_float(r[8 * K + 8 * k + 2 * e + 1]);
            }
            const __nv_bfloat162 p = __floats2bfloat162_rn(v0, v1);
            w[e] = *reinterpret_cast<const uint32_t*>(&p);
          }
          *reinterpret_cast<uint4*>(myrow + ((size_t)k * QT + 16 * g + 8 * half) * 2) = v;
        }
      }
      // accumulator drained: the MMA issuer may reuse the buffer
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty[buf]);
      // staged tile -> y (channels beyond BC and longitudes beyond the ring are clipped)
      tc::fence_proxy_async();
      tc::named_bar_sync(1, 128);
      if (issuer) {
        tc::tma_store_4d(&ymap, sR0, t.q0, t.j, 0, t.ct * kCT);
        tc::bulk_commit();
      }
      t = tn;
    }
    if (issuer) tc::bulk_wait0();
  } else {
    // ---------------------------------------------------------------- epilogue warps (fused)
    const int quad = warp & 3;
    const int m = quad * 32 + lane;  // contraction: channel m % 64 at shift m / 64; mix: output q = m
    const int half = m >> 6;
    const int c = m & 63;
    int sc = 0, items = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x, ++items) {
      const Tile t = decode(a, tile, QT);
      const bool has = t.s_end > t.s_begin;
      // 1. both contraction halves -> y tile (bf16, rounded as the unfused path stores y)
      for (int h = 0; h < NH; ++h, ++sc) {
        const int buf = sc % NB, use = sc / NB;
        ok = tc::named_bar_and(1, 128, tc::mbar_wait(&tfull[buf], use & 1));
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * TN;
#pragma unroll 1
        for (int g = 0; g < T; ++g) {
          uint32_t r[N];
          if (has) {
            tc::tmem_ld_chunks<N / 16>(tb + (uint32_t)(g * N), r);
          } else {
#pragma unroll
            for (int i = 0; i < N; ++i) r[i] = 0u;
          }
          const int qb = 8 * h + 2 * g + half;  // 8-output block of the y tile
#pragma unroll
          for (int k = 0; k < K; ++k) {
            uint4 v;
            uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float v0 = __uint_as_float(r[8 * k + 2 * e]), v1 = __uint_as_float(r[8 * k + 2 * e + 1]);
              if (PARTS == 1) {
                v0 += __uint_as_float(r[8 * K + 8 * k + 2 * e]);
                v1 += __uint_as_float(r[8 * K + 8 * k + 2 * e + 1]);
              }
              const __nv_bfloat162 p = __floats2bfloat162_rn(v0, v1);
              w[e] = *reinterpret_cast<const uint32_t*>(&p);
            }
            *reinterpret_cast<uint4*>(sR0 + (size_t)qb * a.a_sbo + (size_t)(c * K + k) * 16) = v;
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&tempty[buf]);
      }
      if (!ok) break;
      // 2. y tile complete: the mix MMAs may read it (generic -> async proxy, then release)
      tc::fence_proxy_async();
      tc::named_bar_sync(1, 128);
      if (warp == 2 && lane == 0) tc::mbar_arrive(yfull);
      // 3. mix accumulator -> out (+ bias)
      ok = tc::named_bar_and(1, 128, tc::mbar_wait(d2full, items & 1));
      if (!ok) break;
      tc::fence_after_sync();
      const int ct = t.ct, b = ct / a.G, g = ct % a.G;
      const int q = t.q0 + m;
      const uint32_t d2 = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)NB * TN;
      for (int o0 = 0; o0 < a.Og; o0 += 16) {
        float v[16];
        tc::tmem_ld16(d2 + (uint32_t)o0, v);
        if (m < QT && q < a.n_lon) {  // rows beyond the tile's outputs (one-half tiles) are discarded
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int oc = g * a.Og + o0 + i;
            const float bv = a.bias ? __bfloat162float(a.bias[oc]) : 0.0f;
            a.out[(((size_t)b * a.C_out + oc) * a.n_lat_out + t.j) * a.n_lon + q] = __float2bfloat16_rn(v[i] + bv);
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(d2empty);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

namespace {

size_t tz_extra() { return 1024 + 8 * kBars + 4 * kStages * kMetaWords + 16; }

cudaError_t launch_common(const void* kernel, const TzArgs& a, const CUtensorMap& ym, const CUtensorMap& wm,
                          size_t smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(a.n_tiles, sms);
  void* args[] = {const_cast<CUtensorMap*>(&ym), const_cast<CUtensorMap*>(&wm), const_cast<TzArgs*>(&a)};
  e = cudaLaunchKernel(kernel, dim3(grid), dim3(kThreads), args, smem, st);
  count_launch();
  return e;
}

TzArgs base_args(const TzLaunch& L, const void* x, int QT) {
  TzArgs a{};
  a.slabs = reinterpret_cast<const int4*>(L.slabs);
  a.slots = reinterpret_cast<const int4*>(L.slots);
  a.bglob = static_cast<const uint8_t*>(L.b);
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.BC = L.BC;
  a.n_lat_in = L.nlat_in;
  a.n_lon = L.nlon;
  a.n_lat_out = L.nlat_out;
  a.n_seg = (L.nlon + QT - 1) / QT;
  a.n_ctile = (L.BC + kCT - 1) / kCT;
  a.n_tiles = (L.n_slots > 0 ? L.n_slots : L.nlat_out) * a.n_seg * a.n_ctile;
  return a;
}

template <int K, int PARTS>
cudaError_t launch_tz(const TzLaunch& L, const void* x, void* y, cudaStream_t st) {
  using Sh = TzShape<K, PARTS, false>;
  constexpr int N = Sh::N, T = Sh::T;
  if (L.K != K || L.parts != PARTS || L.N != N) return cudaErrorInvalidValue;
  const size_t extra = tz_extra();
  const uint32_t out_bytes = ((uint32_t)(kCT * K * Sh::QT * 2) + 1023u) & ~1023u;
  const uint32_t stage = (uint32_t)((kTcSmemLimit - extra - out_bytes) / kStages) & ~1023u;
  // the largest slab must fit one stage
  const uint32_t max_slab =
      (uint32_t)(2 * T + 2 * kTzSlabK - 1) * kOctBytes + (uint32_t)(PARTS * 2 * kTzSlabK * N * 16);
  if (max_slab > stage) return cudaErrorInvalidValue;
  const size_t smem = (size_t)out_bytes + (size_t)kStages * stage + extra;
  // output as [BC][K][n_lat_out][nlon]: box = QT longitudes x 1 row x K x 64 channels
  CUtensorMap ym, wm;
  std::memset(&wm, 0, sizeof(wm));
  const cuuint64_t dims[4] = {(cuuint64_t)L.nlon, (cuuint64_t)L.nlat_out, (cuuint64_t)K, (cuuint64_t)L.BC};
  const cuuint64_t strides[3] = {(cuuint64_t)L.nlon * 2, (cuuint64_t)L.nlat_out * L.nlon * 2,
                                 (cuuint64_t)K * L.nlat_out * L.nlon * 2};
  const cuuint32_t box[4] = {(cuuint32_t)Sh::QT, 1, (cuuint32_t)K, (cuuint32_t)kCT};
  if (!tc::encode_bf16_map(&ym, y, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorInvalidValue;
  TzArgs a = base_args(L, x, Sh::QT);
  a.stage_bytes = stage;
  a.n_stages = kStages;
  a.r0_bytes = out_bytes;
  a.w_bytes = 0;
  return launch_common(reinterpret_cast<const void*>(&contract_tc_kernel<K, PARTS, false>), a, ym, wm, smem, st);
}

// Shared-memory layout of the fused forward: y tile, w of one group, the stage ring; false when
// the layer does not fit (tensor memory or shared memory).
struct FusedLayout {
  uint32_t a_sbo, r0, w_bytes, stage;
  int stages;
  size_t smem;
};

template <int K, int PARTS>
bool fused_layout(int Og, FusedLayout* f) {
  using Sh = TzShape<K, PARTS, true>;
  constexpr int N = Sh::N, T = Sh::T;
  if (Og % 16 || Og > 256 || Sh::NB * T * N + Og > (int)kTmemCols) return false;
  const int R = kCT * K;
  const size_t extra = tz_extra();
  f->a_sbo = (uint32_t)(R * 16 + 16);
  f->w_bytes = (uint32_t)(K * Og * 128);  // R / 64 = K chunks of [Og][64]
  // the mix reads 16 blocks of 8 outputs: a one-half tile writes 8 of them and the other 8
  // must still lie inside shared memory (they read into the staged w, and are discarded)
  const uint32_t blocks = (uint32_t)(Sh::NH * 8);
  f->r0 = (blocks * f->a_sbo + 1023u) & ~1023u;
  if (16 * f->a_sbo > f->r0 + f->w_bytes) f->r0 = (16 * f->a_sbo - f->w_bytes + 1023u) & ~1023u;
  if (f->r0 + f->w_bytes + extra >= kTcSmemLimit) return false;
  const uint32_t max_slab =
      (uint32_t)(2 * T + 2 * kTzSlabK - 1) * kOctBytes + (uint32_t)(PARTS * 2 * kTzSlabK * N * 16);
  for (f->stages = kStages; f->stages >= 2; --f->stages) {
    f->stage = (uint32_t)((kTcSmemLimit - extra - f->r0 - f->w_bytes) / f->stages) & ~1023u;
    if (max_slab <= f->stage) break;  // the largest slab must fit one stage
  }
  if (f->stages < 2) return false;
  f->smem = (size_t)f->r0 + f->w_bytes + (size_t)f->stages * f->stage + extra;
  return true;
}

// Fused forward: 64 input channels per group (one channel tile), Og outputs per group.
template <int K, int PARTS>
cudaError_t launch_tz_fused(const TzLaunch& L, const TzFused& F, cudaStream_t st) {
  using Sh = TzShape<K, PARTS, true>;
  constexpr int N = Sh::N;
  if (L.K != K || L.parts != PARTS || L.N != N) return cudaErrorInvalidValue;
  const int Og = F.C_out / F.G, R = kCT * K;
  FusedLayout fl;
  if (F.C_in != F.G * kCT || !fused_layout<K, PARTS>(Og, &fl)) return cudaErrorInvalidValue;
  const uint32_t a_sbo = fl.a_sbo, r0 = fl.r0, w_bytes = fl.w_bytes, stage = fl.stage;
  const size_t smem = fl.smem;
  CUtensorMap ym, wm;
  std::memset(&ym, 0, sizeof(ym));
  // w as [C_out][R] (r = c*K + k contiguous): boxes of 64 r x Og rows, 128-byte swizzle
  const cuuint64_t dims[2] = {(cuuint64_t)R, (cuuint64_t)F.C_out};
  const cuuint64_t strides[1] = {(cuuint64_t)R * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)Og};
  if (!tc::encode_bf16_map(&wm, F.w, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  TzArgs a = base_args(L, F.x, Sh::QT);
  a.stage_bytes = stage;
  a.n_stages = fl.stages;
  a.r0_bytes = r0;
  a.w_bytes = w_bytes;
  a.out = static_cast<__nv_bfloat16*>(F.out);
  a.bias = static_cast<const __nv_bfloat16*>(F.bias);
  a.C_in = F.C_in;
  a.C_out = F.C_out;
  a.G = F.G;
  a.Og = Og;
  a.a_sbo = a_sbo;
  a.w_chunks = K;
  return launch_common(reinterpret_cast<const void*>(&contract_tc_kernel<K, PARTS, true>), a, ym, wm, smem, st);
}

}  // namespace

bool toeplitz_geometry(int K, int stride, int nlon_in, int nlon_out) {
  // compiled for K = 1 (the adjoint) and the forward's K = 3, 5, 7, 9; a staged window may
  // wrap around the ring any number of times, so there is no lower bound on nlon
  return stride == 1 && nlon_in == nlon_out && nlon_in % 8 == 0 && (K == 1 || K == 3 || K == 5 || K == 7 || K == 9);
}

bool contract_tc_supported(int K, int stride, int nlon_in, int nlon_out) {
  return tc::encode_tiled_fn() != nullptr && toeplitz_geometry(K, stride, nlon_in, nlon_out);
}

cudaError_t launch_contract_tc(const TzLaunch& L, const void* x, void* y, cudaStream_t st) {
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15)) return cudaErrorInvalidValue;
  switch (L.K) {
    case 1: return launch_tz<1, 1>(L, x, y, st);
    case 3: return launch_tz<3, 1>(L, x, y, st);
    case 5: return launch_tz<5, 1>(L, x, y, st);
    case 7: return launch_tz<7, 1>(L, x, y, st);
    case 9: return launch_tz<9, 2>(L, x, y, st);
    default: return cudaErrorInvalidValue;
  }
}

bool fused_tz_supported(int K, int C_in, int C_out, int G) {
  if (tc::encode_tiled_fn() == nullptr || G <= 0 || C_in != G * kCT || C_out % G) return false;
  FusedLayout f;
  if (K == 3) return fused_layout<3, 1>(C_out / G, &f);
  if (K == 5) return fused_layout<5, 1>(C_out / G, &f);
  if (K == 9) return fused_layout<9, 2>(C_out / G, &f);
  return false;
}

cudaError_t launch_fused_tz(const TzLaunch& L, const TzFused& F, cudaStream_t st) {
  if ((reinterpret_cast<uintptr_t>(F.x) & 15) || (reinterpret_cast<uintptr_t>(F.w) & 15)) return cudaErrorInvalidValue;
  switch (L.K) {
    case 3: return launch_tz_fused<3, 1>(L, F, st);
    case 5: return launch_tz_fused<5, 1>(L, F, st);
    case 9: return launch_tz_fused<9, 2>(L, F, st);
    default: return cudaErrorInvalidValue;
  }
}

int take_contract_tc_status() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
  return v;
}

}  // namespace disco
