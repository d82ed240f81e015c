// Strip-staged tensor-core contraction (tcgen05, sm_100a) for bf16 signals, stride 1.
//
// The contraction of the page "torch_harmonics.DiscreteContinuousConvS2" (class description),
//     y[c, k, j, q] = sum_i sum_p Psi_k(j, i, p) x[c, i, (q + p) mod nlon],
// is, for an output row j and a source row i, a correlation along the longitude ring with the
// same coefficients for every output longitude (the p-shift symmetry).  For 16 consecutive
// outputs it is one product with a banded Toeplitz block of Psi per 16 source longitudes
// (ring_plan.cpp), run here as tcgen05 MMAs:
//   * A = 128 rows x 16 source longitudes from shared memory, staged as octets of
//     [2 groups][64 planes][8 longitudes]; group 0 holds the source row of the output row, group 1
//     either the mirror source row of the mirror output row (whose Toeplitz blocks are the same)
//     or the next 64 planes.  Read K-major without swizzle: core matrices of 8 planes x 8
//     longitudes 128 bytes apart along M, octets 2 KB apart along K.
//   * B = the Toeplitz K-step, [2 octets][N = 16K][8] bf16, one bulk copy per item.
//   * D = fp32 in tensor memory: rows = (group, plane), columns = (k, u) for each block of 16
//     outputs, nb blocks per row buffer.
// A tile is (strip of consecutive output rows, nb*16 output longitudes, plane tile).  The kernel
// replays the plan's script for every tile: four warps copy source-row windows into a ring of
// shared-memory slots as soon as a slot is free (16-byte cp.async, lanes covering 4 octets x 8
// planes so global reads are 64-byte runs; octets are taken modulo the ring, so a window may
// wrap around the longitude ring; planes past the last one read as zeros), another warp copies
// the Toeplitz K-steps of each item into a ring of B slots with bulk copies; a source shared by
// several output rows is loaded once per tile.  The TMA unit is left to the B copies and the y
// stores: boxes with 16-byte rows (one octet of one plane) move about 3 B/cycle per SM there.  One thread issues
// the MMAs, item by item, into the accumulator buffer of the item's row; four epilogue warps
// read finished rows back (each its tensor-memory lane quadrant: 32 planes of one group), round
// them to bf16 into a [32 planes][K][64 outputs] tile (128-byte rows, 128-byte swizzle, so the
// lanes' rows fall in different banks) and write it with one TMA store per row.
// Every mbarrier wait is bounded (tc_common.cuh): on expiry the kernel records the timeout in the
// device status word and stops.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace disco {
namespace {

// Warps: 0..3 epilogue (TMEM lane quadrant = warp), 4..7 MMA issuers (one per SM sub-partition;
// issuer w takes the blocks b with b % 4 == w), 8..11 x copies, 12 B copies and item records.
constexpr int kIssuers = 4;
constexpr int kXWarps = 4;
constexpr int kRingThreads = 416;
constexpr int kRingNb = 4;         // blocks of 16 outputs per tile: 64 outputs, one 128-byte y row
constexpr uint32_t kOct = 2048;    // one staged octet: 2 groups x 64 planes x 8 bf16
constexpr int kMaxSlots = 15, kMaxBufs = 8, kMaxBslots = 12;


struct RingArgs {
  const __nv_bfloat16* x;  // source planes [BC][n_src_rows][nlon]
  int BC, n_src_rows;
  const int4* strips;  // 2 int4 per strip
  const int2* loads;
  const int4* items;
  const int2* rows;
  const uint8_t* b;
  int n_tiles, n_qt, n_pt;
  int nb, ns, nrb, nbs, bk;
  int ring_oct;         // nlon / 8
  int mirror;
  int plane_tile;       // 64 (mirror) or 128
  int nlon;
  uint32_t slot_bytes, bslot_bytes, ystage_bytes;
};

struct TileInfo {
  int item0, item1, load0, load1, row0, row1;
  int q0, plane0;
};

__device__ __forceinline__ TileInfo tile_info(const RingArgs& a, int tile) {
  TileInfo t;
  const int per = a.n_qt * a.n_pt;
  const int st = tile / per, rem = tile % per;
  const int4 s0 = a.strips[2 * st], s1 = a.strips[2 * st + 1];
  t.item0 = s0.x;
  t.item1 = s0.y;
  t.load0 = s0.z;
  t.load1 = s0.w;
  t.row0 = s1.x;
  t.row1 = s1.y;
  t.q0 = (rem / a.n_pt) * a.nb * 16;
  t.plane0 = (rem % a.n_pt) * a.plane_tile;
  return t;
}

__device__ __forceinline__ int4 shfl4(const int4& v, int src) {
  return make_int4(__shfl_sync(0xffffffffu, v.x, src), __shfl_sync(0xffffffffu, v.y, src),
                   __shfl_sync(0xffffffffu, v.z, src), __shfl_sync(0xffffffffu, v.w, src));
}
__device__ __forceinline__ int2 shfl2(const int2& v, int src) {
  return make_int2(__shfl_sync(0xffffffffu, v.x, src), __shfl_sync(0xffffffffu, v.y, src));
}

// Records [begin, end) of a plan array read by a whole warp 32 at a time (one per lane) with the
// next 32 in flight, so that a role walking the script never waits on a global load per record.
// get(n) (n increasing, warp-uniform) returns record n to every lane.
template <typename T>
struct WarpStream {
  const T* p;
  int end, base;
  T cur, nxt;
  __device__ __forceinline__ T fetch(int b) const {
    const int i = b + (int)(threadIdx.x & 31);
    T v{};
    if (i < end) v = p[i];
    return v;
  }
  __device__ __forceinline__ void start(const T* p_, int begin, int end_) {
    p = p_;
    end = end_;
    base = begin;
    cur = fetch(base);
    nxt = fetch(base + 32);
  }
  __device__ __forceinline__ T get(int n) {
    while (n >= base + 32) {
      base += 32;
      cur = nxt;
      nxt = fetch(base + 32);
    }
    if constexpr (sizeof(T) == 16)
      return shfl4(cur, n - base);
    else
      return shfl2(cur, n - base);
  }
};

template <int K>
__global__ void __launch_bounds__(kRingThreads, 1) contract_ring_kernel(const __grid_constant__ CUtensorMap ymap,
                                                                        RingArgs a) {
  constexpr int N = 16 * K;
  constexpr uint32_t kstep_bytes = 2u * N * 16u;  // one Toeplitz K-step: 2 octets x N columns x 16 bytes
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sX = smem;
  uint8_t* sB = sX + (size_t)a.ns * a.slot_bytes;
  // y staging: 1024-byte aligned for the 128-byte swizzle of the stores
  uint8_t* sY = smem + (((size_t)a.ns * a.slot_bytes + (size_t)a.nbs * a.bslot_bytes + 1023) & ~(size_t)1023);
  uint64_t* xfull = reinterpret_cast<uint64_t*>(sY + (size_t)4 * a.ystage_bytes);
  uint64_t* xempty = xfull + kMaxSlots;
  uint64_t* bfull = xempty + kMaxSlots;
  uint64_t* bempty = bfull + kMaxBslots;
  uint64_t* tfull = bempty + kMaxBslots;
  uint64_t* tempty = tfull + kMaxBufs;
  uint64_t* drain = tempty + kMaxBufs;
  int4* sItem = reinterpret_cast<int4*>(drain + 2);  // the record of the item in each B slot
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sItem + kMaxBslots);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxSlots; ++s) {
      tc::mbar_init(&xfull[s], 32 * kXWarps);  // every copy lane's cp.async completions
      tc::mbar_init(&xempty[s], kIssuers);  // every issuer commits its last use
    }
    for (int s = 0; s < kMaxBslots; ++s) {
      tc::mbar_init(&bfull[s], 1);
      tc::mbar_init(&bempty[s], kIssuers);
    }
    for (int s = 0; s < kMaxBufs; ++s) {
      tc::mbar_init(&tfull[s], kIssuers);
      tc::mbar_init(&tempty[s], 4);
    }
    tc::mbar_init(drain, kIssuers);
    tc::fence_barrier_init();
  }
  if (warp == 4) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------------ x copies
    // the strip's loads in order, each as soon as its ring slot is free (its previous load has had
    // its last use).  A load is n_oct octets x 2 groups x 64 planes of 16 bytes; a warp
    // instruction covers 4 octets x 8 planes, and the four copy warps take turns over the
    // (group, plane octet, octet quad) units.  Every lane's copies arrive on the slot's barrier
    // when they land.
    const int pw = warp - 8;
    const int osub = lane & 3, psub = lane >> 2;
    const size_t chan = (size_t)a.n_src_rows * a.nlon;
    uint32_t xpar = 0, xused = 0;  // per ring slot: parity of loads issued, slot used before
    bool ok = true;
    WarpStream<int2> ls;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      const TileInfo t = tile_info(a, tile);
      const int q8 = t.q0 / 8;
      ls.start(a.loads, t.load0, t.load1);
      for (int l = t.load0; l < t.load1 && ok; ++l) {
        const int2 ld = ls.get(l);
        const int s = ld.x & 0xFFFF, sbar = (ld.x >> 16) & 0xFFFF;
        const int o0 = (int)(int16_t)(ld.y & 0xFFFF);
        const int n_oct = (ld.y >> 16) & 0xFF, slot = (ld.y >> 24) & 0xF;
        const uint32_t bit = 1u << slot;
        if (xused & bit) {
          int good = 1;
          if (lane == 0) good = tc::mbar_wait_sleep(&xempty[slot], ((xpar >> slot) & 1u) ^ 1u);
          if (!__shfl_sync(0xffffffffu, good, 0)) {
            ok = false;
            break;
          }
          __syncwarp();  // every lane's copies after lane 0's wait
        }
        xpar ^= bit;
        xused |= bit;
        uint8_t* dst = sX + (size_t)slot * a.slot_bytes;
        const int nq = (n_oct + 3) >> 2;
        for (int u = pw; u < 16 * nq; u += kXWarps) {
          const int g = u & 1, pg = (u >> 1) & 7, oq = u >> 4;
          const int o = 4 * oq + osub;
          if (o < n_oct) {
            int oc = (q8 + o0 + o) % a.ring_oct;
            if (oc < 0) oc += a.ring_oct;
            const int row = (g == 1 && a.mirror) ? sbar : s;
            const int plane = t.plane0 + pg * 8 + psub + ((g == 1 && !a.mirror) ? 64 : 0);
            const bool valid = plane < a.BC;
            const __nv_bfloat16* src = a.x + (valid ? (size_t)plane * chan + (size_t)row * a.nlon + oc * 8 : 0);
            tc::cp_async16(dst + (size_t)o * kOct + g * (kOct / 2) + (pg * 8 + psub) * 16, src, valid ? 16u : 0u);
          }
        }
        tc::cp_async_arrive_noinc(&xfull[slot]);
      }
    }
    // no copy may still be in flight when the CTA exits
    tc::cp_async_wait_all();
  } else if (warp == 12) {
    // ------------------------------------------------------------------ B copies
    // each item's Toeplitz K-steps into the next B slot, as soon as the slot's previous item is done,
    // with the item's record beside it (the MMA issuers read it after the slot's barrier)
    uint32_t nbload = 0;
    bool ok = true;
    WarpStream<int4> is;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      const TileInfo t = tile_info(a, tile);
      is.start(a.items, t.item0, t.item1);
      for (int n = t.item0; n < t.item1 && ok; ++n) {
        const int4 it = is.get(n);
        const int bs = (int)(nbload % (uint32_t)a.nbs);
        int good = 1;
        if (lane == 0) {
          if (nbload >= (uint32_t)a.nbs) good = tc::mbar_wait_sleep(&bempty[bs], ((nbload / a.nbs) - 1) & 1u);
          if (good) {
            const int nkb = (it.z >> 8) & 0xFF;
            const uint32_t bytes = (uint32_t)nkb * kstep_bytes;
            sItem[bs] = it;  // published by the arrival below (release), read after the wait (acquire)
            tc::mbar_arrive_expect_tx(&bfull[bs], bytes);
            tc::bulk_load(sB + (size_t)bs * a.bslot_bytes, a.b + (size_t)(uint32_t)it.w * 16, bytes, &bfull[bs]);
          }
        }
        ok = __shfl_sync(0xffffffffu, good, 0) != 0;
        ++nbload;
      }
    }
    if (lane == 0) {
      const uint32_t first = nbload > (uint32_t)a.nbs ? nbload - a.nbs : 0;
      for (uint32_t m = first; m < nbload; ++m) tc::mbar_wait(&bfull[m % a.nbs], (m / a.nbs) & 1u);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ MMA issuers
    // A thread issuing tcgen05.mma waits about 150-190 cycles per instruction whatever its N, while
    // the tensor core can take an N = 48 MMA every ~45 cycles: four threads (lane 0 of warps 4..7,
    // one per SM sub-partition) issue side by side, each the MMAs of its own blocks of 16 outputs.
    // Each walks all the items, reading an item's record from its B slot after the slot's barrier,
    // and every issuer's commit counts in the barriers that release a B slot, a ring slot or a row.
    if (lane == 0) {
      const int iw = warp - 4;
      constexpr uint32_t idesc = tc::idesc_bf16(128, N, false, false);
      const uint64_t a_fix = tc::desc_noswz(0, kOct, 128);
      const uint64_t b_fix = tc::desc_noswz(0, (uint32_t)N * 16, 128);
      uint32_t xpar = 0;               // per slot: parity of loads consumed
      uint32_t rpar = 0, rused = 0;    // per row buffer: parity of rows started, used before
      unsigned long long started = 0;  // per (buffer, block): accumulator holds a partial sum
      uint32_t nbc = 0;
      const uint32_t sX4 = tc::smem_u32(sX) >> 4, sB4 = tc::smem_u32(sB) >> 4;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
        const TileInfo t = tile_info(a, tile);
        int last_load = -1;
        for (int n = t.item0; n < t.item1; ++n) {
          const int bs = (int)(nbc % (uint32_t)a.nbs);
          if (!tc::mbar_wait_sleep(&bfull[bs], (nbc / a.nbs) & 1u, 64)) {
            ok = false;
            break;
          }
          ++nbc;
          int4 cur;
          asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(cur.x), "=r"(cur.y), "=r"(cur.z), "=r"(cur.w)
                       : "r"(tc::smem_u32(&sItem[bs]))
                       : "memory");
          const int L = cur.x & 0xFFFF;
          const int slot = (cur.z >> 28) & 0xF, rb = (cur.z >> 24) & 0xF;
          const int flags = (cur.y >> 24) & 0xFF;
          if (L > last_load) {
            if (!tc::mbar_wait_sleep(&xfull[slot], (xpar >> slot) & 1u, 64)) {
              ok = false;
              break;
            }
            xpar ^= 1u << slot;
            last_load = L;
          }
          if (flags & kItemRowStart) {
            if ((rused & (1u << rb)) && !tc::mbar_wait_sleep(&tempty[rb], ((rpar >> rb) & 1u) ^ 1u)) {
              ok = false;
              break;
            }
            rpar ^= 1u << rb;
            rused |= 1u << rb;
            started &= ~(0xFFull << (8 * rb));
            tc::fence_after_sync();
          }
          const int a_off = (int)(int16_t)(cur.y & 0xFFFF), ks = (cur.y >> 16) & 0xFF;
          const int kb0 = cur.z & 0xFF, nkb = (cur.z >> 8) & 0xFF, n_oct = (cur.z >> 16) & 0xFF;
          const uint32_t d0 = tmem + (uint32_t)(rb * a.nb * N);
          const uint32_t abase = sX4 + (uint32_t)(slot * a.slot_bytes >> 4);
          const uint32_t bbase = sB4 + (uint32_t)(bs * a.bslot_bytes >> 4);
          for (int b = iw; b < a.nb; b += kIssuers) {
            // K-steps of block b inside this item and this load
            const int base = a_off + 2 * b;                   // octet of K-step 0
            int k_lo = kb0, k_hi = min(kb0 + nkb, ks);
            k_lo = max(k_lo, (-base + 1) >> 1);               // base + 2k >= 0
            k_hi = min(k_hi, ((n_oct - 2 - base) >> 1) + 1);  // base + 2k + 2 <= n_oct
            const unsigned long long sb = 1ull << (8 * rb + b);
            for (int k = k_lo; k < k_hi; ++k) {
              const uint64_t ad = a_fix | (uint64_t)(abase + (uint32_t)((base + 2 * k) * (kOct >> 4)));
              const uint64_t bd = b_fix | (uint64_t)(bbase + (uint32_t)((k - kb0) * (kstep_bytes >> 4)));
              tc::mma_bf16(d0 + (uint32_t)(b * N), ad, bd, idesc, (started & sb) ? 1u : 0u);
              started |= sb;
            }
          }
          tc::mma_commit(&bempty[bs]);
          if (flags & kItemLast) tc::mma_commit(&xempty[slot]);
          if (flags & kItemRowEnd) tc::mma_commit(&tfull[rb]);
        }
      }
      // every MMA issued has completed before tensor memory is released
      tc::mma_commit(drain);
      tc::mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    // each warp drains its TMEM lane quadrant: 32 planes of group quad / 2, into its own
    // [32 planes][K][64] bf16 tile (128-byte rows in the 128-byte swizzle of its TMA store map),
    // one TMA store per row; no cross-warp barrier
    const int quad = warp;
    const int grp = quad >> 1, pl0 = (quad & 1) * 32;
    uint8_t* wy = sY + (size_t)warp * a.ystage_bytes;
    if (lane == 0) tc::prefetch_map(&ymap);
    uint32_t epar = 0;
    bool ok = true;
    WarpStream<int2> rs;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      const TileInfo t = tile_info(a, tile);
      rs.start(a.rows, t.row0, t.row1);
      for (int rr = t.row0; rr < t.row1 && ok; ++rr) {
        const int2 rec = rs.get(rr);
        const int r = rec.x & 0xFFFF, rbar = (rec.x >> 16) & 0xFFFF;
        const bool empty = rec.y & kRowEmpty;
        const int rb = (rec.y >> 8) & 0xF;
        if (!empty) {
          int good = 1;
          if (lane == 0) good = tc::mbar_wait_sleep(&tfull[rb], (epar >> rb) & 1u, 1024);
          ok = __shfl_sync(0xffffffffu, good, 0) != 0;
          if (!ok) break;
          epar ^= 1u << rb;
          tc::fence_after_sync();
        }
        // destination of this warp's planes: the row (group 0, or the next 64 planes) or the
        // mirror row (group 1 with mirror rows; none for the self-mirror equator row)
        int drow = r, dplane = t.plane0 + pl0;
        bool store = true;
        if (grp == 1) {
          if (a.mirror) {
            drow = rbar;
            store = rbar != r && rbar != 0xFFFF;
          } else {
            dplane += 64;
          }
        }
        // the staging tile is free once the previous row's store has read it
        if (lane == 0) tc::bulk_wait_read0();
        __syncwarp();
        const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(rb * kRingNb * N);
#pragma unroll 1
        for (int b = 0; b < kRingNb; ++b) {
#pragma unroll
          for (int k = 0; k < K; ++k) {
            uint32_t v[16];
            if (!empty) {
              tc::tmem_ld_chunks<1>(tb + (uint32_t)(b * N + 16 * k), v);
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = 0u;
            }
            uint4 w0, w1;
            uint32_t* p0 = reinterpret_cast<uint32_t*>(&w0);
            uint32_t* p1 = reinterpret_cast<uint32_t*>(&w1);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
              const __nv_bfloat162 h1 =
                  __floats2bfloat162_rn(__uint_as_float(v[8 + 2 * e]), __uint_as_float(v[8 + 2 * e + 1]));
              p0[e] = *reinterpret_cast<const uint32_t*>(&h0);
              p1[e] = *reinterpret_cast<const uint32_t*>(&h1);
            }
            // row R = (plane, k) of 128 bytes; 16-byte chunk c = 2b (+1) lands at c ^ (R % 8)
            const int R = lane * K + k;
            uint8_t* rowp = wy + (size_t)R * 128;
            *reinterpret_cast<uint4*>(rowp + (((2 * b) ^ (R & 7)) << 4)) = w0;
            *reinterpret_cast<uint4*>(rowp + (((2 * b + 1) ^ (R & 7)) << 4)) = w1;
          }
        }
        if (!empty) {
          // accumulator drained: the MMA issuers may start another row in the buffer
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&tempty[rb]);
        }
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          if (store) tc::tma_store_4d(&ymap, wy, t.q0, drow, 0, dplane);
          tc::bulk_commit();
        }
      }
    }
    if (lane == 0) tc::bulk_wait0();
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 4) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int K>
cudaError_t launch_ring(const RingLaunch& L, const void* src, void* dst, cudaStream_t st) {
  constexpr int N = 16 * K;
  if (L.K != K || L.nb != kRingNb) return cudaErrorInvalidValue;
  if (L.ns > kMaxSlots || L.nrb > kMaxBufs || L.nbs > kMaxBslots || L.nrb * kRingNb * N > 512)
    return cudaErrorInvalidValue;
  RingArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(src);
  a.BC = L.BC;
  a.n_src_rows = L.n_src_rows;
  a.strips = reinterpret_cast<const int4*>(L.strips);
  a.loads = reinterpret_cast<const int2*>(L.loads);
  a.items = reinterpret_cast<const int4*>(L.items);
  a.rows = reinterpret_cast<const int2*>(L.rows);
  a.b = static_cast<const uint8_t*>(L.b);
  a.nb = kRingNb;
  a.ns = L.ns;
  a.nrb = L.nrb;
  a.nbs = L.nbs;
  a.bk = L.bk;
  a.mirror = L.mirror;
  a.plane_tile = L.mirror ? 64 : 128;
  a.nlon = L.nlon;
  a.ring_oct = L.nlon / 8;
  a.n_qt = (L.nlon + 16 * kRingNb - 1) / (16 * kRingNb);
  a.n_pt = (L.BC + a.plane_tile - 1) / a.plane_tile;
  a.n_tiles = L.n_strips * a.n_qt * a.n_pt;
  a.slot_bytes = (uint32_t)L.wmax * kOct;
  a.bslot_bytes = (uint32_t)L.bk * 2u * N * 16u;
  a.ystage_bytes = (uint32_t)(32 * K * 128);  // one warp's row: 32 planes x K x 64 outputs
  const size_t bars = 8 * (2 * kMaxSlots + 2 * kMaxBslots + 2 * kMaxBufs + 2) + 16 * kMaxBslots + 16;
  const size_t smem = 2048 + (size_t)L.ns * a.slot_bytes + (size_t)L.nbs * a.bslot_bytes +
                      (size_t)4 * a.ystage_bytes + bars;
  if (smem > kTcSmemLimit) return cudaErrorInvalidValue;
  // output as [BC][K][n_out_rows][nlon]: boxes of 64 longitudes x 1 row x K x 32 planes, 128-byte
  // swizzle (the staging tile's rows are 128 bytes)
  CUtensorMap ym;
  {
    const cuuint64_t dims[4] = {(cuuint64_t)L.nlon, (cuuint64_t)L.n_out_rows, (cuuint64_t)K, (cuuint64_t)L.BC};
    const cuuint64_t strides[3] = {(cuuint64_t)L.nlon * 2, (cuuint64_t)L.n_out_rows * L.nlon * 2,
                                   (cuuint64_t)K * L.n_out_rows * L.nlon * 2};
    const cuuint32_t box[4] = {16 * kRingNb, 1, (cuuint32_t)K, 32};
    if (!tc::encode_bf16_map(&ym, dst, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  }
  const void* kernel = reinterpret_cast<const void*>(&contract_ring_kernel<K>);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = std::min(a.n_tiles, sms);
  if (grid <= 0) return cudaSuccess;
  void* args[] = {&ym, &a};
  e = cudaLaunchKernel(kernel, dim3(grid), dim3(kRingThreads), args, smem, st);
  count_launch();
  return e;
}

// Self test of the bounded waits: one thread waits on an mbarrier that nothing arrives on, for at
// most limit_ns, and records the timeout in this file's status word like every expired wait.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  tc::mbar_init(&bar, 1);
  tc::fence_barrier_init();
  tc::mbar_wait_for(&bar, 0, limit_ns);
}

}  // namespace

cudaError_t launch_wait_selftest(unsigned int limit_us, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(1000ull * limit_us);
  count_launch();
  return cudaGetLastError();
}

bool ring_kernel_k(int K) { return K == 1 || K == 3 || K == 5 || K == 9; }

cudaError_t launch_contract_ring(const RingLaunch& L, const void* src, void* dst, cudaStream_t st) {
  if ((reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15) || L.nlon % 8)
    return cudaErrorInvalidValue;
  switch (L.K) {
    case 1: return launch_ring<1>(L, src, dst, st);
    case 3: return launch_ring<3>(L, src, dst, st);
    case 5: return launch_ring<5>(L, src, dst, st);
    case 9: return launch_ring<9>(L, src, dst, st);
    default: return cudaErrorInvalidValue;
  }
}

int take_contract_ring_status() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
  return v;
}

}  // namespace disco
