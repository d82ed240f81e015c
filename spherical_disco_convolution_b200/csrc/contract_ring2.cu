// TMA-staged strip contraction (tcgen05, sm_100a) for bf16 signals, stride 1.
//
// The contraction of the page "torch_harmonics.DiscreteContinuousConvS2" (class description),
//     y[c, k, j, q] = sum_i sum_p Psi_k(j, i, p) x[c, i, (q + p) mod nlon],
// is, for an output row j and a source row i, a correlation along the longitude ring with the
// same coefficients for every output longitude (the p-shift symmetry).  For 16 consecutive
// outputs it is one product with a banded Toeplitz block of Psi per 16 source longitudes
// (ring_plan2.cpp), run here as tcgen05 MMAs:
//   * A = 128 rows x 16 source longitudes from a staged chunk: [2 groups][64 planes][64
//     longitudes] bf16, 128-byte rows in the 128-byte swizzle, written by two TMA boxes; group 0
//     holds the source row of the output row, group 1 either the mirror source row of the mirror
//     output row (whose Toeplitz blocks are the same) or the next 64 planes.  A K-step starts at
//     any 16-byte octet of a row that leaves room for two.
//   * B = the Toeplitz K-step, [2 octets][N = 16K][8] bf16 (K-major, no swizzle), copied in
//     batches with bulk copies; a batch's B slot also holds its record (the issuers' MMA lists,
//     the loads and rows that start in it).
//   * D = fp32 in tensor memory: rows = (group, plane), columns = (k, u) for each block of 16
//     outputs, four blocks per row buffer.
// A tile is (strip of consecutive output rows, 64 output longitudes, plane tile); the host wrote
// one script per (strip, longitude tile) with every shared-memory address, seam split and
// synchronisation fixed, and the CTAs take the scripts in the order the host balanced.
// Roles: one thread stages the windows with TMA boxes, one thread copies the B batches, four
// MMA issuers (issuer b: block b) issue the MMA lists of each batch's record, one thread follows the
// completion of the batches, and four epilogue warps read finished rows from tensor memory,
// round them to bf16 and store them with TMA, one kernel index at a time through one staging
// buffer per warp.  The issuers commit once per B batch: the completion of a batch releases its
// B slot, and also every ring slot and finished row whose last use it holds (the host chose the
// batches, slots and row buffers so that none is needed before it is released).
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

constexpr int kIssuers = 4;
constexpr int kThreads = 352;   // warps 0-3 epilogue, 4-7 issuers, 8 x staging, 9 B copies, 10 batch tracking
constexpr int kNb = 4;          // blocks of 16 outputs per tile
constexpr int kMaxSlots = 8, kMaxBufs = 8, kMaxBslots = 8;
constexpr uint32_t kYBuf = 32 * 128;  // one staging buffer: 32 planes x 64 outputs bf16

struct Args {
  const int4* tiles;   // kTileInts ints per script, read as int4 x 4
  const int4* loads;
  const int4* copies;
  const uint32_t* cmds;
  const int2* rows;
  const int* cta_tiles;
  const uint8_t* b;
  int n_ctas, n_qt, n_pt, plane_tile, mirror, BC;
  int ns, nbs, nrb;
  uint32_t bslot_bytes;
  // fused forward: out = W y + bias instead of y
  const __nv_bfloat16* w;     // [C_out][64][K], or [64][C_out][K] with w_t (the adjoint's W^T)
  const __nv_bfloat16* bias;  // [C_out] or null
  int C_out, w_t;
};

__device__ __forceinline__ int4 shfl4(const int4& v, int src) {
  return make_int4(__shfl_sync(0xffffffffu, v.x, src), __shfl_sync(0xffffffffu, v.y, src),
                   __shfl_sync(0xffffffffu, v.z, src), __shfl_sync(0xffffffffu, v.w, src));
}
__device__ __forceinline__ int2 shfl2(const int2& v, int src) {
  return make_int2(__shfl_sync(0xffffffffu, v.x, src), __shfl_sync(0xffffffffu, v.y, src));
}
__device__ __forceinline__ uint32_t shfl1(uint32_t v, int src) { return __shfl_sync(0xffffffffu, v, src); }

// Records [begin, end) of a plan array read by a whole warp 32 at a time (one per lane) with the
// next 32 in flight; get(n) (n increasing, warp-uniform) returns record n to every lane.
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
    else if constexpr (sizeof(T) == 8)
      return shfl2(cur, n - base);
    else
      return shfl1(cur, n - base);
  }
};


// A window of 32 records of a plan array held by a warp (one per lane) with the next 32 in
// flight; at(l) (l increasing, warp-uniform) returns record l + lane to each lane (records past
// the end read as zeros).
template <typename T>
struct WarpWindow {
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
  __device__ __forceinline__ T at(int l) {
    while (l >= base + 32) {
      base += 32;
      cur = nxt;
      nxt = fetch(base + 32);
    }
    const int i = l - base + (int)(threadIdx.x & 31);  // 0 .. 62
    const T a = shfl_any(cur, i & 31), b = shfl_any(nxt, i & 31);
    return i < 32 ? a : b;
  }
  __device__ __forceinline__ static T shfl_any(const T& v, int src) {
    if constexpr (sizeof(T) == 16)
      return shfl4(v, src);
    else
      return shfl2(v, src);
  }
};

struct Script {
  int load0, load1, copy0, copy1, row0, row1, nbatch;
};
__device__ __forceinline__ Script read_script(const Args& a, int si, int) {
  const int4* r = a.tiles + 4 * si;
  const int4 r0 = r[0], r1 = r[1], r2 = r[2];
  Script s;
  s.load0 = r0.x;
  s.load1 = r0.y;
  s.copy0 = r0.z;
  s.copy1 = r0.w;
  s.row0 = r1.x;
  s.row1 = r1.y;
  s.nbatch = r2.w;
  return s;
}

// Prefetch of [p, p + bytes) into L2 (16-byte aligned start and size; no-op for an empty range).
__device__ __forceinline__ void l2_prefetch(const void* p, uint32_t bytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(p) & ~static_cast<uintptr_t>(15);
  const uint32_t n = (uint32_t)((reinterpret_cast<uintptr_t>(p) + bytes + 15 - a0) & ~static_cast<uintptr_t>(15));
  if (bytes == 0) return;
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a0), "r"(n) : "memory");
}

// Batches completed by this CTA (a counter in shared memory written by the tracking thread).
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(tc::smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(tc::smem_u32(p)), "r"(v) : "memory");
}
// Waits (one thread) until at least `target` batches have completed; bounded like every wait.
__device__ __forceinline__ bool wait_batches(const uint32_t* done, uint32_t target, uint32_t max_sleep_ns) {
  if (ld_acquire(done) >= target) return true;
  const unsigned long long t0 = tc::globaltimer();
  if (max_sleep_ns == 0) {
    // no sleep: the x producer and the B warp, whose wake-up would delay the slots they refill
    while (true) {
      for (int i = 0; i < 64; ++i)
        if (ld_acquire(done) >= target) return true;
      if (tc::globaltimer() - t0 > tc::kWaitNs) {
        atomicExch(&g_device_status, 5);
        return false;
      }
    }
  }
  uint32_t ns = 32;
  while (true) {
    if (ld_acquire(done) >= target) return true;
    __nanosleep(ns);
    if (ns < max_sleep_ns) ns <<= 1;
    if (tc::globaltimer() - t0 > tc::kWaitNs) {
      atomicExch(&g_device_status, 5);
      return false;
    }
  }
}

template <int K, bool kFused>
__global__ void __launch_bounds__(kThreads, 1) contract_ring2_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                      const __grid_constant__ CUtensorMap ymap,
                                                                      Args a) {
  // the x producer and the B warp spin on the batch counter in the plain contraction; in the
  // fused forms, whose epilogue warps share their issue slots, they sleep between polls
  constexpr uint32_t kProducerSleepNs = kFused ? 256u : 0u;
  constexpr int N = 16 * K;
  constexpr uint32_t kWBytes = kFused ? (uint32_t)K * 8192u : 0u;  // W_k tiles [64 o][64 c] of the mix
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sX = smem;                                          // ns slots of two chunks
  uint8_t* sB = sX + (size_t)a.ns * kSlotBytes;                // nbs B slots
  uint8_t* sW = sB + (((size_t)a.nbs * a.bslot_bytes + 1023) & ~(size_t)1023);  // fused: the mix weights
  // one buffer per epilogue warp; fused: one per warp and kernel index ([k][warp][32 rows][128 B],
  // the mix's y operand: group g of index k is 64 rows at k * 16 KB + g * 8 KB)
  uint8_t* sY = sW + kWBytes;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(sY + (kFused ? K : 1) * 4 * kYBuf);
  uint64_t* bfull = xfull + kMaxSlots;
  uint64_t* bempty = bfull + kMaxBslots;
  uint64_t* tempty = bempty + kMaxBslots;
  uint64_t* drain = tempty + kMaxBufs;
  uint64_t* mixb = drain + 1;  // fused: the mix MMAs of mirror group 0 / 1 completed
  uint32_t* done = reinterpret_cast<uint32_t*>(mixb + 2);  // batches completed
  uint32_t* tmem_slot = done + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxSlots; ++s) tc::mbar_init(&xfull[s], 1);  // the staging thread, with the box bytes
    for (int s = 0; s < kMaxBslots; ++s) {
      tc::mbar_init(&bfull[s], 1);
      tc::mbar_init(&bempty[s], kIssuers);  // every issuer commits the batch
    }
    for (int s = 0; s < kMaxBufs; ++s) tc::mbar_init(&tempty[s], 4);
    tc::mbar_init(drain, kIssuers);
    tc::mbar_init(&mixb[0], 1);
    tc::mbar_init(&mixb[1], 1);
    *done = 0;
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
  const int* my = a.cta_tiles + (a.n_ctas + 1);
  const int t_begin = a.cta_tiles[blockIdx.x], t_end = a.cta_tiles[blockIdx.x + 1];

  if (warp == 8) {
    // ------------------------------------------------------------------ x staging
    // each load: wait until the batch that held the last use of its slot's previous load has
    // completed, then the chunks' boxes (64 longitudes x 64 planes, both groups) onto the slot's
    // barrier
    if (lane == 0) tc::prefetch_map(&xmap);
    uint32_t rel[kMaxSlots];  // per slot: batches that must complete before it is refilled
#pragma unroll
    for (int s = 0; s < kMaxSlots; ++s) rel[s] = 0;
    uint32_t gbase = 0;  // batches of the scripts before this one
    bool ok = true;
    WarpStream<int4> ls;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Script sc = read_script(a, my[t], -1);
      if (lane == 0 && t + 1 < t_end) {
        const Script nx = read_script(a, my[t + 1], -1);
        l2_prefetch(a.loads + nx.load0, (uint32_t)(nx.load1 - nx.load0) * 16u);
      }
      for (int pt = 0; pt < a.n_pt && ok; ++pt) {
        const int plane0 = pt * a.plane_tile;
        ls.start(a.loads, sc.load0, sc.load1);
        for (int l = sc.load0; l < sc.load1 && ok; ++l) {
          const int4 ld = ls.get(l);
          const int slot = ld.y & 0xFF, mask = (ld.y >> 8) & 3;
          uint32_t need = 0;
#pragma unroll
          for (int s = 0; s < kMaxSlots; ++s)
            if (s == slot) need = rel[s];
          int good = 1;
          if (lane == 0) {
            if (need) good = wait_batches(done, need, kProducerSleepNs);
            if (good) {
              const int src = ld.x & 0xFFFF, sbar = (ld.x >> 16) & 0xFFFF;
              tc::mbar_arrive_expect_tx(&xfull[slot], (uint32_t)__popc(mask) * (uint32_t)kChunkBytes);
              uint8_t* dst = sX + (size_t)slot * kSlotBytes;
#pragma unroll
              for (int c = 0; c < 2; ++c)
                if (mask & (1 << c)) {
                  tc::tma_load_3d(dst + c * kChunkBytes, &xmap, &xfull[slot], ld.z + 56 * c, src, plane0);
                  tc::tma_load_3d(dst + c * kChunkBytes + kChunkBytes / 2, &xmap, &xfull[slot], ld.z + 56 * c,
                                  a.mirror ? sbar : src, a.mirror ? plane0 : plane0 + 64);
                }
            }
          }
          ok = __shfl_sync(0xffffffffu, good, 0) != 0;
          const uint32_t r = gbase + (uint32_t)(ld.w & 0xFFFF) + 1;
#pragma unroll
          for (int s = 0; s < kMaxSlots; ++s)
            if (s == slot) rel[s] = r;
        }
        gbase += (uint32_t)sc.nbatch;
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ B copies
    // each batch: wait until its B slot's previous batch has completed, arm the slot's barrier
    // with the batch's bytes, and issue its copies (the record, then the items' K-steps), one
    // per lane
    int bslot = 0;
    uint32_t nbatch = 0;  // batches started by this CTA
    bool ok = true;
    WarpWindow<int4> win;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Script sc = read_script(a, my[t], -1);
      if (lane == 0 && t + 1 < t_end) {
        const Script nx = read_script(a, my[t + 1], -1);
        l2_prefetch(a.copies + nx.copy0, (uint32_t)(nx.copy1 - nx.copy0) * 16u);
      }
      for (int pt = 0; pt < a.n_pt && ok; ++pt) {
        win.start(a.copies, sc.copy0, sc.copy1);
        for (int c = sc.copy0; c < sc.copy1 && ok;) {
          const int4 cp = win.at(c);  // copy c + lane; copy c is the batch record's
          const int w0 = __shfl_sync(0xffffffffu, cp.w, 0);
          const int n = (w0 >> 24) & 0xFF;
          int good = 1;
          if (lane == 0) {
            if (nbatch >= (uint32_t)a.nbs) good = wait_batches(done, nbatch - a.nbs + 1, kProducerSleepNs);
            if (good) tc::mbar_arrive_expect_tx(&bfull[bslot], (uint32_t)((w0 >> 8) & 0xFFFF));
          }
          ok = __shfl_sync(0xffffffffu, good, 0) != 0;
          if (!ok) break;
          if (lane < n) {
            const uint8_t* src = (cp.w & kCopyMeta) ? reinterpret_cast<const uint8_t*>(a.cmds) : a.b;
            tc::bulk_load(sB + (size_t)bslot * a.bslot_bytes + cp.z, src + (size_t)(uint32_t)cp.x * 16, (uint32_t)cp.y,
                          &bfull[bslot]);
          }
          c += n;
          ++nbatch;
          bslot = (bslot + 1 == a.nbs) ? 0 : bslot + 1;
        }
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------------ batch tracking
    // waits for every batch's completion in order (the issuers' commits) and publishes the count;
    // waiting in order on each B slot's barrier sees every one of its phases
    if (lane == 0) {
      int bslot = 0;
      uint32_t n = 0, bpar = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const Script sc = read_script(a, my[t], -1);
        for (int pt = 0; pt < a.n_pt && ok; ++pt)
          for (int b = 0; b < sc.nbatch; ++b) {
            if (!tc::mbar_wait_sleep(&bempty[bslot], (bpar >> bslot) & 1u, 32)) {
              ok = false;
              break;
            }
            bpar ^= 1u << bslot;
            st_release(done, ++n);
            bslot = (bslot + 1 == a.nbs) ? 0 : bslot + 1;
          }
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ MMA issuers
    // Four issuers (one per SM sub-partition), issuer b the MMAs of block b.  Per batch each waits
    // for the batch's B slot (which holds the batch record and the Toeplitz K-steps), for the
    // loads first used in the batch and for the row buffers whose rows start in it, issues its
    // list of MMAs from the record and commits the batch.
    if (lane == 0) {
      const int iw = warp - 4;
      constexpr uint32_t idesc = tc::idesc_bf16(128, N, false, false);
      // A: 128-byte swizzle, 8-row groups 1024 bytes apart; B: no swizzle, K-octets N*16 apart
      const uint64_t a_fix = tc::desc_sw128(0, 16, 1024);
      const uint64_t b_fix = tc::desc_noswz(0, (uint32_t)N * 16, 128);
      const uint32_t sX4 = tc::smem_u32(sX) >> 4;
      const uint32_t dcol = tmem + (uint32_t)(iw * N);
      uint32_t xpar = 0, bpar = 0, rpar = 0, rused = 0;
      int bcur = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const Script sc = read_script(a, my[t], -1);
        for (int pt = 0; pt < a.n_pt && ok; ++pt)
          for (int bt = 0; bt < sc.nbatch; ++bt) {
            if (!tc::mbar_wait_sleep(&bfull[bcur], (bpar >> bcur) & 1u, 64)) {
              ok = false;
              break;
            }
            bpar ^= 1u << bcur;
            const uint8_t* slotp = sB + (size_t)bcur * a.bslot_bytes;
            const uint32_t* rec = reinterpret_cast<const uint32_t*>(slotp);
            const uint4 h = *reinterpret_cast<const uint4*>(rec);
            const int n = (int)((h.x >> (8 * iw)) & 0xFFu);
            const int off = iw == 0 ? 4 : (int)((h.y >> (10 * (iw - 1))) & 0x3FFu);
            // loads first used in this batch
            const int nls = (int)(h.z & 7u);
            for (int j = 0; j < nls && ok; ++j) {
              const int slot = (int)((h.z >> (3 + 4 * j)) & 0xFu);
              if (!tc::mbar_wait_sleep(&xfull[slot], (xpar >> slot) & 1u, 64)) ok = false;
              xpar ^= 1u << slot;
            }
            // rows that start in this batch: their buffers must have been drained
            const int nrs = (int)(h.w & 7u);
            for (int j = 0; j < nrs && ok; ++j) {
              const int rb = (int)((h.w >> (3 + 3 * j)) & 7u);
              if ((rused & (1u << rb)) && !tc::mbar_wait_sleep(&tempty[rb], ((rpar >> rb) & 1u) ^ 1u, 32)) ok = false;
              rpar ^= 1u << rb;
              rused |= 1u << rb;
            }
            if (!ok) break;
            if (nrs) tc::fence_after_sync();
            const uint32_t bbase = tc::smem_u32(slotp) >> 4;
            const uint32_t* m = rec + off;
            auto issue = [&](uint32_t w) {
              tc::mma_bf16(dcol + ((w >> 24) & 7u) * (uint32_t)(kNb * N), a_fix | (uint64_t)(sX4 + (w & 0x3FFFu)),
                           b_fix | (uint64_t)(bbase + ((w >> 14) & 0x3FFu)), idesc, (w >> 27) & 1u);
            };
            int i = 0;
            for (; i + 2 <= n; i += 2) {
              const uint32_t w0 = m[i], w1 = m[i + 1];
              issue(w0);
              issue(w1);
            }
            if (i < n) issue(m[i]);
            tc::mma_commit(&bempty[bcur]);
            bcur = (bcur + 1 == a.nbs) ? 0 : bcur + 1;
          }
      }
      // every MMA issued has completed before tensor memory is released
      tc::mma_commit(drain);
      tc::mbar_wait(drain, 0);
    }
    __syncwarp();
  } else if (warp < 4 && !kFused) {
    // ------------------------------------------------------------------ epilogue warps
    // each warp drains its TMEM lane quadrant (32 planes of group quad / 2) once the batch that
    // holds the row's last MMA has completed, one kernel index at a time, into a [32 planes][64
    // outputs] bf16 buffer (128-byte rows, 128-byte swizzle) stored with one TMA store
    const int quad = warp;
    const int grp = quad >> 1, pl0 = (quad & 1) * 32;
    uint8_t* wy = sY + (size_t)warp * kYBuf;
    if (lane == 0) tc::prefetch_map(&ymap);
    uint32_t gbase = 0;
    int nst = 0;  // stores issued by this warp
    bool ok = true;
    WarpStream<int2> rs;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const int si = my[t];
      const Script sc = read_script(a, si, -1);
      // the longitude tile of the script: scripts are strip-major, tile-minor
      const int q0 = (si % a.n_qt) * (16 * kNb);
      for (int pt = 0; pt < a.n_pt && ok; ++pt) {
        const int plane0 = pt * a.plane_tile;
        rs.start(a.rows, sc.row0, sc.row1);
        for (int rr = sc.row0; rr < sc.row1 && ok; ++rr) {
          const int2 rec = rs.get(rr);
          const int r = rec.x & 0xFFFF, rbar = (rec.x >> 16) & 0xFFFF;
          const bool empty = rec.y & kRowEmpty;
          const int rb = (rec.y >> 8) & 0xF;
          if (!empty) {
            int good = 1;
            if (lane == 0) good = wait_batches(done, gbase + (uint32_t)(rec.y >> 12) + 1, 64);
            ok = __shfl_sync(0xffffffffu, good, 0) != 0;
            if (!ok) break;
            tc::fence_after_sync();
          }
          // destination of this warp's planes: the row (group 0, or the next 64 planes) or the
          // mirror row (group 1 with mirror rows; none for the self-mirror equator row)
          int drow = r, dplane = plane0 + pl0;
          bool store = true;
          if (grp == 1) {
            if (a.mirror) {
              drow = rbar;
              store = rbar != r && rbar != 0xFFFF;
            } else {
              dplane += 64;
            }
          }
          const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(rb * kNb * N);
          // the row's values as bf16 pairs: pk[k][8b + e] = outputs 16b + 2e, +1 of kernel index k
          // (for K <= 3 all of them are read before the buffer is released, so the MMA issuers
          // may start the buffer's next row while they are staged and stored)
          constexpr int KP = K <= 3 ? K : 1;
          uint32_t pk[KP][32];
          auto load_pack = [&](int k, uint32_t (&dst)[32]) {
            uint32_t v[4 * 16];
#pragma unroll
            for (int b = 0; b < kNb; ++b)
              asm volatile(
                  "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                  "%13, %14, %15}, [%16];"
                  : "=r"(v[16 * b + 0]), "=r"(v[16 * b + 1]), "=r"(v[16 * b + 2]), "=r"(v[16 * b + 3]),
                    "=r"(v[16 * b + 4]), "=r"(v[16 * b + 5]), "=r"(v[16 * b + 6]), "=r"(v[16 * b + 7]),
                    "=r"(v[16 * b + 8]), "=r"(v[16 * b + 9]), "=r"(v[16 * b + 10]), "=r"(v[16 * b + 11]),
                    "=r"(v[16 * b + 12]), "=r"(v[16 * b + 13]), "=r"(v[16 * b + 14]), "=r"(v[16 * b + 15])
                  : "r"(tb + (uint32_t)(b * N + 16 * k)));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int i = 0; i < 64; ++i) asm volatile("" : "+r"(v[i]));
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              dst[i] = *reinterpret_cast<const uint32_t*>(&h);
            }
          };
          auto release = [&]() {
            // accumulator drained: the MMA issuers may start another row in the buffer
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[rb]);
          };
          auto stage_store = [&](int k, const uint32_t (&src)[32]) {
            // the buffer is free once the previous store has read it
            if (lane == 0) tc::bulk_wait_read0();
            __syncwarp();
            uint8_t* buf = wy;
            uint8_t* rowp = buf + (size_t)lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              // row = plane (lane) of 128 bytes; 16-byte chunk c lands at c ^ (lane % 8)
              *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(src[4 * c], src[4 * c + 1], src[4 * c + 2], src[4 * c + 3]);
            }
            tc::fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              if (store) tc::tma_store_4d(&ymap, buf, q0, drow, k, dplane);
              tc::bulk_commit();
            }
            ++nst;
          };
          if constexpr (K <= 3) {
            if (!empty) {
#pragma unroll
              for (int k = 0; k < K; ++k) load_pack(k, pk[k]);
              release();
            } else {
#pragma unroll
              for (int k = 0; k < K; ++k)
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[k][i] = 0u;
            }
#pragma unroll
            for (int k = 0; k < K; ++k) stage_store(k, pk[k]);
          } else {
#pragma unroll 1
            for (int k = 0; k < K; ++k) {
              if (!empty) {
                load_pack(k, pk[0]);
                if (k == K - 1) release();
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[0][i] = 0u;
              }
              stage_store(k, pk[0]);
            }
          }
        }
        gbase += (uint32_t)sc.nbatch;
      }
    }
    if (lane == 0) tc::bulk_wait0();
  } else if (warp < 4) {
    // ------------------------------------------------------------------ fused epilogue warps
    // out[b, o, j, q] = bias[o] + sum_{c, k} W[o, c, k] y[b, c, k, j, q] for the 64 channels c
    // of one batch element (the plane tile); with w_t the same with W[c, o, k] (the input gradient:
    // y is then the transposed contraction of dout, and out is dx).  Per row: each warp drains its TMEM lane quadrant
    // (32 channels of mirror group quad / 2) and releases the buffer; then, one kernel index k
    // at a time, the two warps of a group write y_k of their channels into their staging
    // buffers ([c][64 q], 128-byte swizzle: the MN-major B operand of the mix) and the group's
    // first warp issues the mix MMAs D_g[o, q] += W_k[o, c] y_k[c, q] (M = 128: rows 64..127
    // read past W_k and are never used; N = 64; K = the 64 channels in four steps); finally
    // warps 0 and 1 (TMEM lanes 0..63 = the output channels) read D_0 and D_1, add the bias and
    // store out for the row and its mirror row.
    const int quad = warp;
    const int grp = quad >> 1;
    if (lane == 0) tc::prefetch_map(&ymap);
    // W_k[o][c] into shared memory, K-major with the 128-byte swizzle; rows o >= C_out are zero
    for (int i = threadIdx.x; i < K * 64 * 64; i += 128) {
      const int k = i >> 12, o = (i >> 6) & 63, c = i & 63;
      const size_t wi = a.w_t ? ((size_t)c * a.C_out + o) * K + k : ((size_t)o * 64 + c) * K + k;
      const __nv_bfloat16 v = o < a.C_out ? a.w[wi] : __float2bfloat16(0.0f);
      *reinterpret_cast<__nv_bfloat16*>(sW + (size_t)k * 8192 + o * 128 + ((((c >> 3) ^ (o & 7))) << 4) + (c & 7) * 2) = v;
    }
    tc::fence_proxy_async();
    tc::named_bar_sync(1, 128);
    constexpr uint32_t midesc = tc::idesc_bf16(128, 64, false, true);
    const uint32_t dmix = tmem + (uint32_t)(a.nrb * kNb * N);  // D_0 at +0, D_1 at +64 columns
    const int o_lane = quad * 32 + lane;                        // output channel of this lane (warps 0, 1)
    const float bv = (quad < 2 && a.bias && o_lane < a.C_out) ? __bfloat162float(a.bias[o_lane]) : 0.0f;
    uint32_t gbase = 0, mpar = 0;
    bool ok = true;
    WarpStream<int2> rs;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const int si = my[t];
      const Script sc = read_script(a, si, -1);
      const int q0 = (si % a.n_qt) * (16 * kNb);
      for (int pt = 0; pt < a.n_pt && ok; ++pt) {
        rs.start(a.rows, sc.row0, sc.row1);
        for (int rr = sc.row0; rr < sc.row1 && ok; ++rr) {
          const int2 rec = rs.get(rr);
          const int r = rec.x & 0xFFFF, rbar = (rec.x >> 16) & 0xFFFF;
          const bool empty = rec.y & kRowEmpty;
          const int rb = (rec.y >> 8) & 0xF;
          if (!empty) {
            int good = 1;
            if (lane == 0) good = wait_batches(done, gbase + (uint32_t)(rec.y >> 12) + 1, 64);
            ok = __shfl_sync(0xffffffffu, good, 0) != 0;
          }
          // one decision for the four warps before the named barriers of the row
          ok = tc::named_bar_and(1, 128, ok);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(rb * kNb * N);
          uint32_t pk[K][32];
          if (!empty) {
#pragma unroll
            for (int k = 0; k < K; ++k) {
              uint32_t v[4 * 16];
#pragma unroll
              for (int b = 0; b < kNb; ++b)
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                    "%13, %14, %15}, [%16];"
                    : "=r"(v[16 * b + 0]), "=r"(v[16 * b + 1]), "=r"(v[16 * b + 2]), "=r"(v[16 * b + 3]),
                      "=r"(v[16 * b + 4]), "=r"(v[16 * b + 5]), "=r"(v[16 * b + 6]), "=r"(v[16 * b + 7]),
                      "=r"(v[16 * b + 8]), "=r"(v[16 * b + 9]), "=r"(v[16 * b + 10]), "=r"(v[16 * b + 11]),
                      "=r"(v[16 * b + 12]), "=r"(v[16 * b + 13]), "=r"(v[16 * b + 14]), "=r"(v[16 * b + 15])
                    : "r"(tb + (uint32_t)(b * N + 16 * k)));
              asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
              for (int i = 0; i < 64; ++i) asm volatile("" : "+r"(v[i]));
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const __nv_bfloat162 h =
                    __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                pk[k][i] = *reinterpret_cast<const uint32_t*>(&h);
              }
            }
            // accumulator drained: the MMA issuers may start another row in the buffer
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[rb]);
          } else {
#pragma unroll
            for (int k = 0; k < K; ++k)
#pragma unroll
              for (int i = 0; i < 32; ++i) pk[k][i] = 0u;
          }
          // the mix: y of every kernel index into this warp's buffers (free: the previous row's mix
          // has completed and its out stores from buffers 0 and 1 have read them), then the
          // group's first warp issues all 4K MMAs into the group's accumulator
          if (lane == 0) tc::bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < K; ++k) {
            uint8_t* rowp = sY + (size_t)k * 4 * kYBuf + (size_t)warp * kYBuf + (size_t)lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(pk[k][4 * c], pk[k][4 * c + 1], pk[k][4 * c + 2], pk[k][4 * c + 3]);
          }
          tc::fence_proxy_async();
          tc::named_bar_sync(2 + grp, 64);
          if ((quad & 1) == 0 && lane == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int k = 0; k < K; ++k) {
              const uint32_t wk = tc::smem_u32(sW) + (uint32_t)k * 8192u;
              const uint32_t yg = tc::smem_u32(sY) + (uint32_t)k * 4u * kYBuf + (uint32_t)grp * 8192u;
#pragma unroll
              for (int j = 0; j < 4; ++j)
                tc::mma_bf16(dmix + (uint32_t)(64 * grp), tc::desc_sw128(wk + 32u * j, 16, 1024),
                             tc::desc_sw128(yg + 2048u * j, 16, 1024), midesc, (k > 0 || j > 0) ? 1u : 0u);
            }
            tc::mma_commit(&mixb[grp]);
          }
          {
            int good = 1;
            if (lane == 0) good = tc::mbar_wait_sleep(&mixb[grp], (mpar >> grp) & 1u, 64);
            ok = __shfl_sync(0xffffffffu, good, 0) != 0 && ok;
            mpar ^= 1u << grp;
            tc::fence_after_sync();
          }
          // both groups' mixes are complete (one decision for the four warps): warps 0 and 1 read
          // D_0 and D_1
          tc::fence_before_sync();
          ok = tc::named_bar_and(1, 128, ok);
          if (!ok) break;
          tc::fence_after_sync();
          if (quad < 2) {
            uint32_t d[2][2][32];  // [group][half of the 64 outputs][column]
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tc::tmem_ld_chunks<2>(dmix + ((uint32_t)(quad * 32) << 16) + (uint32_t)(64 * g + 32 * h), d[g][h]);
            // D read: the group-1 issuer (warp 2) may start the next row's mix
            tc::fence_before_sync();
            tc::named_bar_sync(1, 128);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int orow = g == 0 ? r : rbar;
              const bool st = g == 0 || (rbar != r && rbar != 0xFFFF);
              // group g's out tile in this warp's buffer of kernel index g (read by the mix, which
              // has completed)
              uint8_t* ob = sY + (size_t)g * 4 * kYBuf + (size_t)warp * kYBuf;
              uint8_t* rowp = ob + (size_t)lane * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                uint32_t q4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(d[g][c >> 2][8 * (c & 3) + 2 * e]) + bv,
                                                                 __uint_as_float(d[g][c >> 2][8 * (c & 3) + 2 * e + 1]) + bv);
                  q4[e] = *reinterpret_cast<const uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) = make_uint4(q4[0], q4[1], q4[2], q4[3]);
              }
              tc::fence_proxy_async();
              __syncwarp();
              if (lane == 0) {
                if (st && quad * 32 < a.C_out) tc::tma_store_4d(&ymap, ob, q0, orow, quad * 32, pt);
                tc::bulk_commit();
              }
            }
          } else {
            tc::fence_before_sync();
            tc::named_bar_sync(1, 128);
          }
        }
        gbase += (uint32_t)sc.nbatch;
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

template <int K, bool kFused>
cudaError_t launch_k(const Ring2Launch& L, const void* src, void* dst, const Ring2Fused* F, cudaStream_t st) {
  constexpr int N = 16 * K;
  if (L.K != K || L.nb != kNb || L.ns > kMaxSlots || L.nrb > kMaxBufs || L.nbs > kMaxBslots || L.nrb * kNb * N > 512 ||
      L.n_ctas < 1 || L.nlon < 64 || L.bslot_bytes % 16)
    return cudaErrorInvalidValue;
  Args a{};
  a.tiles = reinterpret_cast<const int4*>(L.tiles);
  a.loads = reinterpret_cast<const int4*>(L.loads);
  a.copies = reinterpret_cast<const int4*>(L.copies);
  a.cmds = L.cmds;
  a.rows = reinterpret_cast<const int2*>(L.rows);
  a.cta_tiles = L.cta_tiles;
  a.b = static_cast<const uint8_t*>(L.b);
  a.n_ctas = L.n_ctas;
  a.n_qt = L.n_qt;
  a.mirror = L.mirror;
  a.plane_tile = L.mirror ? 64 : 128;
  a.n_pt = (L.BC + a.plane_tile - 1) / a.plane_tile;
  a.BC = L.BC;
  a.ns = L.ns;
  a.nbs = L.nbs;
  a.nrb = L.nrb;
  a.bslot_bytes = (uint32_t)L.bslot_bytes;
  if (kFused) {
    // one batch element of 64 channels per plane tile, mirror rows, the mix in tensor memory
    // after the row buffers
    if (!F || !L.mirror || L.BC % 64 || F->C_in != 64 || F->C_out < 1 || F->C_out > 64 ||
        L.nrb * kNb * N + 128 > 512 || (reinterpret_cast<uintptr_t>(F->w) & 1))
      return cudaErrorInvalidValue;
    a.w = static_cast<const __nv_bfloat16*>(F->w);
    a.bias = static_cast<const __nv_bfloat16*>(F->bias);
    a.C_out = F->C_out;
    a.w_t = F->w_t;
  }
  const size_t bars = 8 * (kMaxSlots + 2 * kMaxBslots + kMaxBufs + 3) + 16;
  const size_t smem = 1024 + (size_t)L.ns * kSlotBytes + (((size_t)L.nbs * L.bslot_bytes + 1023) & ~(size_t)1023) +
                      (kFused ? (size_t)K * 8192 : 0) + (size_t)(kFused ? K : 1) * 4 * kYBuf + bars;
  if (smem > kTcSmemLimit) return cudaErrorInvalidValue;
  // x as [BC][n_src_rows][nlon]: boxes of 64 longitudes x 1 row x 64 planes, 128-byte swizzle
  CUtensorMap xm, ym;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)L.nlon, (cuuint64_t)L.n_src_rows, (cuuint64_t)L.BC};
    const cuuint64_t strides[2] = {(cuuint64_t)L.nlon * 2, (cuuint64_t)L.n_src_rows * L.nlon * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    if (!tc::encode_bf16_map(&xm, src, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  }
  if (!kFused) {
    // y as [BC][K][n_out_rows][nlon]: boxes of 64 longitudes x 1 row x 1 kernel index x 32 planes
    const cuuint64_t dims[4] = {(cuuint64_t)L.nlon, (cuuint64_t)L.n_out_rows, (cuuint64_t)K, (cuuint64_t)L.BC};
    const cuuint64_t strides[3] = {(cuuint64_t)L.nlon * 2, (cuuint64_t)L.n_out_rows * L.nlon * 2,
                                   (cuuint64_t)K * L.n_out_rows * L.nlon * 2};
    const cuuint32_t box[4] = {64, 1, 1, 32};
    if (!tc::encode_bf16_map(&ym, dst, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  } else {
    // out as [B][C_out][n_out_rows][nlon]: boxes of 64 longitudes x 1 row x 32 channels x 1
    const int Bn = L.BC / 64;
    const cuuint64_t dims[4] = {(cuuint64_t)L.nlon, (cuuint64_t)L.n_out_rows, (cuuint64_t)F->C_out, (cuuint64_t)Bn};
    const cuuint64_t strides[3] = {(cuuint64_t)L.nlon * 2, (cuuint64_t)L.n_out_rows * L.nlon * 2,
                                   (cuuint64_t)F->C_out * L.n_out_rows * L.nlon * 2};
    const cuuint32_t box[4] = {64, 1, 32, 1};
    if (!tc::encode_bf16_map(&ym, dst, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  }
  const void* kernel = reinterpret_cast<const void*>(&contract_ring2_kernel<K, kFused>);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  void* args[] = {&xm, &ym, &a};
  e = cudaLaunchKernel(kernel, dim3(L.n_ctas), dim3(kThreads), args, smem, st);
  count_launch();
  return e;
}

}  // namespace

bool ring2_kernel_k(int K) { return K == 1 || K == 3 || K == 5; }

cudaError_t launch_contract_ring2(const Ring2Launch& L, const void* src, void* dst, cudaStream_t st) {
  if ((reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15) || L.nlon % 8)
    return cudaErrorInvalidValue;
  switch (L.K) {
    case 1: return launch_k<1, false>(L, src, dst, nullptr, st);
    case 3: return launch_k<3, false>(L, src, dst, nullptr, st);
    case 5: return launch_k<5, false>(L, src, dst, nullptr, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused_ring2(const Ring2Launch& L, const Ring2Fused& F, cudaStream_t st) {
  if ((reinterpret_cast<uintptr_t>(F.x) & 15) || (reinterpret_cast<uintptr_t>(F.out) & 15) || L.nlon % 8)
    return cudaErrorInvalidValue;
  switch (L.K) {
    case 1: return launch_k<1, true>(L, F.x, F.out, &F, st);
    case 3: return launch_k<3, true>(L, F.x, F.out, &F, st);
    default: return cudaErrorInvalidValue;
  }
}

int take_contract_ring2_status() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
  return v;
}

}  // namespace disco
