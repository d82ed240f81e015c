// Tensor-core (tcgen05) form of the sparse contraction x -> y for bf16 signals, stride 1.
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
// Persistent CTAs, 6 warps.  Warp 0 (all lanes) fills a ring of stages, each holding as many
// (source row, window slab) pairs of one tile as fit: the x windows by 16-byte cp.async copies
// (lanes cover 4 octets x 8 channels, so global reads are 64-byte runs and shared writes
// 128-byte rows), each Psi slab by one bulk copy, and a table of slab offsets for the MMA
// issuer.  Each lane arrives on a stage's barrier once its copies into it have landed (checked
// one stage later) and after a generic-to-async proxy fence.  Warp 1 lane 0 issues the MMAs;
// warps 2..5 read the accumulator of the previous tile back (each warp its TMEM lane quadrant)
// into a [64 channels][K][16T] bf16 tile in shared memory that one TMA store writes to y.  Every wait is bounded (tc_common.cuh): on expiry the kernel records the timeout
// and stops.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace disco {
namespace {

constexpr int kCT = 64;                       // channels per tile
constexpr uint32_t kOctBytes = kCT * 16;      // one staged octet: 64 channels x 8 bf16
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kStages = 3;
constexpr int kMaxSlabs = 24;                 // slab table entries per stage

struct TzArgs {
  const int4* slabs;  // TzSlab records
  const int* row_begin;
  const int* order;
  const uint8_t* bglob;
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  int BC, K, N, parts, T;
  int n_lat_in, n_lon, n_lat_out;
  int n_seg, n_ctile, n_tiles;
  uint32_t stage_bytes;
  uint32_t out_bytes;  // output staging tile
};

struct Tile {
  int j, q0, ct, s_begin, s_end;
};

__device__ __forceinline__ Tile decode(const TzArgs& a, int tile) {
  Tile t;
  t.ct = tile % a.n_ctile;
  const int r = tile / a.n_ctile;
  t.q0 = (r % a.n_seg) * 16 * a.T;
  t.j = a.order[r / a.n_seg];
  t.s_begin = a.row_begin[t.j];
  t.s_end = a.row_begin[t.j + 1];
  return t;
}

// Stage table: word 0 = slab count | first << 8 | last << 9 (first / last stage of its tile);
// then per slab {nk | x offset << 8, B offset}, offsets in 16-byte units from the stage base.
constexpr int kFirst = 1 << 8, kLast = 1 << 9;
constexpr int kMetaWords = 1 + 2 * kMaxSlabs;

__global__ void __launch_bounds__(kThreads, 1) contract_tc_kernel(const __grid_constant__ CUtensorMap ymap,
                                                                  TzArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sOut = smem;  // output staging tile
  uint8_t* sS = smem + a.out_bytes;  // kStages stages of stage_bytes
  uint64_t* full = reinterpret_cast<uint64_t*>(sS + (size_t)kStages * a.stage_bytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;  // [2] accumulator buffer ready for the epilogue
  uint64_t* tempty = tfull + 2;       // [2] accumulator buffer drained by the epilogue
  int* meta = reinterpret_cast<int*>(tempty + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + kStages * kMetaWords);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ring = a.n_lon / 8;
  const uint32_t TN = (uint32_t)(a.T * a.N);
  const uint32_t bk = (uint32_t)a.N * 16;  // bytes per octet of a Psi block

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 33);  // 32 producer lanes after their copies + the closing arrival
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], 4);
    }
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

  if (warp == 0) {
    // ---------------------------------------------------------------- producer warp
    const size_t chan = (size_t)a.n_lat_in * a.n_lon;
    const int csub = lane >> 2, osub = lane & 3;  // channel within 8, octet within 4
    uint32_t n = 0;                               // stages opened so far
    bool ok = true;
    int st = 0, cnt = 0;
    uint32_t used = 0;                            // bytes of the open stage
    // opens stage n: waits until the MMAs of its previous use are done
    auto open = [&]() -> bool {
      st = (int)(n % kStages);
      cnt = 0;
      used = 0;
      if (n >= (uint32_t)kStages) {
        int good = 1;
        if (lane == 0) good = tc::mbar_wait(&empty[st], ((n / kStages) & 1) ^ 1);
        if (!__shfl_sync(0xffffffffu, good, 0)) return false;
        __syncwarp();  // order every lane's copies after lane 0's wait
      }
      return true;
    };
    // closes stage n; the copies of stage n - 1 are complete once only stage n's group is left
    auto close = [&](int flags) {
      if (lane == 0) {
        meta[st * kMetaWords] = cnt | flags;
        tc::mbar_arrive(&full[st]);
      }
      tc::cp_async_commit();
      if (n >= 1) {
        tc::cp_async_wait<1>();
        tc::fence_proxy_async();
        tc::mbar_arrive(&full[(n - 1) % kStages]);
      }
      ++n;
    };
    int tile = blockIdx.x;
    Tile t, t1;
    if (tile < a.n_tiles) t = decode(a, tile);
    if (tile + (int)gridDim.x < a.n_tiles) t1 = decode(a, tile + gridDim.x);
    int4 mine = make_int4(0, 0, 0, 0);
    if (tile < a.n_tiles && t.s_begin + lane < t.s_end) mine = a.slabs[t.s_begin + lane];
    for (; tile < a.n_tiles && ok; tile += gridDim.x) {
      // prefetch: the tile after next is decoded and the next tile's slabs are loaded while this
      // tile's copies are issued
      const int tile1 = tile + gridDim.x, tile2 = tile1 + gridDim.x;
      Tile t2;
      if (tile2 < a.n_tiles) t2 = decode(a, tile2);
      int4 mine1 = make_int4(0, 0, 0, 0);
      if (tile1 < a.n_tiles && t1.s_begin + lane < t1.s_end) mine1 = a.slabs[t1.s_begin + lane];
      const int nsl = max(t.s_end - t.s_begin, 1);  // a row without slabs still passes one stage
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
        const int n_oct = nk ? 2 * a.T + 2 * nk - 1 : 0;
        const uint32_t xbytes = (uint32_t)n_oct * kOctBytes;
        const uint32_t bbytes = (uint32_t)(a.parts * 2 * nk) * bk;
        if (cnt > 0 && (used + xbytes + bbytes > a.stage_bytes || cnt == kMaxSlabs)) {
          close(first ? kFirst : 0);
          first = false;
          if (!(ok = open())) break;
        }
        uint8_t* base = sS + (size_t)st * a.stage_bytes;
        if (lane == 0) {
          meta[st * kMetaWords + 1 + 2 * cnt] = nk | (int)(used >> 4) << 8;
          meta[st * kMetaWords + 2 + 2 * cnt] = (int)((used + xbytes) >> 4);
          if (nk) {
            tc::mbar_expect_tx(&full[st], bbytes);
            tc::bulk_load(base + used + xbytes, a.bglob + (size_t)boff * 16, bbytes, &full[st]);
          }
        }
        if (nk) {
          int o0 = ((t.q0 + lon_off) / 8) % ring;  // q0 + lon_off is a multiple of 8
          if (o0 < 0) o0 += ring;
          uint8_t* dst = base + used;
          for (int og = 0; og < n_oct; og += 4) {
            const int o = og + osub;
            if (o >= n_oct) continue;
            const int lon = ((o0 + o) % ring) * 8;
#pragma unroll
            for (int cg = 0; cg < kCT; cg += 8) {
              const int ch = cg + csub;
              const int c = t.ct * kCT + ch;
              const __nv_bfloat16* src = c < a.BC ? a.x + (size_t)c * chan + (size_t)si * a.n_lon + lon : a.x;
              tc::cp_async16(dst + o * kOctBytes + ch * 16, src, c < a.BC ? 16u : 0u);
            }
          }
        }
        used += xbytes + bbytes;
        ++cnt;
      }
      if (!ok) break;
      close((first ? kFirst : 0) | kLast);
      t = t1;
      t1 = t2;
      mine = mine1;
    }
    // the last stage's copies still owe their arrivals
    tc::cp_async_wait<0>();
    tc::fence_proxy_async();
    if (n >= 1) tc::mbar_arrive(&full[(n - 1) % kStages]);
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t idesc = tc::idesc_bf16(128, a.N, false, false);
      uint32_t n = 0;
      int tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x, ++tcount) {
        const int buf = tcount & 1, use = tcount >> 1;
        if (tcount >= 2 && !tc::mbar_wait(&tempty[buf], (use & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t d0 = tmem + (uint32_t)buf * TN;
        while (true) {
          const int st = (int)(n % kStages);
          if (!tc::mbar_wait(&full[st], (n / kStages) & 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const volatile int* m = meta + st * kMetaWords;
          const int hdr = m[0];
          const uint32_t sbase = tc::smem_u32(sS + (size_t)st * a.stage_bytes);
          for (int sl = 0; sl < (hdr & 0xFF); ++sl) {
            const int e0 = m[1 + 2 * sl], e1 = m[2 + 2 * sl];
            const int nk = e0 & 0xFF;
            const uint32_t xa = sbase + ((uint32_t)(e0 >> 8) << 4);
            const uint32_t ba = sbase + ((uint32_t)e1 << 4);
            for (int part = 0; part < a.parts; ++part)
              for (int g = 0; g < a.T; ++g)
                for (int kk = 0; kk < nk; ++kk) {
                  const uint64_t ad =
                      tc::desc_noswz(xa + (uint32_t)(2 * g + 2 * kk) * kOctBytes, kOctBytes, 128);
                  const uint64_t bd = tc::desc_noswz(ba + (uint32_t)(2 * (part * nk + kk)) * bk, bk, 128);
                  const bool init = (hdr & kFirst) && sl == 0 && part == 0 && kk == 0;
                  tc::mma_bf16(d0 + (uint32_t)(g * a.N), ad, bd, idesc, init ? 0u : 1u);
                }
          }
          tc::mma_commit(&empty[st]);
          ++n;
          if (hdr & kLast) break;
        }
        if (!ok) break;
        tc::mma_commit(&tfull[buf]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps
    // TMEM lane quadrant (warp % 4); row m = channel (m % 64) at shift m / 64
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    const int half = m >> 6;
    const int QT = 16 * a.T;  // outputs per tile
    const uint32_t lo_off = a.parts == 1 ? (uint32_t)(8 * a.K) : 0u;
    const bool issuer = warp == 2 && lane == 0;
    uint8_t* myrow = sOut + (size_t)(m & 63) * a.K * QT * 2;
    if (warp == 2) tc::prefetch_map(&ymap);
    int tcount = 0;
    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++tcount) {
      const Tile t = decode(a, tile);
      const int buf = tcount & 1, use = tcount >> 1;
      const bool ok = tc::mbar_wait(&tfull[buf], use & 1);
      tc::fence_after_sync();
      // the staging tile is free once the previous store has read it; the four warps leave
      // together when a wait expired
      if (issuer) tc::bulk_wait_read0();
      if (!tc::named_bar_and(1, 128, ok)) break;
      const bool has = t.s_end > t.s_begin;
      const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * TN;
      for (int g = 0; g < a.T; ++g) {
        for (int k = 0; k < a.K; ++k) {
          float hi[8], lo[8];
          if (has) {
            const uint32_t col = tb + (uint32_t)(g * a.N + 8 * k);
            tc::tmem_ld8x2(col, col + lo_off, hi, lo);
          }
          uint4 v;
          uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v0 = 0.0f, v1 = 0.0f;
            if (has) {
              v0 = lo_off ? hi[2 * e] + lo[2 * e] : hi[2 * e];
              v1 = lo_off ? hi[2 * e + 1] + lo[2 * e + 1] : hi[2 * e + 1];
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
        tc::tma_store_4d(&ymap, sOut, t.q0, t.j, 0, t.ct * kCT);
        tc::bulk_commit();
      }
    }
    if (issuer) tc::bulk_wait0();
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int contract_tc_groups(int N) {
  // two accumulator buffers of T*N columns in 512 tensor-memory columns
  return N > 0 ? std::min(8, (int)(kTmemCols / 2) / N) : 0;
}

bool contract_tc_supported(int K, int stride, int nlon_in, int nlon_out) {
  const int N = 16 * K <= 128 ? 16 * K : (8 * K + 15) / 16 * 16;
  // a staged window may wrap around the ring any number of times: no lower bound on nlon
  return tc::encode_tiled_fn() != nullptr && stride == 1 && nlon_in == nlon_out && nlon_in % 8 == 0 &&
         contract_tc_groups(N) >= 1 && N <= 256 && K <= 16;
}

cudaError_t launch_contract_tc(const TzLaunch& L, const void* x, void* y, cudaStream_t st) {
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15)) return cudaErrorInvalidValue;
  const int N = L.N;
  const int T = contract_tc_groups(N);
  const size_t extra = 1024 + 8 * (2 * kStages + 4) + 4 * kStages * kMetaWords + 16;
  const uint32_t out_bytes = ((uint32_t)(kCT * L.K * 16 * T * 2) + 1023u) & ~1023u;
  const uint32_t stage = (uint32_t)((kTcSmemLimit - extra - out_bytes) / kStages) & ~1023u;
  // the largest slab must fit one stage
  const uint32_t max_slab = (uint32_t)(2 * T + 2 * kTzSlabK - 1) * kOctBytes + (uint32_t)(L.parts * 2 * kTzSlabK * N * 16);
  if (max_slab > stage) return cudaErrorInvalidValue;
  const size_t smem = (size_t)out_bytes + (size_t)kStages * stage + extra;
  // y as [BC][K][nlat_out][nlon]: box = 16T longitudes x 1 row x K x 64 channels
  CUtensorMap ym;
  const cuuint64_t dims[4] = {(cuuint64_t)L.nlon, (cuuint64_t)L.nlat_out, (cuuint64_t)L.K, (cuuint64_t)L.BC};
  const cuuint64_t strides[3] = {(cuuint64_t)L.nlon * 2, (cuuint64_t)L.nlat_out * L.nlon * 2,
                                 (cuuint64_t)L.K * L.nlat_out * L.nlon * 2};
  const cuuint32_t box[4] = {(cuuint32_t)(16 * T), 1, (cuuint32_t)L.K, (cuuint32_t)kCT};
  if (!tc::encode_bf16_map(&ym, y, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorInvalidValue;
  TzArgs a;
  a.slabs = reinterpret_cast<const int4*>(L.slabs);
  a.row_begin = L.row_begin;
  a.order = L.order;
  a.bglob = static_cast<const uint8_t*>(L.b);
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.y = static_cast<__nv_bfloat16*>(y);
  a.BC = L.BC;
  a.K = L.K;
  a.N = N;
  a.parts = L.parts;
  a.T = T;
  a.n_lat_in = L.nlat_in;
  a.n_lon = L.nlon;
  a.n_lat_out = L.nlat_out;
  a.n_seg = (L.nlon + 16 * T - 1) / (16 * T);
  a.n_ctile = (L.BC + kCT - 1) / kCT;
  a.n_tiles = L.nlat_out * a.n_seg * a.n_ctile;
  a.stage_bytes = stage;
  a.out_bytes = out_bytes;
  cudaError_t e = cudaFuncSetAttribute(contract_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(a.n_tiles, sms);
  contract_tc_kernel<<<grid, kThreads, smem, st>>>(ym, a);
  count_launch();
  return cudaGetLastError();
}

int take_contract_tc_status() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
  return v;
}

}  // namespace disco
