// Packed tensor-core (tcgen05) contraction for bf16 signals, stride 1.
//
// Same arithmetic as contract_tc.cu (the Toeplitz blocks of Psi, bf16 hi + lo parts, on the
// forward equation of the page "torch_harmonics.DiscreteContinuousConvS2", class description),
// organised by source row instead of by (output row, source row) pair: a source row is staged
// once per tile and one MMA applies it to every output row of the tile that it reaches, with
// those rows' blocks side by side in N (toeplitz_plan.cpp, make_packed_plan).  A tile is a strip
// of consecutive output rows, a group of 16T outputs and 64 channels; each output row
// accumulates in one of NR tensor-memory slots (slot = strip-relative row mod NR, T groups of
// 16 outputs apart by NR*Nr columns) from its first source row to its last.
//
// Roles as in contract_tc.cu (persistent CTAs): warps 0 and 6..8 stage entries (the x window by
// cp.async with copy-completion arrivals, each warp a share of the channels; the packed block
// by one bulk copy from warp 0); lane 0 of warps 1 and 9 (the even and the odd groups of 16
// outputs) each wait until a slot's previous row is drained before the first contribution of
// a new row, issue their MMAs (split in two where the slot range wraps) and commit a "row
// complete" barrier per finished row; warps 2..5 drain finished rows (TMEM -> bf16 -> shared tile -> TMA
// store), write zeros back into the slot and release it.  Every MMA accumulates: slots start at
// zero and are zeroed on release.  Every wait is bounded (tc_common.cuh).
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace disco {
namespace {

constexpr int kCT = 64;
constexpr uint32_t kOctBytes = kCT * 16;
constexpr int kProducers = 4;  // copy warps: 0 and 6..4+kProducers
constexpr int kIssuer2 = 5 + kProducers;  // warp of the second MMA issuer
constexpr int kThreads = 32 * (6 + kProducers);  // producers, two MMA issuers, four epilogue warps
constexpr uint32_t kTmemCols = 512;
constexpr int kStages = 4;
constexpr int kMaxEnt = 24;
constexpr int kEntWords = 5;  // {ks | n_rows << 8 | o_a << 16, new_mask, x_off16, b_off16, done}
constexpr int kMetaWords = 1 + kEntWords * kMaxEnt;
constexpr int kLast = 1 << 8;

struct TpArgs {
  const int4* ent;     // 2 int4 per entry: {s, lon_start, ks|n_rows<<8|o_a<<16, boff}, {new, done, 0, 0}
  const int4* strips;  // {entry_begin, entry_end, first row, rows}
  const uint8_t* bglob;
  const __nv_bfloat16* x;
  int BC, n_src_rows, n_lon;
  int n_seg, n_ctile, n_tiles;
  uint32_t stage_bytes, out_bytes;
};

struct PTile {
  int e0, e1, o0, q0, ct;
};

__device__ __forceinline__ PTile pdecode(const TpArgs& a, int tile, int QT) {
  PTile t;
  t.ct = tile % a.n_ctile;
  const int r = tile / a.n_ctile;
  t.q0 = (r % a.n_seg) * QT;
  const int4 s = a.strips[r / a.n_seg];
  t.e0 = s.x;
  t.e1 = s.y;
  t.o0 = s.z;
  return t;
}

template <int K, int T, int NR>
__global__ void __launch_bounds__(kThreads, 1) contract_tcp_kernel(const __grid_constant__ CUtensorMap ymap,
                                                                   TpArgs a) {
  constexpr int Nr = 16 * K;                   // columns per output row (hi and lo parts)
  constexpr int QT = 16 * T;                   // outputs per tile
  constexpr uint32_t GS = (uint32_t)(NR * Nr);  // columns between groups of 16 outputs
  static_assert(T * NR * Nr <= (int)kTmemCols, "tensor memory");
  static_assert(NR <= 16, "slot masks");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sOut = smem;
  uint8_t* sS = smem + a.out_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sS + (size_t)kStages * a.stage_bytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;  // [NR] row in the slot complete
  uint64_t* tempty = tfull + NR;      // [NR] slot drained, zeroed and free
  int* meta = reinterpret_cast<int*>(tempty + NR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + kStages * kMetaWords);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ring = a.n_lon / 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 32 * kProducers + 1);
      tc::mbar_init(&empty[s], 2);  // both MMA issuers commit
    }
    for (int s = 0; s < NR; ++s) {
      tc::mbar_init(&tfull[s], 2);  // both MMA issuers commit
      tc::mbar_init(&tempty[s], 4);
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
  if (warp >= 2 && warp <= 5) {  // every slot starts at zero
    const uint32_t lb = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    for (uint32_t c = 0; c < kTmemCols; c += 16) tc::tmem_st16_zero(lb + c);
    tc::tmem_wait_st();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  if (warp == 0 || (warp >= 6 && warp < kIssuer2)) {
    // ---------------------------------------------------------------- producer warps
    // kProducers warps run the same stage packing and each copies its share of the 8 channel
    // groups; the first also writes the stage tables, issues the bulk copies and closes stages.
    constexpr int CG = 8 / kProducers;
    const int pw = warp == 0 ? 0 : warp - 5;
    const size_t chan = (size_t)a.n_src_rows * a.n_lon;
    const int csub = lane >> 2, osub = lane & 3;
    uint32_t n = 0;
    bool ok = true;
    int st = 0, cnt = 0;
    uint32_t used = 0;
    auto open = [&]() -> bool {
      st = (int)(n % kStages);
      cnt = 0;
      used = 0;
      if (n >= (uint32_t)kStages) {
        int good = 1;
        if (lane == 0) good = tc::mbar_wait(&empty[st], ((n / kStages) & 1) ^ 1);
        if (!__shfl_sync(0xffffffffu, good, 0)) return false;
        __syncwarp();
      }
      return true;
    };
    auto close = [&](int flags) {
      if (lane == 0 && pw == 0) {
        meta[st * kMetaWords] = cnt | flags;
        tc::mbar_arrive(&full[st]);
      }
      tc::cp_async_arrive_noinc(&full[st]);
      ++n;
    };
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      const PTile t = pdecode(a, tile, QT);
      const __nv_bfloat16* xl = a.x + (size_t)(t.ct * kCT + csub) * chan;
      uint32_t cmask = 0;
#pragma unroll
      for (int cg = 0; cg < 8; ++cg) cmask |= (t.ct * kCT + 8 * cg + csub < a.BC ? 1u : 0u) << cg;
      if (!(ok = open())) break;
      int4 r0 = make_int4(0, 0, 0, 0), r1 = make_int4(0, 0, 0, 0);
      for (int x = t.e0; x < t.e1 && ok; ++x) {
        const int q = (x - t.e0) & 31;
        if (q == 0 && x + lane < t.e1) {
          r0 = a.ent[2 * (x + lane)];
          r1 = a.ent[2 * (x + lane) + 1];
        }
        const int s = __shfl_sync(0xffffffffu, r0.x, q);
        const int lon_start = __shfl_sync(0xffffffffu, r0.y, q);
        const int w2 = __shfl_sync(0xffffffffu, r0.z, q);
        const int boff = __shfl_sync(0xffffffffu, r0.w, q);
        const int newm = __shfl_sync(0xffffffffu, r1.x, q);
        const int done = __shfl_sync(0xffffffffu, r1.y, q);
        const int ks = w2 & 0xFF, nrow = (w2 >> 8) & 0xFF;
        const int n_oct = 2 * T + 2 * ks - 1;
        const uint32_t xbytes = (uint32_t)n_oct * kOctBytes;
        const uint32_t bbytes = (uint32_t)(2 * ks * nrow * Nr * 16);
        if (cnt > 0 && (used + xbytes + bbytes > a.stage_bytes || cnt == kMaxEnt)) {
          close(0);
          if (!(ok = open())) break;
        }
        uint8_t* base = sS + (size_t)st * a.stage_bytes;
        if (lane == 0 && pw == 0) {
          int* m = meta + st * kMetaWords + 1 + kEntWords * cnt;
          m[0] = w2;
          m[1] = newm;
          m[2] = (int)(used >> 4);
          m[3] = (int)((used + xbytes) >> 4);
          m[4] = done;
          tc::mbar_expect_tx(&full[st], bbytes);
          tc::bulk_load(base + used + xbytes, a.bglob + (size_t)boff * 16, bbytes, &full[st]);
        }
        int o0 = ((t.q0 + lon_start) / 8) % ring;  // q0 + lon_start is a multiple of 8
        if (o0 < 0) o0 += ring;
        const __nv_bfloat16* xrow = xl + (size_t)s * a.n_lon;
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
        used += xbytes + bbytes;
        ++cnt;
      }
      if (!ok) break;
      close(kLast);
    }
    tc::cp_async_wait_all();
  } else if (warp == 1 || warp == kIssuer2) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuers
      // two threads issue the MMAs of the even and the odd groups of 16 outputs (disjoint
      // accumulator columns); each waits for the slots it writes and commits its own MMAs
      const int gsel = warp == 1 ? 0 : 1;
      const uint64_t a_fix = tc::desc_noswz(0, kOctBytes, 128);
      const uint32_t a_step = (2 * kOctBytes) >> 4;
      uint32_t n = 0;
      uint32_t occupied = 0, emp_par = 0;  // per slot: had a row before / parity of its next release
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
        while (true) {
          const int st = (int)(n % kStages);
          if (!tc::mbar_wait(&full[st], (n / kStages) & 1)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          tc::fence_proxy_async();  // the stage's cp.async data before the MMA reads
          const volatile int* m = meta + st * kMetaWords;
          const int hdr = m[0];
          const uint32_t sbase4 = tc::smem_u32(sS + (size_t)st * a.stage_bytes) >> 4;
          for (int e = 0; e < (hdr & 0xFF) && ok; ++e) {
            const volatile int* me = m + 1 + kEntWords * e;
            const int w2 = me[0], newm = me[1];
            const uint32_t xo = (uint32_t)me[2], bo = (uint32_t)me[3];
            const int ks = w2 & 0xFF, nrow = (w2 >> 8) & 0xFF, o_a = w2 >> 16;
            // new rows: their slots must have been drained (and zeroed) by the epilogue
            for (int r = 0; r < nrow; ++r) {
              if (!((newm >> r) & 1)) continue;
              const int sl = (o_a + r) % NR;
              if ((occupied >> sl) & 1) {
                if (!tc::mbar_wait(&tempty[sl], (emp_par >> sl) & 1)) {
                  ok = false;
                  break;
                }
                emp_par ^= 1u << sl;
              }
              occupied |= 1u << sl;
            }
            if (!ok) break;
            tc::fence_after_sync();
            const int sl0 = o_a % NR;
            const int n1 = min(nrow, NR - sl0), n2 = nrow - n1;
            const uint32_t NC = (uint32_t)(nrow * Nr);
            const uint32_t id1 = tc::idesc_bf16(128, n1 * Nr, false, false);
            const uint32_t id2 = tc::idesc_bf16(128, n2 > 0 ? n2 * Nr : 16, false, false);
            const uint64_t b_fix = tc::desc_noswz(0, NC * 16, 128);
            const uint32_t b_step = (2 * NC * 16) >> 4;
            const uint32_t b2off = ((uint32_t)(n1 * Nr) * 16) >> 4;  // second column group
#pragma unroll 1
            for (int g = gsel; g < T; g += 2) {
              uint64_t ad = a_fix | (uint64_t)(sbase4 + xo + (uint32_t)g * a_step);
              uint64_t bd = b_fix | (uint64_t)(sbase4 + bo);
              const uint32_t d1 = tmem + (uint32_t)g * GS + (uint32_t)(sl0 * Nr);
              const uint32_t d2 = tmem + (uint32_t)g * GS;
              for (int kk = 0; kk < ks; ++kk) {
                tc::mma_bf16(d1, ad, bd, id1, 1u);
                if (n2 > 0) tc::mma_bf16(d2, ad, bd + b2off, id2, 1u);
                ad += a_step;
                bd += b_step;
              }
            }
          }
          if (!ok) break;
          // rows finished with this stage: their slots are complete once these MMAs are (read
          // the table before releasing the stage, which lets the producer overwrite it)
          for (int e = 0; e < (hdr & 0xFF); ++e) {
            const int done = m[1 + kEntWords * e + 4];
            const int base = done & 0xFFFF;
            for (int b = 0; b < 16; ++b)
              if ((done >> (16 + b)) & 1) tc::mma_commit(&tfull[(base + b) % NR]);
          }
          tc::mma_commit(&empty[st]);
          ++n;
          if (hdr & kLast) break;
        }
      }
    }
  } else if (warp <= 5) {
    // ---------------------------------------------------------------- epilogue warps
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    const int half = m >> 6;
    const bool issuer = warp == 2 && lane == 0;
    uint8_t* myrow = sOut + (size_t)(m & 63) * K * QT * 2;
    const uint32_t lb = tmem + ((uint32_t)(quad * 32) << 16);
    if (warp == 2) tc::prefetch_map(&ymap);
    uint32_t full_par = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      const PTile t = pdecode(a, tile, QT);
      int dn = 0;
      for (int x = t.e0; x < t.e1 && ok; ++x) {
        const int q = (x - t.e0) & 31;
        if (q == 0 && x + lane < t.e1) dn = a.ent[2 * (x + lane) + 1].y;
        const int done = __shfl_sync(0xffffffffu, dn, q);
        const int dbase = done & 0xFFFF;
        for (int b = 0; b < 16; ++b) {
          if (!((done >> (16 + b)) & 1)) continue;
          const int o = dbase + b, sl = o % NR;
          const bool got = tc::mbar_wait(&tfull[sl], (full_par >> sl) & 1);
          full_par ^= 1u << sl;
          tc::fence_after_sync();
          if (issuer) tc::bulk_wait_read0();  // the staging tile is free
          if (!(ok = tc::named_bar_and(1, 128, got))) break;
#pragma unroll 1
          for (int g = 0; g < T; ++g) {
            uint32_t r[Nr];
            const uint32_t col = lb + (uint32_t)g * GS + (uint32_t)(sl * Nr);
            tc::tmem_ld_chunks<Nr / 16>(col, r);
#pragma unroll
            for (int k = 0; k < K; ++k) {
              uint4 v;
              uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float v0 = __uint_as_float(r[8 * k + 2 * e]) + __uint_as_float(r[8 * K + 8 * k + 2 * e]);
                const float v1 =
                    __uint_as_float(r[8 * k + 2 * e + 1]) + __uint_as_float(r[8 * K + 8 * k + 2 * e + 1]);
                const __nv_bfloat162 p = __floats2bfloat162_rn(v0, v1);
                w[e] = *reinterpret_cast<const uint32_t*>(&p);
              }
              *reinterpret_cast<uint4*>(myrow + ((size_t)k * QT + 16 * g + 8 * half) * 2) = v;
            }
#pragma unroll
            for (int c = 0; c < Nr; c += 16) tc::tmem_st16_zero(col + (uint32_t)c);
          }
          tc::tmem_wait_st();
          // slot drained and zeroed: the MMA issuer may give it to the next row
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&tempty[sl]);
          tc::fence_proxy_async();
          tc::named_bar_sync(1, 128);
          if (issuer) {
            tc::tma_store_4d(&ymap, sOut, t.q0, t.o0 + o, 0, t.ct * kCT);
            tc::bulk_commit();
          }
        }
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

template <int K, int T, int NR>
cudaError_t launch_tp(const TpLaunch& L, const void* x, void* y, cudaStream_t st, int grid_cap) {
  constexpr int QT = 16 * T;
  if (L.K != K || L.T != T || L.NR != NR) return cudaErrorInvalidValue;
  const size_t extra = 1024 + 8 * (2 * kStages + 2 * NR) + 4 * kStages * kMetaWords + 16;
  const uint32_t out_bytes = ((uint32_t)(kCT * K * QT * 2) + 1023u) & ~1023u;
  const uint32_t stage = (uint32_t)((kTcSmemLimit - extra - out_bytes) / kStages) & ~1023u;
  const uint32_t max_entry = (uint32_t)(2 * T + 2 * L.ksmax - 1) * kOctBytes + (uint32_t)(2 * L.ksmax * 256 * 16);
  if (max_entry > stage) return cudaErrorInvalidValue;
  const size_t smem = (size_t)out_bytes + (size_t)kStages * stage + extra;
  CUtensorMap ym;
  const cuuint64_t dims[4] = {(cuuint64_t)L.nlon, (cuuint64_t)L.n_out_rows, (cuuint64_t)K, (cuuint64_t)L.BC};
  const cuuint64_t strides[3] = {(cuuint64_t)L.nlon * 2, (cuuint64_t)L.n_out_rows * L.nlon * 2,
                                 (cuuint64_t)K * L.n_out_rows * L.nlon * 2};
  const cuuint32_t box[4] = {(cuuint32_t)QT, 1, (cuuint32_t)K, (cuuint32_t)kCT};
  if (!tc::encode_bf16_map(&ym, y, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorInvalidValue;
  TpArgs a{};
  a.ent = reinterpret_cast<const int4*>(L.ent);
  a.strips = reinterpret_cast<const int4*>(L.strips);
  a.bglob = static_cast<const uint8_t*>(L.b);
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.BC = L.BC;
  a.n_src_rows = L.n_src_rows;
  a.n_lon = L.nlon;
  a.n_seg = (L.nlon + QT - 1) / QT;
  a.n_ctile = (L.BC + kCT - 1) / kCT;
  a.n_tiles = L.n_strips * a.n_seg * a.n_ctile;
  a.stage_bytes = stage;
  a.out_bytes = out_bytes;
  if (a.n_tiles == 0) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(contract_tcp_kernel<K, T, NR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(std::min(a.n_tiles, sms), grid_cap);  // persistent: at most one CTA per SM
  contract_tcp_kernel<K, T, NR><<<grid, kThreads, smem, st>>>(ym, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool packed_shape(int K, bool adjoint, int* T, int* NR) {
  if (adjoint && K == 1) {
    *T = 4;
    *NR = 8;
    return true;
  }
  if (!adjoint && K == 3) {
    *T = 1;
    *NR = 6;
    return true;
  }
  return false;
}

cudaError_t launch_contract_tcp(const TpLaunch& L, const void* x, void* y, cudaStream_t st, int grid_cap) {
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15)) return cudaErrorInvalidValue;
  if (L.K == 1 && L.T == 4 && L.NR == 8) return launch_tp<1, 4, 8>(L, x, y, st, grid_cap);
  if (L.K == 3 && L.T == 1 && L.NR == 6) return launch_tp<3, 1, 6>(L, x, y, st, grid_cap);
  return cudaErrorInvalidValue;
}

int take_contract_tcp_status() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
  return v;
}

}  // namespace disco
