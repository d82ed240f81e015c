// Tensor-core (tcgen05) forms of the dense channel contractions, bf16 in, fp32 accumulate.
//
// The weight einsum of the forward equation on the page
// "torch_harmonics.DiscreteContinuousConvS2" (the sums over c_i and k of
// w_k^{co,ci} times the contracted signal) and the transposed einsum of the
// input gradient are one GEMM per (batch, group):
//     out[g*Mg + m, n] = sum_r wm[g, m, r] * in[g*Rg + r, n]  (+ bias)
// computed here as D[n, m] with M = 128 grid points per tile (A = `in`,
// MN-major: n is contiguous) and N = a tile of up to 256 output channels
// (B = `wm`, K-major: r is contiguous).  The weight gradient is the split-K GEMM
//     part[split, g, o, r] = sum_{n in split} y[g*Rg + r, n] * dout[g*Og + o, n]
// computed as D[r, o] with both operands K-major (n contiguous).
//
// One CTA = 4 warps: lane 0 of warp 0 issues the TMA loads through a ring of
// stages, lane 0 of warp 1 issues the MMAs (fp32 accumulator in tensor
// memory), all four warps read the accumulator back (one TMEM lane per thread)
// and store.  Every wait is bounded (tc_common.cuh).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace disco {
namespace {

constexpr int kStages = 4;
constexpr int kBK = 64;                      // K elements per stage (one 128-byte swizzle row)
constexpr uint32_t kHalfTile = 64 * 128;     // one [64 K][64 M] MN-major box, bytes

struct MixTcArgs {
  void* out;
  const void* bias;
  int G, Mg, Rg, N, BN;
  int S;  // pipeline stages: no more than the K loop has chunks, so small tiles leave room
          // for several CTAs per SM
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__host__ __device__ inline uint32_t tmem_cols(int n) {
  uint32_t c = 32;
  while ((int)c < n) c <<= 1;
  return c;
}

__global__ void __launch_bounds__(128, 2) mix_tc_kernel(const __grid_constant__ CUtensorMap map_in,
                                                        const __grid_constant__ CUtensorMap map_w, MixTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int BN = a.BN;
  const int nst = a.S;  // stages of this launch
  const uint32_t a_bytes = 2 * kHalfTile;
  const uint32_t b_bytes = (uint32_t)BN * 128;
  uint8_t* sA = smem;
  uint8_t* sB = smem + nst * a_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + nst * b_bytes);
  uint64_t* empty = full + nst;
  uint64_t* done = empty + nst;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int n0 = blockIdx.x * 128;
  const int m0 = blockIdx.y * BN;
  const int bg = blockIdx.z;
  const int g = bg % a.G;
  const int nk = (a.Rg + kBK - 1) / kBK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = tmem_cols(BN);

  if (threadIdx.x == 0) {
    tc::prefetch_map(&map_in);
    tc::prefetch_map(&map_w);
    for (int s = 0; s < nst; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (warp == 2) {
    tc::tmem_alloc(tmem_slot, ncols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % nst;
      if (kc >= nst && !tc::mbar_wait(&empty[s], ((kc / nst) & 1) ^ 1)) break;
      tc::mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
      tc::tma_load_3d(sA + s * a_bytes, &map_in, &full[s], n0, kc * kBK, bg);
      tc::tma_load_3d(sA + s * a_bytes + kHalfTile, &map_in, &full[s], n0 + 64, kc * kBK, bg);
      tc::tma_load_2d(sB + s * b_bytes, &map_w, &full[s], kc * kBK, g * a.Mg + m0);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = tc::idesc_bf16(128, BN, true, false);
    bool ok = true;
    for (int kc = 0; kc < nk && ok; ++kc) {
      const int s = kc % nst;
      ok = tc::mbar_wait(&full[s], (kc / nst) & 1);
      if (!ok) break;
      tc::fence_after_sync();
      const uint32_t a0 = tc::smem_u32(sA + s * a_bytes);
      const uint32_t b0 = tc::smem_u32(sB + s * b_bytes);
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        // A (MN-major): 16 K-rows of 128 B per step; the two 64-wide M halves are 8 KB apart
        const uint64_t ad = tc::desc_sw128(a0 + kk * 2048, kHalfTile, 1024);
        // B (K-major): 16 K-elements = 32 B per step inside the 128-byte swizzled rows
        const uint64_t bd = tc::desc_sw128(b0 + kk * 32, 16, 1024);
        tc::mma_bf16(tmem, ad, bd, idesc, (kc | kk) != 0);
      }
      tc::mma_commit(&empty[s]);
    }
    tc::mma_commit(done);
  }
  __syncwarp();
  const bool ok = tc::mbar_wait(done, 0);
  tc::fence_after_sync();
  if (ok) {
    const int row = warp * 32 + lane;
    const int n = n0 + row;
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(a.bias);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + ((size_t)bg * a.Mg) * a.N;
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      if (n < a.N) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = m0 + c + i;
          if (m < a.Mg) {
            const float bv = bias ? __bfloat162float(bias[g * a.Mg + m]) : 0.0f;
            out[(size_t)m * a.N + n] = __float2bfloat16_rn(v[i] + bv);
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) tc::tmem_dealloc(tmem, ncols);
}

// ------------------------------------------------------------------ persistent form
// The same GEMM with one CTA per SM looping over the (batch*group, M-tile of outputs, 128-point)
// tiles, so that the loads of the next tile overlap the epilogue of the last:
//   warp 4 (lane 0)  streams the `in` stages through a ring, and the W chunks of an M tile with
//                    the first stage of a tile whose (group, M tile) differs from the previous
//                    one (after every MMA that read the old W has completed);
//   warp 5 (lane 0)  issues the MMAs into one of two accumulators in tensor memory;
//   warps 0..3       drain an accumulator (TMEM lane = grid point), add the bias, stage the
//                    bf16 tile [m][n] in shared memory and write it with TMA stores.
// W stays in shared memory across the tiles of one (group, M tile), instead of being re-read
// with every tile.  Every wait is bounded.

struct MixPArgs {
  const void* bias;
  int G, Mg, Rg, N, BN, S, NT, MT, T;  // NT point tiles, MT output tiles, T tiles in all
  int NO;                              // out staging buffers (2: a tile's stores overlap the next)
};

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
               "r"(tc::smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

template <int H>  // 128-point halves per tile: a tile reads 128*H consecutive points of each plane
__global__ void __launch_bounds__(192, 1) mix_tc_persistent_kernel(const __grid_constant__ CUtensorMap map_in,
                                                                   const __grid_constant__ CUtensorMap map_w,
                                                                   const __grid_constant__ CUtensorMap map_out,
                                                                   MixPArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int BN = a.BN, S = a.S;
  const int nk = (a.Rg + kBK - 1) / kBK;
  const uint32_t a_bytes = 2 * H * kHalfTile;
  const uint32_t wc_bytes = (uint32_t)BN * 128;  // one 64-wide K chunk of W
  uint8_t* sA = smem;                             // S stages of H x [64 K][128 M], MN-major
  uint8_t* sW = sA + (size_t)S * a_bytes;         // nk chunks of [BN][64 K], K-major
  uint8_t* sO = sW + (size_t)nk * wc_bytes;       // NO out tiles, each 2H quarters [BN][64 n]
  const size_t o_bytes = 2 * H * (size_t)BN * 128;
  float* sBias = reinterpret_cast<float*>(sO + (size_t)a.NO * o_bytes);  // BN floats
  uint64_t* full = reinterpret_cast<uint64_t*>(sBias + 256);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;   // [2]
  uint64_t* tempty = tfull + 2;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = tmem_cols(2 * H * BN);

  if (threadIdx.x == 0) {
    tc::prefetch_map(&map_in);
    tc::prefetch_map(&map_w);
    tc::prefetch_map(&map_out);
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], 4);
    }
    tc::fence_barrier_init();
  }
  if (warp == 5) {
    tc::tmem_alloc(tmem_slot, ncols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  auto wkey = [&](int t) { return t / a.NT; };  // (batch*group, M tile): W and bias change with it
  // a contiguous run of tiles per CTA: consecutive tiles read the next points of the same planes
  const int t_lo = (int)((long)a.T * blockIdx.x / gridDim.x), t_hi = (int)((long)a.T * (blockIdx.x + 1) / gridDim.x);

  if (warp == 4) {
    if (lane == 0) {
      uint32_t gs = 0;  // stages loaded so far
      int prev_key = -1;
      bool ok = true;
      for (int t = t_lo; t < t_hi && ok; ++t) {
        const int nt = t % a.NT, rest = t / a.NT, mt = rest % a.MT, bg = rest / a.MT, g = bg % a.G;
        const bool wload = wkey(t) != prev_key;
        prev_key = wkey(t);
        for (int kc = 0; kc < nk && ok; ++kc, ++gs) {
          const int s = (int)(gs % (uint32_t)S);
          if (gs >= (uint32_t)S) ok = tc::mbar_wait_sleep(&empty[s], ((gs / S) - 1) & 1u);
          if (!ok) break;
          const bool wl = wload && kc == 0;
          if (wl && gs > 0) {
            // every MMA that read the old W has completed: the commit of the last stage loaded
            const uint32_t gp = gs - 1;
            ok = tc::mbar_wait_sleep(&empty[gp % S], (gp / S) & 1u);
            if (!ok) break;
          }
          tc::mbar_arrive_expect_tx(&full[s], a_bytes + (wl ? (uint32_t)nk * wc_bytes : 0u));
          if (wl)
            for (int c = 0; c < nk; ++c)
              tc::tma_load_2d(sW + (size_t)c * wc_bytes, &map_w, &full[s], c * kBK, g * a.Mg + mt * BN);
          for (int q = 0; q < 2 * H; ++q)
            tc::tma_load_3d(sA + (size_t)s * a_bytes + (size_t)q * kHalfTile, &map_in, &full[s], nt * 128 * H + 64 * q,
                            kc * kBK, bg);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(128, BN, true, false);
      uint32_t gs = 0, i = 0;
      bool ok = true;
      for (int t = t_lo; t < t_hi && ok; ++t, ++i) {
        const uint32_t acc = i & 1u, use = i >> 1;
        if (use >= 1) ok = tc::mbar_wait_sleep(&tempty[acc], (use - 1) & 1u);
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t d = tmem + acc * (uint32_t)(H * BN);
        for (int kc = 0; kc < nk && ok; ++kc, ++gs) {
          const int s = (int)(gs % (uint32_t)S);
          ok = tc::mbar_wait(&full[s], (gs / S) & 1u);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t b0 = tc::smem_u32(sW + (size_t)kc * wc_bytes);
#pragma unroll
          for (int hh = 0; hh < H; ++hh) {
            const uint32_t a0 = tc::smem_u32(sA + (size_t)s * a_bytes + (size_t)hh * 2 * kHalfTile);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = tc::desc_sw128(a0 + kk * 2048, kHalfTile, 1024);
              const uint64_t bd = tc::desc_sw128(b0 + kk * 32, 16, 1024);
              tc::mma_bf16(d + (uint32_t)(hh * BN), ad, bd, idesc, (kc | kk) != 0);
            }
          }
          tc::mma_commit(&empty[s]);
        }
        if (ok) tc::mma_commit(&tfull[acc]);
      }
    }
  } else {
    // epilogue: warps 0..3, TMEM lanes 32*warp.., grid point n = 128*nt + 32*warp + lane
    const int row = warp * 32 + lane;
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(a.bias);
    uint32_t i = 0;
    int prev_key = -1;
    bool ok = true;
    for (int t = t_lo; t < t_hi; ++t, ++i) {
      const int nt = t % a.NT, rest = t / a.NT, mt = rest % a.MT, bg = rest / a.MT, g = bg % a.G;
      const uint32_t acc = i & 1u, use = i >> 1;
      if (wkey(t) != prev_key) {
        // the bias of this (group, M tile); the previous tile's readers are past the barrier below
        for (int m = threadIdx.x; m < BN; m += 128) {
          const int o = mt * BN + m;
          sBias[m] = (bias && o < a.Mg) ? __bfloat162float(bias[g * a.Mg + o]) : 0.0f;
        }
        prev_key = wkey(t);
      }
      int good = 1;
      if (lane == 0) good = tc::mbar_wait_sleep(&tfull[acc], use & 1u);
      ok = __shfl_sync(0xffffffffu, good, 0) != 0;
      // this tile's out staging is free once the stores that last read it are done with it (the
      // previous tile's with one buffer, the one before with two); one decision for the four warps
      uint8_t* ob = sO + (size_t)(i % (uint32_t)a.NO) * o_bytes;
      if (threadIdx.x == 0) {
        if (a.NO == 2)
          tc::bulk_wait_read_le<1>();
        else
          tc::bulk_wait_read0();
      }
      ok = tc::named_bar_and(1, 128, ok);
      if (!ok) break;
      tc::fence_after_sync();
      for (int hh = 0; hh < H; ++hh) {
        // point hh*128 + row of the tile: quarter (hh*128 + row) / 64 of the staging
        const uint32_t tb = tmem + ((uint32_t)(warp * 32) << 16) + acc * (uint32_t)(H * BN) + (uint32_t)(hh * BN);
        const int pq = hh * 128 + row;
        uint8_t* orow_p = ob + (size_t)(pq >> 6) * BN * 128 + (size_t)(pq & 63) * 2;
        int c = 0;
        // 64 columns per wait: the loads of a group are in flight together
        for (; c + 64 <= BN; c += 64) {
          uint32_t v[64];
          tc::tmem_ld_chunks<4>(tb + (uint32_t)c, v);
#pragma unroll
          for (int e = 0; e < 64; ++e)
            *reinterpret_cast<__nv_bfloat16*>(orow_p + (size_t)(c + e) * 128) =
                __float2bfloat16_rn(__uint_as_float(v[e]) + sBias[c + e]);
        }
        for (; c < BN; c += 16) {
          uint32_t v[16];
          tc::tmem_ld_chunks<1>(tb + (uint32_t)c, v);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            *reinterpret_cast<__nv_bfloat16*>(orow_p + (size_t)(c + e) * 128) =
                __float2bfloat16_rn(__uint_as_float(v[e]) + sBias[c + e]);
        }
      }
      // accumulator drained: the MMA issuer may reuse it
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty[acc]);
      tc::fence_proxy_async();
      tc::named_bar_sync(1, 128);
      if (threadIdx.x == 0) {
        for (int q = 0; q < 2 * H; ++q)
          tma_store_3d(&map_out, ob + (size_t)q * BN * 128, nt * 128 * H + 64 * q, mt * BN, bg);
        tc::bulk_commit();
      }
    }
    if (threadIdx.x == 0) tc::bulk_wait0();
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) tc::tmem_dealloc(tmem, ncols);
}

struct DwTcArgs {
  float* part;
  float* bpart;  // written here when ones_row (dbias as the product with a row of ones), else null
  int G, Og, Rg, N, nc, nchunk;
  int n_tiles, stages, ones_row;  // M tiles of 128 rows (r = (c, k)); the spare row of the last tile, -1 none
};

// dw partials for one split of the spatial positions: D_t[r][o] = sum_n y[b, g, 128t + r, n] dout[b, g, o, n]
// for every M tile t of the Rg rows in one CTA, so that each dout tile is read once.  With a
// spare row in the last tile (Rg % 128 != 0) that row is set to ones after each stage lands,
// which makes it the split's sum of dout: the dbias partial.
__global__ void __launch_bounds__(128, 1) dw_tc_kernel(const __grid_constant__ CUtensorMap map_y,
                                                       const __grid_constant__ CUtensorMap map_d, DwTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int BN = a.Og, T = a.n_tiles, S = a.stages;
  const uint32_t a_bytes = 128 * 128;            // one M tile: 128 rows x 64 K, 128-byte swizzle
  const uint32_t b_bytes = (uint32_t)BN * 128;
  const uint32_t st_bytes = (uint32_t)T * a_bytes + b_bytes;
  uint8_t* sS = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(sS + (size_t)S * st_bytes);
  uint64_t* empty = full + S;
  uint64_t* done = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int chunk = blockIdx.x;
  const int bg = blockIdx.z;
  const int g = bg % a.G, b = bg / a.G;
  const int nb = chunk * a.nc;
  const int nk = (min(a.N, nb + a.nc) - nb + kBK - 1) / kBK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = tmem_cols(T * BN);

  if (threadIdx.x == 0) {
    tc::prefetch_map(&map_y);
    tc::prefetch_map(&map_d);
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  if (warp == 2) {
    tc::tmem_alloc(tmem_slot, ncols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % S;
      if (kc >= S && !tc::mbar_wait(&empty[s], ((kc / S) & 1) ^ 1)) break;
      tc::mbar_arrive_expect_tx(&full[s], st_bytes);
      uint8_t* st = sS + (size_t)s * st_bytes;
      for (int t = 0; t < T; ++t) tc::tma_load_3d(st + t * a_bytes, &map_y, &full[s], nb + kc * kBK, 128 * t, bg);
      tc::tma_load_3d(st + T * a_bytes, &map_d, &full[s], nb + kc * kBK, 0, bg);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = tc::idesc_bf16(128, BN, false, false);
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % S;
      if (!tc::mbar_wait(&full[s], (kc / S) & 1)) break;
      uint8_t* st = sS + (size_t)s * st_bytes;
      if (a.ones_row >= 0) {
        // the spare row of the last tile: 64 K-elements of 1.0 (the swizzle only permutes them)
        uint4* row = reinterpret_cast<uint4*>(st + (T - 1) * a_bytes + a.ones_row * 128);
        const uint4 one = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
#pragma unroll
        for (int i = 0; i < 8; ++i) row[i] = one;
        tc::fence_proxy_async();
      }
      tc::fence_after_sync();
      const uint32_t a0 = tc::smem_u32(st);
      const uint32_t b0 = tc::smem_u32(st + T * a_bytes);
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk)
        for (int t = 0; t < T; ++t)
          tc::mma_bf16(tmem + (uint32_t)(t * BN), tc::desc_sw128(a0 + t * a_bytes + kk * 32, 16, 1024),
                       tc::desc_sw128(b0 + kk * 32, 16, 1024), idesc, (kc | kk) != 0);
      tc::mma_commit(&empty[s]);
    }
    tc::mma_commit(done);
  }
  __syncwarp();
  const bool ok = tc::mbar_wait(done, 0);
  tc::fence_after_sync();
  if (ok) {
    const size_t split = (size_t)b * a.nchunk + chunk;
    float* P = a.part + ((split * a.G + g) * a.Og) * (size_t)a.Rg;
    for (int t = 0; t < T; ++t) {
      const int rl = warp * 32 + lane, r = 128 * t + rl;
      for (int c = 0; c < BN; c += 16) {
        float v[16];
        tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(t * BN + c), v);
        if (r < a.Rg) {
#pragma unroll
          for (int i = 0; i < 16; ++i) P[(size_t)(c + i) * a.Rg + r] = nk > 0 ? v[i] : 0.0f;
        } else if (t == T - 1 && rl == a.ones_row && a.bpart) {
#pragma unroll
          for (int i = 0; i < 16; ++i) a.bpart[split * (a.G * a.Og) + g * a.Og + c + i] = nk > 0 ? v[i] : 0.0f;
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) tc::tmem_dealloc(tmem, ncols);
}

// bpart[split, g*Og + o] = sum over the split's n of dout[b, g*Og + o, n]; one warp per row,
// fixed lane striding and shuffle tree.
__global__ void __launch_bounds__(256) bias_partial_kernel(const __nv_bfloat16* __restrict__ dout,
                                                           float* __restrict__ bpart, int G, int Og, int N, int nc,
                                                           int nchunk) {
  const int chunk = blockIdx.x, bg = blockIdx.y;
  const int b = bg / G, g = bg % G;
  const int nb = chunk * nc, ne = min(N, nb + nc);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int o = warp; o < Og; o += blockDim.x >> 5) {
    const __nv_bfloat16* row = dout + ((size_t)bg * Og + o) * N;
    float acc = 0.0f;
    for (int n = nb + lane * 8; n < ne; n += 256) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + n));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) acc += __uint_as_float(w[i] << 16) + __uint_as_float(w[i] & 0xffff0000u);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) bpart[((size_t)b * nchunk + chunk) * (G * Og) + g * Og + o] = acc;
  }
}

// ------------------------------------------------------------------- host

// bf16 tensor map with 128-byte swizzle; dims innermost first, strides in bytes for dims 1..
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
              const cuuint32_t* box) {
  return tc::encode_bf16_map(m, base, rank, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

size_t mix_smem(int BN, int S) { return 1024 + S * (2 * kHalfTile + (size_t)BN * 128) + (2 * S + 2) * 8; }

int mix_bn(int Mg) {
  if (Mg <= 256) return Mg;
  for (int bn = 256; bn >= 16; bn -= 16)
    if (Mg % bn == 0) return bn;
  return 256;
}

}  // namespace

bool mix_tc_supported(int Mg, int Rg, int N) {
  return tc::encode_tiled_fn() != nullptr && Mg % 16 == 0 && Rg % 8 == 0 && N % 8 == 0 && (mix_bn(Mg) % 16 == 0);
}

// Shared memory of the persistent form with S stages (the 1 KB alignment slack included).
size_t mixp_smem(int BN, int nk, int S, int NO, int H) {
  return 1024 + (size_t)S * 2 * H * kHalfTile + (size_t)nk * BN * 128 + (size_t)NO * 2 * H * BN * 128 + 256 * 4 +
         (2 * (size_t)S + 4) * 8 + 16;
}

cudaError_t launch_mix_tc(const MixArgs& a, cudaStream_t st) {
  CUtensorMap mi, mw, mo;
  const int BN = mix_bn(a.Mg);
  const int nk = (a.Rg + kBK - 1) / kBK;
  // the wider tile (128*H points, H = 2, else 1) when its two accumulators fit tensor memory and
  // its stages fit shared memory at least twice; two out staging buffers when four stages still
  // fit beside them, else one.  (256 points: weather einsum 0.145 -> 0.134 ms; 512 points, with
  // room for two stages only, 0.137 ms.)
  int H = 2, NO = 2, S = 8;
  for (;; H >>= 1) {
    NO = 2;
    S = 8;
    while (S >= 4 && mixp_smem(BN, nk, S, NO, H) > kTcSmemLimit) --S;
    if (S < 4) {
      NO = 1;
      S = 8;
      while (S >= 2 && mixp_smem(BN, nk, S, NO, H) > kTcSmemLimit) --S;
    }
    if (H == 1 || (2 * H * BN <= 512 && S >= 2)) break;
  }
  // the persistent form where it measured faster: up to 128 outputs per tile (the weight einsum
  // of the 721x1440 and 361x720 layers); the transposed einsum's 192-row tiles keep the
  // one-tile kernel, which ran them faster
  if (S >= 2 && BN <= 128 && !(reinterpret_cast<uintptr_t>(a.out) & 15)) {
    const cuuint64_t di[3] = {(cuuint64_t)a.N, (cuuint64_t)a.Rg, (cuuint64_t)a.B * a.G};
    const cuuint64_t si[2] = {(cuuint64_t)a.N * 2, (cuuint64_t)a.Rg * a.N * 2};
    const cuuint32_t bi[3] = {64, 64, 1};
    const cuuint64_t dw[2] = {(cuuint64_t)a.Rg, (cuuint64_t)a.G * a.Mg};
    const cuuint64_t sw[1] = {(cuuint64_t)a.Rg * 2};
    const cuuint32_t bw[2] = {64, (cuuint32_t)BN};
    const cuuint64_t dq[3] = {(cuuint64_t)a.N, (cuuint64_t)a.Mg, (cuuint64_t)a.B * a.G};
    const cuuint64_t sq[2] = {(cuuint64_t)a.N * 2, (cuuint64_t)a.Mg * a.N * 2};
    const cuuint32_t bq[3] = {64, (cuuint32_t)BN, 1};
    if (!make_map(&mi, a.in, 3, di, si, bi) || !make_map(&mw, a.wm, 2, dw, sw, bw) ||
        !tc::encode_bf16_map(&mo, a.out, 3, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    int dev = 0, n_sm = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int NT = (a.N + 128 * H - 1) / (128 * H), MT = (a.Mg + BN - 1) / BN;
    const long T = (long)NT * MT * a.B * a.G;
    if (T > 0x7FFFFFFFL) return cudaErrorInvalidValue;
    MixPArgs p{a.bias, a.G, a.Mg, a.Rg, a.N, BN, S, NT, MT, (int)T, NO};
    // at least half the shared memory, so that one CTA (and its tensor memory) holds an SM
    const size_t smem = std::max(mixp_smem(BN, nk, S, NO, H), (size_t)kTcSmemLimit / 2 + 1024);
    auto kern = H == 2 ? mix_tc_persistent_kernel<2> : mix_tc_persistent_kernel<1>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(int)std::min<long>(T, n_sm), 192, smem, st>>>(mi, mw, mo, p);
    count_launch();
    return cudaGetLastError();
  }
  const cuuint64_t di[3] = {(cuuint64_t)a.N, (cuuint64_t)a.Rg, (cuuint64_t)a.B * a.G};
  const cuuint64_t si[2] = {(cuuint64_t)a.N * 2, (cuuint64_t)a.Rg * a.N * 2};
  const cuuint32_t bi[3] = {64, 64, 1};
  const cuuint64_t dw[2] = {(cuuint64_t)a.Rg, (cuuint64_t)a.G * a.Mg};
  const cuuint64_t sw[1] = {(cuuint64_t)a.Rg * 2};
  const cuuint32_t bw[2] = {64, (cuuint32_t)BN};
  if (!make_map(&mi, a.in, 3, di, si, bi) || !make_map(&mw, a.wm, 2, dw, sw, bw)) return cudaErrorInvalidValue;
  const int S1 = std::min(kStages, nk);
  MixTcArgs t{a.out, a.bias, a.G, a.Mg, a.Rg, a.N, BN, S1};
  const size_t smem = mix_smem(BN, S1);
  cudaError_t e = cudaFuncSetAttribute(mix_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.N + 127) / 128, (a.Mg + BN - 1) / BN, a.B * a.G);
  mix_tc_kernel<<<grid, 128, smem, st>>>(mi, mw, t);
  count_launch();
  return cudaGetLastError();
}

bool dw_tc_supported(int Og, int Rg, int N) {
  // every M tile's accumulator in tensor memory and at least two stages in shared memory
  const int T = (Rg + 127) / 128;
  const size_t st_bytes = (size_t)T * 128 * 128 + (size_t)Og * 128;
  return tc::encode_tiled_fn() != nullptr && Og % 16 == 0 && Og <= 256 && N % 8 == 0 && Rg >= 1 && T * Og <= 512 &&
         2 * st_bytes + 1280 <= kTcSmemLimit;
}

cudaError_t launch_dw_tc(const DwArgs& a, cudaStream_t st) {
  CUtensorMap my, md;
  const cuuint64_t dy[3] = {(cuuint64_t)a.N, (cuuint64_t)a.Rg, (cuuint64_t)a.B * a.G};
  const cuuint64_t sy[2] = {(cuuint64_t)a.N * 2, (cuuint64_t)a.Rg * a.N * 2};
  const cuuint32_t by[3] = {64, 128, 1};
  const cuuint64_t dd[3] = {(cuuint64_t)a.N, (cuuint64_t)a.Og, (cuuint64_t)a.B * a.G};
  const cuuint64_t sd[2] = {(cuuint64_t)a.N * 2, (cuuint64_t)a.Og * a.N * 2};
  const cuuint32_t bd[3] = {64, (cuuint32_t)a.Og, 1};
  if (!make_map(&my, a.yv, 3, dy, sy, by) || !make_map(&md, a.dout, 3, dd, sd, bd)) return cudaErrorInvalidValue;
  const int T = (a.Rg + 127) / 128;
  const size_t st_bytes = (size_t)T * 128 * 128 + (size_t)a.Og * 128;
  const int S = (int)std::min<size_t>(kStages, (kTcSmemLimit - 1024 - 256) / st_bytes);
  if (S < 2 || T * a.Og > 512) return cudaErrorInvalidValue;
  const int ones = (a.bpart && a.Rg % 128) ? a.Rg % 128 : -1;
  DwTcArgs t{a.part, ones >= 0 ? a.bpart : nullptr, a.G, a.Og, a.Rg, a.N, a.nc, a.nchunk, T, S, ones};
  const size_t smem = 1024 + (size_t)S * st_bytes + (2 * S + 2) * 8;
  cudaError_t e = cudaFuncSetAttribute(dw_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nchunk, 1, a.B * a.G);
  dw_tc_kernel<<<grid, 128, smem, st>>>(my, md, t);
  count_launch();
  if (a.bpart && ones < 0) {
    dim3 g2(a.nchunk, a.B * a.G);
    bias_partial_kernel<<<g2, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a.dout), a.bpart, a.G, a.Og, a.N, a.nc,
                                            a.nchunk);
    count_launch();
  }
  return cudaGetLastError();
}

int take_mix_tc_status() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
  return v;
}

}  // namespace disco
