// Fused DISCO forward on tensor cores (bf16 storage, fp32 accumulate).
//
// The `fused` mode of the page "torch_harmonics.DiscreteContinuousConvS2"
// contracts and mixes in one region so the K-expanded intermediate is never
// stored.  One CTA owns output row j, a block of 128 output longitudes and one
// (batch, group):
//   1. the SIMT gather (gather_common.cuh) contracts the group's input channels
//      into an on-chip y tile Y[q][r], r = c*K + k, rounded to bf16 exactly as
//      the unfused path stores y;
//   2. one thread issues tcgen05.mma: D[q][o] += Y[q][r] * w[g*Og + o][r], with
//      Y as an MN-major operand (no swizzle, one 16-byte row of 8 longitudes per
//      (r, 8-longitude block)) and w staged by TMA (K-major, 128-byte swizzle);
//   3. the eight warps read D from tensor memory and store out (+ bias).
// Channels are taken in passes whose y tile fits in shared memory; the
// accumulator stays in tensor memory across passes.
#include <cuda.h>

#include "gather_common.cuh"
#include "tc_common.cuh"

namespace disco {
namespace {

constexpr int kThreads = 256;
constexpr int kQ = 128;  // outputs per CTA = MMA M

struct FusedTcArgs {
  GatherArgs g;
  const void* x;
  const void* bias;
  void* out;
  int B, C_in, C_out, G, K;
  int pass_ch;       // channels per pass (pass_ch * K a multiple of 16)
  int a_sbo;         // bytes between 8-longitude blocks of the y tile
  int w_chunks;      // 64-wide r chunks of w
};

template <int K, int S>
__global__ void __launch_bounds__(kThreads, 1) fused_tc_kernel(const __grid_constant__ CUtensorMap map_w,
                                                               FusedTcArgs f) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const GatherArgs& a = f.g;
  float* gsm = reinterpret_cast<float*>(smem_raw);
  const GatherSmem s = gather_smem(gsm, a.chunk_cache, K);
  uint8_t* ytile = reinterpret_cast<uint8_t*>(s.stage + a.stage_budget);
  const size_t y_bytes = (size_t)16 * f.a_sbo;
  uint8_t* wsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ytile + y_bytes) + 1023) & ~uintptr_t(1023));
  const int Cg = f.C_in / f.G, Og = f.C_out / f.G;
  uint64_t* bars = reinterpret_cast<uint64_t*>(wsm + (size_t)f.w_chunks * Og * 128);
  uint64_t* w_full = bars;
  uint64_t* mma_done = bars + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

  const RowPlan rp = a.rows[blockIdx.y];
  const int q0 = blockIdx.x * kQ;
  const int bgi = blockIdx.z;
  const int b = bgi / f.G, g = bgi % f.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t ncols = 32;
  while ((int)ncols < Og) ncols <<= 1;

  if (threadIdx.x == 0) {
    tc::prefetch_map(&map_w);
    tc::mbar_init(w_full, 1);
    tc::mbar_init(mma_done, 1);
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, ncols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  const int ch_begin = rp.chunk_start[0], nch = rp.chunk_end[0] - rp.chunk_start[0];
  const int se = gather_prologue(a, rp, ch_begin, rp.chunk_end[0], S, K, s);  // contains __syncthreads
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    tc::mbar_arrive_expect_tx(w_full, (uint32_t)(f.w_chunks * Og * 128));
    for (int t = 0; t < f.w_chunks; ++t) tc::tma_load_2d(wsm + (size_t)t * Og * 128, &map_w, w_full, t * 64, g * Og);
  }

  const int cg_max = max(1, min(kMaxCb, a.stage_budget / max(1, se)));
  const uint32_t idesc = tc::idesc_bf16(kQ, Og, true, false);
  const int cbase = b * f.C_in + g * Cg;
  bool ok = true;
  int pass = 0;
  for (int pc0 = 0; pc0 < Cg; pc0 += f.pass_ch, ++pass) {
    const int pn = min(f.pass_ch, Cg - pc0);
    if (pass > 0) {  // the previous pass's MMAs must be done reading the y tile
      ok = ok && tc::mbar_wait(mma_done, (pass - 1) & 1);
      tc::fence_after_sync();
    }
    for (int c0 = pc0; c0 < pc0 + pn; c0 += cg_max) {
      const int ncg = min(cg_max, pc0 + pn - c0);
      auto sink = [&](int c, int m0, float (&acc)[K][kTaskR]) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
          const int r = (c0 + c - pc0) * K + k;
          __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[k][0], acc[k][1]);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[k][2], acc[k][3]);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[k][4], acc[k][5]);
          __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[k][6], acc[k][7]);
          uint4 pk;
          pk.x = *reinterpret_cast<uint32_t*>(&h0);
          pk.y = *reinterpret_cast<uint32_t*>(&h1);
          pk.z = *reinterpret_cast<uint32_t*>(&h2);
          pk.w = *reinterpret_cast<uint32_t*>(&h3);
          *reinterpret_cast<uint4*>(ytile + (size_t)(m0 / 8) * f.a_sbo + (size_t)r * 16) = pk;
        }
      };
      fwd_block<__nv_bfloat16, K, S>(a, rp, s, se, static_cast<const __nv_bfloat16*>(f.x), cbase + c0, ncg, q0 * S,
                                     ch_begin, nch, sink);  // ends with __syncthreads
    }
    // the y tile was written through the generic proxy; the MMA reads it through the async proxy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc::fence_after_sync();
      if (pass == 0) ok = ok && tc::mbar_wait(w_full, 0);
      const uint32_t a0 = tc::smem_u32(ytile);
      const uint32_t w0 = tc::smem_u32(wsm);
      const int ksteps = pn * K / 16;
      for (int ks = 0; ks < ksteps; ++ks) {
        const int rg = pc0 * K + ks * 16;  // global r of this K step
        const uint64_t ad = tc::desc_sw128(a0 + ks * 256, 128, f.a_sbo) & ~((uint64_t)7 << 61);  // no swizzle
        const uint64_t bd = tc::desc_sw128(w0 + (uint32_t)((rg / 64) * Og * 128 + (rg % 64) * 2), 16, 1024);
        tc::mma_bf16(tmem, ad, bd, idesc, (pass | ks) != 0);
      }
      tc::mma_commit(mma_done);
    }
  }
  ok = ok && tc::mbar_wait(mma_done, (pass - 1) & 1);
  tc::fence_after_sync();
  // epilogue: warp w reads TMEM lanes of quadrant w%4; warps 0-3 take the first half of the columns
  const int quad = warp & 3, half = warp >> 2;
  const int q = q0 + quad * 32 + lane;
  const int cols = Og / 2;
  const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(f.bias);
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(f.out);
  for (int c = half * cols; c < half * cols + cols; c += 16) {
    float v[16];
    tc::tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c, v);
    if (ok && q < a.n_out) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int oc = g * Og + c + i;
        const float bv = bias ? __bfloat162float(bias[oc]) : 0.0f;
        out[(((size_t)b * f.C_out + oc) * a.n_out_rows + rp.row) * a.n_out + q] = __float2bfloat16_rn(v[i] + bv);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, ncols);
}

// Shared memory: [gather layout][y tile: 16 blocks x a_sbo][pad to 1024][w chunks][barriers]
size_t fused_tc_smem(const FusedTcArgs& f, int K) {
  const int Og = f.C_out / f.G;
  size_t n = gather_smem_floats(f.g.chunk_cache, K, f.g.stage_budget) * 4 + (size_t)16 * f.a_sbo;
  n = (n + 1023) & ~size_t(1023);
  return n + (size_t)f.w_chunks * Og * 128 + 64 + 1024;
}

template <int K, int S>
cudaError_t launch_t(const FusedTcArgs& f, const void* w, cudaStream_t st) {
  const int Og = f.C_out / f.G, R = (f.C_in / f.G) * K;
  CUtensorMap mw;
  const cuuint64_t dims[2] = {(cuuint64_t)R, (cuuint64_t)f.C_out};
  const cuuint64_t strides[1] = {(cuuint64_t)R * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)Og};
  if (!tc::encode_bf16_map(&mw, w, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  auto kern = fused_tc_kernel<K, S>;
  const size_t smem = fused_tc_smem(f, K);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(f.g.nblk, f.g.n_rows, f.B * f.G);
  kern<<<grid, kThreads, smem, st>>>(mw, f);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

// Fills the pass layout of a fused tensor-core launch; false when the layer does not fit it.
bool fused_tc_plan(int C_in, int C_out, int G, int K, int chunk_cache, int stage_floats, int* pass_ch, int* a_sbo,
                   int* w_chunks, size_t* smem) {
  const int Cg = C_in / G, Og = C_out / G, R = Cg * K;
  if (Og % 32 || Og > 256 || Cg % 16 || R % 8) return false;
  int pc = 16;
  while (pc + 16 <= Cg && (size_t)16 * ((pc + 16) * K * 16 + 16) <= 80 * 1024) pc += 16;
  *pass_ch = pc;
  *a_sbo = pc * K * 16 + 16;
  *w_chunks = (R + 63) / 64;
  if ((size_t)*w_chunks * Og * 128 > 96 * 1024) return false;
  FusedTcArgs f{};
  f.g.chunk_cache = chunk_cache;
  f.g.stage_budget = stage_floats;
  f.C_in = C_in;
  f.C_out = C_out;
  f.G = G;
  f.a_sbo = *a_sbo;
  f.w_chunks = *w_chunks;
  *smem = fused_tc_smem(f, K);
  return *smem <= 227 * 1024;
}

int take_fused_tc_status() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (v) cudaMemcpyToSymbol(g_device_status, &z, sizeof(int));
  return v;
}

cudaError_t launch_fused_tc(int K, int S, const GatherArgs& g, const void* x, const void* w, const void* bias,
                            void* out, int B, int C_in, int C_out, int G, int pass_ch, int a_sbo, int w_chunks,
                            cudaStream_t st) {
  FusedTcArgs f;
  f.g = g;
  f.x = x;
  f.bias = bias;
  f.out = out;
  f.B = B;
  f.C_in = C_in;
  f.C_out = C_out;
  f.G = G;
  f.K = K;
  f.pass_ch = pass_ch;
  f.a_sbo = a_sbo;
  f.w_chunks = w_chunks;
#define DISCO_FTC_CASE(KK)                             \
  if (K == KK) {                                       \
    if (S == 1) return launch_t<KK, 1>(f, w, st);      \
    if (S == 2) return launch_t<KK, 2>(f, w, st);      \
  }
  DISCO_FTC_CASE(3)
  DISCO_FTC_CASE(5)
  DISCO_FTC_CASE(7)
  DISCO_FTC_CASE(9)
#undef DISCO_FTC_CASE
  return cudaErrorNotSupported;
}

}  // namespace disco
