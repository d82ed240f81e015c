// Fused DISCO forward, SIMT form (used for fp32 layers).
//
// The `fused` mode of the page "torch_harmonics.DiscreteContinuousConvS2"
// fuses the sparse contraction and the weight einsum so that the K-expanded
// intermediate y is never stored.  One CTA owns output row j, a block of qb
// output longitudes and one (batch, group): it contracts every input channel
// of the group into an on-chip y tile [Cg*K][qb] (rounded to the storage type,
// exactly as the unfused path stores y), then mixes the tile with w into the
// out block.  y never reaches device memory.
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace disco {
namespace {

constexpr int kThreads = 256;

template <int K, int S, int W>
__device__ __forceinline__ void chunk_fma(float (&acc)[K][kTaskR], const float* __restrict__ win_ptr,
                                          const float* __restrict__ v, int kmask) {
  constexpr int NW = (kTaskR - 1) * S + W;
  float win[NW];
#pragma unroll
  for (int t = 0; t < NW; ++t) win[t] = win_ptr[t];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (kmask & (1 << k)) {
#pragma unroll
      for (int u = 0; u < W; ++u) {
        const float vv = __ldg(v + k * kChunkW + u);
#pragma unroll
        for (int r = 0; r < kTaskR; ++r) acc[k][r] = fmaf(vv, win[r * S + u], acc[k][r]);
      }
    }
  }
}

template <typename T, int K, int S>
__global__ void __launch_bounds__(kThreads) fused_simt_kernel(FusedArgs f) {
  extern __shared__ float smem[];
  int* soff = reinterpret_cast<int*>(smem);
  float* ytile = smem + kMaxSrc + 4;
  float* stage = ytile + f.ytile_floats;
  const GatherArgs& a = f.g;
  const T* x = static_cast<const T*>(f.x);
  const T* w = static_cast<const T*>(f.w);
  const T* bias = static_cast<const T*>(f.bias);
  T* out = static_cast<T*>(f.out);
  const RowPlan rp = a.rows[blockIdx.y];
  const int q0 = blockIdx.x * a.qb;
  const int b = blockIdx.z / f.G, g = blockIdx.z % f.G;
  const int Cg = f.C_in / f.G, Og = f.C_out / f.G;
  int stage_elems;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int s = rp.src_begin; s < rp.src_end; ++s) {
      soff[s - rp.src_begin] = acc;
      acc += staged_len(a.srcs[s].span, a.qb, S);
    }
    soff[rp.src_end - rp.src_begin] = acc;
  }
  __syncthreads();
  stage_elems = soff[rp.src_end - rp.src_begin];
  const int cg = max(1, min(Cg, a.stage_budget / max(1, stage_elems)));
  const int tasks_per_ch = a.qb / kTaskR;
  const size_t x_chan = (size_t)a.n_src_rows * a.n_src;
  const int cbase = b * f.C_in + g * Cg;
  for (int c0 = 0; c0 < Cg; c0 += cg) {
    const int ncg = min(cg, Cg - c0);
    for (int s = rp.src_begin; s < rp.src_end; ++s) {
      const SrcRow sr = a.srcs[s];
      const int len = staged_len(sr.span, a.qb, S);
      const int first = q0 * S + sr.start;
      for (int c = 0; c < ncg; ++c) {
        const T* row = x + (size_t)(cbase + c0 + c) * x_chan + (size_t)sr.row * a.n_src;
        float* dst = stage + (size_t)c * stage_elems + soff[s - rp.src_begin];
        for (int t = threadIdx.x; t < len; t += blockDim.x) dst[t] = to_f32(row[wrap_mod(first + t, a.n_src)]);
      }
    }
    __syncthreads();
    for (int task = threadIdx.x; task < ncg * tasks_per_ch; task += blockDim.x) {
      const int c = task / tasks_per_ch;
      const int m0 = (task - c * tasks_per_ch) * kTaskR;
      const float* sb = stage + (size_t)c * stage_elems + m0 * S;
      float acc[K][kTaskR];
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int r = 0; r < kTaskR; ++r) acc[k][r] = 0.0f;
      for (int ch = rp.chunk_start[0]; ch < rp.chunk_end[0]; ++ch) {
        const Chunk cc = a.chunks[ch];
        const float* wp = sb + soff[cc.src] + cc.t0;
        const float* v = a.vals + cc.voff;
        const int kmask = cc.wk >> 8;
        switch (cc.wk & 0xff) {
          case 1: chunk_fma<K, S, 1>(acc, wp, v, kmask); break;
          case 2: chunk_fma<K, S, 2>(acc, wp, v, kmask); break;
          case 3: chunk_fma<K, S, 3>(acc, wp, v, kmask); break;
          case 4: chunk_fma<K, S, 4>(acc, wp, v, kmask); break;
          case 5: chunk_fma<K, S, 5>(acc, wp, v, kmask); break;
          case 6: chunk_fma<K, S, 6>(acc, wp, v, kmask); break;
          case 7: chunk_fma<K, S, 7>(acc, wp, v, kmask); break;
          default: chunk_fma<K, S, 8>(acc, wp, v, kmask); break;
        }
      }
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int r = 0; r < kTaskR; ++r)
          ytile[((size_t)(c0 + c) * K + k) * a.qb + m0 + r] = round_trip<T>(acc[k][r]);
    }
    __syncthreads();
  }
  const int R = Cg * K;
  for (int idx = threadIdx.x; idx < Og * a.qb; idx += blockDim.x) {
    const int o = idx / a.qb, m = idx - o * a.qb;
    if (q0 + m >= a.n_out) continue;
    const int oc = g * Og + o;
    const T* wr = w + (size_t)oc * R;
    float acc = 0.0f;
    for (int r = 0; r < R; ++r) acc = fmaf(to_f32(wr[r]), ytile[(size_t)r * a.qb + m], acc);
    if (bias) acc += to_f32(bias[oc]);
    out[(((size_t)b * f.C_out + oc) * a.n_out_rows + rp.row) * a.n_out + q0 + m] = from_f32<T>(acc);
  }
}

template <typename T, int K, int S>
cudaError_t launch_t(const FusedArgs& f, cudaStream_t st) {
  auto kern = fused_simt_kernel<T, K, S>;
  const size_t smem = (size_t)(kMaxSrc + 4 + f.ytile_floats + f.g.stage_budget) * 4;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(f.g.nblk, f.g.n_rows, f.B * f.G);
  kern<<<grid, kThreads, smem, st>>>(f);
  count_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_k(int K, int S, const FusedArgs& f, cudaStream_t st) {
#define DISCO_FUSED_CASE(KK)                          \
  if (K == KK) {                                      \
    if (S == 1) return launch_t<T, KK, 1>(f, st);     \
    if (S == 2) return launch_t<T, KK, 2>(f, st);     \
  }
  DISCO_FUSED_CASE(3)
  DISCO_FUSED_CASE(5)
  DISCO_FUSED_CASE(7)
  DISCO_FUSED_CASE(9)
#undef DISCO_FUSED_CASE
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_fused_simt(bool bf16, int K, int S, const FusedArgs& f, cudaStream_t st) {
  return bf16 ? launch_k<__nv_bfloat16>(K, S, f, st) : launch_k<float>(K, S, f, st);
}

}  // namespace disco
