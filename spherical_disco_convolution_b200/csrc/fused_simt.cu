// Fused DISCO forward, SIMT form (used for fp32 layers).
//
// The `fused` mode of the page "torch_harmonics.DiscreteContinuousConvS2"
// fuses the sparse contraction and the weight einsum so that the K-expanded
// intermediate y is never stored.  One CTA owns output row j, a block of qb
// output longitudes and one (batch, group): it contracts every input channel
// of the group into an on-chip y tile [Cg*K][qb] (rounded to the storage type,
// exactly as the unfused path stores y), then mixes the tile with w into the
// out block.  y never reaches device memory.
#include "gather_common.cuh"

namespace disco {
namespace {

constexpr int kThreads = 256;

template <typename T, int K, int S>
__global__ void __launch_bounds__(kThreads) fused_simt_kernel(FusedArgs f) {
  extern __shared__ __align__(16) float smem[];
  const GatherArgs& a = f.g;
  const GatherSmem s = gather_smem(smem, a.chunk_cache, K);
  float* ytile = s.stage + a.stage_budget;
  const T* x = static_cast<const T*>(f.x);
  const T* w = static_cast<const T*>(f.w);
  const T* bias = static_cast<const T*>(f.bias);
  T* out = static_cast<T*>(f.out);
  const RowPlan rp = a.rows[blockIdx.y];
  const int q0 = blockIdx.x * a.qb;
  const int b = blockIdx.z / f.G, g = blockIdx.z % f.G;
  const int Cg = f.C_in / f.G, Og = f.C_out / f.G;
  const int ch_begin = rp.chunk_start[0], nch = rp.chunk_end[0] - rp.chunk_start[0];
  const int se = gather_prologue(a, rp, ch_begin, rp.chunk_end[0], S, K, s);
  const int cg = max(1, min(min(Cg, kMaxCb), a.stage_budget / max(1, se)));
  const int cbase = b * f.C_in + g * Cg;
  for (int c0 = 0; c0 < Cg; c0 += cg) {
    const int ncg = min(cg, Cg - c0);
    auto sink = [&](int c, int m0, float (&acc)[K][kTaskR]) {
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int r = 0; r < kTaskR; ++r)
          ytile[((size_t)(c0 + c) * K + k) * a.qb + m0 + r] = round_trip<T>(acc[k][r]);
    };
    fwd_block<T, K, S>(a, rp, s, se, x, cbase + c0, ncg, q0 * S, ch_begin, nch, sink);
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
  const size_t smem = (gather_smem_floats(f.g.chunk_cache, K, f.g.stage_budget) + f.ytile_floats) * 4;
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
