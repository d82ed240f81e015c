// Sparse Psi contraction kernels (SIMT gather form).
//
// Forward (page "torch_harmonics.DiscreteContinuousConvS2", forward equation):
//   y[bc, k, j, q] = sum_{(i,d)} Psi[k, j, (i, d)] * x[bc, i, (q*s + d) mod nlon_in]
// Adjoint of that map summed over k, used for dx after the weight einsum has
// been transposed (dy = w^T dout):
//   dx[bc, i, l] = sum_{(k, j, d) : (l - d) = s*q (mod nlon_in)} Psi[k, j, (i, d)] * dy[bc, k, j, q]
// which for l = s*m + rho reads dy[bc, k, j, m + e] with e = (rho - d)/s.
//
// One CTA owns one output row, a block of qb consecutive outputs and a block
// of channel planes.  It stages the source rows that the output row reaches
// in shared memory (fp32, wrap-around already unrolled, 16-byte vector moves),
// then every thread owns kTaskR consecutive outputs of one channel plane and
// walks the row's chunks: a window of (kTaskR-1)*step + w staged values is
// loaded once into registers and reused by all non-zero basis functions of
// the chunk.
#include "gather_common.cuh"

namespace disco {
namespace {

constexpr int kThreads = 256;

template <typename T, int K, int S>
__global__ void __launch_bounds__(kThreads) fwd_gather_kernel(GatherArgs a, const T* __restrict__ x,
                                                              T* __restrict__ y) {
  extern __shared__ __align__(16) float smem[];
  const GatherSmem s = gather_smem(smem, a.chunk_cache, K);
  const RowPlan rp = a.rows[blockIdx.z];
  const int q0 = blockIdx.y * a.qb;
  const int c_begin = blockIdx.x * a.cb;
  const int c_end = min(a.BC, c_begin + a.cb);
  const int ch_begin = rp.chunk_start[0], nch = rp.chunk_end[0] - rp.chunk_start[0];
  const int se = gather_prologue(a, rp, ch_begin, rp.chunk_end[0], S, K, s);
  const int cg = max(1, min(a.cb, a.stage_budget / max(1, se)));
  const int tasks_per_ch = a.qb / kTaskR;
  for (int c0 = c_begin; c0 < c_end; c0 += cg) {
    const int ncg = min(cg, c_end - c0);
    stage_rows<T>(a, rp, s, se, x, c0, ncg, q0 * S, S);
    __syncthreads();
    for (int task = threadIdx.x; task < ncg * tasks_per_ch; task += blockDim.x) {
      const int c = task / tasks_per_ch;
      const int m0 = (task - c * tasks_per_ch) * kTaskR;
      if (q0 + m0 >= a.n_out) continue;
      float acc[K][kTaskR];
      fwd_task<K, S>(acc, a, s, s.stage + (size_t)c * se + m0 * S, ch_begin, nch);
      const int n = min(kTaskR, a.n_out - (q0 + m0));
#pragma unroll
      for (int k = 0; k < K; ++k) {
        T* dst = y + (((size_t)(c0 + c) * K + k) * a.n_out_rows + rp.row) * a.n_out + q0 + m0;
        store_run<T, kTaskR>(dst, acc[k], n);
      }
    }
    __syncthreads();
  }
}

template <int W>
__device__ __forceinline__ void adj_chunk(float (&acc)[kTaskR], const float* __restrict__ win_ptr,
                                          const float* __restrict__ v) {
  constexpr int NW = kTaskR - 1 + W;
  float win[NW];
#pragma unroll
  for (int t = 0; t < NW; ++t) win[t] = win_ptr[t];
#pragma unroll
  for (int u = 0; u < W; ++u) {
    const float vv = v[u];
#pragma unroll
    for (int r = 0; r < kTaskR; ++r) acc[r] = fmaf(vv, win[r + u], acc[r]);
  }
}

template <typename T, int S>
__global__ void __launch_bounds__(kThreads) adj_gather_kernel(GatherArgs a, const T* __restrict__ dy,
                                                              T* __restrict__ dx) {
  extern __shared__ __align__(16) float smem[];
  const GatherSmem s = gather_smem(smem, a.chunk_cache, 1);
  const RowPlan rp = a.rows[blockIdx.z];
  const int m_blk = blockIdx.y * a.qb;
  const int c_begin = blockIdx.x * a.cb;
  const int c_end = min(a.BC, c_begin + a.cb);
  const int ch_begin = rp.chunk_start[0];
  const int se = gather_prologue(a, rp, ch_begin, rp.chunk_end[S - 1], 1, 1, s);
  const int cg = max(1, min(a.cb, a.stage_budget / max(1, se)));
  const int tasks_per_ch = a.qb / kTaskR;
  const int n_m = a.n_out / S;  // outputs l = S*m + rho, m < n_m
  for (int c0 = c_begin; c0 < c_end; c0 += cg) {
    const int ncg = min(cg, c_end - c0);
    stage_rows<T>(a, rp, s, se, dy, c0, ncg, m_blk, 1);
    __syncthreads();
    for (int task = threadIdx.x; task < ncg * tasks_per_ch; task += blockDim.x) {
      const int c = task / tasks_per_ch;
      const int m0 = (task - c * tasks_per_ch) * kTaskR;
      if (m_blk + m0 >= n_m) continue;
      const float* sb = s.stage + (size_t)c * se + m0;
      float acc[S][kTaskR];
#pragma unroll
      for (int rho = 0; rho < S; ++rho) {
#pragma unroll
        for (int r = 0; r < kTaskR; ++r) acc[rho][r] = 0.0f;
        for (int ch = rp.chunk_start[rho] - ch_begin; ch < rp.chunk_end[rho] - ch_begin; ++ch) {
          Chunk cc;
          const float* v;
          chunk_at(a, s, ch_begin, ch, 1, &cc, &v);
          const float* wp = sb + s.soff[cc.src] + cc.t0;
          switch (cc.wk & 0xff) {
            case 1: adj_chunk<1>(acc[rho], wp, v); break;
            case 2: adj_chunk<2>(acc[rho], wp, v); break;
            case 3: adj_chunk<3>(acc[rho], wp, v); break;
            case 4: adj_chunk<4>(acc[rho], wp, v); break;
            case 5: adj_chunk<5>(acc[rho], wp, v); break;
            case 6: adj_chunk<6>(acc[rho], wp, v); break;
            case 7: adj_chunk<7>(acc[rho], wp, v); break;
            default: adj_chunk<8>(acc[rho], wp, v); break;
          }
        }
      }
      const int nm = min(kTaskR, n_m - (m_blk + m0));
      T* dst = dx + ((size_t)(c0 + c) * a.n_out_rows + rp.row) * a.n_out + (size_t)S * (m_blk + m0);
      if constexpr (S == 1) {
        store_run<T, kTaskR>(dst, acc[0], nm);
      } else {
#pragma unroll
        for (int r = 0; r < kTaskR; ++r)
#pragma unroll
          for (int rho = 0; rho < S; ++rho)
            if (r < nm) dst[r * S + rho] = from_f32<T>(acc[rho][r]);
      }
    }
    __syncthreads();
  }
}

template <typename T, int K, int S>
cudaError_t launch_fwd_t(const GatherArgs& a, const void* x, void* y, cudaStream_t st) {
  auto kern = fwd_gather_kernel<T, K, S>;
  const size_t smem = gather_smem_floats(a.chunk_cache, K, a.stage_budget) * 4;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.BC + a.cb - 1) / a.cb, a.nblk, a.n_rows);
  kern<<<grid, kThreads, smem, st>>>(a, static_cast<const T*>(x), static_cast<T*>(y));
  count_launch();
  return cudaGetLastError();
}

template <typename T, int S>
cudaError_t launch_adj_t(const GatherArgs& a, const void* dy, void* dx, cudaStream_t st) {
  auto kern = adj_gather_kernel<T, S>;
  const size_t smem = gather_smem_floats(a.chunk_cache, 1, a.stage_budget) * 4;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.BC + a.cb - 1) / a.cb, a.nblk, a.n_rows);
  kern<<<grid, kThreads, smem, st>>>(a, static_cast<const T*>(dy), static_cast<T*>(dx));
  count_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fwd_k(int K, int S, const GatherArgs& a, const void* x, void* y, cudaStream_t st) {
#define DISCO_FWD_CASE(KK)                                           \
  if (K == KK) {                                                     \
    if (S == 1) return launch_fwd_t<T, KK, 1>(a, x, y, st);          \
    if (S == 2) return launch_fwd_t<T, KK, 2>(a, x, y, st);          \
  }
  DISCO_FWD_CASE(3)
  DISCO_FWD_CASE(5)
  DISCO_FWD_CASE(7)
  DISCO_FWD_CASE(9)
#undef DISCO_FWD_CASE
  return cudaErrorNotSupported;
}

}  // namespace

bool gather_supports(int K, int stride) {
  return (K == 3 || K == 5 || K == 7 || K == 9) && (stride == 1 || stride == 2);
}

cudaError_t launch_fwd_gather(bool bf16, int K, int S, const GatherArgs& a, const void* x, void* y, cudaStream_t st) {
  return bf16 ? launch_fwd_k<__nv_bfloat16>(K, S, a, x, y, st) : launch_fwd_k<float>(K, S, a, x, y, st);
}

cudaError_t launch_adj_gather(bool bf16, int S, const GatherArgs& a, const void* dy, void* dx, cudaStream_t st) {
  if (bf16) {
    if (S == 1) return launch_adj_t<__nv_bfloat16, 1>(a, dy, dx, st);
    if (S == 2) return launch_adj_t<__nv_bfloat16, 2>(a, dy, dx, st);
  } else {
    if (S == 1) return launch_adj_t<float, 1>(a, dy, dx, st);
    if (S == 2) return launch_adj_t<float, 2>(a, dy, dx, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace disco
