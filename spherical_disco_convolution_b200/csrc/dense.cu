// Dense channel contractions of the DISCO layer (SIMT fp32-accumulate forms).
//
// The weight einsum of the forward equation on the page
// "torch_harmonics.DiscreteContinuousConvS2" (sum over c_i and k of
// w_k^{co,ci} times the contracted signal) is, per batch and group, a GEMM
//   out[g*Mg + m, n] = sum_r wm[g, m, r] * in[g*Rg + r, n]  (+ bias)
// with n running over the output grid.  The same kernel serves the transposed
// einsum of the backward pass (dy = w^T dout).  The weight gradient is the
// split-K GEMM dw[o, r] = sum_n dout[o, n] * y[r, n] reduced in a fixed order.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace disco {
namespace {

constexpr int kBM = 64, kBN = 128, kBK = 16;

// C tile 64 x 128 per CTA, 4 x 8 per thread.
template <typename T>
__global__ void __launch_bounds__(256) mix_kernel(MixArgs a) {
  __shared__ __align__(16) float As[kBK][kBM];
  __shared__ __align__(16) float Bs[kBK][kBN];
  const T* in = static_cast<const T*>(a.in);
  const T* wm = static_cast<const T*>(a.wm);
  const T* bias = static_cast<const T*>(a.bias);
  T* out = static_cast<T*>(a.out);
  const int n0 = blockIdx.x * kBN;
  const int m0 = blockIdx.y * kBM;
  const int bg = blockIdx.z;
  const int b = bg / a.G, g = bg - b * a.G;
  const T* A = wm + (size_t)g * a.Mg * a.Rg;
  const T* Bm = in + ((size_t)b * a.G + g) * a.Rg * (size_t)a.N;
  const int tid = threadIdx.x;
  const int tm = tid / 16, tn = tid % 16;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int r0 = 0; r0 < a.Rg; r0 += kBK) {
    for (int t = tid; t < kBK * kBM; t += 256) {
      const int kk = t % kBK, mm = t / kBK;
      const int m = m0 + mm, r = r0 + kk;
      As[kk][mm] = (m < a.Mg && r < a.Rg) ? to_f32(A[(size_t)m * a.Rg + r]) : 0.0f;
    }
    for (int t = tid; t < kBK * kBN; t += 256) {
      const int kk = t / kBN, nn = t % kBN;
      const int n = n0 + nn, r = r0 + kk;
      Bs[kk][nn] = (n < a.N && r < a.Rg) ? to_f32(Bm[(size_t)r * a.N + n]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][tm * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tn * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][tn * 8 + 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tm * 4 + i;
    if (m >= a.Mg) continue;
    const float bv = bias ? to_f32(bias[g * a.Mg + m]) : 0.0f;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = acc[i][j] + bv;
    const int n = n0 + tn * 8;
    if (n >= a.N) continue;
    T* dst = out + (((size_t)b * a.G + g) * a.Mg + m) * (size_t)a.N + n;
    store_run<T, 8>(dst, v, min(8, a.N - n));
  }
}

template <typename T>
__global__ void transpose_weight_kernel(const T* __restrict__ w, T* __restrict__ wt, int G, int Og, int Cg, int K) {
  const int total = G * Og * Cg * K;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < total; t += gridDim.x * blockDim.x) {
    // t indexes wt[g][c*K + k][o]
    const int o = t % Og;
    const int ck = (t / Og) % (Cg * K);
    const int g = t / (Og * Cg * K);
    wt[t] = w[((size_t)(g * Og + o)) * Cg * K + ck];
  }
}

constexpr int kDM = 64, kDN = 64, kDK = 32;

// Partial weight gradient for one split (b, chunk), tile 64 (o) x 64 (r).
template <typename T>
__global__ void __launch_bounds__(256) dw_partial_kernel(DwArgs a) {
  __shared__ __align__(16) float As[kDK][kDM + 4];
  __shared__ __align__(16) float Bs[kDK][kDN + 4];
  const T* dout = static_cast<const T*>(a.dout);
  const T* yv = static_cast<const T*>(a.yv);
  const int chunk = blockIdx.x;
  const int ntile_r = (a.Rg + kDN - 1) / kDN;
  const int ot = blockIdx.y / ntile_r, rt = blockIdx.y % ntile_r;
  const int b = blockIdx.z / a.G, g = blockIdx.z % a.G;
  const int o0 = ot * kDM, r0 = rt * kDN;
  const int nb = chunk * a.nc, ne = min(a.N, nb + a.nc);
  const T* A = dout + ((size_t)b * a.G + g) * a.Og * (size_t)a.N;
  const T* Bm = yv + ((size_t)b * a.G + g) * a.Rg * (size_t)a.N;
  const int tid = threadIdx.x;
  const int to = tid / 16, tr = tid % 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  float bsum = 0.0f;
  const bool do_bias = a.bpart && rt == 0;
  for (int n0 = nb; n0 < ne; n0 += kDK) {
    for (int t = tid; t < kDK * kDM; t += 256) {
      const int kk = t % kDK, mm = t / kDK;
      const int o = o0 + mm, n = n0 + kk;
      As[kk][mm] = (o < a.Og && n < ne) ? to_f32(A[(size_t)o * a.N + n]) : 0.0f;
    }
    for (int t = tid; t < kDK * kDN; t += 256) {
      const int kk = t % kDK, rr = t / kDK;
      const int r = r0 + rr, n = n0 + kk;
      Bs[kk][rr] = (r < a.Rg && n < ne) ? to_f32(Bm[(size_t)r * a.N + n]) : 0.0f;
    }
    __syncthreads();
    if (do_bias && tid < kDM) {
      for (int kk = 0; kk < kDK; ++kk) bsum += As[kk][tid];
    }
#pragma unroll 8
    for (int kk = 0; kk < kDK; ++kk) {
      float ar[4], br[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) ar[i] = As[kk][to * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) br[j] = Bs[kk][tr * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
    __syncthreads();
  }
  const size_t split = (size_t)b * a.nchunk + chunk;
  float* P = a.part + ((split * a.G + g) * a.Og) * (size_t)a.Rg;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int o = o0 + to * 4 + i;
    if (o >= a.Og) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + tr * 4 + j;
      if (r < a.Rg) P[(size_t)o * a.Rg + r] = acc[i][j];
    }
  }
  if (do_bias && tid < kDM && o0 + tid < a.Og) a.bpart[split * (a.G * a.Og) + g * a.Og + o0 + tid] = bsum;
}

template <typename T>
__global__ void dw_reduce_kernel(const float* __restrict__ part, const float* __restrict__ bpart, T* __restrict__ dw,
                                 T* __restrict__ dbias, int nsplit, int G, int Og, int Rg) {
  const int per = G * Og * Rg;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < per) {
    float acc = 0.0f;
    for (int s = 0; s < nsplit; ++s) acc += part[(size_t)s * per + t];
    dw[t] = from_f32<T>(acc);  // part index (g, o, r) == dw index (g*Og + o, r)
  }
  if (dbias && t < G * Og) {
    float acc = 0.0f;
    for (int s = 0; s < nsplit; ++s) acc += bpart[(size_t)s * G * Og + t];
    dbias[t] = from_f32<T>(acc);
  }
}

}  // namespace

cudaError_t launch_mix_simt(bool bf16, const MixArgs& a, cudaStream_t st) {
  dim3 grid((a.N + kBN - 1) / kBN, (a.Mg + kBM - 1) / kBM, a.B * a.G);
  if (bf16)
    mix_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  else
    mix_kernel<float><<<grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_transpose_weight(bool bf16, const void* w, void* wt, int G, int Og, int Cg, int K, cudaStream_t st) {
  const int total = G * Og * Cg * K;
  const int blocks = (total + 255) / 256;
  if (bf16)
    transpose_weight_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w),
                                                                   static_cast<__nv_bfloat16*>(wt), G, Og, Cg, K);
  else
    transpose_weight_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(w), static_cast<float*>(wt), G,
                                                           Og, Cg, K);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_dw_partial_simt(bool bf16, const DwArgs& a, cudaStream_t st) {
  dim3 grid(a.nchunk, ((a.Og + kDM - 1) / kDM) * ((a.Rg + kDN - 1) / kDN), a.B * a.G);
  if (bf16)
    dw_partial_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  else
    dw_partial_kernel<float><<<grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

namespace {
// t[p][rows[r]][0..n) = 0 for every plane p: one CTA per (row, plane block), 16-byte stores.
// With vec (base address and row length multiples of 16 bytes) 16-byte stores, else bytes.
__global__ void zero_rows_kernel(uint8_t* t, const int* __restrict__ rows, int n_rows, int planes, int nrows,
                                 size_t row_bytes, bool vec) {
  const int r = rows[blockIdx.x];
  for (int p = blockIdx.y; p < planes; p += gridDim.y) {
    uint8_t* base = t + ((size_t)p * nrows + r) * row_bytes;
    if (vec) {
      for (size_t o = (size_t)threadIdx.x * 16; o < row_bytes; o += (size_t)blockDim.x * 16)
        *reinterpret_cast<uint4*>(base + o) = make_uint4(0u, 0u, 0u, 0u);
    } else {
      for (size_t o = threadIdx.x; o < row_bytes; o += blockDim.x) base[o] = 0;
    }
  }
}
}  // namespace

cudaError_t launch_zero_rows(void* t, int elem_bytes, const int* rows, int n_rows, int planes, int nrows, int nlon,
                             cudaStream_t st) {
  if (n_rows <= 0 || planes <= 0) return cudaSuccess;
  const size_t row_bytes = (size_t)nlon * elem_bytes;
  const bool vec = !(reinterpret_cast<uintptr_t>(t) & 15) && !(row_bytes & 15);
  dim3 grid(n_rows, std::min(planes, 64));
  zero_rows_kernel<<<grid, 128, 0, st>>>(static_cast<uint8_t*>(t), rows, n_rows, planes, nrows, row_bytes, vec);
  count_launch();
  return cudaGetLastError();
}

namespace {
// t[p][rows[r]][0..nlon) = bias[p % C] for every plane p (a plane is one (b, output channel))
template <typename T>
__global__ void fill_rows_kernel(T* t, const int* __restrict__ rows, int planes, int nrows, int nlon,
                                 const T* __restrict__ bias, int C) {
  const int r = rows[blockIdx.x];
  for (int p = blockIdx.y; p < planes; p += gridDim.y) {
    const T v = bias[p % C];
    T* base = t + ((size_t)p * nrows + r) * nlon;
    for (int q = threadIdx.x; q < nlon; q += blockDim.x) base[q] = v;
  }
}
}  // namespace

cudaError_t launch_fill_rows(bool bf16, void* t, const int* rows, int n_rows, int planes, int nrows, int nlon,
                             const void* bias, int C, cudaStream_t st) {
  if (!bias) return launch_zero_rows(t, bf16 ? 2 : 4, rows, n_rows, planes, nrows, nlon, st);
  if (n_rows <= 0 || planes <= 0) return cudaSuccess;
  dim3 grid(n_rows, std::min(planes, 64));
  if (bf16)
    fill_rows_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(static_cast<__nv_bfloat16*>(t), rows, planes, nrows, nlon,
                                                          static_cast<const __nv_bfloat16*>(bias), C);
  else
    fill_rows_kernel<float><<<grid, 128, 0, st>>>(static_cast<float*>(t), rows, planes, nrows, nlon,
                                                  static_cast<const float*>(bias), C);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_dw_reduce(bool bf16, const float* part, const float* bpart, void* dw, void* dbias, int nsplit,
                             int G, int Og, int Rg, cudaStream_t st) {
  const int per = G * Og * Rg;
  const int blocks = (per + 255) / 256;
  if (bf16)
    dw_reduce_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(part, bpart, static_cast<__nv_bfloat16*>(dw),
                                                            static_cast<__nv_bfloat16*>(dbias), nsplit, G, Og, Rg);
  else
    dw_reduce_kernel<float><<<blocks, 256, 0, st>>>(part, bpart, static_cast<float*>(dw), static_cast<float*>(dbias),
                                                    nsplit, G, Og, Rg);
  count_launch();
  return cudaGetLastError();
}

}  // namespace disco
