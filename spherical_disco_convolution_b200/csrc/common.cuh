// Device helpers shared by the libdisco kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace disco {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Value after a round trip through the storage type (what a store then load gives).
template <typename T>
__device__ __forceinline__ float round_trip(float v) { return to_f32(from_f32<T>(v)); }

__device__ __forceinline__ int wrap_mod(int a, int n) {
  int r = a % n;
  return r < 0 ? r + n : r;
}

// Stores n (<= R) consecutive values; vectorised when the run is full and aligned.
template <typename T, int R>
__device__ __forceinline__ void store_run(T* dst, const float (&v)[R], int n) {
  if (n == R && (reinterpret_cast<uintptr_t>(dst) % (R * sizeof(T))) == 0) {
    if constexpr (sizeof(T) == 2 && R == 8) {
      uint4 pk;
      __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
      __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
      pk.x = *reinterpret_cast<uint32_t*>(&h0);
      pk.y = *reinterpret_cast<uint32_t*>(&h1);
      pk.z = *reinterpret_cast<uint32_t*>(&h2);
      pk.w = *reinterpret_cast<uint32_t*>(&h3);
      *reinterpret_cast<uint4*>(dst) = pk;
      return;
    } else if constexpr (sizeof(T) == 4 && R == 8) {
      reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
      return;
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (r < n) dst[r] = from_f32<T>(v[r]);
}

}  // namespace disco
