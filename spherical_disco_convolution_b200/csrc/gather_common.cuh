// Shared pieces of the gather kernels: staging, ring sums, the chunk cache and
// the sliced per-row accumulation.
#pragma once

#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace disco {

constexpr int kMaxCb = 16;  // channel planes staged at once

// Dynamic shared memory layout of a gather CTA:
//   int   soff[kMaxSrc + 4]              staging offset of every source row (+ total)
//   Ring  rings[kMaxRing]                the row's ring terms
//   float rsum[kMaxCb * kMaxRing]        source-row sums of the rings, per staged channel
//   Chunk cch[chunk_cache]               the first chunk_cache chunks of the row
//   float cval[chunk_cache * nk * 8]     their values
//   float stage[...]                     staged source rows, channel after channel
struct GatherSmem {
  int* soff;
  Ring* rings;
  float* rsum;
  Chunk* cch;
  float* cval;
  float* stage;
};

__host__ __device__ inline size_t gather_fixed_floats(int chunk_cache, int nk) {
  return (size_t)(kMaxSrc + 4) + (size_t)kMaxRing * 4 + (size_t)kMaxCb * kMaxRing + (size_t)chunk_cache * 4 +
         (size_t)chunk_cache * nk * kChunkW;
}

__host__ __device__ inline size_t gather_smem_floats(int chunk_cache, int nk, int stage_floats) {
  return gather_fixed_floats(chunk_cache, nk) + stage_floats;
}

__device__ __forceinline__ GatherSmem gather_smem(float* smem, int chunk_cache, int nk) {
  GatherSmem s;
  s.soff = reinterpret_cast<int*>(smem);
  s.rings = reinterpret_cast<Ring*>(smem + kMaxSrc + 4);
  s.rsum = reinterpret_cast<float*>(s.rings + kMaxRing);
  s.cch = reinterpret_cast<Chunk*>(s.rsum + kMaxCb * kMaxRing);
  s.cval = reinterpret_cast<float*>(s.cch + chunk_cache);
  s.stage = s.cval + (size_t)chunk_cache * nk * kChunkW;
  return s;
}

// Staging offsets of the row's source rows; returns the elements staged per channel.
// Also copies the row's ring terms, first chunks and their values into shared memory.
__device__ __forceinline__ int gather_prologue(const GatherArgs& a, const RowPlan& rp, int ch_begin, int ch_end,
                                               int step, int nk, const GatherSmem& s) {
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int t = rp.src_begin; t < rp.src_end; ++t) {
      s.soff[t - rp.src_begin] = acc;
      acc += staged_words(staged_len(a.srcs[t].span, a.qb, step));
    }
    s.soff[rp.src_end - rp.src_begin] = acc;
  }
  for (int t = threadIdx.x; t < rp.ring_end - rp.ring_begin; t += blockDim.x) s.rings[t] = a.rings[rp.ring_begin + t];
  const int ncache = min(ch_end - ch_begin, a.chunk_cache);
  for (int t = threadIdx.x; t < ncache; t += blockDim.x) s.cch[t] = a.chunks[ch_begin + t];
  if (ncache > 0) {
    const float* v0 = a.vals + a.chunks[ch_begin].voff;  // a row's chunk values are contiguous
    for (int t = threadIdx.x; t < ncache * nk * kChunkW; t += blockDim.x) s.cval[t] = __ldg(v0 + t);
  }
  __syncthreads();
  return s.soff[rp.src_end - rp.src_begin];
}

// Chunk ch (row-relative) and its values: from the cache, else from global memory.
__device__ __forceinline__ void chunk_at(const GatherArgs& a, const GatherSmem& s, int ch_begin, int ch, int nk,
                                         Chunk* c, const float** v) {
  if (ch < a.chunk_cache) {
    *c = s.cch[ch];
    *v = s.cval + (size_t)ch * nk * kChunkW;
  } else {
    *c = a.chunks[ch_begin + ch];
    *v = a.vals + c->voff;
  }
}

__device__ __forceinline__ void bf16x8_to_floats(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Stages every source row of the output row for channel planes c0 .. c0+ncg-1.
// Staged element t of a source row holds source longitude (base + start + t) mod n_src and
// lives at word t + t/8 of the row (see staged_words).  With vec_stage, starts are multiples
// of kAlign (the plan guarantees it) and n_src is a multiple of the 16-byte vector, so whole
// vectors are read.
template <typename T>
__device__ __forceinline__ void stage_rows(const GatherArgs& a, const RowPlan& rp, const GatherSmem& s, int se,
                                           const T* __restrict__ src, int c0, int ncg, int base, int step) {
  const size_t chan = (size_t)a.n_src_rows * a.n_src;
  const int n = a.n_src;
  for (int t = rp.src_begin; t < rp.src_end; ++t) {
    const SrcRow sr = a.srcs[t];
    const int len = staged_len(sr.span, a.qb, step);
    const int first = wrap_mod(base + sr.start, n);
    float* dst0 = s.stage + s.soff[t - rp.src_begin];
    const T* row0 = src + (size_t)sr.row * n;
    if (a.vec_stage) {
      constexpr int V = 16 / sizeof(T);
      const int ng = len / V;
#pragma unroll 4
      for (int idx = threadIdx.x; idx < ncg * ng; idx += blockDim.x) {
        const int c = idx / ng, g = idx - c * ng;
        int l = first + g * V;
        while (l >= n) l -= n;
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(row0 + (size_t)(c0 + c) * chan + l));
        const int e = g * V;
        float* dst = dst0 + (size_t)c * se + e + (e >> 3);
        if constexpr (sizeof(T) == 2) {
          float f[8];
          bf16x8_to_floats(u, f);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = f[i];
        } else {
          dst[0] = __uint_as_float(u.x);
          dst[1] = __uint_as_float(u.y);
          dst[2] = __uint_as_float(u.z);
          dst[3] = __uint_as_float(u.w);
        }
      }
    } else {
      for (int idx = threadIdx.x; idx < ncg * len; idx += blockDim.x) {
        const int c = idx / len, e = idx - c * len;
        int l = first + e;
        while (l >= n) l -= n;
        dst0[(size_t)c * se + e + (e >> 3)] = to_f32(row0[(size_t)(c0 + c) * chan + l]);
      }
    }
  }
}

// rsum[c * nring + t] = sum over the whole source row of ring t, channel c0 + c.  One warp per
// (ring, channel) pair; lanes stride the row and combine with a fixed shuffle tree, so the
// result does not depend on scheduling.
template <typename T>
__device__ __forceinline__ void ring_sums(const GatherArgs& a, const GatherSmem& s, int nring,
                                          const T* __restrict__ src, int c0, int ncg) {
  const size_t chan = (size_t)a.n_src_rows * a.n_src;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  for (int pr = warp; pr < nring * ncg; pr += nwarp) {
    const int c = pr / nring, t = pr - c * nring;
    const T* row = src + (size_t)(c0 + c) * chan + (size_t)s.rings[t].row * a.n_src;
    float acc = 0.0f;
    if (a.vec_stage) {
      constexpr int V = 16 / sizeof(T);
      for (int g = lane; g < a.n_src / V; g += 32) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + g);
        if constexpr (sizeof(T) == 2) {
          float f[8];
          bf16x8_to_floats(u, f);
          acc += ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
        } else {
          acc += (__uint_as_float(u.x) + __uint_as_float(u.y)) + (__uint_as_float(u.z) + __uint_as_float(u.w));
        }
      }
    } else {
      for (int l = lane; l < a.n_src; l += 32) acc += to_f32(row[l]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) s.rsum[c * nring + t] = acc;
  }
}

// Loads NW staged elements e0 .. e0+NW-1 of a padded row (word e + e/8); p points at the
// word of e0 and LO = e0 mod 8, so the pad words inside the window sit at compile-time offsets.
template <int NW, int LO>
__device__ __forceinline__ void load_window(float (&win)[NW], const float* __restrict__ p) {
#pragma unroll
  for (int t = 0; t < NW; ++t) win[t] = p[t + (LO + t) / 8];
}

template <int NW>
__device__ __forceinline__ void load_window_any(float (&win)[NW], const float* __restrict__ row, int e0) {
  const float* p = row + e0 + (e0 >> 3);
  switch (e0 & 7) {
    case 0: load_window<NW, 0>(win, p); break;
    case 1: load_window<NW, 1>(win, p); break;
    case 2: load_window<NW, 2>(win, p); break;
    case 3: load_window<NW, 3>(win, p); break;
    case 4: load_window<NW, 4>(win, p); break;
    case 5: load_window<NW, 5>(win, p); break;
    case 6: load_window<NW, 6>(win, p); break;
    default: load_window<NW, 7>(win, p); break;
  }
}

// acc[k][r] += sum_u v[k][u] * win[r*S + u] for the basis functions set in kmask.
template <int K, int S, int W, int NW>
__device__ __forceinline__ void fwd_chunk(float (&acc)[K][kTaskR], const float (&win)[NW],
                                          const float* __restrict__ v, int kmask) {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (kmask & (1 << k)) {
#pragma unroll
      for (int u = 0; u < W; ++u) {
        const float vv = v[k * kChunkW + u];
#pragma unroll
        for (int r = 0; r < kTaskR; ++r) acc[k][r] = fmaf(vv, win[r * S + u], acc[k][r]);
      }
    }
  }
}

// Chunks [c_lo, c_hi) of the row for one task (kTaskR outputs of one channel plane whose
// staging starts at `sc`; the task's first output is m0 of the block).
template <int K, int S>
__device__ __forceinline__ void fwd_task(float (&acc)[K][kTaskR], const GatherArgs& a, const GatherSmem& s,
                                         const float* sc, int m0, int ch_begin, int c_lo, int c_hi) {
  constexpr int NW = (kTaskR - 1) * S + kChunkW;
#pragma unroll
  for (int k = 0; k < K; ++k)
#pragma unroll
    for (int r = 0; r < kTaskR; ++r) acc[k][r] = 0.0f;
  for (int ch = c_lo; ch < c_hi; ++ch) {
    Chunk cc;
    const float* v;
    chunk_at(a, s, ch_begin, ch, K, &cc, &v);
    float win[NW];
    load_window_any<NW>(win, sc + s.soff[cc.src], cc.t0 + m0 * S);
    const int kmask = cc.wk >> 8;
    switch (cc.wk & 0xff) {
      case 1: fwd_chunk<K, S, 1>(acc, win, v, kmask); break;
      case 2: fwd_chunk<K, S, 2>(acc, win, v, kmask); break;
      case 3: fwd_chunk<K, S, 3>(acc, win, v, kmask); break;
      case 4: fwd_chunk<K, S, 4>(acc, win, v, kmask); break;
      case 5: fwd_chunk<K, S, 5>(acc, win, v, kmask); break;
      case 6: fwd_chunk<K, S, 6>(acc, win, v, kmask); break;
      case 7: fwd_chunk<K, S, 7>(acc, win, v, kmask); break;
      default: fwd_chunk<K, S, 8>(acc, win, v, kmask); break;
    }
  }
}

// Chunk slices per task: split a heavy row's chunk list over otherwise idle threads.  The
// partial sums are combined through shared memory (the staging area, once it is consumed).
__device__ __forceinline__ int slice_count(int tasks, int nch, int red_floats_per_task, int stage_budget) {
  if (tasks >= (int)blockDim.x || nch < 16) return 1;
  int nsl = min((int)blockDim.x / tasks, nch / 8);
  nsl = min(nsl, stage_budget / max(1, tasks * red_floats_per_task));
  return max(1, nsl);
}

// Forward accumulation of one output row over a block of outputs for ncg channel planes
// (c0 .. c0+ncg-1 of the source tensor).  Stages, computes ring sums, accumulates every
// chunk, then hands each finished task to sink(c, m0, acc) (acc already holds the rings).
template <typename T, int K, int S, typename Sink>
__device__ __forceinline__ void fwd_block(const GatherArgs& a, const RowPlan& rp, const GatherSmem& s, int se,
                                          const T* __restrict__ x, int c0, int ncg, int base, int ch_begin,
                                          int nch, Sink& sink, bool rings_ready = false) {
  const int nring = rp.ring_end - rp.ring_begin;
  stage_rows<T>(a, rp, s, se, x, c0, ncg, base, S);
  if (!rings_ready) ring_sums<T>(a, s, nring, x, c0, ncg);
  __syncthreads();
  const int tpc = a.qb / kTaskR;
  const int tasks = ncg * tpc;
  const int nsl = slice_count(tasks, nch, K * kTaskR, a.stage_budget);
  auto add_rings = [&](float (&acc)[K][kTaskR], int c) {
    for (int t = 0; t < nring; ++t) {
      const Ring rg = s.rings[t];
      const float add = rg.v * s.rsum[c * nring + t];
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (rg.k == k)
#pragma unroll
          for (int r = 0; r < kTaskR; ++r) acc[k][r] += add;
    }
  };
  if (nsl == 1) {
    for (int task = threadIdx.x; task < tasks; task += blockDim.x) {
      const int c = task / tpc, m0 = (task - c * tpc) * kTaskR;
      float acc[K][kTaskR];
      fwd_task<K, S>(acc, a, s, s.stage + (size_t)c * se, m0, ch_begin, 0, nch);
      add_rings(acc, c);
      sink(c, m0, acc);
    }
    __syncthreads();
    return;
  }
  // one (slice, task) per thread
  const int tg = threadIdx.x;
  const bool active = tg < nsl * tasks;
  const int sl = tg / tasks, task = tg - sl * tasks;
  float acc[K][kTaskR];
  if (active) {
    const int c = task / tpc, m0 = (task - c * tpc) * kTaskR;
    fwd_task<K, S>(acc, a, s, s.stage + (size_t)c * se, m0, ch_begin, (sl * nch) / nsl, ((sl + 1) * nch) / nsl);
  }
  __syncthreads();  // staging consumed: reuse it for the partial sums
  float* red = s.stage;
  if (active)
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int r = 0; r < kTaskR; ++r) red[((size_t)(sl * tasks + task) * K + k) * kTaskR + r] = acc[k][r];
  __syncthreads();
  for (int t = threadIdx.x; t < tasks; t += blockDim.x) {
    const int c = t / tpc, m0 = (t - c * tpc) * kTaskR;
    float sum[K][kTaskR];
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int r = 0; r < kTaskR; ++r) {
        float v = 0.0f;
        for (int q = 0; q < nsl; ++q) v += red[((size_t)(q * tasks + t) * K + k) * kTaskR + r];
        sum[k][r] = v;
      }
    add_rings(sum, c);
    sink(c, m0, sum);
  }
  __syncthreads();
}

}  // namespace disco
