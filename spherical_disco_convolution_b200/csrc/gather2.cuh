// Forward gather over pairs of channel planes with packed fp32 FMAs (sm_100 fma.rn.f32x2).
//
// A thread owns kTaskR consecutive outputs of TWO channel planes.  The staged
// rows hold (plane a, plane b) as float2 at word2 index e + e/8 (the same pad
// rule as the single-plane layout, so 16 threads 8 outputs apart still hit 16
// different bank pairs), the chunk values are cached as (v, v) pairs, and each
// tap is one __ffma2_rn on the two planes.  Against one plane per thread this
// halves the window loads, the value loads, the per-chunk bookkeeping and the
// FMA instructions per useful multiply-add.
#pragma once

#include "gather_common.cuh"

namespace disco {

// Shared memory of the paired gather (float2 = 8 bytes):
//   [soff ints][rings][rsum][chunk cache][pair values: cache*nk*8 float2][stage: float2]
struct Gather2Smem {
  int* soff;
  Ring* rings;
  float* rsum;
  Chunk* cch;
  float2* cval;
  float2* stage;
};

__host__ __device__ inline size_t gather2_smem_bytes(int chunk_cache, int nk, int stage_f2) {
  return 4 * ((size_t)(kMaxSrc + 4) + (size_t)kMaxRing * 4 + (size_t)kMaxCb * kMaxRing + (size_t)chunk_cache * 4) +
         8 * ((size_t)chunk_cache * nk * kChunkW + (size_t)stage_f2);
}

__device__ __forceinline__ Gather2Smem gather2_smem(float* smem, int chunk_cache, int nk) {
  Gather2Smem s;
  s.soff = reinterpret_cast<int*>(smem);
  s.rings = reinterpret_cast<Ring*>(smem + kMaxSrc + 4);
  s.rsum = reinterpret_cast<float*>(s.rings + kMaxRing);
  s.cch = reinterpret_cast<Chunk*>(s.rsum + kMaxCb * kMaxRing);
  s.cval = reinterpret_cast<float2*>(s.cch + chunk_cache);
  s.stage = s.cval + (size_t)chunk_cache * nk * kChunkW;
  return s;
}

// Offsets (float2 units) of the row's source rows, rings and the duplicated chunk values.
__device__ __forceinline__ int gather2_prologue(const GatherArgs& a, const RowPlan& rp, int ch_begin, int ch_end,
                                                int step, int nk, const Gather2Smem& s) {
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
    const float* v0 = a.vals + a.chunks[ch_begin].voff;
    for (int t = threadIdx.x; t < ncache * nk * kChunkW; t += blockDim.x) {
      const float v = __ldg(v0 + t);
      s.cval[t] = make_float2(v, v);
    }
  }
  __syncthreads();
  return s.soff[rp.src_end - rp.src_begin];
}

// Stages planes c0 .. c0+ncg-1 as pairs (an odd last plane is paired with zeros).
template <typename T>
__device__ __forceinline__ void stage_rows2(const GatherArgs& a, const RowPlan& rp, const Gather2Smem& s, int se,
                                            const T* __restrict__ src, int c0, int ncg, int base, int step) {
  const size_t chan = (size_t)a.n_src_rows * a.n_src;
  const int n = a.n_src;
  const int npair = (ncg + 1) >> 1;
  for (int t = rp.src_begin; t < rp.src_end; ++t) {
    const SrcRow sr = a.srcs[t];
    const int len = staged_len(sr.span, a.qb, step);
    const int first = wrap_mod(base + sr.start, n);
    float2* dst0 = s.stage + s.soff[t - rp.src_begin];
    const T* row0 = src + (size_t)sr.row * n;
    if (a.vec_stage) {
      constexpr int V = 16 / sizeof(T);
      const int ng = len / V;
#pragma unroll 2
      for (int idx = threadIdx.x; idx < npair * ng; idx += blockDim.x) {
        const int p = idx / ng, g = idx - p * ng;
        int l = first + g * V;
        while (l >= n) l -= n;
        const bool has_b = 2 * p + 1 < ncg;
        const uint4 ua = __ldg(reinterpret_cast<const uint4*>(row0 + (size_t)(c0 + 2 * p) * chan + l));
        const uint4 ub = has_b ? __ldg(reinterpret_cast<const uint4*>(row0 + (size_t)(c0 + 2 * p + 1) * chan + l))
                               : make_uint4(0, 0, 0, 0);
        const int e = g * V;
        float2* dst = dst0 + (size_t)p * se + e + (e >> 3);
        if constexpr (sizeof(T) == 2) {
          float fa[8], fb[8];
          bf16x8_to_floats(ua, fa);
          bf16x8_to_floats(ub, fb);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float2(fa[i], fb[i]);
        } else {
          dst[0] = make_float2(__uint_as_float(ua.x), __uint_as_float(ub.x));
          dst[1] = make_float2(__uint_as_float(ua.y), __uint_as_float(ub.y));
          dst[2] = make_float2(__uint_as_float(ua.z), __uint_as_float(ub.z));
          dst[3] = make_float2(__uint_as_float(ua.w), __uint_as_float(ub.w));
        }
      }
    } else {
      for (int idx = threadIdx.x; idx < npair * len; idx += blockDim.x) {
        const int p = idx / len, e = idx - p * len;
        int l = first + e;
        while (l >= n) l -= n;
        const float va = to_f32(row0[(size_t)(c0 + 2 * p) * chan + l]);
        const float vb = 2 * p + 1 < ncg ? to_f32(row0[(size_t)(c0 + 2 * p + 1) * chan + l]) : 0.0f;
        dst0[(size_t)p * se + e + (e >> 3)] = make_float2(va, vb);
      }
    }
  }
}

template <int NW, int LO>
__device__ __forceinline__ void load_window2(float2 (&win)[NW], const float2* __restrict__ p) {
#pragma unroll
  for (int t = 0; t < NW; ++t) win[t] = p[t + (LO + t) / 8];
}

template <int NW>
__device__ __forceinline__ void load_window2_any(float2 (&win)[NW], const float2* __restrict__ row, int e0) {
  const float2* p = row + e0 + (e0 >> 3);
  switch (e0 & 7) {
    case 0: load_window2<NW, 0>(win, p); break;
    case 1: load_window2<NW, 1>(win, p); break;
    case 2: load_window2<NW, 2>(win, p); break;
    case 3: load_window2<NW, 3>(win, p); break;
    case 4: load_window2<NW, 4>(win, p); break;
    case 5: load_window2<NW, 5>(win, p); break;
    case 6: load_window2<NW, 6>(win, p); break;
    default: load_window2<NW, 7>(win, p); break;
  }
}

// Values of a chunk as (v, v) pairs: from the shared cache, or read from the plan and
// duplicated on the fly for chunks beyond the cache.
struct CachedValues {
  const float2* v;
  __device__ __forceinline__ float2 operator()(int i) const { return v[i]; }
};
struct GlobalValues {
  const float* v;
  __device__ __forceinline__ float2 operator()(int i) const {
    const float x = __ldg(v + i);
    return make_float2(x, x);
  }
};

template <int K, int S, int W, int NW, typename Vals>
__device__ __forceinline__ void fwd_chunk2(float2 (&acc)[K][kTaskR], const float2 (&win)[NW], const Vals& v,
                                           int kmask) {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (kmask & (1 << k)) {
#pragma unroll
      for (int u = 0; u < W; ++u) {
        const float2 vv = v(k * kChunkW + u);
#pragma unroll
        for (int r = 0; r < kTaskR; ++r) acc[k][r] = __ffma2_rn(vv, win[r * S + u], acc[k][r]);
      }
    }
  }
}

template <int K, int S, typename Vals>
__device__ __forceinline__ void apply_chunk2(float2 (&acc)[K][kTaskR], const float2* sc, const Gather2Smem& s,
                                             const Chunk& cc, int m0, const Vals& v) {
  constexpr int NW = (kTaskR - 1) * S + kChunkW;
  float2 win[NW];
  load_window2_any<NW>(win, sc + s.soff[cc.src], cc.t0 + m0 * S);
  const int kmask = cc.wk >> 8;
  switch (cc.wk & 0xff) {
    case 1: fwd_chunk2<K, S, 1>(acc, win, v, kmask); break;
    case 2: fwd_chunk2<K, S, 2>(acc, win, v, kmask); break;
    case 3: fwd_chunk2<K, S, 3>(acc, win, v, kmask); break;
    case 4: fwd_chunk2<K, S, 4>(acc, win, v, kmask); break;
    case 5: fwd_chunk2<K, S, 5>(acc, win, v, kmask); break;
    case 6: fwd_chunk2<K, S, 6>(acc, win, v, kmask); break;
    case 7: fwd_chunk2<K, S, 7>(acc, win, v, kmask); break;
    default: fwd_chunk2<K, S, 8>(acc, win, v, kmask); break;
  }
}

template <int K, int S>
__device__ __forceinline__ void fwd_task2(float2 (&acc)[K][kTaskR], const GatherArgs& a, const Gather2Smem& s,
                                          const float2* sc, int m0, int ch_begin, int c_lo, int c_hi) {
#pragma unroll
  for (int k = 0; k < K; ++k)
#pragma unroll
    for (int r = 0; r < kTaskR; ++r) acc[k][r] = make_float2(0.0f, 0.0f);
  const int c_mid = max(c_lo, min(c_hi, a.chunk_cache));
  for (int ch = c_lo; ch < c_mid; ++ch)
    apply_chunk2<K, S>(acc, sc, s, s.cch[ch], m0, CachedValues{s.cval + (size_t)ch * K * kChunkW});
  for (int ch = c_mid; ch < c_hi; ++ch) {
    const Chunk cc = a.chunks[ch_begin + ch];
    apply_chunk2<K, S>(acc, sc, s, cc, m0, GlobalValues{a.vals + cc.voff});
  }
}

// Paired forward accumulation of one output row over a block of outputs for planes c0 ..
// c0+ncg-1; sink(p, m0, acc) receives pair p (planes c0+2p, c0+2p+1; the second is absent when
// 2p+1 == ncg) with the rings added.
template <typename T, int K, int S, typename Sink>
__device__ __forceinline__ void fwd_block2(const GatherArgs& a, const RowPlan& rp, const Gather2Smem& s, int se,
                                           const T* __restrict__ x, int c0, int ncg, int base, int ch_begin,
                                           int nch, Sink& sink) {
  const int nring = rp.ring_end - rp.ring_begin;
  stage_rows2<T>(a, rp, s, se, x, c0, ncg, base, S);
  GatherSmem s1;
  s1.soff = s.soff;
  s1.rings = s.rings;
  s1.rsum = s.rsum;
  ring_sums<T>(a, s1, nring, x, c0, ncg);
  __syncthreads();
  const int tpc = a.qb / kTaskR;
  const int npair = (ncg + 1) >> 1;
  const int tasks = npair * tpc;
  const int nsl = slice_count(tasks, nch, 2 * K * kTaskR, 2 * a.stage_budget);
  auto add_rings = [&](float2 (&acc)[K][kTaskR], int p) {
    for (int t = 0; t < nring; ++t) {
      const Ring rg = s.rings[t];
      const float ra = rg.v * s.rsum[(2 * p) * nring + t];
      const float rb = 2 * p + 1 < ncg ? rg.v * s.rsum[(2 * p + 1) * nring + t] : 0.0f;
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (rg.k == k)
#pragma unroll
          for (int r = 0; r < kTaskR; ++r) {
            acc[k][r].x += ra;
            acc[k][r].y += rb;
          }
    }
  };
  if (nsl == 1) {
    for (int task = threadIdx.x; task < tasks; task += blockDim.x) {
      const int p = task / tpc, m0 = (task - p * tpc) * kTaskR;
      float2 acc[K][kTaskR];
      fwd_task2<K, S>(acc, a, s, s.stage + (size_t)p * se, m0, ch_begin, 0, nch);
      add_rings(acc, p);
      sink(p, m0, acc);
    }
    __syncthreads();
    return;
  }
  const int tg = threadIdx.x;
  const bool active = tg < nsl * tasks;
  const int sl = tg / tasks, task = tg - sl * tasks;
  float2 acc[K][kTaskR];
  if (active) {
    const int p = task / tpc, m0 = (task - p * tpc) * kTaskR;
    fwd_task2<K, S>(acc, a, s, s.stage + (size_t)p * se, m0, ch_begin, (sl * nch) / nsl, ((sl + 1) * nch) / nsl);
  }
  __syncthreads();  // staging consumed: reuse it for the partial sums
  float2* red = s.stage;
  if (active)
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int r = 0; r < kTaskR; ++r) red[((size_t)(sl * tasks + task) * K + k) * kTaskR + r] = acc[k][r];
  __syncthreads();
  for (int t = threadIdx.x; t < tasks; t += blockDim.x) {
    const int p = t / tpc, m0 = (t - p * tpc) * kTaskR;
    float2 sum[K][kTaskR];
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int r = 0; r < kTaskR; ++r) {
        float2 v = make_float2(0.0f, 0.0f);
        for (int q = 0; q < nsl; ++q) {
          const float2 w = red[((size_t)(q * tasks + t) * K + k) * kTaskR + r];
          v.x += w.x;
          v.y += w.y;
        }
        sum[k][r] = v;
      }
    add_rings(sum, p);
    sink(p, m0, sum);
  }
  __syncthreads();
}

}  // namespace disco
