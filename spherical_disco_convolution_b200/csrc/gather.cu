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
// the chunk.  Full circles of one constant value (rings) enter as value x
// row sum.  Rows with many chunks and few staged channels split their chunk
// list over idle threads and combine the partial sums in a fixed order.
#include "gather2.cuh"
#include "gather_common.cuh"

namespace disco {
namespace {

constexpr int kThreads = 256;

template <typename T, int K>
struct YSink {
  T* y;
  int c0, n_out_rows, row, n_out, q0;
  __device__ __forceinline__ void operator()(int c, int m0, float (&acc)[K][kTaskR]) const {
    if (q0 + m0 >= n_out) return;
    const int n = min(kTaskR, n_out - (q0 + m0));
#pragma unroll
    for (int k = 0; k < K; ++k) {
      T* dst = y + (((size_t)(c0 + c) * K + k) * n_out_rows + row) * n_out + q0 + m0;
      store_run<T, kTaskR>(dst, acc[k], n);
    }
  }
};

template <typename T, int K, int S>
__global__ void __launch_bounds__(kThreads, (K <= 3 ? 3 : (K <= 5 ? 2 : 1))) fwd_gather_kernel(GatherArgs a, const T* __restrict__ x,
                                                              T* __restrict__ y) {
  extern __shared__ __align__(16) float smem[];
  const GatherSmem s = gather_smem(smem, a.chunk_cache, K);
  const RowPlan rp = a.rows[blockIdx.z];
  const int q0 = blockIdx.y * a.qb;
  const int c_begin = blockIdx.x * a.cb;
  const int c_end = min(a.BC, c_begin + a.cb);
  const int ch_begin = rp.chunk_start[0], nch = rp.chunk_end[0] - rp.chunk_start[0];
  const int se = gather_prologue(a, rp, ch_begin, rp.chunk_end[0], S, K, s);
  const int cg = max(1, min(min(a.cb, kMaxCb), a.stage_budget / max(1, se)));
  for (int c0 = c_begin; c0 < c_end; c0 += cg) {
    const int ncg = min(cg, c_end - c0);
    YSink<T, K> sink{y, c0, a.n_out_rows, rp.row, a.n_out, q0};
    fwd_block<T, K, S>(a, rp, s, se, x, c0, ncg, q0 * S, ch_begin, nch, sink);
  }
}

template <typename T, int K>
struct YSink2 {
  T* y;
  int c0, ncg, n_out_rows, row, n_out, q0;
  __device__ __forceinline__ void operator()(int p, int m0, float2 (&acc)[K][kTaskR]) const {
    if (q0 + m0 >= n_out) return;
    const int n = min(kTaskR, n_out - (q0 + m0));
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float va[kTaskR], vb[kTaskR];
#pragma unroll
      for (int r = 0; r < kTaskR; ++r) {
        va[r] = acc[k][r].x;
        vb[r] = acc[k][r].y;
      }
      const size_t off = ((size_t)k * n_out_rows + row) * n_out + q0 + m0;
      store_run<T, kTaskR>(y + (size_t)(c0 + 2 * p) * K * n_out_rows * n_out + off, va, n);
      if (2 * p + 1 < ncg) store_run<T, kTaskR>(y + (size_t)(c0 + 2 * p + 1) * K * n_out_rows * n_out + off, vb, n);
    }
  }
};

// Paired form of the forward gather (K <= 5): 128 threads, each owning 8 outputs of two
// channel planes; the stage budget counts float2 words.
template <typename T, int K, int S>
__global__ void __launch_bounds__(128, 3) fwd_gather2_kernel(GatherArgs a, const T* __restrict__ x,
                                                              T* __restrict__ y) {
  extern __shared__ __align__(16) float smem[];
  const Gather2Smem s = gather2_smem(smem, a.chunk_cache, K);
  const RowPlan rp = a.rows[blockIdx.z];
  const int q0 = blockIdx.y * a.qb;
  const int c_begin = blockIdx.x * a.cb;
  const int c_end = min(a.BC, c_begin + a.cb);
  const int ch_begin = rp.chunk_start[0], nch = rp.chunk_end[0] - rp.chunk_start[0];
  const int se = gather2_prologue(a, rp, ch_begin, rp.chunk_end[0], S, K, s);
  const int cg = max(1, min(min(a.cb, kMaxCb), 2 * (a.stage_budget / max(1, se))));
  for (int c0 = c_begin; c0 < c_end; c0 += cg) {
    const int ncg = min(cg, c_end - c0);
    YSink2<T, K> sink{y, c0, ncg, a.n_out_rows, rp.row, a.n_out, q0};
    fwd_block2<T, K, S>(a, rp, s, se, x, c0, ncg, q0 * S, ch_begin, nch, sink);
  }
}

// Banded paired forward gather: the rows of a band share their staged source rows.
template <typename T, int K, int S>
__global__ void __launch_bounds__(128, 3) fwd_gather2_band_kernel(GatherArgs a, const T* __restrict__ x,
                                                                   T* __restrict__ y) {
  extern __shared__ __align__(16) float smem[];
  __shared__ int brow[8][3];  // row, first chunk, end chunk (band-relative) of each member row
  const Gather2Smem s = gather2_smem(smem, a.chunk_cache, K);
  const BandPlan bp = a.bands[a.band0 + blockIdx.z];
  const int nr = bp.rp_end - bp.rp_begin;
  const RowPlan r0 = a.rows[bp.rp_begin];
  const int ch_begin = r0.chunk_start[0];
  const int ch_end = a.rows[bp.rp_end - 1].chunk_end[0];
  if (threadIdx.x < nr) {
    const RowPlan& rr = a.rows[bp.rp_begin + threadIdx.x];
    brow[threadIdx.x][0] = rr.row;
    brow[threadIdx.x][1] = rr.chunk_start[0] - ch_begin;
    brow[threadIdx.x][2] = rr.chunk_end[0] - ch_begin;
  }
  const int q0 = blockIdx.y * a.qb;
  const int c_begin = blockIdx.x * a.cb;
  const int c_end = min(a.BC, c_begin + a.cb);
  const int se = gather2_prologue(a, r0, ch_begin, ch_end, S, K, s);
  const int cg = max(1, min(min(a.cb, kMaxCb), 2 * (a.stage_budget / max(1, se))));
  const int tpc = a.qb / kTaskR;
  for (int c0 = c_begin; c0 < c_end; c0 += cg) {
    const int ncg = min(cg, c_end - c0);
    if (nr == 1) {
      YSink2<T, K> sink{y, c0, ncg, a.n_out_rows, r0.row, a.n_out, q0};
      fwd_block2<T, K, S>(a, r0, s, se, x, c0, ncg, q0 * S, ch_begin, ch_end - ch_begin, sink);
      continue;
    }
    stage_rows2<T>(a, r0, s, se, x, c0, ncg, q0 * S, S);
    __syncthreads();
    const int npair = (ncg + 1) >> 1;
    const int per_row = npair * tpc;
    for (int t = threadIdx.x; t < nr * per_row; t += blockDim.x) {
      const int r = t / per_row, rem = t - r * per_row;
      const int p = rem / tpc, m0 = (rem - p * tpc) * kTaskR;
      float2 acc[K][kTaskR];
      fwd_task2<K, S>(acc, a, s, s.stage + (size_t)p * se, m0, ch_begin, brow[r][1], brow[r][2]);
      YSink2<T, K> sink{y, c0, ncg, a.n_out_rows, brow[r][0], a.n_out, q0};
      sink(p, m0, acc);
    }
    __syncthreads();
  }
}

template <int W, int NW>
__device__ __forceinline__ void adj_chunk(float (&acc)[kTaskR], const float (&win)[NW],
                                          const float* __restrict__ v) {
#pragma unroll
  for (int u = 0; u < W; ++u) {
    const float vv = v[u];
#pragma unroll
    for (int r = 0; r < kTaskR; ++r) acc[r] = fmaf(vv, win[r + u], acc[r]);
  }
}

template <int S>
__device__ __forceinline__ void adj_task(float (&acc)[S][kTaskR], const GatherArgs& a, const GatherSmem& s,
                                         const RowPlan& rp, const float* sc, int m0, int ch_begin, int sl, int nsl) {
  constexpr int NW = kTaskR - 1 + kChunkW;
#pragma unroll
  for (int rho = 0; rho < S; ++rho) {
#pragma unroll
    for (int r = 0; r < kTaskR; ++r) acc[rho][r] = 0.0f;
    const int lo = rp.chunk_start[rho] - ch_begin, n = rp.chunk_end[rho] - rp.chunk_start[rho];
    for (int ch = lo + (sl * n) / nsl; ch < lo + ((sl + 1) * n) / nsl; ++ch) {
      Chunk cc;
      const float* v;
      chunk_at(a, s, ch_begin, ch, 1, &cc, &v);
      float win[NW];
      load_window_any<NW>(win, sc + s.soff[cc.src], cc.t0 + m0);
      switch (cc.wk & 0xff) {
        case 1: adj_chunk<1>(acc[rho], win, v); break;
        case 2: adj_chunk<2>(acc[rho], win, v); break;
        case 3: adj_chunk<3>(acc[rho], win, v); break;
        case 4: adj_chunk<4>(acc[rho], win, v); break;
        case 5: adj_chunk<5>(acc[rho], win, v); break;
        case 6: adj_chunk<6>(acc[rho], win, v); break;
        case 7: adj_chunk<7>(acc[rho], win, v); break;
        default: adj_chunk<8>(acc[rho], win, v); break;
      }
    }
  }
}

template <typename T, int S>
__global__ void __launch_bounds__(kThreads, 3) adj_gather_kernel(GatherArgs a, const T* __restrict__ dy,
                                                              T* __restrict__ dx) {
  extern __shared__ __align__(16) float smem[];
  const GatherSmem s = gather_smem(smem, a.chunk_cache, 1);
  const RowPlan rp = a.rows[blockIdx.z];
  const int m_blk = blockIdx.y * a.qb;
  const int c_begin = blockIdx.x * a.cb;
  const int c_end = min(a.BC, c_begin + a.cb);
  const int ch_begin = rp.chunk_start[0], nch = rp.chunk_end[S - 1] - rp.chunk_start[0];
  const int se = gather_prologue(a, rp, ch_begin, rp.chunk_end[S - 1], 1, 1, s);
  const int cg = max(1, min(min(a.cb, kMaxCb), a.stage_budget / max(1, se)));
  const int tpc = a.qb / kTaskR;
  const int n_m = a.n_out / S;  // outputs l = S*m + rho, m < n_m
  const int nring = rp.ring_end - rp.ring_begin;
  for (int c0 = c_begin; c0 < c_end; c0 += cg) {
    const int ncg = min(cg, c_end - c0);
    stage_rows<T>(a, rp, s, se, dy, c0, ncg, m_blk, 1);
    ring_sums<T>(a, s, nring, dy, c0, ncg);
    __syncthreads();
    const int tasks = ncg * tpc;
    const int nsl = slice_count(tasks, nch, S * kTaskR, a.stage_budget);
    auto finish = [&](int c, int m0, float (&acc)[S][kTaskR]) {
      if (m_blk + m0 >= n_m) return;
      float ring = 0.0f;
      for (int t = 0; t < nring; ++t) ring += s.rings[t].v * s.rsum[c * nring + t];
      const int nm = min(kTaskR, n_m - (m_blk + m0));
      T* dst = dx + ((size_t)(c0 + c) * a.n_out_rows + rp.row) * a.n_out + (size_t)S * (m_blk + m0);
      if constexpr (S == 1) {
#pragma unroll
        for (int r = 0; r < kTaskR; ++r) acc[0][r] += ring;
        store_run<T, kTaskR>(dst, acc[0], nm);
      } else {
#pragma unroll
        for (int r = 0; r < kTaskR; ++r)
#pragma unroll
          for (int rho = 0; rho < S; ++rho)
            if (r < nm) dst[r * S + rho] = from_f32<T>(acc[rho][r] + ring);
      }
    };
    if (nsl == 1) {
      for (int task = threadIdx.x; task < tasks; task += blockDim.x) {
        const int c = task / tpc, m0 = (task - c * tpc) * kTaskR;
        float acc[S][kTaskR];
        adj_task<S>(acc, a, s, rp, s.stage + (size_t)c * se, m0, ch_begin, 0, 1);
        finish(c, m0, acc);
      }
    } else {
      const int tg = threadIdx.x;
      const bool active = tg < nsl * tasks;
      const int sl = tg / tasks, task = tg - sl * tasks;
      float acc[S][kTaskR];
      if (active) {
        const int c = task / tpc, m0 = (task - c * tpc) * kTaskR;
        adj_task<S>(acc, a, s, rp, s.stage + (size_t)c * se, m0, ch_begin, sl, nsl);
      }
      __syncthreads();  // staging consumed: reuse it for the partial sums
      float* red = s.stage;
      if (active)
#pragma unroll
        for (int rho = 0; rho < S; ++rho)
#pragma unroll
          for (int r = 0; r < kTaskR; ++r) red[((size_t)(sl * tasks + task) * S + rho) * kTaskR + r] = acc[rho][r];
      __syncthreads();
      for (int t = threadIdx.x; t < tasks; t += blockDim.x) {
        const int c = t / tpc, m0 = (t - c * tpc) * kTaskR;
        float sum[S][kTaskR];
#pragma unroll
        for (int rho = 0; rho < S; ++rho)
#pragma unroll
          for (int r = 0; r < kTaskR; ++r) {
            float v = 0.0f;
            for (int q = 0; q < nsl; ++q) v += red[((size_t)(q * tasks + t) * S + rho) * kTaskR + r];
            sum[rho][r] = v;
          }
        finish(c, m0, sum);
      }
    }
    __syncthreads();
  }
}

// ---- paired, banded adjoint gather (dx) ----

template <int W, int NW, typename Vals>
__device__ __forceinline__ void adj_chunk2(float2 (&acc)[kTaskR], const float2 (&win)[NW], const Vals& v) {
#pragma unroll
  for (int u = 0; u < W; ++u) {
    const float2 vv = v(u);
#pragma unroll
    for (int r = 0; r < kTaskR; ++r) acc[r] = __ffma2_rn(vv, win[r + u], acc[r]);
  }
}

template <typename Vals>
__device__ __forceinline__ void adj_apply2(float2 (&acc)[kTaskR], const float2* sc, const Gather2Smem& s,
                                           const Chunk& cc, int m0, const Vals& v) {
  constexpr int NW = kTaskR - 1 + kChunkW;
  float2 win[NW];
  load_window2_any<NW>(win, sc + s.soff[cc.src], cc.t0 + m0);
  switch (cc.wk & 0xff) {
    case 1: adj_chunk2<1>(acc, win, v); break;
    case 2: adj_chunk2<2>(acc, win, v); break;
    case 3: adj_chunk2<3>(acc, win, v); break;
    case 4: adj_chunk2<4>(acc, win, v); break;
    case 5: adj_chunk2<5>(acc, win, v); break;
    case 6: adj_chunk2<6>(acc, win, v); break;
    case 7: adj_chunk2<7>(acc, win, v); break;
    default: adj_chunk2<8>(acc, win, v); break;
  }
}

// Chunk ranges are relative to the band's first chunk; lo/hi per residue class.
template <int S>
__device__ __forceinline__ void adj_task2(float2 (&acc)[S][kTaskR], const GatherArgs& a, const Gather2Smem& s,
                                          const float2* sc, int m0, int ch_begin, const int* lo, const int* hi,
                                          int sl, int nsl) {
#pragma unroll
  for (int rho = 0; rho < S; ++rho) {
#pragma unroll
    for (int r = 0; r < kTaskR; ++r) acc[rho][r] = make_float2(0.0f, 0.0f);
    const int n = hi[rho] - lo[rho];
    const int ca = lo[rho] + (sl * n) / nsl, cb = lo[rho] + ((sl + 1) * n) / nsl;
    const int cm = max(ca, min(cb, a.chunk_cache));
    for (int ch = ca; ch < cm; ++ch) adj_apply2(acc[rho], sc, s, s.cch[ch], m0, CachedValues{s.cval + (size_t)ch * kChunkW});
    for (int ch = cm; ch < cb; ++ch) {
      const Chunk cc = a.chunks[ch_begin + ch];
      adj_apply2(acc[rho], sc, s, cc, m0, GlobalValues{a.vals + cc.voff});
    }
  }
}

template <typename T, int S>
__global__ void __launch_bounds__(128, 4) adj_gather2_band_kernel(GatherArgs a, const T* __restrict__ dy,
                                                                   T* __restrict__ dx) {
  extern __shared__ __align__(16) float smem[];
  __shared__ int brow[8][1 + 2 * kMaxStride];  // row, then [lo, hi) of each residue class
  const Gather2Smem s = gather2_smem(smem, a.chunk_cache, 1);
  const BandPlan bp = a.bands[a.band0 + blockIdx.z];
  const int nr = bp.rp_end - bp.rp_begin;
  const RowPlan r0 = a.rows[bp.rp_begin];
  const int ch_begin = r0.chunk_start[0];
  const int ch_end = a.rows[bp.rp_end - 1].chunk_end[S - 1];
  if (threadIdx.x < nr) {
    const RowPlan& rr = a.rows[bp.rp_begin + threadIdx.x];
    brow[threadIdx.x][0] = rr.row;
    for (int rho = 0; rho < S; ++rho) {
      brow[threadIdx.x][1 + 2 * rho] = rr.chunk_start[rho] - ch_begin;
      brow[threadIdx.x][2 + 2 * rho] = rr.chunk_end[rho] - ch_begin;
    }
  }
  const int m_blk = blockIdx.y * a.qb;
  const int c_begin = blockIdx.x * a.cb;
  const int c_end = min(a.BC, c_begin + a.cb);
  const int se = gather2_prologue(a, r0, ch_begin, ch_end, 1, 1, s);
  const int cg = max(1, min(min(a.cb, kMaxCb), 2 * (a.stage_budget / max(1, se))));
  const int tpc = a.qb / kTaskR;
  const int n_m = a.n_out / S;  // outputs l = S*m + rho, m < n_m
  const int nring = nr == 1 ? r0.ring_end - r0.ring_begin : 0;
  GatherSmem s1;
  s1.soff = s.soff;
  s1.rings = s.rings;
  s1.rsum = s.rsum;
  for (int c0 = c_begin; c0 < c_end; c0 += cg) {
    const int ncg = min(cg, c_end - c0);
    stage_rows2<T>(a, r0, s, se, dy, c0, ncg, m_blk, 1);
    if (nring) ring_sums<T>(a, s1, nring, dy, c0, ncg);
    __syncthreads();
    const int npair = (ncg + 1) >> 1;
    const int per_row = npair * tpc;
    const int tasks = nr * per_row;
    const int nsl = nr == 1 ? slice_count(tasks, ch_end - ch_begin, 2 * S * kTaskR, 2 * a.stage_budget) : 1;
    auto finish = [&](int r, int p, int m0, float2 (&acc)[S][kTaskR]) {
      if (m_blk + m0 >= n_m) return;
      float ra = 0.0f, rb = 0.0f;
      for (int t = 0; t < nring; ++t) {
        ra += s.rings[t].v * s.rsum[(2 * p) * nring + t];
        if (2 * p + 1 < ncg) rb += s.rings[t].v * s.rsum[(2 * p + 1) * nring + t];
      }
      const int nm = min(kTaskR, n_m - (m_blk + m0));
      const size_t off = (size_t)brow[r][0] * a.n_out + (size_t)S * (m_blk + m0);
      T* da = dx + (size_t)(c0 + 2 * p) * a.n_out_rows * a.n_out + off;
      T* db = dx + (size_t)(c0 + 2 * p + 1) * a.n_out_rows * a.n_out + off;
      const bool has_b = 2 * p + 1 < ncg;
      if constexpr (S == 1) {
        float va[kTaskR], vb[kTaskR];
#pragma unroll
        for (int q = 0; q < kTaskR; ++q) {
          va[q] = acc[0][q].x + ra;
          vb[q] = acc[0][q].y + rb;
        }
        store_run<T, kTaskR>(da, va, nm);
        if (has_b) store_run<T, kTaskR>(db, vb, nm);
      } else {
#pragma unroll
        for (int q = 0; q < kTaskR; ++q)
#pragma unroll
          for (int rho = 0; rho < S; ++rho)
            if (q < nm) {
              da[q * S + rho] = from_f32<T>(acc[rho][q].x + ra);
              if (has_b) db[q * S + rho] = from_f32<T>(acc[rho][q].y + rb);
            }
      }
    };
    if (nsl == 1) {
      for (int t = threadIdx.x; t < tasks; t += blockDim.x) {
        const int r = t / per_row, rem = t - r * per_row;
        const int p = rem / tpc, m0 = (rem - p * tpc) * kTaskR;
        float2 acc[S][kTaskR];
        int lo[S], hi[S];
#pragma unroll
        for (int rho = 0; rho < S; ++rho) {
          lo[rho] = brow[r][1 + 2 * rho];
          hi[rho] = brow[r][2 + 2 * rho];
        }
        adj_task2<S>(acc, a, s, s.stage + (size_t)p * se, m0, ch_begin, lo, hi, 0, 1);
        finish(r, p, m0, acc);
      }
    } else {
      const int tg = threadIdx.x;
      const bool active = tg < nsl * tasks;
      const int sl = tg / tasks, task = tg - sl * tasks;
      const int p = task / tpc, m0 = (task - p * tpc) * kTaskR;
      float2 acc[S][kTaskR];
      if (active) {
        int lo[S], hi[S];
#pragma unroll
        for (int rho = 0; rho < S; ++rho) {
          lo[rho] = brow[0][1 + 2 * rho];
          hi[rho] = brow[0][2 + 2 * rho];
        }
        adj_task2<S>(acc, a, s, s.stage + (size_t)p * se, m0, ch_begin, lo, hi, sl, nsl);
      }
      __syncthreads();  // staging consumed: reuse it for the partial sums
      float2* red = s.stage;
      if (active)
#pragma unroll
        for (int rho = 0; rho < S; ++rho)
#pragma unroll
          for (int q = 0; q < kTaskR; ++q) red[((size_t)(sl * tasks + task) * S + rho) * kTaskR + q] = acc[rho][q];
      __syncthreads();
      for (int t = threadIdx.x; t < tasks; t += blockDim.x) {
        const int pp = t / tpc, mm = (t - pp * tpc) * kTaskR;
        float2 sum[S][kTaskR];
#pragma unroll
        for (int rho = 0; rho < S; ++rho)
#pragma unroll
          for (int q = 0; q < kTaskR; ++q) {
            float2 v = make_float2(0.0f, 0.0f);
            for (int z = 0; z < nsl; ++z) {
              const float2 w = red[((size_t)(z * tasks + t) * S + rho) * kTaskR + q];
              v.x += w.x;
              v.y += w.y;
            }
            sum[rho][q] = v;
          }
        finish(0, pp, mm, sum);
      }
    }
    __syncthreads();
  }
}

template <typename T, int S>
cudaError_t launch_adj2b_t(const GatherArgs& a, const void* dy, void* dx, cudaStream_t st) {
  auto kern = adj_gather2_band_kernel<T, S>;
  const size_t smem = gather2_smem_bytes(a.chunk_cache, 1, a.stage_budget);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.BC + a.cb - 1) / a.cb, a.nblk, a.n_bands);
  kern<<<grid, 128, smem, st>>>(a, static_cast<const T*>(dy), static_cast<T*>(dx));
  count_launch();
  return cudaGetLastError();
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

template <typename T, int K, int S>
cudaError_t launch_fwd2_t(const GatherArgs& a, const void* x, void* y, cudaStream_t st) {
  auto kern = fwd_gather2_kernel<T, K, S>;
  const size_t smem = gather2_smem_bytes(a.chunk_cache, K, a.stage_budget);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.BC + a.cb - 1) / a.cb, a.nblk, a.n_rows);
  kern<<<grid, 128, smem, st>>>(a, static_cast<const T*>(x), static_cast<T*>(y));
  count_launch();
  return cudaGetLastError();
}

template <typename T, int K, int S>
cudaError_t launch_fwd2b_t(const GatherArgs& a, const void* x, void* y, cudaStream_t st) {
  auto kern = fwd_gather2_band_kernel<T, K, S>;
  const size_t smem = gather2_smem_bytes(a.chunk_cache, K, a.stage_budget);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.BC + a.cb - 1) / a.cb, a.nblk, a.n_bands);
  kern<<<grid, 128, smem, st>>>(a, static_cast<const T*>(x), static_cast<T*>(y));
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

cudaError_t launch_fwd_gather2(bool bf16, int K, int S, const GatherArgs& a, const void* x, void* y,
                               cudaStream_t st) {
#define DISCO_FWD2_CASE(TT, KK)                                      \
  if (K == KK) {                                                     \
    if (S == 1) return launch_fwd2_t<TT, KK, 1>(a, x, y, st);        \
    if (S == 2) return launch_fwd2_t<TT, KK, 2>(a, x, y, st);        \
  }
  if (bf16) {
    DISCO_FWD2_CASE(__nv_bfloat16, 3)
  } else {
    DISCO_FWD2_CASE(float, 3)
  }
#undef DISCO_FWD2_CASE
  return cudaErrorNotSupported;
}

cudaError_t launch_fwd_gather2_band(bool bf16, int K, int S, const GatherArgs& a, const void* x, void* y,
                                    cudaStream_t st) {
  if (K != 3) return cudaErrorNotSupported;
  if (bf16) {
    if (S == 1) return launch_fwd2b_t<__nv_bfloat16, 3, 1>(a, x, y, st);
    if (S == 2) return launch_fwd2b_t<__nv_bfloat16, 3, 2>(a, x, y, st);
  } else {
    if (S == 1) return launch_fwd2b_t<float, 3, 1>(a, x, y, st);
    if (S == 2) return launch_fwd2b_t<float, 3, 2>(a, x, y, st);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_adj_gather2_band(bool bf16, int S, const GatherArgs& a, const void* dy, void* dx,
                                    cudaStream_t st) {
  if (bf16) {
    if (S == 1) return launch_adj2b_t<__nv_bfloat16, 1>(a, dy, dx, st);
    if (S == 2) return launch_adj2b_t<__nv_bfloat16, 2>(a, dy, dx, st);
  } else {
    if (S == 1) return launch_adj2b_t<float, 1>(a, dy, dx, st);
    if (S == 2) return launch_adj2b_t<float, 2>(a, dy, dx, st);
  }
  return cudaErrorNotSupported;
}

size_t gather2_bytes(int chunk_cache, int nk, int stage_f2) { return gather2_smem_bytes(chunk_cache, nk, stage_f2); }

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
