// Launch interfaces of the libdisco kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include "plan.h"

namespace disco {

// Counts a kernel launch (reported by disco_launch_count).
void count_launch();

struct GatherArgs {
  const RowPlan* rows;
  const SrcRow* srcs;
  const Chunk* chunks;
  const float* vals;
  const Ring* rings;
  const BandPlan* bands;  // banded plans only
  int n_bands;            // bands of this launch: bands[band0 .. band0 + n_bands)
  int band0;
  int n_rows;        // output rows in the plan (grid.z)
  int BC;            // channel planes (batch * channels)
  int cb;            // channel planes per CTA
  int qb, nblk;      // outputs per block, blocks per row
  int n_src, n_src_rows;  // source row length, source rows per channel plane
  int n_out, n_out_rows;  // output row length, output rows per channel plane
  int stage_budget;  // staged floats per CTA (>= the largest row's per-channel need)
  int chunk_cache;   // chunks (and their values) of a row kept in shared memory
  int vec_stage;     // 1: stage whole 16-byte vectors (n_src a multiple of the vector)
};

bool gather_supports(int K, int stride);
cudaError_t launch_fwd_gather(bool bf16, int K, int S, const GatherArgs& a, const void* x, void* y, cudaStream_t st);
cudaError_t launch_adj_gather(bool bf16, int S, const GatherArgs& a, const void* dy, void* dx, cudaStream_t st);
// Paired-plane forward gather (packed fp32 FMAs) for K = 3; stage_budget in float2 words.
cudaError_t launch_fwd_gather2(bool bf16, int K, int S, const GatherArgs& a, const void* x, void* y,
                               cudaStream_t st);
// Same over a banded plan (a.bands): one CTA per band, block of outputs and channel block.
cudaError_t launch_fwd_gather2_band(bool bf16, int K, int S, const GatherArgs& a, const void* x, void* y,
                                    cudaStream_t st);
size_t gather2_bytes(int chunk_cache, int nk, int stage_f2);
// Paired, banded adjoint gather (dx) over a banded adjoint plan; stage_budget in float2 words.
cudaError_t launch_adj_gather2_band(bool bf16, int S, const GatherArgs& a, const void* dy, void* dx,
                                    cudaStream_t st);

// Tensor-core (Toeplitz) contraction x -> y for bf16, stride 1 (contract_tc.cu).
constexpr size_t kTcSmemLimit = 227 * 1024;
struct TzLaunch {
  const TzSlab* slabs;   // device arrays of the Toeplitz plan
  const int* row_begin;
  const int* slots;     // {row, first slab, end slab, 0} per row position, heaviest rows first
  const void* b;         // expanded Psi blocks (bf16)
  int K, parts, N;
  int BC, nlat_in, nlat_out, nlon;
  int n_slots = 0;       // row records to process (0: all nlat_out rows)
};
// Layers the Toeplitz plan serves (host-side geometry only) / that the device can run.
bool toeplitz_geometry(int K, int stride, int nlon_in, int nlon_out);
bool contract_tc_supported(int K, int stride, int nlon_in, int nlon_out);
cudaError_t launch_contract_tc(const TzLaunch& L, const void* x, void* y, cudaStream_t st);
// Strip-staged tensor-core contraction over a ring plan (contract_ring.cu, RingPlan in
// psi_builder.h); src is [BC][n_src_rows][nlon], dst [BC][K][n_out_rows][nlon], bf16.
struct RingLaunch {
  const int* strips;   // device arrays of the ring plan
  const int* loads;
  const int* items;
  const int* rows;
  const void* b;
  int n_strips;
  int K, nb, wmax, ns, nrb, bk, nbs, mirror;
  int BC, n_src_rows, n_out_rows, nlon;
};
// TMA-staged strip contraction over a tile-script plan (contract_ring2.cu, TilePlan in
// psi_builder.h); src is [BC][n_src_rows][nlon], dst [BC][K][n_out_rows][nlon], bf16.
struct Ring2Launch {
  const int* tiles;  // device arrays of the tile-script plan
  const int* loads;
  const int* copies;
  const uint32_t* cmds;
  const int* rows;
  const int* cta_tiles;
  const void* b;
  int n_ctas, n_qt;
  int K, nb, ns, nrb, nbs, bslot_bytes, mirror;
  int BC, n_src_rows, n_out_rows, nlon;
};
// Fused forward on the same kernel (mirror rows, C_in = 64 channels per batch element, groups 1,
// C_out <= 64): out [B][C_out][n_out_rows][nlon] = bias + the channel mix of the contraction.
// With w_t, over the transposed-Psi plan and dout as the source, it is the input gradient dx.
struct Ring2Fused {
  const void* x;
  const void* w;     // [C_out][64][K] bf16, or [64][C_out][K] with w_t
  const void* bias;  // [C_out] bf16 or null
  void* out;
  int C_in, C_out;
  int w_t = 0;       // 1: mix with the transposed weights (the input gradient)
};
cudaError_t launch_fused_ring2(const Ring2Launch& L, const Ring2Fused& F, cudaStream_t st);
bool ring2_kernel_k(int K);
cudaError_t launch_contract_ring2(const Ring2Launch& L, const void* src, void* dst, cudaStream_t st);
int take_contract_ring2_status();
bool ring_kernel_k(int K);
// One-thread kernel whose wait on an mbarrier nothing arrives on expires after limit_us; the
// expiry is reported by take_contract_ring_status like any bounded wait of the ring kernel.
cudaError_t launch_wait_selftest(unsigned int limit_us, cudaStream_t st);
cudaError_t launch_contract_ring(const RingLaunch& L, const void* src, void* dst, cudaStream_t st);
int take_contract_ring_status();

// Fused forward on the same plan: out = bias + mix(w, contraction(x)) with the y tile kept in
// shared memory; for K = 3 or 5 and 64 input channels per group (bf16, stride 1).
struct TzFused {
  const void* x;
  const void* w;     // (C_out, C_in / G, K)
  const void* bias;  // may be null
  void* out;
  int C_in, C_out, G;
};
bool fused_tz_supported(int K, int C_in, int C_out, int G);
cudaError_t launch_fused_tz(const TzLaunch& L, const TzFused& F, cudaStream_t st);
int take_contract_tc_status();

// Grouped channel mix (SIMT):
//   out[b, g*Mg + m, n] = bias[g*Mg + m] + sum_{r < Rg} wm[g, m, r] * in[b, g*Rg + r, n]
struct MixArgs {
  const void* in;
  const void* wm;
  const void* bias;  // may be null
  void* out;
  int B, G, Mg, Rg, N;
};
cudaError_t launch_mix_simt(bool bf16, const MixArgs& a, cudaStream_t st);
// Tensor-core (tcgen05) form for bf16: needs Mg % 16 == 0, Rg % 8 == 0 and N % 8 == 0
// (TMA rows start on 16-byte boundaries).
bool mix_tc_supported(int Mg, int Rg, int N);
cudaError_t launch_mix_tc(const MixArgs& a, cudaStream_t st);
// Device status word of the tensor-core kernels (5 after an expired wait); read and clear.
int take_mix_tc_status();
int take_fused_tc_status();

// wt[g, c*K + k, o] = w[g*Og + o, c, k]   (the transposed weight of the dx einsum)
cudaError_t launch_transpose_weight(bool bf16, const void* w, void* wt, int G, int Og, int Cg, int K, cudaStream_t st);

// Split-K weight gradient partials (SIMT):
//   part[split, g, o, r] = sum_{n in chunk} dout[b, g*Og + o, n] * yv[b, g*Rg + r, n]
//   bpart[split, g*Og + o] = sum_{n in chunk} dout[b, g*Og + o, n]          (when bpart != null)
// split = b * nchunk + chunk, chunk covers n in [chunk*nc, chunk*nc + nc).
struct DwArgs {
  const void* dout;
  const void* yv;
  float* part;
  float* bpart;
  int B, G, Og, Rg, N, nc, nchunk;
};
cudaError_t launch_dw_partial_simt(bool bf16, const DwArgs& a, cudaStream_t st);
// Tensor-core form for bf16 (Og % 16 == 0, Og <= 256, N % 8 == 0); nc must be a multiple of 64.
bool dw_tc_supported(int Og, int Rg, int N);
cudaError_t launch_dw_tc(const DwArgs& a, cudaStream_t st);
// t[p][rows[i]][0..nlon) = 0 for p < planes, t being [planes][nrows][nlon] of elem_bytes elements.
cudaError_t launch_zero_rows(void* t, int elem_bytes, const int* rows, int n_rows, int planes, int nrows, int nlon,
                             cudaStream_t st);
// Rows `rows` of every plane set to bias[plane % C] (zero when bias is NULL).
cudaError_t launch_fill_rows(bool bf16, void* t, const int* rows, int n_rows, int planes, int nrows, int nlon,
                             const void* bias, int C, cudaStream_t st);
// dw[g*Og + o, r] = sum_split part[split, g, o, r]; dbias[o] = sum_split bpart[split, o]; fixed order.
cudaError_t launch_dw_reduce(bool bf16, const float* part, const float* bpart, void* dw, void* dbias, int nsplit,
                             int G, int Og, int Rg, cudaStream_t st);

// Fused forward (SIMT): contraction into an on-chip y tile, then the channel mix.
struct FusedArgs {
  GatherArgs g;       // forward gather plan; BC unused, qb/nblk for the fused block
  const void* x;
  const void* w;      // (C_out, Cg, K)
  const void* bias;   // may be null
  void* out;
  int B, C_in, C_out, G, K;
  int ytile_floats;   // Cg*K*qb
};
cudaError_t launch_fused_simt(bool bf16, int K, int S, const FusedArgs& a, cudaStream_t st);

// Fused forward with the channel mix on tensor cores (bf16).  fused_tc_plan decides whether the
// layer fits (Og a multiple of 32 up to 256, C_in/G a multiple of 16, w staged in <= 96 KB) and
// fills the pass layout and the shared memory size for a gather block of 128 outputs.
bool fused_tc_plan(int C_in, int C_out, int G, int K, int chunk_cache, int stage_floats, int* pass_ch, int* a_sbo,
                   int* w_chunks, size_t* smem);
cudaError_t launch_fused_tc(int K, int S, const GatherArgs& g, const void* x, const void* w, const void* bias,
                            void* out, int B, int C_in, int C_out, int G, int pass_ch, int a_sbo, int w_chunks,
                            cudaStream_t st);

}  // namespace disco
