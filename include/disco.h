/*
 * disco.h -- C ABI of libdisco, the B200 (sm_100a) DISCO convolution on the 2-sphere.
 *
 * The operation is the discrete-continuous convolution of the page
 * "torch_harmonics.DiscreteContinuousConvS2" (forward equation and the
 * definition of Psi below it):
 *
 *   out[b,o,j,q] = bias[o] + sum_{c in group(o)} sum_k w[o,c',k] * y[b,c,k,j,q]
 *   y[b,c,k,j,q] = sum_{(i,p)} Psi[k,j,(i,p)] * x[b,c,i,(q*s + p) mod nlon_in]
 *
 * with s = nlon_in / nlon_out.  Psi is the filter basis evaluated at the
 * input grid points rotated so that output point (j, 0) sits at the north
 * pole, times the quadrature weights, normalised per (k, j) row ("nodal");
 * equispaced longitudes make it independent of the output longitude
 * (p-shift symmetry).  The constructor arguments of that page map onto
 * disco_spec_t; input (B, C_in, nlat_in, nlon_in) and output
 * (B, C_out, nlat_out, nlon_out) shapes are as printed there.
 *
 * Conventions for every compute call:
 *   - Tensors are dense row-major (C order) in device memory, base 16-byte
 *     aligned, in the storage dtype given (fp32 or bf16); the caller owns them.
 *       x    (B, C_in, nlat_in, nlon_in)
 *       w    (C_out, C_in/groups, K)
 *       bias (C_out)                      may be NULL (no bias)
 *       y    (B, C_in, K, nlat_out, nlon_out)   the K-expanded intermediate
 *       out  (B, C_out, nlat_out, nlon_out)
 *       dout like out, dx like x, dw like w, dbias like bias
 *   - Output channel o belongs to group o / (C_out/groups) and reads input
 *     channels of the same group (standard grouped convolution).
 *   - Arithmetic is fp32 accumulate.  bf16 layers store x, w, y, out, dout,
 *     dx, dw and dbias in bf16 (round to nearest even on store).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream).  They never synchronise and never
 *     allocate device memory; scratch comes in through `workspace` of at
 *     least disco_workspace_size() bytes (256-byte aligned).
 *   - Errors are reported as a disco_status; nothing is thrown across the
 *     ABI.  disco_last_error() returns a thread-local message for the last
 *     non-OK status on the calling thread.
 *   - A launch error is reported as DISCO_ERR_CUDA.  Faults that surface
 *     later (asynchronously) are seen by the caller's next synchronisation.
 */
#ifndef DISCO_H
#define DISCO_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DISCO_OK = 0,
  DISCO_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, groups not dividing C_in/C_out,
                                theta_cutoff <= 0, nlat < 2, n_r < 2 */
  DISCO_ERR_UNSUPPORTED = 2, /* grid/basis/normalisation other than the ones below; nlon_in not a
                                multiple of nlon_out (the p-shift needs output longitudes on input
                                longitudes); stride nlon_in/nlon_out above 4; channel counts or
                                K beyond the kernels' limits */
  DISCO_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  DISCO_ERR_ALLOC = 4,       /* host allocation or the one-off Psi upload failed */
  DISCO_ERR_TIMEOUT = 5,     /* a bounded device-side wait expired */
  DISCO_ERR_GEOMETRY = 6     /* a distance or basis value fell inside the tie reject band
                                (see disco_psi_build) */
} disco_status;

typedef enum { DISCO_F32 = 0, DISCO_BF16 = 1 } disco_dtype;

/* Latitude grids (grid_in / grid_out).  The DISCO constructor takes grid_in / grid_out (page
 * "torch_harmonics.DiscreteContinuousConvS2", signature; default "equiangular"); the four
 * names are listed with the same parameters on the page of the module
 * "torch_harmonics.distributed.distributed_spectral_convolution" (class docstring,
 * Parameters).  Neither page defines them; they are read as the textbook rules on
 * t = cos(theta).  Nodes run north to south and the quadrature weights sum to 2 (times
 * 2*pi/nlon_in per point). */
enum {
  DISCO_GRID_EQUIANGULAR = 0,             /* theta_i = pi*i/(nlat-1), poles included;
                                             Clenshaw-Curtis weights */
  DISCO_GRID_LEGENDRE_GAUSS = 1,          /* the nlat Gauss-Legendre nodes and weights; no poles */
  DISCO_GRID_LOBATTO = 2,                 /* the nlat Gauss-Lobatto-Legendre nodes (poles
                                             included) and weights; nlat >= 2 */
  DISCO_GRID_EQUIANGULAR_TRAPEZOIDAL = 3  /* equiangular nodes, trapezoidal weights in t:
                                             w_i = (t_{i-1} - t_{i+1}) / 2, ends one-sided */
};
enum { DISCO_BASIS_PIECEWISE_LINEAR = 0 };
enum { DISCO_NORM_NODAL = 0 };                 /* every (k, j) row of Psi sums to one */

/* Operation codes for disco_workspace_size. */
enum {
  DISCO_OP_FWD = 0,
  DISCO_OP_FWD_FUSED = 1,
  DISCO_OP_BWD_INPUT = 2,
  DISCO_OP_BWD_WEIGHT = 3,           /* with y given */
  DISCO_OP_BWD_WEIGHT_RECOMPUTE = 4, /* with y == NULL: y is recomputed from x */
  DISCO_OP_EINSUM_ADJOINT = 5        /* disco_einsum_adjoint */
};

/* Layer geometry: the in_shape / out_shape / kernel_shape / basis_type /
 * basis_norm_mode / grid_in / grid_out / theta_cutoff arguments of the
 * DiscreteContinuousConvS2 constructor.  kernel_shape = {n_r, n_alpha};
 * n_alpha == 1 is the isotropic basis with K = n_r radial hats at
 * r_k = k*theta_cutoff/(n_r-1); n_alpha > 1 is the anisotropic basis with
 * K = 1 + (n_r-1)*n_alpha (the r = 0 hat merged, the outer radial hats times
 * n_alpha azimuthal hats of the bearing east of local north).  The pages give
 * no default cutoff, so theta_cutoff is required. */
typedef struct {
  int nlat_in, nlon_in, nlat_out, nlon_out;
  int grid_in, grid_out;      /* DISCO_GRID_* (any of the four) */
  int kernel_shape[2];        /* {n_r, n_alpha} */
  int basis_type;             /* DISCO_BASIS_PIECEWISE_LINEAR only */
  int basis_norm_mode;        /* DISCO_NORM_NODAL only */
  double theta_cutoff;        /* radians, > 0 */
} disco_spec_t;

/* Opaque Psi: owns a host copy (fp64 values) and the device plans. */
typedef struct disco_psi disco_psi;

/* Builds Psi on the host (synchronous; Clenshaw-Curtis quadrature, inclusive
 * cutoff r <= theta_c + 1e-10, entries kept when phi_k > 1e-10, a computed
 * r - theta_c or phi inside [1e-11, 1e-9] is DISCO_ERR_GEOMETRY) and uploads
 * the kernels' plans to `device`.  On success *out owns everything until
 * disco_psi_destroy.  On failure *out is NULL. */
disco_status disco_psi_build(const disco_spec_t* spec, int device, disco_psi** out);

/* Psi of one polar band: the output latitudes j_begin <= j < j_end of the layer spec describes,
 * as a layer of its own.  This is the per-rank layer of the "halo-exchange" polar mode on the page
 * "torch_harmonics.distributed.DistributedDiscreteContinuousConvS2" (parameter polar_mode): a
 * rank computes the output latitudes it owns outright from the input rows they reach.
 *   j_begin, j_end : output latitude range, 0 <= j_begin < j_end <= spec->nlat_out.
 *   i_begin, i_end : (out, host) the input rows [i_begin, i_end) the band's Psi reaches.
 * The handle is a layer with nlat_out = j_end - j_begin and nlat_in = i_end - i_begin (the same
 * longitudes, K and grids): every compute call takes x restricted to input rows
 * [i_begin, i_end) and gives out rows [j_begin, j_end); disco_bwd_input gives the band's
 * contribution to dx on rows [i_begin, i_end), to be summed with the other bands' contributions
 * over shared rows; disco_bwd_weight gives the band's part of dw / dbias, to be summed over
 * bands.  Its rows are exactly the full Psi's rows j_begin..j_end-1, re-indexed.  Errors as
 * disco_psi_build, and INVALID_ARG for an empty or out-of-range row range or NULL i_begin /
 * i_end.  The caller owns the handle (disco_psi_destroy). */
disco_status disco_psi_build_band(const disco_spec_t* spec, int j_begin, int j_end, int device, disco_psi** out,
                                  int* i_begin, int* i_end);

/* Psi of one band of input latitudes: the entries of the layer spec describes whose input row i
 * lies in [i_begin, i_end), for every output latitude.  This is the per-rank layer of the
 * "reduce-scatter" polar mode on the page "torch_harmonics.distributed.
 * DistributedDiscreteContinuousConvS2" (parameter polar_mode): every rank computes a partial sum
 * over all output latitudes from the input rows it owns, and a reduce-scatter completes and
 * splits it.  The handle is a layer with nlat_in = i_end - i_begin (its rows re-indexed from 0)
 * and the full nlat_out: disco_contract / disco_fwd / disco_einsum give the band's partial y and
 * out (sum them over bands; add the bias once), disco_bwd_input takes dout on every output row
 * and gives dx on the band's rows, disco_bwd_weight the band's part of dw (sum over bands).
 * Output rows that no entry of the band reaches are written as zeros by the contraction, as the
 * bias (zeros without one) by disco_fwd_fused, and input rows no entry reaches as zeros by the
 * adjoint.  Errors as disco_psi_build, and INVALID_ARG for an
 * empty or out-of-range row range.  The caller owns the handle (disco_psi_destroy). */
disco_status disco_psi_build_inputs(const disco_spec_t* spec, int i_begin, int i_end, int device, disco_psi** out);

/* Frees host and device memory of a Psi (synchronises the device first).  NULL is a no-op. */
disco_status disco_psi_destroy(disco_psi* psi);

/* K (number of basis functions) and nnz (number of non-zero Psi entries). */
disco_status disco_psi_info(const disco_psi* psi, int* K, long long* nnz);

/* Copies the nnz Psi entries to caller-owned HOST arrays of length nnz,
 * sorted by (j, k, i, p), p in [0, nlon_in), values in fp64. */
disco_status disco_psi_export(const disco_psi* psi, int* k, int* j, int* i, int* p, double* val);

/* Bytes of scratch the operation needs (0 when none). */
disco_status disco_workspace_size(const disco_psi* psi, int op, int B, int C_in, int C_out, int groups,
                                  disco_dtype dtype, size_t* bytes);

/* The sparse Psi contraction alone (the first sum of the forward equation):
 *   y[b,c,k,j,q] = sum_{(i,p)} Psi[k,j,(i,p)] * x[b,c,i,(q*s + p) mod nlon_in]
 * x (B, C, nlat_in, nlon_in) -> y (B, C, K, nlat_out, nlon_out).  No scratch. */
disco_status disco_contract(const disco_psi* psi, int B, int C, disco_dtype dtype, const void* x, void* y,
                            void* stream);

/* The weight einsum alone (the sums over c_i and k of the forward equation):
 *   out[b,o,j,q] = bias[o] + sum_{c in group(o), k} w[o,c',k] * y[b,c,k,j,q]
 * y (B, C_in, K, nlat_out, nlon_out), w, bias (nullable) -> out.  No scratch. */
disco_status disco_einsum(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                          const void* y, const void* w, const void* bias, void* out, void* stream);

/* Forward, unfused: writes the K-expanded y (saved for backward) and out;
 * the same as disco_contract followed by disco_einsum. */
disco_status disco_fwd(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                       const void* x, const void* w, const void* bias, void* y, void* out,
                       void* workspace, size_t ws_bytes, void* stream);

/* Forward, fused: out only; the K-expanded y is formed tile by tile on chip
 * and never written to device memory (the `fused=True` mode of the page). */
disco_status disco_fwd_fused(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                             const void* x, const void* w, const void* bias, void* out,
                             void* workspace, size_t ws_bytes, void* stream);

/* Backward with respect to x: dx = A^T dout, A the forward map without bias
 * (the exact adjoint of contraction followed by the weight einsum). */
disco_status disco_bwd_input(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                             const void* dout, const void* w, void* dx,
                             void* workspace, size_t ws_bytes, void* stream);

/* The two halves of disco_bwd_input, for callers that keep dy or time the steps apart.
 *
 * disco_einsum_adjoint: the transposed weight einsum (the adjoint of disco_einsum without bias)
 *   dy[b,c,k,j,q] = sum_{o in group(c)} w[o,c',k] * dout[b,o,j,q]
 * dout (B, C_out, nlat_out, nlon_out), w (C_out, C_in/groups, K) -> dy (B, C_in, K, nlat_out,
 * nlon_out), all caller-owned device memory.  Scratch (the transposed w) comes in through
 * `workspace`, sized by disco_workspace_size(DISCO_OP_EINSUM_ADJOINT, ...).
 *
 * disco_contract_adjoint: the adjoint of the sparse Psi contraction (disco_contract), that is
 * the transpose of the forward equation's first sum on the page
 * "torch_harmonics.DiscreteContinuousConvS2", section "Forward":
 *   dx[b,c,i,l] = sum_{k,j,q,p : (q*s + p) mod nlon_in = l} Psi[k,j,(i,p)] * dy[b,c,k,j,q]
 * dy (B, C, K, nlat_out, nlon_out) -> dx (B, C, nlat_in, nlon_in).  No scratch.
 *
 * Both are asynchronous on `stream` and allocate nothing; errors as for disco_bwd_input.
 * disco_bwd_input(..) is disco_einsum_adjoint followed by disco_contract_adjoint. */
disco_status disco_einsum_adjoint(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                                  const void* dout, const void* w, void* dy, void* workspace, size_t ws_bytes,
                                  void* stream);
disco_status disco_contract_adjoint(const disco_psi* psi, int B, int C, disco_dtype dtype, const void* dy, void* dx,
                                    void* stream);

/* Backward with respect to w and bias:
 *   dw[o,c',k] = sum_{b,j,q} dout[b,o,j,q] * y[b,c,k,j,q],  dbias[o] = sum_{b,j,q} dout[b,o,j,q].
 * When y is NULL it is recomputed from x (the fused mode's one extra
 * contraction).  dbias may be NULL.  The reduction order is fixed, so results
 * are bitwise reproducible from run to run. */
disco_status disco_bwd_weight(const disco_psi* psi, int B, int C_in, int C_out, int groups, disco_dtype dtype,
                              const void* dout, const void* y, const void* x, void* dw, void* dbias,
                              void* workspace, size_t ws_bytes, void* stream);

/* The weight einsum, its transpose and the weight gradient on a set of points, without a Psi
 * handle.  They compute the channel-mixing sums of the forward equation on the page
 * "torch_harmonics.DiscreteContinuousConvS2", section "Forward", and of its adjoint, at each of
 * npts points of every (b, channel) plane, the points contiguous in the plane:
 *
 *   disco_mix:          out[b,o,n] = bias[o] + sum_{c in group(o), k} w[o,c',k] * y[b,c,k,n]
 *   disco_mix_adjoint:  dy[b,c,k,n] = sum_{o in group(c)} w[o,c',k] * dout[b,o,n]
 *   disco_mix_weight:   dw[o,c',k] = sum_{b,n} dout[b,o,n] * y[b,c,k,n],  dbias[o] = sum_{b,n} dout[b,o,n]
 *
 * y and dy are (B, C_in, K, npts), out and dout (B, C_out, npts), w and dw (C_out, C_in/groups,
 * K), bias and dbias (C_out), all caller-owned device memory on the current device, in `dtype`.
 * bias and dbias may be NULL.  The page's distributed layer needs them on the longitudes that
 * one azimuth rank owns (page "torch_harmonics.distributed.DistributedDiscreteContinuousConvS2",
 * class description: the einsum runs after the transpose back to longitude shards), a set of
 * points no Psi handle describes.
 *
 * disco_mix_adjoint and disco_mix_weight take scratch through `workspace`, sized by
 * disco_mix_workspace_size with op DISCO_OP_EINSUM_ADJOINT or DISCO_OP_BWD_WEIGHT (no other op).
 * All three are asynchronous on `stream` and allocate nothing.  Errors: DISCO_ERR_INVALID_ARG for
 * a non-positive size, groups not dividing both channel counts, npts above 2^31 - 1, a NULL
 * required pointer, an unknown dtype or a missing or short workspace; DISCO_ERR_CUDA for a
 * failed launch.  The weight gradient's reduction order is fixed (bitwise reproducible). */
disco_status disco_mix_workspace_size(int op, int B, int C_in, int C_out, int groups, int K, long long npts,
                                      disco_dtype dtype, size_t* bytes);
disco_status disco_mix(int B, int C_in, int C_out, int groups, int K, long long npts, disco_dtype dtype,
                       const void* y, const void* w, const void* bias, void* out, void* stream);
disco_status disco_mix_adjoint(int B, int C_in, int C_out, int groups, int K, long long npts, disco_dtype dtype,
                               const void* dout, const void* w, void* dy, void* workspace, size_t ws_bytes,
                               void* stream);
disco_status disco_mix_weight(int B, int C_in, int C_out, int groups, int K, long long npts, disco_dtype dtype,
                              const void* dout, const void* y, void* dw, void* dbias, void* workspace, size_t ws_bytes,
                              void* stream);

/* Weight gradient that allocates nothing (the pages have no counterpart to this entry point).
 *
 * disco_bwd_weight needs a caller-provided workspace for its split-K partial sums.  Some
 * callers cannot provide one: code that runs inside a host application whose device
 * memory is all owned by that application's allocator, and code that must not allocate
 * once it has started (a cudaMalloc can synchronise the device, fail under memory
 * pressure, or be forbidden by the surrounding framework).  This variant computes the
 * same dw and dbias with its partial sums in a fixed 8 MiB array built into the library;
 * every GPU that loads the library holds that array until the process exits.  It calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *
 *   - Arguments as for disco_bwd_weight, except that y is required (no recompute from x:
 *     that would need a y-sized buffer) and there is no workspace.
 *   - Limit: B * (C_out * (C_in/groups) * K + C_out) <= 2^21 (floats of the array);
 *     larger layers get DISCO_ERR_UNSUPPORTED with a message, and nothing is launched.
 *   - Results equal disco_bwd_weight's up to the order of the split-K additions (this
 *     variant may use fewer, longer splits); the order is fixed, so repeated calls give
 *     identical bits.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call before any
 *     stream capture.  The address is kept together with the device's current context and
 *     looked up again when that context changes (after cudaDeviceReset, for example), so
 *     the first call after such a change also belongs before any capture.
 *   - DISCO_ERR_CUDA when cudaGetDevice or the address lookup fails.
 *   - All calls share the one array and each call overwrites every entry it later reads,
 *     so nothing from an earlier call leaks into a result.  Calls that can overlap on the
 *     GPU (on different streams, or from threads that do not order their streams) race on
 *     the array and produce wrong results: serialise them. */
disco_status disco_bwd_weight_noalloc(const disco_psi* psi, int B, int C_in, int C_out, int groups,
                                      disco_dtype dtype, const void* dout, const void* y, void* dw, void* dbias,
                                      void* stream);

/* Diagnostics: the host copy of a gather plan, for inspection by tests.
 * which = 0 is the forward contraction plan (output rows j), which = 1 the
 * adjoint plan used by disco_bwd_input (output rows i), which = 2 and 3 the
 * banded forms of those two (consecutive light rows sharing their staged
 * source rows; each row record carries its band's source range).  disco_plan_info fills
 * dims[9] = {rows, source rows, chunks, values, value sets per chunk, source
 * step per output, residue classes, ints per row record, ring terms}.
 * disco_plan_export copies the records into caller-owned HOST arrays sized
 * from dims: rows (rows x ints-per-row: row, src_begin, src_end,
 * chunk_start[4], chunk_end[4], ring_begin, ring_end, cost as float bits),
 * source rows (x4: row, start, span, 0), chunks (x4: src, t0, voff,
 * width | kmask << 8), values, and ring terms (x4: source row, k, value as
 * float bits, 0). */
disco_status disco_plan_info(const disco_psi* psi, int which, int* dims);
disco_status disco_plan_export(const disco_psi* psi, int which, int* rows, int* srcs, int* chunks, float* vals,
                               int* rings);

/* Toeplitz plans of the tensor-core kernels (bf16 layers with nlon_in == nlon_out, a
 * multiple of 8): which = 0 the forward plan (output rows j, source rows i of x), which = 1
 * the adjoint plan (output rows i, source rows k*nlat_out + j of dy, one basis function).
 * For an output row and a source row, the correlation along the longitude ring of the
 * forward equation on the page "torch_harmonics.DiscreteContinuousConvS2" (class
 * description) has the same coefficients for every output longitude; for 8 outputs q0 + u
 * and 16*nk input longitudes q0 + lon_off + p' it is the banded block
 * B[p', (h, k, u)] = part h of Psi_k(lon_off + p' - u), h = 0 the bf16 rounding of the
 * value and h = 1 the bf16 rounding of the remainder.
 * disco_toeplitz_info fills dims[8] = {K, parts, N, slabs, row records, bf16 values, most
 * K-steps per slab, K-steps}.  disco_toeplitz_export copies into caller-owned HOST arrays:
 * slabs (x4: source row, lon_off, nk, offset of the block in 16-byte units), row records
 * (x4: output row, first slab, end slab, 0; heaviest rows first) and the blocks (bf16
 * bits, [parts][2*nk][N][8] per slab; column n = (h*K + k)*8 + u when parts = 1,
 * n = k*8 + u in part h when parts = 2).  Both return DISCO_ERR_UNSUPPORTED for layers
 * without a Toeplitz plan.  Host-only handles (device < 0) build the plans too. */
disco_status disco_toeplitz_info(const disco_psi* psi, int which, int* dims);
disco_status disco_toeplitz_export(const disco_psi* psi, int which, int* slabs, int* slots, unsigned short* b);

/* Ring plans of the strip-staged tensor-core kernel (bf16 layers with nlon_in == nlon_out, a
 * multiple of 8): which = 0 the forward plan with mirror rows, 1 the forward plan with plane
 * pairs, 2 and 3 the same for the adjoint (output rows i of dx, source rows k*nlat_out + j of
 * dy, one basis function).  For an output row r and a source row s, the forward equation on the
 * page "torch_harmonics.DiscreteContinuousConvS2" (class description) is a correlation along
 * the longitude ring with the same coefficients for every output longitude; for 16 outputs
 * q0 + u and 16*ks source longitudes starting at q0 + 8*lo (lo = floor(pmin / 8)) it is the
 * banded block B[p', (k, u)] = bf16(Psi_k(8*lo + p' - u)).  A plan is a script replayed for
 * every tile (a strip of output rows, nb*16 output longitudes, 64 or 128 planes): loads put
 * windows of source octets (8 longitudes) into ring slots, items apply a range of one block's
 * K-steps to one load for every block of 16 outputs of the tile.  With mirror rows, M rows
 * 64..127 of each MMA hold the north-south mirror of the output row and of each source row
 * (built only when every mirror row's entries equal the row's own, mirrored, to 1e-12).
 * disco_ring_info fills dims[16] = {K, N = 16K, mirror, nb, wmax (octets per slot), ring slots,
 * row buffers, K-steps per B slot, B slots, grouped by source (0/1), strips, loads, items,
 * rows, bf16 values, MMAs of one tile column}.  disco_ring_export copies into caller-owned
 * HOST arrays: strips (x8: first item, end item, first load, end load, first row, end row,
 * cost, 0; heaviest first), loads (x2: source row | mirror source row << 16, first octet
 * relative to q0/8 (signed 16 bits) | octets << 16 | ring slot << 24), items (x4: load |
 * row << 16 (strip-relative); a_off (signed 16 bits) | ks << 16 | flags << 24 (1 last use of
 * the load, 2 last item of the row, 4 first item of the row); kb0 | nkb << 8 | octets of the
 * load << 16 | row buffer << 24 | ring slot << 28; B offset of K-step kb0 in 16-byte units),
 * rows (x2: r | mirror row
 * << 16 (0xFFFF none); flags (1 no entries) | row buffer << 8) and the blocks ([ks][2][N][8]
 * bf16 bits per (row, source) pair, column k*16 + u).  Block b, K-step k of an item reads
 * octets a_off + 2b + 2k and the next of its load when both lie inside it.  Both return
 * DISCO_ERR_UNSUPPORTED when that plan was not built.  Host-only handles build them too. */
/* Tile-script plans of the TMA-staged strip kernel (bf16 layers with nlon_in == nlon_out, a
 * multiple of 8 and at least 64; K in {1, 3, 5}), same four kinds as the ring plans.  They
 * hold the same products as the ring plans (Toeplitz blocks of Psi on 16 outputs, strips of
 * output rows, 64 output longitudes per tile), with one script per (strip, longitude tile)
 * (scripts strip-major, tile-minor):
 *   tiles (x16: first load, end load, first copy, end copy, first row, end row, start of the
 *     command stream of issuers 0..3 and its end, B batches, cost, 0, 0, 0);
 *   loads (x4: source row | mirror source row << 16; ring slot | chunk mask << 8; first
 *     longitude of chunk 0 (may be negative or past nlon: the staged box reads zeros there);
 *     the script's batch that holds the load's last use).  Chunk c (bit c of the mask) stages the 64 longitudes from x0 + 56c of the row (M
 *     rows 0..63) and of the mirror row or the next 64 planes (M rows 64..127), as 64 x 128-byte
 *     rows in the 128-byte swizzle, at byte 32768*slot + 16384*c (+8192 for rows 64..127);
 *   copies (x4: B offset in 16-byte units; bytes; byte offset in the B slot; flags (1 first of
 *     a batch, 2 last of a batch) | bytes of the batch << 8);
 *   cmds (issuer words: bit 31 clear: an MMA, A at 16*(bits 0-13) in the ring, B at
 *     16*(bits 14-23) in the current B slot, row buffer bits 24-26, accumulate bit 27; bit 31
 *     set: the commit of the current batch (8), then waits for the next batch (1), for the load
 *     of slot bits 8-11 (2), for row buffer bits 12-14 to be free (4)).  The completion of a
 *     batch releases its B slot and every ring slot and finished row whose last use it holds;
 *   rows (x2: r | mirror row << 16; flags (1 no entries) | row buffer << 8 | the script's
 *     batch that holds the row's last MMA << 12);
 *   cta_tiles (n_ctas + 1 offsets, then the scripts of each CTA);
 *   b (the Toeplitz blocks, [ks][2][N][8] bf16 bits per (row, source) pair).
 * disco_tile_info fills dims[20] = {K, N, mirror, nb, ring slots, row buffers, B slots, bytes
 * per B slot, grouped by source, strips, longitude tiles, CTAs, loads, copies, command words,
 * rows, bf16 values, MMAs, TMA boxes, cta_tiles ints}; disco_tile_export copies every array
 * into caller-owned HOST arrays of those sizes (tiles: 12 x strips x tiles).  Both return
 * DISCO_ERR_UNSUPPORTED when that plan was not built.  Host-only handles build them too. */
disco_status disco_tile_info(const disco_psi* psi, int which, int* dims);
disco_status disco_tile_export(const disco_psi* psi, int which, int* tiles, int* loads, int* copies, unsigned int* cmds,
                               int* rows, int* cta_tiles, unsigned short* b);

disco_status disco_ring_info(const disco_psi* psi, int which, int* dims);
disco_status disco_ring_export(const disco_psi* psi, int which, int* strips, int* loads, int* items, int* rows,
                               unsigned short* b);

/* Self test of the failure path of the bounded device-side waits (the pages have no
 * counterpart; it exercises the timeout status that every compute call can report).  Launches
 * on `stream` a one-thread kernel that waits on an mbarrier nothing ever arrives on, gives up
 * after limit_us microseconds (1 to 1000000) and records DISCO_ERR_TIMEOUT the way an expired
 * wait inside a compute kernel does; the kernel then exits, so nothing is left waiting and the
 * context stays usable.  A following disco_sync_status on the stream reports
 * DISCO_ERR_TIMEOUT and clears the status.  INVALID_ARG for a limit out of range, CUDA for a
 * launch error.  Asynchronous; allocates nothing. */
disco_status disco_wait_selftest(unsigned int limit_us, void* stream);

/* Synchronises `stream` and reports device-side failures of the calls queued on it
 * before: DISCO_ERR_CUDA for an asynchronous CUDA error, DISCO_ERR_TIMEOUT when a
 * tensor-core kernel gave up a bounded wait (its results are then invalid).  Clears the
 * timeout record. */
disco_status disco_sync_status(void* stream);

/* Number of kernels this library has launched in the process so far (all
 * devices, all threads); a diagnostic for benchmarks. */
unsigned long long disco_launch_count(void);

/* Thread-local description of the last non-OK status on this thread. */
const char* disco_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DISCO_H */
