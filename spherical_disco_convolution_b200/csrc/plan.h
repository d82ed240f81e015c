// Host/device plan structures of the DISCO gather kernels.
//
// A "plan" is Psi re-laid out for one kernel family.  Psi itself (page
// "torch_harmonics.DiscreteContinuousConvS2", definition below the forward
// equation) is a sparse tensor Psi[k, j, (i, p)]; the p-shift symmetry stated
// there means one row per output latitude j serves every output longitude q.
//
// Gather plans group the entries of one output row into "source rows" (the
// rows of the source tensor it reaches) and "chunks" (windows of at most
// kChunkW consecutive longitude offsets of one source row, holding the values
// of all nk basis functions densely, zeros included).  A CTA stages every
// source row of its output row in shared memory as a straight run of
// longitudes that already contains the wrap-around, so the inner loop never
// takes a modulo.
//
// For a block of outputs starting at m0 (0 <= m < qb), staged element t of a
// source row holds source longitude  (m0*step + start + t) mod n_src, and a
// chunk with column offset t0 reads, for block-relative output m, the staged
// elements  t0 + m*step + u,  u = 0 .. w-1  (step = s for the forward, where
// output q reads input longitude q*s + d; step = 1 for the adjoint).
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define DISCO_HD __host__ __device__
#else
#define DISCO_HD
#endif

namespace disco {

constexpr int kChunkW = 8;      // longitude offsets per chunk
constexpr int kTaskR = 8;       // consecutive outputs per thread
constexpr int kMaxStride = 4;   // nlon_in / nlon_out supported by the kernels
constexpr int kMaxK = 16;       // basis functions supported by the kernels
constexpr int kMaxSrc = 512;    // source rows per output row supported by the kernels
constexpr int kMaxRing = 64;    // ring terms per output row supported by the kernels
constexpr int kAlign = 8;       // staged rows start on a multiple of 8 longitudes (16 bytes of bf16)

struct SrcRow {
  int row;     // row index into the source tensor's (row, longitude) plane of one channel
  int start;   // offset of staged element 0 relative to m0*step (may be negative)
  int span;    // longitude offsets covered by the row's chunks
  int pad;
};

struct Chunk {
  int src;     // source row, relative to RowPlan::src_begin
  int t0;      // first column (staged element for m = 0)
  int voff;    // offset (floats) of the values, laid out [nk][kChunkW]
  int wk;      // width (1..kChunkW) in bits 0..7, kmask (bit k: basis k non-zero) from bit 8
};

// A full longitude circle of one source row that enters with one constant
// value (an input pole row, or any row seen from an output pole with an
// isotropic basis): its contribution is value * (sum of the source row), the
// same for every output longitude.
struct Ring {
  int row;     // source row index (as SrcRow::row)
  int k;       // accumulator (basis function; 0 for the adjoint)
  float v;     // the constant value
  int pad;
};

// One output row of a gather plan.
struct RowPlan {
  int row;                      // output row (j for the forward, i for the adjoint)
  int src_begin, src_end;
  int chunk_start[kMaxStride];  // chunk list of residue class rho: [chunk_start[rho], chunk_end[rho])
  int chunk_end[kMaxStride];    // (the forward plan only has rho = 0)
  int ring_begin, ring_end;     // ring terms of the row
  float cost;                   // relative work, used to order heavy rows first
};

// A band of consecutive output rows that share their staged source rows: the RowPlans
// rows[rp_begin .. rp_end) all carry the band's source range and their chunks refer to it.
struct BandPlan {
  int rp_begin, rp_end;
  float cost;
  int pad;
};

// One slab of the tensor-core (Toeplitz) contraction: a window of 16*nk consecutive source
// longitudes of source row i, starting lon_off longitudes after the first output of a step
// (lon_off a multiple of 8), together with its expanded Psi block in global memory at 16-byte
// unit boff: [parts][2*nk octets][N columns][8 longitudes] bf16.  Column n of part h holds the
// hi (h = 0) or lo (h = 1) bf16 part of Psi_k at offset lon_off + p' - u for output u, with
// n = (h*K + k)*8 + u when both parts share one block (parts = 1), n = k*8 + u otherwise.
struct TzSlab {
  int i, lon_off, nk, boff;
};
constexpr int kTzSlabK = 4;  // most 16-longitude K-steps in one slab

// Flags of the ring plan records (RingPlan in psi_builder.h, contract_ring.cu).
constexpr int kRowEmpty = 1;      // row flag: no entries, the epilogue writes zeros
constexpr int kItemLast = 1;      // item flag: last use of its load (the slot may be refilled)
constexpr int kItemRowEnd = 2;    // item flag: last item of its row (the accumulator is complete)
constexpr int kItemRowStart = 4;  // item flag: first item of its row

// Tile-script plan (TilePlan in psi_builder.h, contract_ring2.cu).
constexpr int kTileInts = 16;  // per script: load0, load1, copy0, copy1, row0, row1, record0, record1, 0, 0, 0,
                               // batches, cost, 0, 0, 0
// Copy flags: first / last copy of a batch, the copy of the batch record (source: the records).
// The record's copy carries the batch's total bytes << 8 and its number of copies << 24.
constexpr int kCopyBatchStart = 1, kCopyBatchEnd = 2, kCopyMeta = 4;
// A batch's B slot holds its record in the first kMetaBytes: a header of four words (MMA counts
// of issuers 0..3 in bytes 0..3; word offsets of the lists of issuers 1..3 in 10-bit fields;
// load starts: count | ring slots << 3 + 4i; row starts: count | row buffers << 3 + 3i) and
// each issuer's MMA words.  MMA word: A address >> 4 relative to the x ring (bits 0-13), B
// offset >> 4 in the B slot (bits 14-23), row buffer (bits 24-26), accumulate (bit 27).
constexpr int kMetaBytes = 1024;
constexpr int kMaxMetaWords = kMetaBytes / 4;
constexpr int kMaxLoadStarts = 6, kMaxRowStarts = 4;
constexpr int kChunkBytes = 16384;  // one staged chunk: 2 groups x 64 planes x 128 bytes
constexpr int kSlotBytes = 2 * kChunkBytes;

// Staged elements of one source row for a block of qb outputs (a multiple of kAlign).  A task's
// window starts at t0 + m0*step (t0 <= span - 1, m0 <= qb - kTaskR) and holds
// (kTaskR - 1)*step + kChunkW elements, so the last element read is span + (qb - 1)*step + 6.
DISCO_HD inline int staged_len(int span, int qb, int step) {
  return ((qb - 1) * step + span + kChunkW - 1 + kAlign - 1) & ~(kAlign - 1);
}

// Shared-memory words of a staged row: one pad word after every 8 elements, so that the
// windows of 32 threads 8 outputs apart fall into 32 different banks.
DISCO_HD inline int staged_words(int len) { return len + (len >> 3); }

}  // namespace disco
