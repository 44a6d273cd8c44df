// Internal definitions shared by the library's kernels and host code.
//
// Storage of a prepared matrix W [I x O] (binary16).  Row i's order is |w|
// descending with ties to the lower column, and its first n = floor(keep * O
// + 1/2) entries are kept.  The columns are cut into panels of kPW (2048)
// columns; panel p holds columns [kPW p, kPW p + kPW).
//   * lists: for every (row i, panel p), the kept entries of row i whose
//     column lies in panel p, in row i's order.  Only the leading
//     ceil(n_ip * kStoreNum / kStoreDen) of them are stored (n_ip = the list's
//     kept entries); a call that needs more of a list reads the row from the
//     dense copy instead.  The stored part is cut into chunks of kCS slots.
//     A chunk holds a run of consecutive ranks, sorted by column, as binary16
//     value bits (vals) and 8-bit column gaps (gaps): the first gap counts
//     from column -1 of the panel, every further one from the previous slot.
//     A gap of more than 255 is bridged by filler slots (value +0, gap 255);
//     the chunk is padded to kCS slots with (value +0, gap 0).  Fillers and
//     pads have magnitude 0, so no call with a positive cutoff uses them, and
//     at cutoff 0 they add +0 to a column of the panel.
//   * head: per chunk, the magnitude bits of its first (largest) rank.
//   * lst:  per (i, p) {first chunk, stored chunks, tail, n_ip}, where tail
//     is the magnitude bits of the first rank that is not stored (0 when the
//     whole list is stored) and n_ip the list's kept entries.
//   * wdense: [I][dstride] fp16, kept weights at their columns, +0 elsewhere
//     (dstride = O rounded up to a multiple of 256).
//   * probes: [I][16] |w| bits at the midpoint ranks of 16 equal segments of
//     the kept list (the `get_probes` step of the pages' pseudo-code).
//   * wmax_bits: the largest kept |w| (bounds every partial sum of a call).
//
// Q8 matrices (int8 q and one binary16 scale s_i per row, w = s_i q) use the
// same layout with int8 values (vals8, wdense8) and the row scales; heads,
// tails and probes hold the binary16 bits of |q| (0 on a zero-scale row),
// and wmax_bits the fp32 bits of the largest |s_i| |q|.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace effort {

constexpr int kP = 16;            // probes per row
constexpr int kPW = 2048;         // panel width (columns)
constexpr int kStripe = 256;      // dense stripe: 32 lanes x 8 columns
constexpr int kCS = 64;           // slots per chunk: 8 lanes x 8 slots
constexpr int kLanesPerChunk = kCS / 8;
constexpr int kStoreNum = 3, kStoreDen = 8;  // stored share of every list
// Matvec kernel: one block per SM, all resident at once; 16 warps, which
// stream the block's work units with plain 16-byte loads (dense units: warp w
// owns 256-column stripe w mod 8 of half the units; sparse chunks: 8 lanes per
// chunk).
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kUnitCap = kThreads;    // work units of a block handled per round (one per thread)
constexpr int kChunkCap = 8192;       // sparse chunks of a round (more: the rest are read dense)
constexpr int kDenseBatch = 8;        // dense units a warp has in flight
constexpr int kSparseBatch = 8;       // sparse chunks a lane group has in flight
constexpr int kPrepThreads = 1024;
constexpr int kDenseThreads = 256;
constexpr int kDenseRowsPerItem = 8;  // dense rows a warp accumulates per stripe item
constexpr int kMaxPanels = 16;        // 32768 / 2048

// weight kinds of a prepared matrix
enum : int { kWeightF16 = 0, kWeightQ8 = 1 };

// call modes decided on the host from K and the kept count
enum : int { kModeSelect = 0, kModeAll = 1, kModeNone = 2 };
// device status bits
enum : unsigned { kStatusNonfiniteV = 1u, kStatusNonfiniteW = 2u, kStatusInternal = 4u, kStatusTimeout = 8u };

// radix-select digits of the non-negative fp32 chart: bits [30:19], [18:9], [8:0]
constexpr int kBins0 = 4096, kBins1 = 1024, kBins2 = 512;
constexpr int kCandCap = 4096;     // crossing-bin candidates resolved in one block's shared memory
constexpr int kMaxGrid = 512;      // blocks of a matvec grid (one per SM) the crossing-bin gather handles
// chart entries of one block: 16-bit offsets in the bin descriptors, and the
// ranks of two charts' entries share the chunk-index area
constexpr int kMaxSegEntries = kChunkCap;
static_assert(kMaxSegEntries <= 65535 && 2 * kMaxSegEntries * 2 <= kChunkCap * 4, "segment entry bound");
static_assert(2 * kBins0 * 4 <= kCandCap * 8, "two charts' bin counts share the candidate area");
static_assert(2 * (kMaxGrid + 1) * 4 <= kChunkCap * 2, "the gather offsets share the chunk-unit area");

// Device-resident description of a prepared matrix (passed by value).
struct HandleDesc {
  const uint16_t* vals;    // [total chunks * kCS]
  const uint8_t* gaps;     // [total chunks * kCS]
  const uint16_t* head;    // [total chunks]
  const uint4* lst;        // [I][P]
  const uint16_t* wdense;  // [I][dstride]
  const uint16_t* probes;  // [I][kP]
  int I, O, n, P, dstride;
  unsigned total_chunks;
  unsigned wmax_bits;      // binary16 bits of the largest kept |w| (Q8: fp32 bits)
  int wk;                  // kWeightF16 or kWeightQ8
  const int8_t* vals8;     // Q8: [total chunks * kCS] (vals is null)
  const int8_t* wdense8;   // Q8: [I][dstride] (wdense is null)
  const uint16_t* scales;  // Q8: [I] binary16 row scales
  unsigned long long kept_total;
  int pw[kP];              // probe weights (entries each probe stands for)
};

// Per-call scratch in device memory.  The header words, the histograms and
// the bin descriptors must be zero before a call (the library clears them at
// allocation and every call leaves them zero, except after a timeout).
struct WsPtrs {
  unsigned* hdr;              // see kHdr* below
  unsigned long long* bar;    // grid-barrier counter (monotonic)
  unsigned long long* count;  // running |S| (vector 0's: bits [39:0], the finished blocks above)
  unsigned* ghist0;           // [kBins0]
  unsigned* ghist1;           // [kBins1]
  unsigned* ghist2;           // [kBins2]
  unsigned* desc;             // [kBins0][grid]: block b's entries of first-digit bin h, (start << 16) | count
  uint2* seg;                 // [grid][rows_per_block * kP]: block b's chart entries {bits, weight}, grouped by bin
};
// header words: status (word 0), the running sum of |v| over the blocks
// (word 3, fp32 bits), and the 64-bit dense and sparse bytes the last call
// planned to read (words 12..15, added up by the blocks as they finish)
enum : int { kHdrStatus = 0, kHdrVsum = 3, kHdrBytesLast = 12, kHdrWords = 64 };

struct Job {
  HandleDesc hd;
  unsigned barrier_nb;  // blocks each grid-wide barrier waits for (the grid size)
  const void* v;
  float* out;
  float* cutoff_out;
  unsigned long long* count_out;
  unsigned int* rowlen_out;
  WsPtrs ws;
  unsigned long long K;
  int mode;
  int vdtype;  // 0 f32, 1 f16
  unsigned long long* marks;  // nullable: [grid][kMarks] phase times (measurement entry point)
  // the second vector of a two-vector launch (same matrix, each its own
  // cutoff; both in select mode; no row lengths): its v, out, reported
  // cutoff and count, scratch and target count
  const void* v2;
  float* out2;
  float* cutoff_out2;
  unsigned long long* count_out2;
  WsPtrs ws2;
  unsigned long long K2;
  int accumulate_bytes;  // 1: add the planned bytes to the last-call words (a batched call's launches)
  float* out_mirror;     // nullable: page-locked host memory mapped for the device; the finished out is
                         // written there by the last block (host-buffer entry point)
};
constexpr int kMarks = 16;

// Rows of the chart each block of an nb-block grid owns during the cutoff.
__host__ __device__ inline int rows_per_block(int I, int nb) { return (I + nb - 1) / nb; }

// Shared memory of the matvec kernel (byte offsets) for V vectors per launch
// (V = 2: two vectors on one matrix read the union of their prefixes once).
struct SmemLayout {
  size_t iacc, chart, absv, hist, hist2, cand, ulst, uhead, uv, utau, dlist, cidx, cunit, ctl, us, cscale, total;
};
__host__ __device__ inline SmemLayout smem_layout(int I, int nb, int V = 1) {
  SmemLayout L;
  const size_t rp = (size_t)rows_per_block(I, nb);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = (o + bytes + 15) / 16 * 16;
    return at;
  };
  L.iacc = take((size_t)V * kPW * 4);                 // fixed-point panel accumulators
  L.chart = take((size_t)V * rp * kP * 4);            // chart bits of the cutoff rows
  L.absv = take((size_t)V * rp * 4);                  // |v| of the cutoff rows
  L.hist = take((size_t)V * kBins0 * 4);              // first-digit histograms
  L.hist2 = take((size_t)(kBins1 + kBins2) * 4);      // second- and third-digit histograms
  L.cand = take((size_t)kCandCap * 8);                // per-bin entry counts of the charts, then the
                                                      // gathered crossing-bin candidates
  L.ulst = take((size_t)kUnitCap * 16);               // list records of the round's (row, panel) units
  L.uhead = take((size_t)kUnitCap * 32);              // their first 16 stored chunks' first magnitudes
  L.uv = take((size_t)V * kUnitCap * 4);              // v of the unit's row
  L.utau = take((size_t)V * kUnitCap * 4);            // threshold of the unit's row
  L.dlist = take((size_t)kUnitCap * 2);               // units read dense
  L.cidx = take((size_t)kChunkCap * 4);               // sparse chunks to read (chunk index)
  L.cunit = take((size_t)kChunkCap * 2);              // and the unit of each (before the dispatch: the
                                                      // crossing-bin gather's per-block offsets)
  L.ctl = take(256 * 4);                              // control words
  L.us = take((size_t)kUnitCap * 4);                  // Q8: scale of the unit's row
  L.cscale = take(rp * 4);                            // Q8: |scale| of the cutoff rows
  L.total = o;
  return L;
}

}  // namespace effort
