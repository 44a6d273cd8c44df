// Internal definitions shared by the library's kernels and host code.
//
// Storage of a prepared matrix W [I x O] (binary16), per row i with kept count
// n = floor(keep * O + 1/2):
//   * buckets: tile t covers columns [256 t, 256 t + 256).  Bucket (i, t) holds
//     the kept entries of row i in tile t, ordered by |w| descending (ties:
//     lower column first), as fp16 value bits + u8 local column, at entry
//     offset (t * I + i) * kCap.  Unused slots are +0.0 / 0.
//   * wdense: [I][T * 256] fp16, kept weights at their columns, 0 elsewhere.
//   * probes: [I][16] |w| bits at the midpoint ranks of 16 equal segments of
//     the kept list (the `get_probes` step of the pages' pseudo-code).
//   * ckmag: [I][C + 1]: rank-0 magnitude, then the magnitude at the last rank
//     of each checkpoint block of H ranks (block k ends at min((k+1)H, n)).
//   * cnt: [I][C][T] u8: entries of tile t among the ranks before the end of
//     checkpoint block k, saturated at 255.
// Per call (one "job"): a cutoff c, per-row dispatch records grouped by 32
// rows, and split-K partial sums of each output tile.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace effort {

constexpr int kTW = 256;         // output-tile width (u8 local column)
constexpr int kCap = 256;        // bucket capacity (entries)
constexpr int kP = 16;           // probes per row
constexpr int kCutThreads = 1024;
#ifndef EFFORT_MAC_THREADS
#define EFFORT_MAC_THREADS 384  // multiply kernel block size
#endif
#ifndef EFFORT_MAC_BLOCKS_PER_SM
#define EFFORT_MAC_BLOCKS_PER_SM 2  // resident multiply blocks per SM the register budget is sized for
#endif
constexpr int kMacThreads = EFFORT_MAC_THREADS;
constexpr int kMacBlocksPerSM = EFFORT_MAC_BLOCKS_PER_SM;
constexpr int kMacWarps = kMacThreads / 32;
constexpr int kPrepThreads = 1024;
constexpr int kDenseThreads = 256;
constexpr int kMaxJobs = 16;     // pairs per launch
constexpr int kGroupRows = 32;   // dispatch records are grouped by 32 rows
constexpr int kRecPerGroup = 32; // one 8-byte record per row of a group

// call modes decided on the host from K and the kept count
enum : int { kModeSelect = 0, kModeAll = 1, kModeNone = 2 };
// device status bits
enum : unsigned { kStatusNonfiniteV = 1u, kStatusNonfiniteW = 2u, kStatusInternal = 4u };
// dispatch classes
enum : int { kClassOff = 0, kClassSparse = 1, kClassDense = 2 };

// Device-resident description of a prepared matrix (written once at prepare).
struct HandleDesc {
  const uint16_t* vals;
  const uint8_t* idx;
  const uint16_t* wdense;
  const uint16_t* probes;
  const uint16_t* ckmag;
  const uint8_t* cnt;
  int I, O, T, n, C, H, dstride;
  int pad0;
  unsigned long long kept_total;
  int prank[kP];  // probe ranks (-1 for empty segments)
  int pw[kP];     // probe weights (entries each probe stands for)
};

// Per-job scratch.
struct WsPtrs {
  float* c;                     // the cutoff
  unsigned long long* count;    // running |S|
  unsigned int* done;           // CTAs of the multiply kernel that finished
  unsigned int* tilecnt;        // [T] split-K arrivals per tile
  uint2* rec;                   // [G][32] dispatch records {v bits, tau (fp16 bits) | row << 16}:
                                //   sparse rows at [0, ns), dense rows at [ns, ns + nd)
  unsigned int* gcnt;           // [G] ns | nd << 8
  unsigned char* ut;            // [G][T][32]: read bound U of sparse slot p of group g in tile t
  float* part;                  // per-tile partial sums of the CTAs that share a tile
  unsigned int* status;         // sticky device status bits
};

struct Job {
  HandleDesc hd;  // by value: kernels read it from the parameter bank
  const void* v;
  float* out;
  float* cutoff_out;
  unsigned long long* count_out;
  unsigned int* rowlen_out;
  WsPtrs ws;
  unsigned long long K;
  int mode;
  int vdtype;     // 0 f32, 1 f16
  int dense_q16;  // a row is read densely once this share (x 65536) of it is surely used
  int pad0;
};

template <int NJ>
struct Jobs {
  Job j[NJ];
};

// Cutoff cluster geometry: rows per CTA rounded to whole 32-row groups.
__host__ __device__ inline int cut_rows_per_cta(int I, int cl) {
  int rp = (I + cl - 1) / cl;
  return (rp + kGroupRows - 1) / kGroupRows * kGroupRows;
}
// radix-select digits: bits [30:19], [18:9], [8:0] of the non-negative fp32 chart
constexpr int kBins0 = 4096, kBins1 = 1024, kBins2 = 512;
constexpr int kCandLocal = 2048;  // crossing-bin candidates one cutoff CTA can hold
constexpr int kCandTotal = 4096;  // candidates gathered from the whole cluster
// dynamic shared memory of a cutoff CTA: chart, v, the first-pass histogram,
// its candidate list, and one area shared by the merged histogram, the
// gathered candidates and the fallback passes
__host__ __device__ inline size_t cut_union_bytes() {
  const size_t merged = (size_t)kBins0 * 4;
  const size_t gathered = (size_t)kCandTotal * 6;
  const size_t fallback = 2 * (size_t)(kBins1 + kBins2) * 4;
  size_t m = merged > gathered ? merged : gathered;
  return m > fallback ? m : fallback;
}
__host__ __device__ inline size_t cut_smem_bytes(int I, int cl) {
  const size_t rp = (size_t)cut_rows_per_cta(I, cl);
  return rp * kP * 4 + rp * 4 + (size_t)kBins0 * 4 + (size_t)kCandLocal * 6 + cut_union_bytes() + 64;
}

}  // namespace effort
