// Offline preprocessing: the `precompute(W)` step of the pages' pseudo-code
// (Hacker News item 40067677, "Show HN: Speeding up LLM inference 2x times
// (possibly)": transpose, probes, sortMatrixRows).  Here W already arrives
// [in_dim x out_dim] (row i multiplies v[i]), so no transpose is needed.
//
// One thread block per row:
//   1. keys = (0x7FFF - |w| bits) << 16 | column: ascending order of the keys
//      is |w| descending with ties broken by the lower column (the author's
//      CSR reply: rows are stored from the largest absolute value down);
//      bitonic sort in shared memory.
//   2. the first n ranks are kept (the post text: the least important weights
//      of a row can be left out of memory altogether); probes at the midpoint
//      ranks of 16 equal segments; the dense copy of the kept weights.
//   3. per output panel of 2048 columns, one warp takes the row's kept entries
//      of that panel in rank order (the author's reply on the format: each
//      row is split into parts and only the needed parts are read), keeps the
//      leading 3/8 of them, and cuts those into chunks of 64 slots: a chunk is
//      a run of consecutive ranks, stored sorted by column with 8-bit column
//      gaps (filler slots bridge gaps above 255, pad slots fill the chunk).
//      The greedy cut takes as many ranks as fit in 64 slots.  Chunks are
//      placed through a global counter; the host then copies the used part
//      into storage of the exact size.
//
// Q8 weights (int8 q and a binary16 scale s_i per row, w = s_i q exactly)
// take the same steps: the sort key holds the binary16 bits of |q| (0 for a
// row whose scale is 0, where every |w| is 0), so lists, chunks, heads,
// tails and probes come out as for fp16 weights of magnitude |q|; the
// values (dense copy and chunk slots) are the int8 q.
#include "effort_internal.cuh"

#define EFFORT_PREP_KEYS_MAX 32768
#define EFFORT_PREP_LIST_MAX 800  // >= ceil(3 * 2048 / 8) + 1 entries of one panel list

namespace effort {

struct PrepArgs {
  const void* W;             // [I][O] binary16 bits, or int8 (Q8)
  const uint16_t* scales;    // Q8: [I] binary16 row scales; null for fp16
  int wk;                    // kWeightF16 or kWeightQ8
  int I, O, n, P, dstride, Np;
  void* wdense;              // [I][dstride] of the weight type
  uint16_t* probes;
  void* vals;                // capacity cap_chunks * kCS, of the weight type
  uint8_t* gaps;         // capacity cap_chunks * kCS
  uint16_t* head;        // capacity cap_chunks
  uint4* lst;            // [I][P]
  unsigned* chunk_count; // global chunk allocator; chunk_count[1] receives max |w| bits of the kept weights
  unsigned cap_chunks;
  unsigned* status;
  int prank[kP];         // probe ranks (-1 for empty segments)
};

__device__ __forceinline__ void bitonic_sort_u32(uint32_t* s, int Np) {
  for (int k = 2; k <= Np; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < (Np >> 1); t += blockDim.x) {
        const int lo = ((t & ~(j - 1)) << 1) | (t & (j - 1));
        const int hi = lo + j;
        const uint32_t a = s[lo], b = s[hi];
        const bool asc = (lo & k) == 0;
        if ((a > b) == asc) {
          s[lo] = b;
          s[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

// Ascending bitonic sort of 64 values held by a warp: element `lane` in a0,
// element `lane + 32` in a1.
__device__ __forceinline__ void warp_sort64(unsigned& a0, unsigned& a1) {
  const int lane = threadIdx.x & 31;
  for (int k = 2; k <= 64; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {
        const unsigned lo = min(a0, a1), hi = max(a0, a1);
        a0 = lo;
        a1 = hi;
      } else {
        const unsigned b0 = __shfl_xor_sync(0xFFFFFFFFu, a0, j), b1 = __shfl_xor_sync(0xFFFFFFFFu, a1, j);
        const bool lower = (lane & j) == 0;
        const bool asc0 = (lane & k) == 0, asc1 = ((lane + 32) & k) == 0;
        a0 = (lower == asc0) ? min(a0, b0) : max(a0, b0);
        a1 = (lower == asc1) ? min(a1, b1) : max(a1, b1);
      }
    }
  }
}

// For t <= 64 panel-local columns of a chunk (sorted ascending in s0/s1, the
// positions >= t hold 0xFFFFFFFF), the per-position gap from the previous
// column (from -1 for position 0) and the filler slots it needs.
__device__ __forceinline__ void chunk_gaps(unsigned s0, unsigned s1, int t, int& g0, int& g1, int& f0, int& f1) {
  const int lane = threadIdx.x & 31;
  const unsigned up0 = __shfl_up_sync(0xFFFFFFFFu, s0, 1), up1 = __shfl_up_sync(0xFFFFFFFFu, s1, 1);
  const unsigned last0 = __shfl_sync(0xFFFFFFFFu, s0, 31);
  const int prev0 = (lane == 0) ? -1 : (int)up0;
  const int prev1 = (lane == 0) ? (int)last0 : (int)up1;
  g0 = (lane < t) ? (int)s0 - prev0 : 0;
  g1 = (lane + 32 < t) ? (int)s1 - prev1 : 0;
  f0 = (lane < t) ? (g0 - 1) / 255 : 0;
  f1 = (lane + 32 < t) ? (g1 - 1) / 255 : 0;
}

__device__ __forceinline__ int warp_sum(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

// Slots a chunk of the list entries [q, q + t) takes (entries plus fillers).
__device__ __forceinline__ int chunk_slots(const uint32_t* list, int q, int t, int pbase) {
  const int lane = threadIdx.x & 31;
  unsigned s0 = (lane < t) ? (list[q + lane] & 0xFFFFu) - pbase : 0xFFFFFFFFu;
  unsigned s1 = (lane + 32 < t) ? (list[q + lane + 32] & 0xFFFFu) - pbase : 0xFFFFFFFFu;
  warp_sort64(s0, s1);
  int g0, g1, f0, f1;
  chunk_gaps(s0, s1, t, g0, g1, f0, f1);
  return t + warp_sum(f0 + f1);
}

// Chunk slot `slot` gets the weight at column j of the row (or +0 when the
// row pointers are null: fillers and pads).
__device__ __forceinline__ void put_val(const PrepArgs& a, size_t slot, const uint16_t* row, const int8_t* row8, int j) {
  if (a.wk == kWeightQ8) static_cast<int8_t*>(a.vals)[slot] = row8 ? row8[j] : (int8_t)0;
  else static_cast<uint16_t*>(a.vals)[slot] = row ? row[j] : (uint16_t)0;
}

__global__ void __launch_bounds__(kPrepThreads, 1) k_prep_rows(const __grid_constant__ PrepArgs a) {
  extern __shared__ uint32_t keys[];  // Np keys, then the per-warp list buffers
  __shared__ int panel_n[kMaxPanels];
  const int O = a.O, n = a.n, P = a.P;
  const int i = blockIdx.x;
  const bool q8 = a.wk == kWeightQ8;
  const uint16_t* row = q8 ? nullptr : static_cast<const uint16_t*>(a.W) + (size_t)i * O;
  const int8_t* row8 = q8 ? static_cast<const int8_t*>(a.W) + (size_t)i * O : nullptr;
  uint32_t* lists = keys + a.Np;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  if (threadIdx.x < kMaxPanels) panel_n[threadIdx.x] = 0;
  bool bad = false;
  unsigned sbits = 0;
  if (q8) {
    sbits = a.scales[i];
    if ((sbits & 0x7C00u) == 0x7C00u) bad = true;
  }
  const bool szero = q8 && (sbits & 0x7FFFu) == 0u;
  for (int j = threadIdx.x; j < a.Np; j += blockDim.x) {
    uint32_t key = 0xFFFFFFFFu;
    if (j < O) {
      uint32_t mag;
      if (q8) {
        // |q| as binary16 bits (exact for 0..128); every |w| of a zero-scale row is 0
        mag = szero ? 0u : (uint32_t)__half_as_ushort(__int2half_rn(abs((int)row8[j])));
      } else {
        const uint32_t b = row[j];
        if ((b & 0x7C00u) == 0x7C00u) bad = true;
        mag = b & 0x7FFFu;
      }
      key = ((0x7FFFu - mag) << 16) | (uint32_t)j;
    }
    keys[j] = key;
  }
  if (bad) atomicOr(a.status, kStatusNonfiniteW);
  __syncthreads();
  bitonic_sort_u32(keys, a.Np);

  // dense copy of the kept weights (dropped ones stay +0.0 from the memset)
  for (int r = threadIdx.x; r < n; r += blockDim.x) {
    const int j = (int)(keys[r] & 0xFFFFu);
    if (q8) static_cast<int8_t*>(a.wdense)[(size_t)i * a.dstride + j] = row8[j];
    else static_cast<uint16_t*>(a.wdense)[(size_t)i * a.dstride + j] = row[j];
    atomicAdd(&panel_n[j / kPW], 1);
  }
  // the largest kept |w|: binary16 bits (fp16), or fp32 bits of |s_i| max |q| (Q8, exact)
  if (threadIdx.x == 0) {
    const unsigned m = 0x7FFFu - (keys[0] >> 16);
    atomicMax(a.chunk_count + 1,
              q8 ? __float_as_uint(fabsf(__half2float(__ushort_as_half((unsigned short)sbits))) *
                                   __half2float(__ushort_as_half((unsigned short)m)))
                 : m);
  }
  if (threadIdx.x < kP) {
    const int r = a.prank[threadIdx.x];
    a.probes[(size_t)i * kP + threadIdx.x] = (r >= 0) ? (uint16_t)(0x7FFFu - (keys[r] >> 16)) : (uint16_t)0;
  }
  __syncthreads();

  for (int p = warp; p < P; p += kPrepThreads / 32) {
    uint32_t* list = lists + (size_t)warp * EFFORT_PREP_LIST_MAX;
    const int pbase = p * kPW;
    const int np = panel_n[p];
    const int nstore = (np * kStoreNum + kStoreDen - 1) / kStoreDen;
    const int want = min(np, nstore + 1);  // stored entries plus the first unstored one
    // the panel's kept entries in rank order
    int got = 0;
    for (int r0 = 0; r0 < n && got < want; r0 += 32) {
      const int r = r0 + lane;
      const uint32_t key = (r < n) ? keys[r] : 0xFFFFFFFFu;
      const bool in = (r < n) && ((int)(key & 0xFFFFu) / kPW == p);
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, in);
      const int pos = got + __popc(bal & ((1u << lane) - 1u));
      if (in && pos < want) list[pos] = key;
      got += __popc(bal);
    }
    __syncwarp();
    const unsigned tail = (np > nstore) ? (0x7FFFu - (list[nstore] >> 16)) : 0u;
    // plan: greedy chunks of at most kCS slots
    int nchunks = 0;
    for (int q = 0; q < nstore;) {
      int t = min(kCS, nstore - q);
      int s = chunk_slots(list, q, t, pbase);
      while (s > kCS) {
        t -= s - kCS;
        s = chunk_slots(list, q, t, pbase);
      }
      q += t;
      ++nchunks;
    }
    unsigned base = 0;
    if (lane == 0) base = atomicAdd(a.chunk_count, (unsigned)nchunks);
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
    if (base + (unsigned)nchunks > a.cap_chunks) {
      if (lane == 0) atomicOr(a.status, kStatusInternal);
      continue;
    }
    // emit: the same cut again, now writing the slots
    int k = 0;
    for (int q = 0; q < nstore; ++k) {
      int t = min(kCS, nstore - q);
      int s = chunk_slots(list, q, t, pbase);
      while (s > kCS) {
        t -= s - kCS;
        s = chunk_slots(list, q, t, pbase);
      }
      unsigned s0 = (lane < t) ? (list[q + lane] & 0xFFFFu) - pbase : 0xFFFFFFFFu;
      unsigned s1 = (lane + 32 < t) ? (list[q + lane + 32] & 0xFFFFu) - pbase : 0xFFFFFFFFu;
      warp_sort64(s0, s1);
      int g0, g1, f0, f1;
      chunk_gaps(s0, s1, t, g0, g1, f0, f1);
      // slot of each entry: entries and fillers before it, plus its own fillers
      int inc0 = (lane < t) ? 1 + f0 : 0, inc1 = (lane + 32 < t) ? 1 + f1 : 0;
      int x0 = inc0, x1 = inc1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y0 = __shfl_up_sync(0xFFFFFFFFu, x0, o), y1 = __shfl_up_sync(0xFFFFFFFFu, x1, o);
        if (lane >= o) {
          x0 += y0;
          x1 += y1;
        }
      }
      const int tot0 = __shfl_sync(0xFFFFFFFFu, x0, 31);
      x1 += tot0;
      const int used = __shfl_sync(0xFFFFFFFFu, x1, 31);
      const size_t slot0 = (size_t)(base + k) * kCS;
      if (lane < t) {
        const int e = x0 - inc0;  // first slot of this entry's fillers
        for (int f = 0; f < f0; ++f) {
          put_val(a, slot0 + e + f, nullptr, nullptr, 0);
          a.gaps[slot0 + e + f] = 255;
        }
        put_val(a, slot0 + e + f0, row, row8, pbase + (int)s0);
        a.gaps[slot0 + e + f0] = (uint8_t)(g0 - 255 * f0);
      }
      if (lane + 32 < t) {
        const int e = x1 - inc1;
        for (int f = 0; f < f1; ++f) {
          put_val(a, slot0 + e + f, nullptr, nullptr, 0);
          a.gaps[slot0 + e + f] = 255;
        }
        put_val(a, slot0 + e + f1, row, row8, pbase + (int)s1);
        a.gaps[slot0 + e + f1] = (uint8_t)(g1 - 255 * f1);
      }
      for (int z = used + lane; z < kCS; z += 32) {
        put_val(a, slot0 + z, nullptr, nullptr, 0);
        a.gaps[slot0 + z] = 0;
      }
      if (lane == 0) a.head[base + k] = (uint16_t)(0x7FFFu - (list[q] >> 16));
      q += t;
    }
    if (lane == 0) a.lst[(size_t)i * P + p] = make_uint4(base, (unsigned)nchunks, tail, (unsigned)np);
  }
}

size_t prep_smem_bytes(int Np) {
  return (size_t)Np * 4 + (size_t)kMaxPanels * EFFORT_PREP_LIST_MAX * 4;  // list buffers of warps 0..P-1
}

cudaError_t prep_attributes() {
  return cudaFuncSetAttribute(k_prep_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)prep_smem_bytes(EFFORT_PREP_KEYS_MAX));
}

cudaError_t launch_prep(const void* W, const uint16_t* scales, int wk, int I, int O, int n, int P, int dstride,
                        const int* prank, void* wdense, uint16_t* probes, void* vals, uint8_t* gaps, uint16_t* head,
                        uint4* lst, unsigned* chunk_count, unsigned cap_chunks, unsigned* status, cudaStream_t stream) {
  PrepArgs a;
  a.W = W;
  a.scales = scales;
  a.wk = wk;
  a.I = I;
  a.O = O;
  a.n = n;
  a.P = P;
  a.dstride = dstride;
  int Np = 1;
  while (Np < O) Np <<= 1;
  a.Np = Np;
  a.wdense = wdense;
  a.probes = probes;
  a.vals = vals;
  a.gaps = gaps;
  a.head = head;
  a.lst = lst;
  a.chunk_count = chunk_count;
  a.cap_chunks = cap_chunks;
  a.status = status;
  for (int k = 0; k < kP; ++k) a.prank[k] = prank[k];
  cudaError_t e = prep_attributes();
  if (e != cudaSuccess) return e;
  k_prep_rows<<<I, kPrepThreads, prep_smem_bytes(Np), stream>>>(a);
  return cudaGetLastError();
}

// Upper bound on the chunks of one row: per panel, the stored entries over the
// fewest entries a full chunk holds (kCS minus the fillers a panel's span can
// need).
unsigned long long prep_chunk_bound_per_row(int O, int n) {
  unsigned long long total = 0;
  const int P = (O + kPW - 1) / kPW;
  for (int p = 0; p < P; ++p) {
    const int w = (p == P - 1) ? O - p * kPW : kPW;
    const int np = n < w ? n : w;
    const int nstore = (np * kStoreNum + kStoreDen - 1) / kStoreDen;
    const int per = kCS - (w / 255 + 1);
    total += (unsigned long long)((nstore + per - 1) / per);
  }
  return total;
}

}  // namespace effort
