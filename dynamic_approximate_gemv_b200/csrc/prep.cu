// Offline preprocessing: the `precompute(W)` step of the pages' pseudo-code
// (Hacker News item 40067677, "Show HN: Speeding up LLM inference 2x times
// (possibly)": transpose, probes, sortMatrixRows).  Here W already arrives
// [in_dim x out_dim] (row i multiplies v[i]), so no transpose is needed.
//
// One thread block per row:
//   1. keys = (0x7FFF - |w| bits) << 16 | column: ascending order of the keys
//      is |w| descending with ties broken by the lower column (the author's
//      CSR reply: rows are stored from the largest absolute value down).
//   2. bitonic sort of the keys in shared memory.
//   3. the first n ranks are kept (the post text: the least important weights
//      of a row can be left out of memory altogether).
//   4. probes at the midpoint ranks of 16 equal segments; checkpoint
//      magnitudes every H ranks; the dense copy of the kept weights.
//   5. one warp per output tile walks the sorted row in rank order and
//      appends the tile's entries to its bucket (stable, so each bucket is
//      sorted the same way), recording the running count at every
//      checkpoint.
#include "effort_internal.cuh"

#define EFFORT_PREP_SMEM_MAX (32768 * 4)  // keys of the widest supported row

namespace effort {

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

__global__ void __launch_bounds__(kPrepThreads, 1)
    k_prep_rows(const uint16_t* __restrict__ W, const HandleDesc* __restrict__ hdp, int Np, uint16_t* vals,
                uint8_t* idx, uint16_t* wdense, uint16_t* probes, uint16_t* ckmag, uint8_t* cnt,
                unsigned int* status) {
  extern __shared__ uint32_t keys[];  // Np entries
  const int I = hdp->I, O = hdp->O, T = hdp->T, n = hdp->n, C = hdp->C, H = hdp->H;
  const int dstride = hdp->dstride;
  const int i = blockIdx.x;
  const uint16_t* row = W + (size_t)i * O;

  bool bad = false;
  for (int j = threadIdx.x; j < Np; j += blockDim.x) {
    uint32_t key = 0xFFFFFFFFu;
    if (j < O) {
      const uint32_t b = row[j];
      if ((b & 0x7C00u) == 0x7C00u) bad = true;
      key = ((0x7FFFu - (b & 0x7FFFu)) << 16) | (uint32_t)j;
    }
    keys[j] = key;
  }
  if (bad) atomicOr(status, kStatusNonfiniteW);
  __syncthreads();
  bitonic_sort_u32(keys, Np);

  // dense copy of the kept weights (dropped ones stay +0.0 from the memset)
  for (int r = threadIdx.x; r < n; r += blockDim.x) {
    const int j = (int)(keys[r] & 0xFFFFu);
    wdense[(size_t)i * dstride + j] = row[j];
  }
  if (threadIdx.x < kP) {
    const int k = threadIdx.x, r = hdp->prank[k];
    probes[(size_t)i * kP + k] = (r >= 0) ? (uint16_t)(0x7FFFu - (keys[r] >> 16)) : (uint16_t)0;
  }
  for (int k = threadIdx.x; k <= C; k += blockDim.x) {
    const int r = (k == 0) ? 0 : min(k * H, n) - 1;
    ckmag[(size_t)i * (C + 1) + k] = (uint16_t)(0x7FFFu - (keys[r] >> 16));
  }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int t = warp; t < T; t += nwarps) {
    int running = 0;
    const size_t bbase = ((size_t)t * I + i) * kCap;
    for (int cb = 0; cb < n; cb += 32) {
      const int r = cb + lane;
      int j = 0;
      bool m = false;
      if (r < n) {
        j = (int)(keys[r] & 0xFFFFu);
        m = (j >> 8) == t;
      }
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, m);
      if (m) {
        const int pos = running + __popc(bal & ((1u << lane) - 1u));
        vals[bbase + pos] = row[j];
        idx[bbase + pos] = (uint8_t)(j & 255);
      }
      running += __popc(bal);
      const int end = cb + 32;
      if (lane == 0 && end <= n && end % H == 0) {
        cnt[((size_t)i * C + (end / H - 1)) * T + t] = (uint8_t)min(running, 255);
      }
    }
    if (lane == 0 && n % H != 0) cnt[((size_t)i * C + (C - 1)) * T + t] = (uint8_t)min(running, 255);
  }
}

cudaError_t prep_attributes() {
  return cudaFuncSetAttribute(k_prep_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, EFFORT_PREP_SMEM_MAX);
}

cudaError_t launch_prep(const uint16_t* W, const HandleDesc* d_desc, int I, int O, uint16_t* vals, uint8_t* idx,
                        uint16_t* wdense, uint16_t* probes, uint16_t* ckmag, uint8_t* cnt, unsigned int* status,
                        cudaStream_t stream) {
  int Np = 1;
  while (Np < O) Np <<= 1;
  const size_t smem = (size_t)Np * 4;
  k_prep_rows<<<I, kPrepThreads, smem, stream>>>(W, d_desc, Np, vals, idx, wdense, probes, ckmag, cnt, status);
  return cudaGetLastError();
}

}  // namespace effort
