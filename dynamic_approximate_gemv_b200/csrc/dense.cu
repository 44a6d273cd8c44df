// Dense baseline: out = W^T v over every weight (the full multiplication the
// method is measured against; the post text of Hacker News item 40067677
// compares the approximation with the regular matrix multiply).
//
// Grid (T * S): CTA (t, s) streams the 256 columns of tile t for the rows of
// slice s, 16 B (8 fp16) per lane per row, 8 rows per warp in flight, fp32
// accumulation in registers; the S partial tiles are summed in fixed order by
// the last CTA of each tile to arrive.
#include "effort_internal.cuh"

namespace effort {

constexpr int kTW = 256;  // columns of one output tile

template <typename VT>
__global__ void __launch_bounds__(kDenseThreads, 4) k_dense_gemv(const uint16_t* __restrict__ W, int I, int O,
                                                              const VT* __restrict__ v, float* out, float* part,
                                                              unsigned* tilecnt, int T, int S) {
  constexpr int kW = kDenseThreads / 32;
  constexpr int kU = 8;
  __shared__ float acc[kW][kTW];
  __shared__ int is_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x % T, s = blockIdx.x / T;
  const int r0 = (int)((long long)I * s / S), r1 = (int)((long long)I * (s + 1) / S);
  const int col0 = t * kTW + 8 * lane;
  const bool active = col0 < O;
  float a8[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) a8[m] = 0.0f;
  for (int r = r0 + warp; r < r1; r += kU * kW) {
    uint4 wv[kU];
    float vv[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int rr = r + u * kW;
      if (active && rr < r1) {
        wv[u] = __ldg(reinterpret_cast<const uint4*>(W + (size_t)rr * O + col0));
        vv[u] = (float)v[rr];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int rr = r + u * kW;
      if (active && rr < r1) {
        const __half* h = reinterpret_cast<const __half*>(&wv[u]);
#pragma unroll
        for (int m = 0; m < 8; ++m) a8[m] += vv[u] * __half2float(h[m]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) acc[warp][8 * lane + m] = a8[m];
  __syncthreads();
  float sum = 0.0f;
  if (threadIdx.x < kTW) {
#pragma unroll
    for (int w = 0; w < kW; ++w) sum += acc[w][threadIdx.x];
  }
  const int col = t * kTW + threadIdx.x;
  const int TWT = T * kTW;
  if (S == 1) {
    if (threadIdx.x < kTW && col < O) out[col] = sum;
    return;
  }
  if (threadIdx.x < kTW) part[(size_t)s * TWT + col] = sum;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(&tilecnt[t], 1u) == (unsigned)(S - 1));
  __syncthreads();
  if (is_last) {
    __threadfence();
    if (threadIdx.x < kTW) {
      float tot = 0.0f;
      for (int ss = 0; ss < S; ++ss) tot += __ldcg(&part[(size_t)ss * TWT + col]);
      if (col < O) out[col] = tot;
    }
    if (threadIdx.x == 0) tilecnt[t] = 0u;
  }
}

// Resident CTAs of the dense baseline per SM (its registers allow fewer than
// its thread count would).
int dense_ctas_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_dense_gemv<float>, kDenseThreads, 0) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  return n > 0 ? n : 1;
}

cudaError_t launch_dense(const uint16_t* W, int I, int O, const void* v, int vdtype, float* out, float* part,
                         unsigned* tilecnt, int T, int S, cudaStream_t stream) {
  const dim3 grid((unsigned)(T * S));
  if (vdtype == 1)
    k_dense_gemv<__half><<<grid, kDenseThreads, 0, stream>>>(W, I, O, reinterpret_cast<const __half*>(v), out, part,
                                                              tilecnt, T, S);
  else
    k_dense_gemv<float><<<grid, kDenseThreads, 0, stream>>>(W, I, O, reinterpret_cast<const float*>(v), out, part,
                                                             tilecnt, T, S);
  return cudaGetLastError();
}

}  // namespace effort
