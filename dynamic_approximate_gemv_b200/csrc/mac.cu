// Multiply-accumulate: the multiply step of `approxMul` in the pages'
// pseudo-code (Hacker News item 40067677).  For every used pair the vector
// element v_i is multiplied by w_ij and added into out_j (the CSR-style walk
// of the write-up quoted in that thread); the author's complexity reply
// (item 40095016) counts O(effort * inDim * outDim) such multiplications.
//
// Grid: (T * S) x jobs.  CTA (t, s) owns output tile t (256 columns) and the
// 32-row groups g = s, s + S, ... of the dispatch.  For each of its rows:
//   dense rows   lanes read the row's 256 weights of the tile from the dense
//                copy (16 B per lane, coalesced), apply the exact predicate
//                fl32(|v_i| * |w|) >= c and accumulate in registers (8
//                columns per lane);
//   sparse rows  lanes read the bucket's leading U entries (U from the
//                checkpoint count table: an upper bound on the used length,
//                at most about H / T entries above it), apply the same
//                predicate and add into a warp-private shared-memory copy of
//                the tile.  The entries of one bucket have distinct columns,
//                so a warp updates its copy with plain loads and stores; a
//                __syncwarp separates buckets.
// Warp copies and registers are summed per CTA; the S partial tiles are summed
// in fixed order by the last CTA of each tile to arrive (no float atomics, so
// results are reproducible run to run).
#include "effort_internal.cuh"

namespace effort {

constexpr int kChunkGroups = 16;                  // groups staged per chunk
constexpr int kChunkRecs = kChunkGroups * 32;     // per list

struct MacShared {
  float acc[kMacWarps][kTW];
  uint4 recD[kChunkRecs];
  uint4 recS[kChunkRecs];
  int offD[kChunkGroups + 1];
  int offS[kChunkGroups + 1];
  unsigned long long warp_cnt[kMacWarps];
  int is_last;
  int all_last;
};

__device__ __forceinline__ float sel_product(float av, unsigned short wbits, float c, bool vneg, bool& sel) {
  const float w = __half2float(__ushort_as_half(wbits));
  const float p = __fmul_rn(av, fabsf(w));
  sel = p >= c;
  return (vneg != (bool)(wbits >> 15)) ? -p : p;
}

template <int NJ>
__global__ void __launch_bounds__(kMacThreads) k_mac(const __grid_constant__ Jobs<NJ> jobs, int S) {
  __shared__ HandleDesc d;
  __shared__ MacShared sh;
  const Job& jb = jobs.j[blockIdx.y];
  if (threadIdx.x < (int)(sizeof(HandleDesc) / 4))
    reinterpret_cast<int*>(&d)[threadIdx.x] = reinterpret_cast<const int*>(jb.hd)[threadIdx.x];
  for (int k = threadIdx.x; k < kMacWarps * kTW; k += blockDim.x) (&sh.acc[0][0])[k] = 0.0f;
  __syncthreads();

  const int T = d.T, I = d.I, C = d.C, O = d.O;
  const int t = blockIdx.x % T, s = blockIdx.x / T;
  const int G = (I + kGroupRows - 1) / kGroupRows;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // wait for the cutoff/dispatch grid of this call (programmatic dependent launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const float c = *reinterpret_cast<volatile float*>(jb.ws.c);
  const bool count_all = (__float_as_uint(c) == 0u);  // c == 0: every kept product is used
  const bool want_rowlen = (jb.rowlen_out != nullptr) && !count_all;
  float a8[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) a8[m] = 0.0f;
  unsigned nsel = 0;
  float* myacc = sh.acc[warp];
  const uint16_t* wd_tile = d.wdense + (size_t)t * kTW + 8 * lane;

  const int nq = (G > s) ? (G - s + S - 1) / S : 0;  // groups of this slice
  for (int q0 = 0; q0 < nq; q0 += kChunkGroups) {
    const int ng = min(kChunkGroups, nq - q0);
    // offsets of this chunk's records
    if (warp == 0) {
      unsigned gc = 0;
      if (lane < ng) gc = jb.ws.gcnt[s + (size_t)(q0 + lane) * S];
      int ns = (int)(gc & 0xFFu), nd = (int)((gc >> 8) & 0xFFu);
      int is = ns, id = nd;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ys = __shfl_up_sync(0xFFFFFFFFu, is, o), yd = __shfl_up_sync(0xFFFFFFFFu, id, o);
        if (lane >= o) {
          is += ys;
          id += yd;
        }
      }
      if (lane < kChunkGroups) {
        sh.offS[lane + 1] = is;
        sh.offD[lane + 1] = id;
      }
      if (lane == 0) {
        sh.offS[0] = 0;
        sh.offD[0] = 0;
      }
    }
    __syncthreads();
    // stage the chunk's records; sparse records get their read bound U in .w
    {
      const int gq = threadIdx.x >> 4, slot = threadIdx.x & 15;  // 16 groups x 16 threads
      if (gq < ng) {
        const size_t g = s + (size_t)(q0 + gq) * S;
        const uint4* grec = jb.ws.rec + g * kRecPerGroup;
        const int nsq = sh.offS[gq + 1] - sh.offS[gq], ndq = sh.offD[gq + 1] - sh.offD[gq];
        for (int p = slot; p < ndq; p += 16) sh.recD[sh.offD[gq] + p] = grec[32 + p];
        for (int p = slot; p < nsq; p += 16) {
          uint4 r = grec[p];
          const int kk = min((int)r.z, C - 1);
          unsigned u = d.cnt[((size_t)r.x * C + kk) * T + t];
          r.w = (u == 255u) ? (unsigned)kCap : u;
          sh.recS[sh.offS[gq] + p] = r;
        }
      }
    }
    __syncthreads();
    const int ND = sh.offD[ng], NS = sh.offS[ng];

    // ---- dense rows: 4 rows per warp in flight, register accumulation
    for (int f = warp; f < ND; f += 4 * kMacWarps) {
      uint4 wv[4];
      uint4 rr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ff = f + u * kMacWarps;
        if (ff < ND) {
          rr[u] = sh.recD[ff];
          wv[u] = __ldg(reinterpret_cast<const uint4*>(wd_tile + (size_t)rr[u].x * d.dstride));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ff = f + u * kMacWarps;
        if (ff < ND) {
          const float vi = __uint_as_float(rr[u].y);
          const float av = fabsf(vi);
          const bool vneg = signbit(vi);
          const unsigned short* h = reinterpret_cast<const unsigned short*>(&wv[u]);
          unsigned rowsel = 0;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            bool sl;
            const float p = sel_product(av, h[m], c, vneg, sl);
            if (sl) {
              a8[m] += p;
              ++rowsel;
            }
          }
          nsel += rowsel;
          if (want_rowlen) {
            unsigned tot = rowsel;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xFFFFFFFFu, tot, o);
            if (lane == 0 && tot) atomicAdd(&jb.rowlen_out[rr[u].x], tot);
          }
        }
      }
    }

    // ---- sparse rows: 4 rows per warp in flight, 4 entries per lane per round
    for (int f = warp; f < NS; f += 4 * kMacWarps) {
      uint2 wv[4];
      unsigned ix[4];
      uint4 rr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ff = f + u * kMacWarps;
        rr[u] = make_uint4(0, 0, 0, 0);
        if (ff < NS) {
          rr[u] = sh.recS[ff];
          const size_t base = ((size_t)t * I + rr[u].x) * kCap + 4 * lane;
          if (4 * lane < (int)rr[u].w) {
            wv[u] = __ldg(reinterpret_cast<const uint2*>(d.vals + base));
            ix[u] = __ldg(reinterpret_cast<const unsigned*>(d.idx + base));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ff = f + u * kMacWarps;
        if (ff < NS) {
          const float vi = __uint_as_float(rr[u].y);
          const float av = fabsf(vi);
          const bool vneg = signbit(vi);
          const int U = (int)rr[u].w;
          const size_t rbase = ((size_t)t * I + rr[u].x) * kCap;
          unsigned rowsel = 0;
          for (int e0 = 0; e0 < U; e0 += 128) {
            const int e = e0 + 4 * lane;
            if (e < U) {
              uint2 w2;
              unsigned i4;
              if (e0 == 0) {
                w2 = wv[u];
                i4 = ix[u];
              } else {
                w2 = __ldg(reinterpret_cast<const uint2*>(d.vals + rbase + e));
                i4 = __ldg(reinterpret_cast<const unsigned*>(d.idx + rbase + e));
              }
              const unsigned short* h = reinterpret_cast<const unsigned short*>(&w2);
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                if (e + m < U) {
                  bool sl;
                  const float p = sel_product(av, h[m], c, vneg, sl);
                  if (sl) {
                    myacc[(i4 >> (8 * m)) & 255u] += p;
                    ++rowsel;
                  }
                }
              }
            }
          }
          nsel += rowsel;
          if (want_rowlen) {
            unsigned tot = rowsel;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xFFFFFFFFu, tot, o);
            if (lane == 0 && tot) atomicAdd(&jb.rowlen_out[rr[u].x], tot);
          }
          __syncwarp();
        }
      }
    }
    __syncthreads();  // records of the next chunk overwrite this chunk's
  }

  // fold the dense registers into this warp's copy, then sum the copies
#pragma unroll
  for (int m = 0; m < 8; ++m) myacc[8 * lane + m] += a8[m];
  unsigned long long wc = nsel;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wc += __shfl_xor_sync(0xFFFFFFFFu, wc, o);
  if (lane == 0) sh.warp_cnt[warp] = wc;
  __syncthreads();

  const int TWT = T * kTW;
  float tile_sum = 0.0f;
  if (threadIdx.x < kTW) {
#pragma unroll
    for (int w = 0; w < kMacWarps; ++w) tile_sum += sh.acc[w][threadIdx.x];
  }
  const int col = t * kTW + threadIdx.x;
  if (S == 1) {
    if (threadIdx.x < kTW && col < O) jb.out[col] = tile_sum;
  } else {
    if (threadIdx.x < kTW) jb.ws.part[(size_t)s * TWT + col] = tile_sum;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) sh.is_last = (atomicAdd(&jb.ws.tilecnt[t], 1u) == (unsigned)(S - 1));
    __syncthreads();
    if (sh.is_last) {
      __threadfence();
      if (threadIdx.x < kTW) {
        float sum = 0.0f;
        for (int ss = 0; ss < S; ++ss) sum += __ldcg(&jb.ws.part[(size_t)ss * TWT + col]);
        if (col < O) jb.out[col] = sum;
      }
      if (threadIdx.x == 0) jb.ws.tilecnt[t] = 0u;
    }
  }

  // used-product count: summed over CTAs; the last CTA publishes it
  if (threadIdx.x == 0) {
    unsigned long long bc = 0;
    for (int w = 0; w < kMacWarps; ++w) bc += sh.warp_cnt[w];
    if (!count_all && bc) atomicAdd(jb.ws.count, bc);
    __threadfence();
    const unsigned total_ctas = (unsigned)(T * S);
    sh.all_last = (atomicAdd(jb.ws.done, 1u) == total_ctas - 1u);
    if (sh.all_last) {
      __threadfence();
      const unsigned long long cnt = count_all ? d.kept_total : atomicAdd(jb.ws.count, 0ull);
      if (jb.count_out) jb.count_out[0] = cnt;
      jb.ws.done[0] = 0u;
    }
  }
}

template <int NJ>
cudaError_t launch_mac_t(const Jobs<NJ>& jobs, int njobs, int T, int S, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(T * S), (unsigned)njobs, 1);
  cfg.blockDim = dim3(kMacThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_mac<NJ>, jobs, S);
}

cudaError_t launch_mac(const Jobs<1>& jobs, int T, int S, cudaStream_t stream) {
  return launch_mac_t<1>(jobs, 1, T, S, stream);
}
cudaError_t launch_mac_batch(const Jobs<kMaxJobs>& jobs, int njobs, int T, int S, cudaStream_t stream) {
  return launch_mac_t<kMaxJobs>(jobs, njobs, T, S, stream);
}

int mac_ctas_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_mac<1>, kMacThreads, 0) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

}  // namespace effort
