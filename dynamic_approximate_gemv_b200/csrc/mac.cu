// Multiply-accumulate: the multiply step of `approxMul` in the pages'
// pseudo-code (Hacker News item 40067677).  For every used pair the vector
// element v_i multiplies w_ij and the product is added into out_j (the
// CSR-style walk of the write-up quoted in that thread); the author's
// complexity reply (item 40095016) counts O(effort * inDim * outDim) such
// multiplications.
//
// Selection test.  For row i the dispatch computed tau_i, the smallest fp16
// magnitude m with fl32(|v_i| * m) >= c.  Because fl32(a * m) does not
// decrease as m grows, "|w| >= tau_i" holds exactly for the weights whose
// product passes the cutoff; the kernel compares magnitudes and never forms
// the compare product.
//
// Work split (stream-K style).  The units are (tile t, 32-row group g), tile
// major; CTA c of P takes units [c*TU/P, (c+1)*TU/P).  For each tile it
// touches, a CTA stages the dispatch records of its groups in shared memory
// with one round of loads, then streams the rows:
//   dense rows   the row's 256 weights of the tile come from the dense copy
//                and are accumulated in registers, 8 columns per lane, with a
//                predicated FMA;
//   sparse rows  the bucket's leading U entries (U from the dispatch's read
//                bound table) are scattered into a warp-private shared copy of
//                the tile.  One bucket's columns are distinct, so a warp updates
//                its copy with plain loads and stores; a __syncwarp separates
//                buckets.
// Each warp streams its rows through an 8-slot ring of 512 B in shared memory
// filled with cp.async (16 B per lane), so 7 rows per warp are in flight
// without holding registers.  When a CTA leaves a tile it sums its warp copies
// and registers into one partial tile; the last CTA to arrive at a tile adds
// the partials in CTA order (no float atomics: results are reproducible run to
// run).
#include "effort_internal.cuh"

namespace effort {

constexpr int kSlots = 8;
constexpr int kSlotBytes = 512;    // one dense tile-row, or 128 bucket entries + their columns
constexpr int kSparseStage = 128;  // bucket entries staged per sparse row
constexpr int kSegGroups = 24;     // groups staged per round
constexpr int kSegRecs = kSegGroups * 32;
constexpr int kStagePairs = (kSegGroups * kRecPerGroup + kMacThreads - 1) / kMacThreads;

// Staged records.  dense: {first element of the row's tile in the dense copy,
// v bits, tau as float bits, row}; sparse: {first bucket entry, v bits,
// tau as float bits, U}.
struct MacSmem {
  float acc[kMacWarps][kTW];
  uint4 recD[kSegRecs];
  uint4 recS[kSegRecs];
  int offD[kSegGroups + 1];
  int offS[kSegGroups + 1];
  unsigned long long warp_cnt[kMacWarps];
  int flag;
  alignas(16) unsigned char ring[kMacWarps][kSlots][kSlotBytes];
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// owner CTA of unit u when TU units are split evenly over P CTAs
__device__ __forceinline__ int unit_owner(long long u, long long TU, int P) {
  return (int)(((u + 1) * (long long)P - 1) / TU);
}

template <int NJ, bool STATS>
__global__ void __launch_bounds__(kMacThreads, 2) k_mac(const __grid_constant__ Jobs<NJ> jobs, int maxC) {
  extern __shared__ __align__(16) unsigned char dyn_smem[];
  MacSmem& sh = *reinterpret_cast<MacSmem*>(dyn_smem);
  const Job& jb = jobs.j[blockIdx.y];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // every field used below is read once from the parameter bank into registers
  const uint16_t* __restrict__ wdense = jb.hd.wdense;
  const uint16_t* __restrict__ vals = jb.hd.vals;
  const uint8_t* __restrict__ idxs = jb.hd.idx;
  const int dstride = jb.hd.dstride;
  const unsigned long long kept_total = jb.hd.kept_total;
  const unsigned* __restrict__ gcnt = jb.ws.gcnt;
  const uint4* __restrict__ grec_all = jb.ws.rec;
  const unsigned char* __restrict__ ut = jb.ws.ut;
  float* __restrict__ part_all = jb.ws.part;
  unsigned* tilecnt = jb.ws.tilecnt;
  unsigned* __restrict__ rowlen_out = jb.rowlen_out;
  float* __restrict__ out = jb.out;
  const int T = jb.hd.T, I = jb.hd.I, O = jb.hd.O;
  const int G = (I + kGroupRows - 1) / kGroupRows;
  const long long TU = (long long)T * G;
  const int P = gridDim.x, cta = blockIdx.x;
  const long long u0 = (long long)cta * TU / P, u1 = (long long)(cta + 1) * TU / P;

  for (int k = threadIdx.x; k < kMacWarps * kTW; k += blockDim.x) (&sh.acc[0][0])[k] = 0.0f;

  // wait for this call's cutoff/dispatch grid (programmatic dependent launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const float c = *reinterpret_cast<volatile float*>(jb.ws.c);
  const bool count_all = (__float_as_uint(c) == 0u);
  const bool want_rowlen = STATS && rowlen_out != nullptr && !count_all;
  float a8[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) a8[m] = 0.0f;
  unsigned nsel = 0;
  float* myacc = sh.acc[warp];
  unsigned char* ring = sh.ring[warp][0];

  for (int t = (int)(u0 / G); (long long)t * G < u1; ++t) {
    const int gb = (int)(max(u0, (long long)t * G) - (long long)t * G);
    const int ge = (int)(min(u1, (long long)(t + 1) * G) - (long long)t * G);

    for (int q0 = gb; q0 < ge; q0 += kSegGroups) {
      const int ng = min(kSegGroups, ge - q0);
      // ---- stage: one round of independent loads (counts, records, read bounds)
      uint4 r4[kStagePairs];
      unsigned u8v[kStagePairs];
#pragma unroll
      for (int z = 0; z < kStagePairs; ++z) {
        const int pr = threadIdx.x + z * kMacThreads;  // (group, slot) pair
        const int gq = pr >> 6, p = pr & 63;
        r4[z] = make_uint4(0, 0, 0, 0);
        u8v[z] = 0;
        if (gq < ng) {
          r4[z] = grec_all[(size_t)(q0 + gq) * kRecPerGroup + p];
          if (p < 32) u8v[z] = ut[((size_t)(q0 + gq) * T + t) * 32 + p];
        }
      }
      if (warp == 0) {
        unsigned gc = 0;
        if (lane < ng) gc = gcnt[q0 + lane];
        int is = (int)(gc & 0xFFu), id = (int)((gc >> 8) & 0xFFu);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int ys = __shfl_up_sync(0xFFFFFFFFu, is, o), yd = __shfl_up_sync(0xFFFFFFFFu, id, o);
          if (lane >= o) {
            is += ys;
            id += yd;
          }
        }
        if (lane < kSegGroups) {
          sh.offS[lane + 1] = is;
          sh.offD[lane + 1] = id;
        }
        if (lane == 0) sh.offS[0] = sh.offD[0] = 0;
      }
      __syncthreads();
#pragma unroll
      for (int z = 0; z < kStagePairs; ++z) {
        const int pr = threadIdx.x + z * kMacThreads;
        const int gq = pr >> 6, p = pr & 63;
        if (gq < ng) {
          const uint4 r = r4[z];
          const float tau = __half2float(__ushort_as_half((unsigned short)r.z));
          if (p < 32) {
            if (p < sh.offS[gq + 1] - sh.offS[gq]) {
              const unsigned U = (u8v[z] == 255u) ? (unsigned)kCap : u8v[z];
              sh.recS[sh.offS[gq] + p] =
                  make_uint4((unsigned)(((size_t)t * I + r.x) * kCap), r.y, __float_as_uint(tau), U);
            }
          } else if (p - 32 < sh.offD[gq + 1] - sh.offD[gq]) {
            sh.recD[sh.offD[gq] + p - 32] =
                make_uint4((unsigned)((size_t)r.x * dstride + (size_t)t * kTW), r.y, __float_as_uint(tau), r.x);
          }
        }
      }
      __syncthreads();
      const int ND = sh.offD[ng], NS = sh.offS[ng];
      const int NI = ND + NS;
      // this warp's items: j = warp, warp + NW, ...; j < ND dense, else sparse
      const int nmine = (NI > warp) ? (NI - warp + kMacWarps - 1) / kMacWarps : 0;

      auto issue = [&](int q) {  // the warp's q-th item into ring slot q % kSlots
        if (q < nmine) {
          const int j = warp + q * kMacWarps;
          unsigned char* slot = ring + (q % kSlots) * kSlotBytes;
          if (j < ND) {
            cp_async16(slot + 16 * lane, wdense + sh.recD[j].x + 8 * lane);
          } else {
            const uint4 r = sh.recS[j - ND];
            const unsigned U = min(r.w, (unsigned)kSparseStage);
            const unsigned nv = (U + 7u) >> 3, ni = (U + 15u) >> 4;
            // lanes 0..15 copy values, lanes 16..23 copy columns
            const bool is_v = lane < 16;
            const unsigned k = is_v ? (unsigned)lane : (unsigned)lane - 16u;
            if (k < (is_v ? nv : ni)) {
              if (is_v) cp_async16(slot + 16 * k, vals + r.x + 8 * k);
              else cp_async16(slot + 256 + 16 * k, idxs + r.x + 16 * k);
            }
          }
        }
        cp_async_commit();
      };

#pragma unroll
      for (int q = 0; q < kSlots - 1; ++q) issue(q);
      for (int q = 0; q < nmine; ++q) {
        cp_async_wait<kSlots - 2>();
        __syncwarp();
        const int j = warp + q * kMacWarps;
        const unsigned char* slot = ring + (q % kSlots) * kSlotBytes;
        if (j < ND) {
          const uint4 r = sh.recD[j];
          const float vi = __uint_as_float(r.y), tau = __uint_as_float(r.z);
          const uint4 wv = *reinterpret_cast<const uint4*>(slot + 16 * lane);
          const __half* h = reinterpret_cast<const __half*>(&wv);
          unsigned rs = 0;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float w = __half2float(h[m]);
            if (fabsf(w) >= tau) {
              a8[m] = fmaf(vi, w, a8[m]);
              if (STATS) ++rs;
            }
          }
          if (STATS) {
            nsel += rs;
            if (want_rowlen) {
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xFFFFFFFFu, rs, o);
              if (lane == 0 && rs) atomicAdd(&rowlen_out[r.w], rs);
            }
          }
        } else {
          const uint4 r = sh.recS[j - ND];
          const float vi = __uint_as_float(r.y), tau = __uint_as_float(r.z);
          const int U = (int)r.w;
          const __half* sv = reinterpret_cast<const __half*>(slot);
          const unsigned char* si = slot + 256;
          unsigned rs = 0;
#pragma unroll
          for (int m = 0; m < kSparseStage / 32; ++m) {
            const int e = lane + 32 * m;
            if (e < U) {
              const float w = __half2float(sv[e]);
              if (fabsf(w) >= tau) {
                const int col = si[e];
                myacc[col] = fmaf(vi, w, myacc[col]);
                if (STATS) ++rs;
              }
            }
          }
          if (U > kSparseStage) {  // long buckets: the rest straight from global memory
            for (int e = kSparseStage + lane; e < U; e += 32) {
              const float w = __half2float(__ushort_as_half(__ldg(vals + r.x + e)));
              if (fabsf(w) >= tau) {
                const int col = __ldg(idxs + r.x + e);
                myacc[col] = fmaf(vi, w, myacc[col]);
                if (STATS) ++rs;
              }
            }
          }
          if (STATS) {
            nsel += rs;
            if (want_rowlen) {
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xFFFFFFFFu, rs, o);
              if (lane == 0 && rs) atomicAdd(&rowlen_out[(r.x / kCap) % I], rs);
            }
          }
        }
        __syncwarp();  // slot and warp copy are free for the next item
        issue(q + kSlots - 1);
      }
      cp_async_wait<0>();
      __syncthreads();  // records of the next round overwrite this round's
    }

    // ---- leave tile t: one partial tile per CTA, summed in CTA order by the last to arrive
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      myacc[8 * lane + m] += a8[m];
      a8[m] = 0.0f;
    }
    __syncthreads();
    float s = 0.0f;
    if (threadIdx.x < kTW) {
#pragma unroll
      for (int w = 0; w < kMacWarps; ++w) {
        s += sh.acc[w][threadIdx.x];
        sh.acc[w][threadIdx.x] = 0.0f;
      }
    }
    const int cfirst = unit_owner((long long)t * G, TU, P);
    const int clast = unit_owner((long long)(t + 1) * G - 1, TU, P);
    const int ncontrib = clast - cfirst + 1;
    const int col = t * kTW + threadIdx.x;
    if (ncontrib == 1) {
      if (threadIdx.x < kTW && col < O) out[col] = s;
    } else {
      float* part = part_all + (size_t)t * maxC * kTW;
      if (threadIdx.x < kTW) part[(size_t)(cta - cfirst) * kTW + threadIdx.x] = s;
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) sh.flag = (atomicAdd(&tilecnt[t], 1u) == (unsigned)(ncontrib - 1));
      __syncthreads();
      if (sh.flag) {
        __threadfence();
        if (threadIdx.x < kTW) {
          float tot = 0.0f;
          for (int k = 0; k < ncontrib; ++k) tot += __ldcg(&part[(size_t)k * kTW + threadIdx.x]);
          if (col < O) out[col] = tot;
        }
        if (threadIdx.x == 0) tilecnt[t] = 0u;
      }
    }
    __syncthreads();
  }

  if (STATS) {  // used-product count, published by the last CTA of the call
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nsel += __shfl_xor_sync(0xFFFFFFFFu, nsel, o);
    if (lane == 0) sh.warp_cnt[warp] = nsel;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long bc = 0;
      for (int w = 0; w < kMacWarps; ++w) bc += sh.warp_cnt[w];
      if (!count_all && bc) atomicAdd(jb.ws.count, bc);
      __threadfence();
      if (atomicAdd(jb.ws.done, 1u) == (unsigned)(P - 1)) {
        __threadfence();
        const unsigned long long total = count_all ? kept_total : atomicAdd(jb.ws.count, 0ull);
        if (jb.count_out) jb.count_out[0] = total;
        jb.ws.done[0] = 0u;
      }
    }
  }
}

template <int NJ, bool STATS>
cudaError_t launch_mac_t(const Jobs<NJ>& jobs, int njobs, int P, int maxC, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P, (unsigned)njobs, 1);
  cfg.blockDim = dim3(kMacThreads, 1, 1);
  cfg.dynamicSmemBytes = sizeof(MacSmem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_mac<NJ, STATS>, jobs, maxC);
}

bool jobs_want_stats(const Job* j, int n) {
  for (int k = 0; k < n; ++k)
    if (j[k].count_out || j[k].rowlen_out) return true;
  return false;
}

cudaError_t launch_mac(const Jobs<1>& jobs, int P, int maxC, cudaStream_t stream) {
  return jobs_want_stats(jobs.j, 1) ? launch_mac_t<1, true>(jobs, 1, P, maxC, stream)
                                    : launch_mac_t<1, false>(jobs, 1, P, maxC, stream);
}
cudaError_t launch_mac_batch(const Jobs<kMaxJobs>& jobs, int njobs, int P, int maxC, cudaStream_t stream) {
  return jobs_want_stats(jobs.j, njobs) ? launch_mac_t<kMaxJobs, true>(jobs, njobs, P, maxC, stream)
                                        : launch_mac_t<kMaxJobs, false>(jobs, njobs, P, maxC, stream);
}

cudaError_t cutoff_attributes();
cudaError_t prep_attributes();

// One-time per-device setup of kernel attributes (not a stream operation).
cudaError_t init_kernel_attributes() {
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  const int smem = (int)sizeof(MacSmem);
  e = cudaFuncSetAttribute(k_mac<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_mac<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_mac<kMaxJobs, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_mac<kMaxJobs, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cutoff_attributes();
  if (e == cudaSuccess) e = prep_attributes();
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

int mac_ctas_per_sm() {
  int n = 0;
  if (init_kernel_attributes() != cudaSuccess) return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_mac<1, false>, kMacThreads, sizeof(MacSmem)) !=
      cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

}  // namespace effort
