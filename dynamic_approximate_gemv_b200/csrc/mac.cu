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
// Work split.  CTA (t, s) of a T x S grid owns output tile t and the 32-row
// groups [s*G/S, (s+1)*G/S).  It stages the dispatch records of its groups in
// shared memory (16 groups per round, one round of loads each), then streams
// the rows:
//   dense rows   the row's 256 weights of the tile come from the dense copy
//                and are accumulated in registers, 8 columns per lane, with a
//                predicated FMA;
//   sparse rows  the bucket's leading U entries (U from the dispatch's read
//                bound table) are cut into chunks of up to 64 entries; a ring
//                slot holds two chunks and each half-warp scatters one of them,
//                4 entries per lane, into its own shared copy of the tile.  The
//                entries of one bucket have distinct columns, so a half-warp
//                updates its copy with plain loads and stores; a __syncwarp
//                separates slots.
// Each warp streams its items through a ring of 512 B slots in shared memory
// filled with cp.async (16 B per lane), so several items per warp are in
// flight without holding registers.  At the end a CTA sums its warp copies and
// registers into one partial tile; the last of the S CTAs of a tile to arrive
// adds the partials in slice order (no float atomics: results are
// reproducible run to run).
#include "effort_internal.cuh"

namespace effort {

constexpr int kSlots = 6;
constexpr int kSlotBytes = 512;    // one dense tile-row, or two chunks (64 values + 64 columns each)
constexpr int kChunk = 64;         // bucket entries per sparse chunk
constexpr int kSegGroups = 16;     // groups staged per round
constexpr int kSegRecs = kSegGroups * 32;
constexpr int kMaxChunks = 1024;   // a round takes only the leading groups whose chunks fit
constexpr int kStagePairs = (kSegGroups * kRecPerGroup + kMacThreads - 1) / kMacThreads;

// Staged work.  dense rows: {first element of the row's tile in the dense
// copy, v bits, tau as float bits, row}; sparse chunks: {first entry of the
// chunk, v bits, tau as float bits, entries in the chunk | row << 8}.
struct MacSmem {
  float acc[kMacWarps][2][kTW];  // a shared copy of the tile per half-warp
  uint4 recD[kSegRecs];
  uint4 chunk[kMaxChunks];
  unsigned short nchk[kSegRecs];  // chunks of each staged sparse row, then their start
  int offD[kSegGroups + 1];
  int offS[kSegGroups + 1];
  unsigned warp_tot[kMacWarps];
  unsigned long long warp_cnt[kMacWarps];
  int nchunks;
  int ngroups;  // groups the round takes
  int flag;
  alignas(16) unsigned char ring[kMacWarps][kSlots][kSlotBytes];
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(gsrc) : "memory");
}
// copies `bytes` (0..16) and zero-fills the rest of the 16-byte destination
__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gsrc, unsigned bytes) {
  const unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(gsrc), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <int NJ, bool STATS>
__global__ void __launch_bounds__(kMacThreads, 2) k_mac(const __grid_constant__ Jobs<NJ> jobs, int S) {
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
  const int t = blockIdx.x % T, sl = blockIdx.x / T;
  const int gb = (int)((long long)G * sl / S), ge = (int)((long long)G * (sl + 1) / S);

  for (int k = threadIdx.x; k < kMacWarps * 2 * kTW; k += blockDim.x) (&sh.acc[0][0][0])[k] = 0.0f;

  // wait for this call's cutoff/dispatch grid (programmatic dependent launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const float c = *reinterpret_cast<volatile float*>(jb.ws.c);
  const bool count_all = (__float_as_uint(c) == 0u);
  const bool want_rowlen = STATS && rowlen_out != nullptr && !count_all;
  float a8[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) a8[m] = 0.0f;
  unsigned nsel = 0;
  unsigned char* ring = sh.ring[warp][0];

  {
    for (int q0 = gb; q0 < ge; q0 += sh.ngroups) {
      const int ng_load = min(kSegGroups, ge - q0);
      // ---- stage: one round of independent loads (counts, records, read bounds)
      uint4 r4[kStagePairs];
      unsigned u8v[kStagePairs];
#pragma unroll
      for (int z = 0; z < kStagePairs; ++z) {
        const int pr = threadIdx.x + z * kMacThreads;  // (group, slot) pair
        const int gq = pr >> 6, p = pr & 63;
        r4[z] = make_uint4(0, 0, 0, 0);
        u8v[z] = 0;
        if (gq < ng_load) {
          r4[z] = grec_all[(size_t)(q0 + gq) * kRecPerGroup + p];
          if (p < 32) u8v[z] = ut[((size_t)(q0 + gq) * T + t) * 32 + p];
        }
      }
      if (warp == 0) {
        unsigned gc = 0;
        if (lane < ng_load) gc = gcnt[q0 + lane];
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
      // dense rows go to their list; sparse rows note how many chunks they need
#pragma unroll
      for (int z = 0; z < kStagePairs; ++z) {
        const int pr = threadIdx.x + z * kMacThreads;
        const int gq = pr >> 6, p = pr & 63;
        if (gq < ng_load) {
          if (p < 32) {
            if (p < sh.offS[gq + 1] - sh.offS[gq]) {
              const unsigned U = (u8v[z] == 255u) ? (unsigned)kCap : u8v[z];
              sh.nchk[sh.offS[gq] + p] = (unsigned short)((U + kChunk - 1) / kChunk);
            }
          } else if (p - 32 < sh.offD[gq + 1] - sh.offD[gq]) {
            const uint4 r = r4[z];
            const float tau = __half2float(__ushort_as_half((unsigned short)r.z));
            sh.recD[sh.offD[gq] + p - 32] =
                make_uint4((unsigned)((size_t)r.x * dstride + (size_t)t * kTW), r.y, __float_as_uint(tau), r.x);
          }
        }
      }
      __syncthreads();
      const int NS = sh.offS[ng_load];
      {  // exclusive scan of the chunk counts (NS <= kSegRecs <= kMacThreads)
        unsigned x = (threadIdx.x < NS) ? sh.nchk[threadIdx.x] : 0u;
        unsigned incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) sh.warp_tot[warp] = incl;
        __syncthreads();
        unsigned before = 0;
        for (int w = 0; w < warp; ++w) before += sh.warp_tot[w];
        if (threadIdx.x < NS) sh.nchk[threadIdx.x] = (unsigned short)(before + incl - x);
        if (threadIdx.x == kMacThreads - 1) sh.nchunks = (int)(before + incl);
      }
      __syncthreads();
      if (threadIdx.x == 0) {  // the leading groups whose chunks fit the chunk list
        int take = ng_load, nc = sh.nchunks;
        while (nc > kMaxChunks) {
          --take;
          nc = (sh.offS[take] < NS) ? (int)sh.nchk[sh.offS[take]] : sh.nchunks;
        }
        sh.ngroups = take;
        sh.nchunks = nc;
      }
      __syncthreads();
      const int ng = sh.ngroups;
      // sparse rows: their chunks go to the chunk list
#pragma unroll
      for (int z = 0; z < kStagePairs; ++z) {
        const int pr = threadIdx.x + z * kMacThreads;
        const int gq = pr >> 6, p = pr & 63;
        if (gq < ng && p < 32 && p < sh.offS[gq + 1] - sh.offS[gq]) {
          const uint4 r = r4[z];
          const unsigned U = (u8v[z] == 255u) ? (unsigned)kCap : u8v[z];
          const float tau = __half2float(__ushort_as_half((unsigned short)r.z));
          const unsigned first = (unsigned)(((size_t)t * I + r.x) * kCap);
          int slot = sh.nchk[sh.offS[gq] + p];
          for (unsigned e0 = 0; e0 < U; e0 += kChunk, ++slot)
            sh.chunk[slot] = make_uint4(first + e0, r.y, __float_as_uint(tau), min(U - e0, (unsigned)kChunk) | (r.x << 8));
        }
      }
      __syncthreads();
      const int ND = sh.offD[ng];
      const int NC = sh.nchunks;
      const int NI = ND + (NC + 1) / 2;  // dense rows, then pairs of chunks
      // this warp's items: j = warp, warp + NW, ...
      const int nmine = (NI > warp) ? (NI - warp + kMacWarps - 1) / kMacWarps : 0;

      // A pair slot holds two chunks: values at [256 h, 256 h + 128), columns at
      // [256 h + 128, 256 h + 192).  Lanes 0..15 copy values (8 per chunk), lanes
      // 16..23 copy columns (4 per chunk); bytes past a chunk's length are
      // zero-filled, so those entries carry weight 0 and never pass tau > 0.
      const bool cp_val = lane < 16;
      const int cp_h = cp_val ? (lane >> 3) : ((lane - 16) >> 2);
      const int cp_k = cp_val ? (lane & 7) : ((lane - 16) & 3);
      const int cp_dst = 256 * cp_h + (cp_val ? 16 * cp_k : 128 + 16 * cp_k);
      auto issue = [&](int q) {  // the warp's q-th item into ring slot q % kSlots
        if (q < nmine) {
          const int j = warp + q * kMacWarps;
          unsigned char* slot = ring + (q % kSlots) * kSlotBytes;
          if (j < ND) {
            cp_async16(slot + 16 * lane, wdense + sh.recD[j].x + 8 * lane);
          } else if (lane < 24) {
            const int ch = 2 * (j - ND) + cp_h;
            const uint4 r = (ch < NC) ? sh.chunk[ch] : make_uint4(0, 0, 0, 0);
            const int len = (int)(r.w & 0xFFu);
            const int nb = cp_val ? 2 * len - 16 * cp_k : len - 16 * cp_k;
            const void* src = cp_val ? (const void*)(vals + r.x + 8 * cp_k) : (const void*)(idxs + r.x + 16 * cp_k);
            cp_async16_zfill(slot + cp_dst, src, (unsigned)max(0, min(16, nb)));
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
            const bool sel = fabsf(w) >= tau;
            a8[m] = sel ? fmaf(vi, w, a8[m]) : a8[m];
            if (STATS) rs += sel ? 1u : 0u;
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
          // half-warp h scatters chunk 2 (j - ND) + h, 4 entries per lane
          const int h = lane >> 4, hl = lane & 15;
          const int ch = 2 * (j - ND) + h;
          const uint4 r = (ch < NC) ? sh.chunk[ch] : make_uint4(0, 0, 0x7F800000u, 0);  // missing: tau = inf
          const float vi = __uint_as_float(r.y), tau = __uint_as_float(r.z);
          const uint2 w4 = *reinterpret_cast<const uint2*>(slot + 256 * h + 8 * hl);
          const unsigned c4 = *reinterpret_cast<const unsigned*>(slot + 256 * h + 128 + 4 * hl);
          const __half* hw = reinterpret_cast<const __half*>(&w4);
          float* acc = sh.acc[warp][h];
          unsigned rs = 0;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float w = __half2float(hw[m]);
            const bool sel = fabsf(w) >= tau;
            float* a = acc + ((c4 >> (8 * m)) & 255u);
            const float nv = fmaf(vi, w, *a);
            if (sel) *a = nv;
            if (STATS) rs += sel ? 1u : 0u;
          }
          if (STATS) {
            nsel += rs;
            if (want_rowlen) {
#pragma unroll
              for (int o = 8; o > 0; o >>= 1) rs += __shfl_xor_sync(0xFFFFFFFFu, rs, o);
              if (hl == 0 && rs) atomicAdd(&rowlen_out[r.w >> 8], rs);
            }
          }
        }
        __syncwarp();  // slot and tile copies are free for the next item
        issue(q + kSlots - 1);
      }
      cp_async_wait<0>();
      __syncthreads();  // the next round's staging overwrites this round's lists
    }

    // ---- leave tile t: one partial tile per CTA, summed in CTA order by the last to arrive
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      sh.acc[warp][0][8 * lane + m] += a8[m];
      a8[m] = 0.0f;
    }
    __syncthreads();
    float s = 0.0f;
    if (threadIdx.x < kTW) {
#pragma unroll
      for (int w = 0; w < kMacWarps; ++w) {
        s += sh.acc[w][0][threadIdx.x] + sh.acc[w][1][threadIdx.x];
        sh.acc[w][0][threadIdx.x] = 0.0f;
        sh.acc[w][1][threadIdx.x] = 0.0f;
      }
    }
    const int col = t * kTW + threadIdx.x;
    if (S == 1) {
      if (threadIdx.x < kTW && col < O) out[col] = s;
    } else {
      float* part = part_all + (size_t)t * S * kTW;
      if (threadIdx.x < kTW) part[(size_t)sl * kTW + threadIdx.x] = s;
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) sh.flag = (atomicAdd(&tilecnt[t], 1u) == (unsigned)(S - 1));
      __syncthreads();
      if (sh.flag) {
        __threadfence();
        if (threadIdx.x < kTW) {
          float tot = 0.0f;
          for (int k = 0; k < S; ++k) tot += __ldcg(&part[(size_t)k * kTW + threadIdx.x]);
          if (col < O) out[col] = tot;
        }
        if (threadIdx.x == 0) tilecnt[t] = 0u;
      }
    }
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
      if (atomicAdd(jb.ws.done, 1u) == (unsigned)(T * S - 1)) {
        __threadfence();
        const unsigned long long total = count_all ? kept_total : atomicAdd(jb.ws.count, 0ull);
        if (jb.count_out) jb.count_out[0] = total;
        jb.ws.done[0] = 0u;
      }
    }
  }
}

template <int NJ, bool STATS>
cudaError_t launch_mac_t(const Jobs<NJ>& jobs, int njobs, int T, int S, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(T * S), (unsigned)njobs, 1);
  cfg.blockDim = dim3(kMacThreads, 1, 1);
  cfg.dynamicSmemBytes = sizeof(MacSmem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_mac<NJ, STATS>, jobs, S);
}

bool jobs_want_stats(const Job* j, int n) {
  for (int k = 0; k < n; ++k)
    if (j[k].count_out || j[k].rowlen_out) return true;
  return false;
}

cudaError_t launch_mac(const Jobs<1>& jobs, int T, int S, cudaStream_t stream) {
  return jobs_want_stats(jobs.j, 1) ? launch_mac_t<1, true>(jobs, 1, T, S, stream)
                                    : launch_mac_t<1, false>(jobs, 1, T, S, stream);
}
cudaError_t launch_mac_batch(const Jobs<kMaxJobs>& jobs, int njobs, int T, int S, cudaStream_t stream) {
  return jobs_want_stats(jobs.j, njobs) ? launch_mac_t<kMaxJobs, true>(jobs, njobs, T, S, stream)
                                        : launch_mac_t<kMaxJobs, false>(jobs, njobs, T, S, stream);
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
