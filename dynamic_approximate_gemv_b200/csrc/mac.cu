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
// product passes the cutoff; the kernel compares fp16 magnitudes (two per
// instruction) and never forms the compare product.
//
// Work split.  CTA (t, s) of a T x S grid owns output tile t and the 32-row
// groups [s*G/S, (s+1)*G/S).  It stages the dispatch records of up to 32
// groups per round in shared memory (one warp per group, two block barriers
// per round), then streams the rows:
//   dense rows   the row's 256 weights of the tile come from the dense copy
//                and are accumulated in registers, 8 columns per lane: a
//                packed magnitude mask zeroes the unused weights, then a
//                packed fp32 FMA adds v_i * w;
//   sparse rows  the bucket's leading U entries (U from the dispatch's read
//                bound table) are cut into chunks of up to 32 entries.  A work
//                item holds four chunks; each half-warp takes two of them in
//                turn, 2 entries per lane, and adds the selected products into
//                its own shared copy of the tile.  The entries of one bucket
//                have distinct columns, so a half-warp updates its copy with
//                plain loads and stores; a __syncwarp separates its chunks.
// Each warp loads a batch of items straight into registers (16 bytes per lane
// for a dense tile row, 4 + 2 bytes per lane for a chunk step), so several
// items per warp are in flight, then works through the batch.  At the end a
// CTA sums its warp copies and registers into
// one partial tile; the last of the S CTAs of a tile to arrive adds the
// partials in slice order (no float atomics: results are reproducible run to
// run).
#include "effort_internal.cuh"

namespace effort {

constexpr int kChunk = 32;          // bucket entries per sparse chunk
constexpr int kDenseBatch = 8;      // dense tile rows a warp has in flight
constexpr int kSparseBatch = 8;     // chunk steps a warp has in flight
constexpr int kRoundGroups = 32;    // groups staged per round
constexpr int kGroupsPerWarp = (kRoundGroups + kMacWarps - 1) / kMacWarps;
constexpr int kRoundRows = kRoundGroups * 32;
constexpr int kMaxChunks = 2048;    // a round takes only the leading groups whose chunks fit

// Staged work of one round:
//   dense row  {v bits, tau | row << 16}
//   chunk      {first entry, entries, v bits, tau | row << 16}; the list is
//              padded to whole items with empty chunks (no entries, tau = +inf)
struct MacSmem {
  float acc[kMacWarps][2][kTW];  // a shared copy of the tile per half-warp
  uint2 recD[kRoundRows];
  uint4 chunk[kMaxChunks];
  int gtot[2][kRoundGroups];     // per staged group: dense rows, chunks
  unsigned long long warp_cnt[kMacWarps];
  int flag;
};

// Streamed weights are read once per call: they bypass L1 and carry an L2
// evict-first policy so that they do not push the kernels' code, the dispatch
// records and the tables out of L2.
__device__ __forceinline__ unsigned long long evict_first_policy() {
  unsigned long long p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ld_stream_v4(const void* p, unsigned long long pol) {
  uint4 x;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
               : "l"(p), "l"(pol));
  return x;
}
__device__ __forceinline__ unsigned ld_stream_u32(const void* p, unsigned long long pol) {
  unsigned x;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u32 %0, [%1], %2;" : "=r"(x) : "l"(p), "l"(pol));
  return x;
}
__device__ __forceinline__ unsigned ld_stream_u16(const void* p, unsigned long long pol) {
  unsigned short x;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u16 %0, [%1], %2;" : "=h"(x) : "l"(p), "l"(pol));
  return x;
}
// mask with 0xFFFF in each half whose magnitude is >= tau (both halves hold tau)
__device__ __forceinline__ unsigned ge_mask(unsigned w2, unsigned tau2) {
  const unsigned mag = w2 & 0x7FFF7FFFu;
  return __hge2_mask(*reinterpret_cast<const __half2*>(&mag), *reinterpret_cast<const __half2*>(&tau2));
}


template <int NJ, bool STATS>
__global__ void __launch_bounds__(kMacThreads, kMacBlocksPerSM) k_mac(const __grid_constant__ Jobs<NJ> jobs, int S) {
  extern __shared__ __align__(16) unsigned char dyn_smem[];
  MacSmem& sh = *reinterpret_cast<MacSmem*>(dyn_smem);
  const Job& jb = jobs.j[NJ == 1 ? 0 : blockIdx.y];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // every field used below is read once from the parameter bank into registers
  const uint16_t* __restrict__ wdense = jb.hd.wdense;
  const uint16_t* __restrict__ vals = jb.hd.vals;
  const uint8_t* __restrict__ idxs = jb.hd.idx;
  const int dstride = jb.hd.dstride;
  const unsigned long long kept_total = jb.hd.kept_total;
  const unsigned* __restrict__ gcnt = jb.ws.gcnt;
  const uint2* __restrict__ grec_all = jb.ws.rec;
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
  // the next grid of the stream may launch once every CTA of this one is
  // resident (each has passed this point); it waits for this grid's completion
  // before touching what this grid reads or writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const float c = *reinterpret_cast<volatile float*>(jb.ws.c);
  const bool count_all = (__float_as_uint(c) == 0u);
  const bool want_rowlen = STATS && rowlen_out != nullptr && !count_all;
  float2 acc2[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc2[u] = make_float2(0.0f, 0.0f);
  unsigned nsel = 0;
  const unsigned long long pol = evict_first_policy();
  const int h = lane >> 4, hl = lane & 15;
  float* acc_h = sh.acc[warp][h];

  for (int q0 = gb; q0 < ge;) {
    const int ng_load = min(kRoundGroups, ge - q0);
    // ---- stage: warp w reads groups q0 + w, q0 + w + NW, ... (records, read
    // bounds and counts in one round of loads; records past a group's counts
    // are stale and ignored)
    uint2 rr[kGroupsPerWarp];
    unsigned uu[kGroupsPerWarp], gc[kGroupsPerWarp];
#pragma unroll
    for (int z = 0; z < kGroupsPerWarp; ++z) {
      const int gq = warp + kMacWarps * z;
      rr[z] = make_uint2(0, 0);
      uu[z] = gc[z] = 0;
      if (gq < ng_load) {
        const size_t g = (size_t)(q0 + gq);
        gc[z] = gcnt[g];
        rr[z] = grec_all[g * kRecPerGroup + lane];
        uu[z] = ut[(g * T + t) * 32 + lane];
      }
    }
    int nck[kGroupsPerWarp], cincl[kGroupsPerWarp];
#pragma unroll
    for (int z = 0; z < kGroupsPerWarp; ++z) {
      const int gq = warp + kMacWarps * z;
      const int ns = (int)(gc[z] & 0xFFu), nd = (int)((gc[z] >> 8) & 0xFFu);
      const unsigned U = (uu[z] == 255u) ? (unsigned)kCap : uu[z];
      nck[z] = (lane < ns) ? (int)((U + kChunk - 1) / kChunk) : 0;
      int x = nck[z];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
      }
      cincl[z] = x;
      if (lane == 31 && gq < ng_load) {
        sh.gtot[0][gq] = nd;
        sh.gtot[1][gq] = x;
      }
    }
    __syncthreads();
    // every warp: offsets of the staged groups, and how many leading groups
    // the round takes (their chunks must fit the chunk list)
    int od = (lane < ng_load) ? sh.gtot[0][lane] : 0;
    int oc = (lane < ng_load) ? sh.gtot[1][lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yd = __shfl_up_sync(0xFFFFFFFFu, od, o);
      const int yc = __shfl_up_sync(0xFFFFFFFFu, oc, o);
      if (lane >= o) {
        od += yd;
        oc += yc;
      }
    }
    const unsigned over = __ballot_sync(0xFFFFFFFFu, lane < ng_load && oc > kMaxChunks - 3);
    const int take = over ? (__ffs(over) - 1) : ng_load;  // >= 1: one group has at most 256 chunks
    const int ND = __shfl_sync(0xFFFFFFFFu, od, take - 1);
    const int NC0 = __shfl_sync(0xFFFFFFFFu, oc, take - 1);  // chunks of the taken groups
    const int NC = (NC0 + 3) & ~3;                            // padded to whole items
#pragma unroll
    for (int z = 0; z < kGroupsPerWarp; ++z) {
      const int gq = warp + kMacWarps * z;
      if (gq < take) {  // warp-uniform
        const int src = gq > 0 ? gq - 1 : 0;
        const int xd = __shfl_sync(0xFFFFFFFFu, od, src), xc = __shfl_sync(0xFFFFFFFFu, oc, src);
        const int offD = gq > 0 ? xd : 0, offC = gq > 0 ? xc : 0;
        const int ns = (int)(gc[z] & 0xFFu), nd = (int)((gc[z] >> 8) & 0xFFu);
        if (lane >= ns && lane < ns + nd) sh.recD[offD + lane - ns] = rr[z];
        if (lane < ns) {
          const unsigned U = (uu[z] == 255u) ? (unsigned)kCap : uu[z];
          const unsigned first = (unsigned)(((size_t)t * I + (rr[z].y >> 16)) * kCap);
          const int cpos = offC + cincl[z] - nck[z];
          for (int k = 0; k < nck[z]; ++k)
            sh.chunk[cpos + k] = make_uint4(first + (unsigned)(k * kChunk), min(U - (unsigned)(k * kChunk), (unsigned)kChunk),
                                            rr[z].x, rr[z].y);
        }
      }
    }
    if (threadIdx.x < NC - NC0) sh.chunk[NC0 + threadIdx.x] = make_uint4(0u, 0u, 0u, 0x7C00u);
    __syncthreads();
    // ---- dense rows: warp w takes rows j = w, w + NW, ... in batches, each
    // lane reading 16 bytes (8 columns) of every row's tile
    for (int j0 = warp; j0 < ND; j0 += kDenseBatch * kMacWarps) {
      uint4 wv[kDenseBatch];
      uint2 rd[kDenseBatch];
#pragma unroll
      for (int u = 0; u < kDenseBatch; ++u) {
        const int j = j0 + u * kMacWarps;
        rd[u] = make_uint2(0u, 0x7C00u);  // past the list: tau = +inf, nothing passes
        wv[u] = make_uint4(0u, 0u, 0u, 0u);
        if (j < ND) {
          rd[u] = sh.recD[j];
          wv[u] = ld_stream_v4(wdense + (size_t)(rd[u].y >> 16) * dstride + (size_t)t * kTW + 8 * lane, pol);
        }
      }
#pragma unroll
      for (int u = 0; u < kDenseBatch; ++u) {
        const float vi = __uint_as_float(rd[u].x);
        const unsigned tau2 = (rd[u].y & 0xFFFFu) * 0x10001u;
        const unsigned wr[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
        const float2 v2 = make_float2(vi, vi);
        unsigned rsel = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const unsigned m = ge_mask(wr[k], tau2);
          const unsigned wk = wr[k] & m;  // unused weights become +0
          acc2[k] = __ffma2_rn(v2, __half22float2(*reinterpret_cast<const __half2*>(&wk)), acc2[k]);
          if (STATS) rsel += (unsigned)__popc(m) >> 4;
        }
        if (STATS) {
          nsel += rsel;
          if (want_rowlen) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) rsel += __shfl_xor_sync(0xFFFFFFFFu, rsel, o);
            if (lane == 0 && rsel) atomicAdd(&rowlen_out[rd[u].y >> 16], rsel);
          }
        }
      }
    }
    // ---- sparse chunks: step s takes chunk 2s for half-warp 0 and 2s + 1 for
    // half-warp 1; each lane reads 2 entries (values and columns) of its chunk
    const int NS = NC / 2;
    for (int s0 = warp; s0 < NS; s0 += kSparseBatch * kMacWarps) {
      unsigned w2[kSparseBatch], ix[kSparseBatch];
      uint2 vr[kSparseBatch];  // {v bits, tau | row << 16}
#pragma unroll
      for (int u = 0; u < kSparseBatch; ++u) {
        const int st = s0 + u * kMacWarps;
        w2[u] = 0u;
        ix[u] = 0u;
        vr[u] = make_uint2(0u, 0x7C00u);
        if (st < NS) {
          const uint4 cr = sh.chunk[2 * st + h];  // {first entry, entries, v bits, tau | row << 16}
          vr[u] = make_uint2(cr.z, cr.w);
          // entries past the chunk are not read; the odd one that shares a
          // lane's 4 bytes lies past the read bound, so its |w| < tau
          if (2 * hl < (int)cr.y) {
            w2[u] = ld_stream_u32(vals + cr.x + 2 * hl, pol);
            ix[u] = ld_stream_u16(idxs + cr.x + 2 * hl, pol);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kSparseBatch; ++u) {
        const float vi = __uint_as_float(vr[u].x);
        const unsigned tau2 = (vr[u].y & 0xFFFFu) * 0x10001u;
        const unsigned m = ge_mask(w2[u], tau2);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w2[u]));
        if (m & 0xFFFFu) {
          float* a = acc_h + (ix[u] & 0xFFu);
          *a = fmaf(vi, f.x, *a);
        }
        if (m >> 16) {
          float* a = acc_h + (ix[u] >> 8);
          *a = fmaf(vi, f.y, *a);
        }
        if (STATS) {
          unsigned rsel = (unsigned)__popc(m) >> 4;
          nsel += rsel;
          if (want_rowlen) {
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) rsel += __shfl_xor_sync(0xFFFFFFFFu, rsel, o);
            if (hl == 0 && rsel) atomicAdd(&rowlen_out[vr[u].y >> 16], rsel);
          }
        }
        __syncwarp();  // the half-warp's next chunk may touch the same columns
      }
    }
    __syncthreads();  // the next round's staging overwrites this round's lists
    q0 += take;
  }

  // ---- leave tile t: one partial tile per CTA, summed in CTA order by the last to arrive
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    sh.acc[warp][0][8 * lane + 2 * u] += acc2[u].x;
    sh.acc[warp][0][8 * lane + 2 * u + 1] += acc2[u].y;
  }
  __syncthreads();
  float s = 0.0f;
  if (threadIdx.x < kTW) {
#pragma unroll
    for (int w = 0; w < kMacWarps; ++w) s += sh.acc[w][0][threadIdx.x] + sh.acc[w][1][threadIdx.x];
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
