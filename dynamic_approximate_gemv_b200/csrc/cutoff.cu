// Cutoff and dispatch: the `cutoff_chart = v * probes` and
// `cutoff = topK(cutoff_chart, effort)` steps of the pages' pseudo-code
// (Hacker News item 40067677), and the per-row dispatch whose cost the
// author's complexity reply (Hacker News item 40095016) puts at O(inDim).
//
// One thread-block cluster per job.  CTA r of the cluster owns rows
// [r * RP, (r + 1) * RP).
//   chart   x_ik = fl32(|v_i| * p_ik), kept in shared memory as fp32 bit
//           patterns (non-negative floats order like their bit patterns).
//   topK    c = max{x : sum of probe weights of chart entries >= x is >= K}.
//           Weighted radix select over the bit patterns.  The first digit
//           (bits 30..19) is chosen cluster-wide: CTA-local weighted
//           histograms are summed into per-CTA slices through distributed
//           shared memory, and every CTA reads the slices to find the
//           crossing bin.  Each CTA then lists its chart entries that fall in the
//           chosen bin, every CTA gathers all lists and finishes the select
//           locally (bits 18..9, then 8..0); all CTAs reach the same c.  If the
//           bin holds too many entries, the last two digits are also chosen
//           cluster-wide.
//   dispatch per row: the probes that pass c narrow the rank range of the
//           row's selection boundary; the checkpoint magnitudes inside that
//           range give k_i, the number of checkpoint blocks of H ranks that are
//           used entirely.  The row's exact fp16 threshold tau_i (smallest
//           magnitude whose product with |v_i| reaches c) turns the product
//           rule into a magnitude compare.  Rows with k_i * H >= f * n (f the
//           dense fraction, 0.2 by default) are "dense" (read from the dense
//           copy), other active rows are "sparse" (read from the sorted
//           buckets), rows whose largest product is below c are off.  Records
//           {v_i, tau_i, row} of a 32-row group are written sparse rows first,
//           then dense rows.
//
// Launch: programmatic, behind the preceding grid of the stream.  Before
// waiting on that grid the kernel touches only the prepared matrix (probes,
// checkpoint rows) and its shared memory; v, which that grid may produce, and
// the scratch, which an earlier call's multiply may still read, come after.
#include <cooperative_groups.h>

#include "effort_internal.cuh"

namespace cg = cooperative_groups;

namespace effort {

struct CutShared {
  unsigned warp_tot[32];
  unsigned sel_digit;
  unsigned sel_krem;
  unsigned ncand;       // this CTA's entries in the first-pass bin
  unsigned ncnt[16];    // every cluster CTA's ncand, stored here by that CTA
  unsigned cand_off[17];
  unsigned cand_total;
};

// Over a complete histogram of B digits (B a multiple of kCutThreads / 32 ...
// any B up to 4 * kCutThreads): D = max{d : weight of digits >= d reaches
// krem}, and the weight still needed inside digit D.  Two block barriers; the
// caller passes at least one more barrier before cs.sel_* or cs.warp_tot is
// written again.
template <int B>
__device__ void find_crossing(const unsigned* hist, unsigned krem, CutShared& cs, unsigned& digit, unsigned& knew) {
  constexpr int q = (B + kCutThreads - 1) / kCutThreads;  // digits per thread, highest digits first
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // thread j owns digits [B - q (j + 1), B - q j): thread 0 the highest
  const int hi = B - q * (int)threadIdx.x, lo = max(0, hi - q);
  unsigned local = 0;
#pragma unroll
  for (int u = 0; u < q; ++u)
    if (hi - 1 - u >= lo) local += hist[hi - 1 - u];
  // inclusive scan over threads in order (= descending digits)
  unsigned x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) cs.warp_tot[warp] = x;
  __syncthreads();
  // every warp scans the 32 warp totals itself (no second barrier)
  unsigned wt = cs.warp_tot[lane];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, wt, o);
    if (lane >= o) wt += y;
  }
  const unsigned before = __shfl_sync(0xFFFFFFFFu, wt, warp > 0 ? warp - 1 : 0) * (warp > 0 ? 1u : 0u);
  unsigned cum = before + x - local;  // weight of all digits above this thread's
  if (cum < krem && cum + local >= krem) {
    for (int d = hi - 1; d >= lo; --d) {
      const unsigned nb = hist[d];
      if (cum + nb >= krem) {
        cs.sel_digit = (unsigned)d;
        cs.sel_krem = krem - cum;
        break;
      }
      cum += nb;
    }
  }
  __syncthreads();
  digit = cs.sel_digit;
  knew = cs.sel_krem;
}

// Cluster-wide radix pass (used when the first-pass bin is crowded).
template <int B>
__device__ void cluster_radix_pass(cg::cluster_group& cluster, int cl, int crank, int shift, const unsigned* chart,
                                   int RP, int nr, const int* pw, unsigned* lh, unsigned* mg, unsigned& prefix,
                                   unsigned& pmask, unsigned& krem, CutShared& cs) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) lh[b] = 0u;
  __syncthreads();
  for (int k = 0; k < kP; ++k) {
    const int w = pw[k];
    if (w == 0) continue;
    for (int r = threadIdx.x; r < nr; r += blockDim.x) {
      const unsigned x = chart[(size_t)k * RP + r];
      if ((x & pmask) == prefix) atomicAdd(&lh[(x >> shift) & (B - 1)], (unsigned)w);
    }
  }
  __syncthreads();
  cluster.sync();
  const int per = B / cl;
  for (int b = threadIdx.x; b < per; b += blockDim.x) {
    const int bin = crank * per + b;
    unsigned s = 0;
    for (int r = 0; r < cl; ++r) s += cluster.map_shared_rank(lh, r)[bin];
    for (int r = 0; r < cl; ++r) cluster.map_shared_rank(mg, r)[bin] = s;
  }
  cluster.sync();
  unsigned digit, knew;
  find_crossing<B>(mg, krem, cs, digit, knew);
  prefix |= digit << shift;
  pmask |= (unsigned)(B - 1) << shift;
  krem = knew;
}

// Local radix pass over gathered (value, weight) candidates.  `hist` (B bins)
// was zeroed before the last block barrier.
template <int B>
__device__ void local_radix_pass(int shift, const unsigned* val, const unsigned short* wt, int n, unsigned* hist,
                                 unsigned& prefix, unsigned& pmask, unsigned& krem, CutShared& cs) {
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const unsigned x = val[e];
    if ((x & pmask) == prefix) atomicAdd(&hist[(x >> shift) & (B - 1)], (unsigned)wt[e]);
  }
  __syncthreads();
  unsigned digit, knew;
  find_crossing<B>(hist, krem, cs, digit, knew);
  prefix |= digit << shift;
  pmask |= (unsigned)(B - 1) << shift;
  krem = knew;
}

template <int NJ>
__global__ void __launch_bounds__(kCutThreads, 1) k_cutoff_dispatch(const __grid_constant__ Jobs<NJ> jobs, int cl) {
  // let the multiply kernel of this call get onto the idle SMs early; it waits
  // for this grid's completion before touching anything written here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const Job& jb = jobs.j[blockIdx.x / cl];
  __shared__ CutShared cs;
  __shared__ int s_prank[kP], s_pw[kP];
  // every field used below is read once from the parameter bank into registers
  const int I = jb.hd.I, n = jb.hd.n, C = jb.hd.C, H = jb.hd.H;
  const uint16_t* __restrict__ ckmag = jb.hd.ckmag;
  const uint16_t* __restrict__ probes = jb.hd.probes;
  const void* vptr = jb.v;
  const int vdtype = jb.vdtype, dense_q16 = jb.dense_q16;
  unsigned* __restrict__ status = jb.ws.status;
  uint2* __restrict__ rec = jb.ws.rec;
  unsigned* __restrict__ gcnt = jb.ws.gcnt;
  unsigned char* __restrict__ ut = jb.ws.ut;
  const uint8_t* __restrict__ cntt = jb.hd.cnt;
  const int T = jb.hd.T;
  unsigned* __restrict__ rowlen_out = jb.rowlen_out;
  const unsigned Kt = (unsigned)jb.K;
  if (threadIdx.x < kP) {
    s_prank[threadIdx.x] = jb.hd.prank[threadIdx.x];
    s_pw[threadIdx.x] = jb.hd.pw[threadIdx.x];
  }
  const int RP = cut_rows_per_cta(I, cl);
  const int i0 = crank * RP;
  const int nr = max(0, min(I, i0 + RP) - i0);
  const int G = (I + kGroupRows - 1) / kGroupRows;

  extern __shared__ __align__(16) unsigned smem[];
  unsigned* chart = smem;                                                    // [kP][RP], column k at k * RP
  float* vs = reinterpret_cast<float*>(chart + (size_t)RP * kP);             // RP
  unsigned* h0 = reinterpret_cast<unsigned*>(vs + RP);                       // kBins0
  unsigned* cval = h0 + kBins0;                                              // kCandLocal
  unsigned short* cwt = reinterpret_cast<unsigned short*>(cval + kCandLocal);  // kCandLocal
  unsigned* uni = reinterpret_cast<unsigned*>(cwt + kCandLocal);             // shared area
  unsigned* mg0 = uni;                                                       // merged first-pass histogram
  unsigned* gval = uni;                                                      // gathered candidates
  unsigned short* gwt = reinterpret_cast<unsigned short*>(uni + kCandTotal);
  unsigned* h1 = uni;                                                        // fallback passes
  unsigned* m1 = h1 + kBins1;
  unsigned* h2 = m1 + kBins1;
  unsigned* m2 = h2 + kBins2;

  int mode = jb.mode;
  if (threadIdx.x == 0) cs.ncand = 0u;
  // the first-pass histogram and this CTA's merged slice, zeroed first: the
  // block barrier after the chart orders the histogram's zeroing before its
  // atomics, the split cluster barrier below orders the slice's zeroing
  // before other CTAs add into it
  const int per = kBins0 / cl;
  unsigned* own = mg0;  // this CTA's merged slice lives at the start of the shared area
  if (mode == kModeSelect) {
    for (int b = threadIdx.x; b < kBins0; b += blockDim.x) h0[b] = 0u;
    for (int b = threadIdx.x; b < per; b += blockDim.x) own[b] = 0u;
    // split cluster barrier: arrive now (this CTA's slice is zeroed), wait
    // just before the first remote atomic into another CTA's slice
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
  }
  // ---- before the preceding grid of the stream has completed: only the
  // prepared matrix (never written by a call) and shared memory are touched.
  // The probes go into the chart area as floats; the rows' checkpoint
  // magnitudes are prefetched into L2 for the dispatch.
  for (int r = threadIdx.x; r < nr; r += blockDim.x) {
    const int i = i0 + r;
    if (mode == kModeSelect) {
      const uint4 p0 = reinterpret_cast<const uint4*>(probes + (size_t)i * kP)[0];
      const uint4 p1 = reinterpret_cast<const uint4*>(probes + (size_t)i * kP)[1];
      const unsigned short* ph0 = reinterpret_cast<const unsigned short*>(&p0);
      const unsigned short* ph1 = reinterpret_cast<const unsigned short*>(&p1);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        chart[(size_t)k * RP + r] = __float_as_uint(__half2float(__ushort_as_half(ph0[k])));
        chart[(size_t)(8 + k) * RP + r] = __float_as_uint(__half2float(__ushort_as_half(ph1[k])));
      }
    }
    const char* ck = reinterpret_cast<const char*>(ckmag + (size_t)i * (C + 1));
    for (int b = 0; b < (C + 1) * 2; b += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(ck + b));
  }
  // the preceding grid may produce v and may still read this call's scratch:
  // everything below comes after its completion
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // ---- v, and the chart x_ik = fl32(|v_i| * p_ik) (each thread rescales the
  // probes of its own rows in place)
  bool bad = false;
  for (int r = threadIdx.x; r < nr; r += blockDim.x) {
    const int i = i0 + r;
    const float x = (vdtype == 1) ? __half2float(reinterpret_cast<const __half*>(vptr)[i])
                                  : reinterpret_cast<const float*>(vptr)[i];
    if (!isfinite(x)) bad = true;
    vs[r] = x;
    if (mode == kModeSelect) {
      const float av = fabsf(x);
#pragma unroll
      for (int k = 0; k < kP; ++k)
        chart[(size_t)k * RP + r] = __float_as_uint(__fmul_rn(av, __uint_as_float(chart[(size_t)k * RP + r])));
    }
  }
  if (bad) atomicOr(status, kStatusNonfiniteV);
  __syncthreads();

  unsigned prefix = 0u, pmask = 0u;
  unsigned krem = Kt;
  bool split_exit = false;  // cluster barrier arrived early, to be waited on at exit
  if (mode == kModeSelect) {
    // ---- first digit, cluster-wide.  Local weighted histogram; its nonzero
    // bins are added into the owner CTA's slice (bin / (kBins0 / cl)) with
    // distributed shared memory atomics; after one cluster barrier each thread
    // reads its four bins of the merged histogram from their owner's slice.
    // chart entry e = k * RP + r (column-major); k from a float reciprocal,
    // exact for e < 2^16 and RP <= 2^12
    const int ne = kP * RP;
    const float rcp_rp = 1.0f / (float)RP;
    for (int e = threadIdx.x; e < ne; e += blockDim.x) {
      const int k = __float2int_rd(((float)e + 0.5f) * rcp_rp);
      const int r = e - k * RP;
      const int wk = s_pw[k];
      if (r < nr && wk > 0) atomicAdd(&h0[(chart[e] >> 19) & (kBins0 - 1)], (unsigned)wk);
    }
    __syncthreads();  // the local histogram is complete
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");  // every CTA's slice is zeroed
    for (int b = threadIdx.x; b < kBins0; b += blockDim.x) {
      const unsigned x = h0[b];
      if (x) atomicAdd(cluster.map_shared_rank(own, b / per) + (b % per), x);
    }
    cluster.sync();  // merged slices complete
    {
      // The crossing of the merged histogram, read straight from the owners'
      // slices: thread j owns digits [kBins0 - 4 (j + 1), kBins0 - 4 j) (thread
      // 0 the highest), four adjacent bins of one slice fetched with one
      // 16-byte remote load and scanned in registers.
      static_assert(kBins0 == 4 * kCutThreads, "four first-digit bins per thread");
      const int ln = threadIdx.x & 31, wp = threadIdx.x >> 5;
      const int hi = kBins0 - 4 * (int)threadIdx.x, b0 = hi - 4;
      const uint4 q = *reinterpret_cast<const uint4*>(cluster.map_shared_rank(own, b0 / per) + (b0 % per));
      const unsigned local = q.x + q.y + q.z + q.w;
      unsigned x = local;  // inclusive scan over threads in order (= descending digits)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (ln >= o) x += y;
      }
      if (ln == 31) cs.warp_tot[wp] = x;
      __syncthreads();
      unsigned wt = cs.warp_tot[ln];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xFFFFFFFFu, wt, o);
        if (ln >= o) wt += y;
      }
      const unsigned before = __shfl_sync(0xFFFFFFFFu, wt, wp > 0 ? wp - 1 : 0) * (wp > 0 ? 1u : 0u);
      unsigned cum = before + x - local;  // weight of all digits above this thread's
      if (cum < Kt && cum + local >= Kt) {
        const unsigned hv[4] = {q.w, q.z, q.y, q.x};  // digits hi - 1 ... hi - 4
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (cum + hv[u] >= Kt) {
            cs.sel_digit = (unsigned)(hi - 1 - u);
            cs.sel_krem = Kt - cum;
            break;
          }
          cum += hv[u];
        }
      }
      __syncthreads();
    }
    prefix = cs.sel_digit << 19;
    pmask = (unsigned)(kBins0 - 1) << 19;
    krem = cs.sel_krem;
    // the local passes' histograms (h0 is free since the merge barrier)
    static_assert(kBins1 + kBins2 <= kBins0, "local-pass histograms fit the first-pass one");
    for (int b = threadIdx.x; b < kBins1 + kBins2; b += blockDim.x) h0[b] = 0u;
    // ---- this CTA's entries in the chosen bin (one atomic per warp)
    for (int e = threadIdx.x; e < ne; e += blockDim.x) {
      const int k = __float2int_rd(((float)e + 0.5f) * rcp_rp);
      const int r = e - k * RP;
      const int wk = s_pw[k];
      const unsigned x = chart[e];
      const bool in = r < nr && wk > 0 && (x & pmask) == prefix;
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, in);
      if (bal) {
        const int ln = threadIdx.x & 31;
        unsigned base = 0;
        if (ln == 0) base = atomicAdd(&cs.ncand, (unsigned)__popc(bal));
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        const unsigned slot = base + (unsigned)__popc(bal & ((1u << ln) - 1u));
        if (in && slot < (unsigned)kCandLocal) {
          cval[slot] = x;
          cwt[slot] = (unsigned short)wk;
        }
      }
    }
    __syncthreads();
    // this CTA's list length into every CTA's table (the barrier below
    // publishes it), so that no CTA reads the lengths remotely afterwards
    if ((int)threadIdx.x < cl) *cluster.map_shared_rank(&cs.ncnt[crank], (int)threadIdx.x) = cs.ncand;
    cluster.sync();  // every list complete; no CTA reads another's merged slice any more
    if (threadIdx.x < 32) {  // the cl list lengths and their offsets
      const int ln = threadIdx.x;
      const unsigned nc = (ln < cl) ? cs.ncnt[ln] : 0u;
      const bool over = __any_sync(0xFFFFFFFFu, nc > (unsigned)kCandLocal);
      unsigned incl = nc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (ln >= o) incl += y;
      }
      if (ln < cl) cs.cand_off[ln + 1] = incl;
      if (ln == 0) cs.cand_off[0] = 0u;
      if (ln == 31) cs.cand_total = over ? 0xFFFFFFFFu : incl;
    }
    __syncthreads();
    const unsigned total = cs.cand_total;
    if (total <= (unsigned)kCandTotal) {
      // gather every CTA's list and finish locally (same multiset, same c everywhere)
      for (unsigned q0 = 0; q0 < total; q0 += 4u * kCutThreads) {
        unsigned v4[4];
        unsigned short w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // issue the remote loads of four candidates together
          const unsigned q = q0 + threadIdx.x + (unsigned)u * kCutThreads;
          v4[u] = 0u;
          w4[u] = 0;
          if (q < total) {
            int r = 0;
            while (q >= cs.cand_off[r + 1]) ++r;
            const unsigned k = q - cs.cand_off[r];
            v4[u] = cluster.map_shared_rank(cval, r)[k];
            w4[u] = cluster.map_shared_rank(cwt, r)[k];
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const unsigned q = q0 + threadIdx.x + (unsigned)u * kCutThreads;
          if (q < total) {
            gval[q] = v4[u];
            gwt[q] = w4[u];
          }
        }
      }
      asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
      split_exit = true;
      __syncthreads();
      local_radix_pass<kBins1>(9, gval, gwt, (int)total, h0, prefix, pmask, krem, cs);
      local_radix_pass<kBins2>(0, gval, gwt, (int)total, h0 + kBins1, prefix, pmask, krem, cs);
    } else {
      cluster_radix_pass<kBins1>(cluster, cl, crank, 9, chart, RP, nr, s_pw, h1, m1, prefix, pmask, krem, cs);
      cluster_radix_pass<kBins2>(cluster, cl, crank, 0, chart, RP, nr, s_pw, h2, m2, prefix, pmask, krem, cs);
    }
  }
  const float c = (mode == kModeAll) ? 0.0f : (mode == kModeNone) ? __int_as_float(0x7F800000) : __uint_as_float(prefix);
  const unsigned cbits = __float_as_uint(c);
  if (mode == kModeSelect && cbits == 0u) mode = kModeAll;  // every kept product passes c = 0

  if (crank == 0 && threadIdx.x == 0) {
    jb.ws.c[0] = c;
    jb.ws.count[0] = 0ull;
    if (jb.cutoff_out) jb.cutoff_out[0] = c;
  }

  // ---- dispatch: one thread per row; a warp covers one 32-row group
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < RP; base += blockDim.x) {
    const int r = base + threadIdx.x;
    const int i = i0 + r;
    const bool valid = r < nr;
    int cls = kClassOff, ki = 0;
    unsigned tau = 0x7C00u;
    float vi = 0.0f;
    if (valid) {
      vi = vs[r];
      if (mode == kModeAll) {
        cls = kClassDense;
        ki = C;
        tau = 0u;
      } else if (mode == kModeSelect) {
        const float av = fabsf(vi);
        // tau: the smallest fp16 magnitude m with fl32(|v_i| * m) >= c (0x7C00 if
        // none); fl32(|v_i| * m) is non-decreasing in m, so |w| >= tau <=> used.
        // Start from the fp16 rounding of c / |v_i| and settle it with exact
        // product tests; a bisection over all magnitudes covers the rest.
        const float q = __fdividef(c, av);  // a guess only (inf when av == 0; c > 0 here)
        unsigned lo = 0u, hi = 0x7C00u;
        if (q < 65504.0f) {
          const unsigned g = (unsigned)__half_as_ushort(__float2half_rd(q)) & 0x7FFFu;
          const unsigned a = g > 2u ? g - 2u : 0u, b = min(g + 3u, 0x7C00u);
          // [a, b) brackets the answer when the guess is within two ulps
          const bool a_fails = (a == 0u) || (__fmul_rn(av, __half2float(__ushort_as_half((unsigned short)(a - 1u)))) < c);
          const bool b_passes = (b == 0x7C00u) || (__fmul_rn(av, __half2float(__ushort_as_half((unsigned short)b))) >= c);
          if (a_fails && b_passes) {
            lo = a;
            hi = b;
          }
        }
        while (lo < hi) {
          const unsigned mid = (lo + hi) >> 1;
          if (__fmul_rn(av, __half2float(__ushort_as_half((unsigned short)mid))) >= c) hi = mid;
          else lo = mid + 1u;
        }
        tau = lo;
        // probes narrow the rank range of the row's boundary
        int last_sel = -1, first_unsel = n;
#pragma unroll
        for (int k = 0; k < kP; ++k) {
          const int rk = s_prank[k];
          if (rk < 0) continue;
          if (chart[(size_t)k * RP + r] >= cbits) last_sel = rk;
          else if (first_unsel == n) first_unsel = rk;
        }
        const int known = min(C, (last_sel + 1) / H);
        const int kend = (first_unsel >= n) ? C : min(C - 1, (first_unsel + 1 + H - 1) / H - 1);
        ki = known;
        const uint16_t* ck = ckmag + (size_t)i * (C + 1);
        // checkpoints in the window, loaded together; the used ones lead the window
        for (int k0 = known; k0 < kend; k0 += 16) {
          unsigned short m[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) m[u] = (k0 + u < kend) ? ck[1 + k0 + u] : (unsigned short)0;
          int cnt = 0;
#pragma unroll
          for (int u = 0; u < 16; ++u) cnt += (k0 + u < kend && (unsigned)m[u] >= tau) ? 1 : 0;
          ki += cnt;
          if (cnt < 16) break;
        }
        const bool active = (ki > 0) || (last_sel >= 0) || ((unsigned)ck[0] >= tau);
        if (active)
          cls = ((long long)ki * H * 65536 >= (long long)n * dense_q16) ? kClassDense : kClassSparse;
      }
      if (rowlen_out) rowlen_out[i] = (mode == kModeAll) ? (unsigned)n : 0u;
    }
    const unsigned bs = __ballot_sync(0xFFFFFFFFu, cls == kClassSparse);
    const unsigned bd = __ballot_sync(0xFFFFFFFFu, cls == kClassDense);
    const int g = (i0 + base) / kGroupRows + warp;
    // a group is written only by the CTA whose row range holds it
    if (base + warp * kGroupRows < RP && g < G) {
      const unsigned lt = (1u << lane) - 1u;
      const uint2 r2 = make_uint2(__float_as_uint(vi), (tau & 0xFFFFu) | ((unsigned)i << 16));
      if (cls == kClassSparse) rec[(size_t)g * kRecPerGroup + __popc(bs & lt)] = r2;
      if (cls == kClassDense) rec[(size_t)g * kRecPerGroup + __popc(bs) + __popc(bd & lt)] = r2;
      if (lane == 0) gcnt[g] = (unsigned)__popc(bs) | ((unsigned)__popc(bd) << 8);
      // read bounds of the group's sparse rows in every tile: entries of the tile
      // among the first min((k+1) H, n) ranks (255 saturates: read the whole
      // bucket).  Each lane loads its row's count row in one batch of 4-byte
      // loads; then, tile by tile, the 32 lanes store one contiguous 32-byte
      // line ut[g][t][0..31] (lane = sparse slot).
      const int p = __popc(bs & lt);
      const bool sp = cls == kClassSparse;
      const uint8_t* crow = cntt + ((size_t)i * C + min(ki, C - 1)) * T;
      unsigned char* ug = ut + (size_t)g * T * 32;
      for (int t0 = 0; t0 < T; t0 += 32) {
        unsigned w[8];
        const int nt = min(32, T - t0);
        if ((T & 3) == 0) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            w[u] = (sp && 4 * u < nt) ? *reinterpret_cast<const unsigned*>(crow + t0 + 4 * u) : 0u;
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            unsigned x = 0u;
#pragma unroll
            for (int b = 0; b < 4; ++b)
              if (sp && 4 * u + b < nt) x |= (unsigned)crow[t0 + 4 * u + b] << (8 * b);
            w[u] = x;
          }
        }
        // lane p's byte for tile t goes to ug[t * 32 + p]; lanes of unused slots
        // leave their byte untouched
#pragma unroll
        for (int tt = 0; tt < 32; ++tt) {
          if (tt < nt && sp) ug[(size_t)(t0 + tt) * 32 + p] = (unsigned char)((w[tt >> 2] >> (8 * (tt & 3))) & 0xFFu);
        }
      }
    }
  }
  // other CTAs may still be reading this CTA's candidate list
  if (split_exit) asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Largest dynamic shared memory a cutoff CTA may use on this device: the
// opt-in limit minus the kernel's static shared memory.
size_t cutoff_max_dynamic_smem() {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
  cudaFuncAttributes fa1, fa16;
  if (cudaFuncGetAttributes(&fa1, k_cutoff_dispatch<1>) != cudaSuccess) return 0;
  if (cudaFuncGetAttributes(&fa16, k_cutoff_dispatch<kMaxJobs>) != cudaSuccess) return 0;
  const size_t st = fa1.sharedSizeBytes > fa16.sharedSizeBytes ? fa1.sharedSizeBytes : fa16.sharedSizeBytes;
  return (size_t)optin > st ? (size_t)optin - st : 0;
}

// Kernel attributes are set once per device (outside any stream capture):
// the largest dynamic shared memory the chart may need and 16-CTA clusters.
cudaError_t cutoff_attributes() {
  const int dyn = (int)cutoff_max_dynamic_smem();
  if (dyn <= 0) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_cutoff_dispatch<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_cutoff_dispatch<kMaxJobs>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_cutoff_dispatch<1>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_cutoff_dispatch<kMaxJobs>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

// How many clusters of `cl` CTAs with `smem` bytes each the device can hold
// at once (0: this cluster shape cannot be launched here).
int cutoff_max_clusters(int cl, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cl, 1, 1);
  cfg.blockDim = dim3(kCutThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_cutoff_dispatch<1>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int NJ>
cudaError_t launch_cutoff_t(const Jobs<NJ>& jobs, int njobs, int I, int cl, cudaStream_t stream) {
  const size_t smem = cut_smem_bytes(I, cl);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(cl * njobs), 1, 1);
  cfg.blockDim = dim3(kCutThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // may start once the preceding grid allows it (the multiply of an earlier
  // call does so as soon as all its CTAs run); the kernel waits for that
  // grid's completion before it reads v or touches the scratch
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_cutoff_dispatch<NJ>, jobs, cl);
}

cudaError_t launch_cutoff(const Jobs<1>& jobs, int I, int cl, cudaStream_t stream) {
  return launch_cutoff_t<1>(jobs, 1, I, cl, stream);
}
cudaError_t launch_cutoff_batch(const Jobs<kMaxJobs>& jobs, int njobs, int I, int cl, cudaStream_t stream) {
  return launch_cutoff_t<kMaxJobs>(jobs, njobs, I, cl, stream);
}

}  // namespace effort
