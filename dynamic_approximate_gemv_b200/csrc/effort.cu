// One approximate matvec in one kernel: the `approxMul` step of the pages'
// pseudo-code (Hacker News item 40067677, "Show HN: Speeding up LLM inference
// 2x times (possibly)": cutoff_chart = v * probes, cutoff = topK(chart,
// effort), then the multiply over the leading part of every sorted row), with
// the cost split the author gives in Hacker News item 40095016 (about
// O(inDim log inDim) for the cutoff, O(inDim) for the dispatch,
// O(effort inDim outDim) multiplications).
//
// Grid: one block of 1024 threads per SM, all resident at once; the blocks
// meet at two grid-wide barriers (a monotonic 64-bit counter in the scratch,
// polled with a time limit; on timeout the kernel sets a status bit and
// returns).
//
//   Cutoff (rows a2).  Block b owns rows [b rp, b rp + rp) of the chart
//   x_ik = fl32(|v_i| p_ik).  The chart's fp32 patterns are non-negative and
//   order like unsigned integers, so c is found by a weighted radix select:
//   every block adds its entries' probe weights into a global histogram of
//   bits [30:19] (barrier B1), every block finds the bin where the weight
//   counted from the top reaches K, lists its entries of that bin (barrier
//   B2), and every block resolves bits [18:0] over the gathered candidates in
//   shared memory.  With more candidates than fit, two more grid-wide
//   histogram passes resolve the other digits.
//
//   Dispatch (row a3).  Between B1 and B2 every block knows that c lies in
//   the crossing bin [lo, hi).  For its rows and every output panel it
//   computes tau_i(lo), the smallest fp16 magnitude m with fl32(|v_i| m) >=
//   lo, the number of stored chunks whose first magnitude reaches it, and the
//   bytes the (row, panel) will cost: the row's stripes of the dense copy
//   when the stored part of the list does not reach tau (or the list is
//   used too deeply), else the chunks.  Since lo <= c, this covers every used
//   product.  The block publishes per-row prefix sums of those bytes and its
//   totals, and asks L2 to prefetch the bytes (bulk prefetch, so DRAM is busy
//   while the select finishes).  After B2 the whole work space (panel by
//   panel, row by row) is split into nb equal byte ranges, one per block: the
//   prefix sum of the dispatch lengths turned into a work partition.
//
//   Multiply (row a4).  A block takes its byte range one panel at a time.
//   The exact per-row threshold tau_i(c) decides each product: |w| >= tau_i
//   holds exactly when fl32(|v_i| |w|) >= c, because the product does not
//   decrease as |w| grows.
//     dense units: warps own 256-column stripes and accumulate 8 columns per
//     lane in registers over groups of 4 rows (16-byte loads, packed fp16
//     magnitude mask, packed fp32 FMA);
//     sparse chunks: 8 lanes per chunk, 8 slots per lane (16-byte value and
//     8-byte gap loads), segmented scan of the gaps to the columns, and a
//     shared-memory atomic add of each used product into the panel
//     accumulator.
//   Each block adds its panel accumulator into out with float4 reductions
//   (out was cleared by its column owners before B2); the last block to
//   finish (a counter, no wait) publishes |S| and resets the scratch words.
//   The order of the fp32 additions varies from call to call, so out is
//   reproducible to rounding, c, |S| and the L_i bit for bit.
#include "effort_internal.cuh"

namespace effort {

// ------------------------------------------------------------------ helpers
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
__device__ __forceinline__ uint2 ld_stream_v2(const void* p, unsigned long long pol) {
  uint2 x;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
               : "=r"(x.x), "=r"(x.y)
               : "l"(p), "l"(pol));
  return x;
}
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// mask with 0xFFFF in each half whose magnitude is >= tau (both halves hold tau)
__device__ __forceinline__ unsigned ge_mask(unsigned w2, unsigned tau2) {
  const unsigned mag = w2 & 0x7FFF7FFFu;
  return __hge2_mask(*reinterpret_cast<const __half2*>(&mag), *reinterpret_cast<const __half2*>(&tau2));
}
__device__ __forceinline__ float h2f(unsigned bits16) { return __half2float(__ushort_as_half((unsigned short)bits16)); }

// Smallest binary16 magnitude m (0..0x7BFF) with fl32(a * m) >= x; 0x7C00 if
// none.  fl32(a * m) does not decrease as m grows, so a binary search over
// the magnitude patterns (which order like the values) is exact.
__device__ __forceinline__ unsigned tau_of(float a, float x) {
  if (!(x > 0.0f)) return 0u;
  if (!(__fmul_rn(a, 65504.0f) >= x)) return 0x7C00u;
  unsigned lo = 0, hi = 0x7BFFu;
  while (lo < hi) {
    const unsigned mid = (lo + hi) >> 1;
    if (__fmul_rn(a, h2f(mid)) >= x) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

// Debug builds (-DEFFORT_DEBUG) check every index a kernel takes from data
// (rows, chunks, decoded columns) before using it; a bad one sets
// kStatusInternal (effort_check then returns EFFORT_ERR_DEVICE) and the
// access is skipped.  Release builds rely on the prepared format, whose
// indices are in range by construction.
#ifdef EFFORT_DEBUG
#define EFFORT_IN_RANGE(cond, status) ((cond) ? true : (atomicOr((status), kStatusInternal), false))
#else
#define EFFORT_IN_RANGE(cond, status) true
#endif

// Phase marks (measurement entry point only): thread 0 of every block stores
// the global timer at fixed points of the call into marks[block][k].
#define EFFORT_MARK(k)                                                              \
  do {                                                                              \
    if (jb.marks && tid == 0) jb.marks[(size_t)blockIdx.x * kMarks + (k)] = global_ns(); \
  } while (0)

constexpr unsigned long long kBarrierLimitNs = 200ull * 1000 * 1000;  // 0.2 s

// Grid-wide barrier over a monotonic counter: the k-th barrier of the
// counter's life completes when the counter reaches (k + 1) nb.  Returns
// false (and sets kStatusTimeout) if the wait ran out of time.
__device__ __forceinline__ bool grid_barrier(unsigned long long* bar, unsigned nb, unsigned* status, int* flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    const unsigned long long old = atomicAdd(bar, 1ull);
    const unsigned long long target = (old / nb + 1ull) * nb;
    const unsigned long long t0 = global_ns();
    for (;;) {
      unsigned long long cur;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(cur) : "l"(bar) : "memory");
      if (cur >= target) break;
      if (global_ns() - t0 > kBarrierLimitNs) {
        atomicOr(status, kStatusTimeout);
        ok = 0;
        break;
      }
    }
    __threadfence();
    *flag = ok;
  }
  __syncthreads();
  return *flag != 0;
}

// Block-wide: every thread passes the summed weight s of its bins (a
// contiguous range, thread 0 lowest); returns in *above the weight of the
// bins of all higher threads.
__device__ __forceinline__ unsigned block_suffix_excl(unsigned s, unsigned* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned x = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_down_sync(0xFFFFFFFFu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) wsum[warp] = x;
  __syncthreads();
  unsigned hiw = 0;
  for (int w = warp + 1; w < kWarps; ++w) hiw += wsum[w];
  __syncthreads();
  return hiw + (x - s);
}

// Block-wide exclusive prefix sum (thread order); *total receives the sum.
__device__ __forceinline__ unsigned block_prefix_excl(unsigned s, unsigned* wsum, unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned x = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  unsigned low = 0, all = 0;
  for (int w = 0; w < kWarps; ++w) {
    const unsigned t = wsum[w];
    if (w < warp) low += t;
    all += t;
  }
  __syncthreads();
  *total = all;
  return low + x - s;
}

// The bin where the weight counted from the top reaches K.  Thread t holds
// the weights of bins [t q, t q + q) in h[0..q).  Writes the bin and K minus
// the weight of all higher bins to ctl[0], ctl[1] (when some bin qualifies).
template <int Q>
__device__ __forceinline__ void find_crossing(const unsigned (&h)[Q], unsigned K, unsigned* wsum, unsigned* ctl) {
  unsigned s = 0;
#pragma unroll
  for (int k = 0; k < Q; ++k) s += h[k];
  const unsigned above = block_suffix_excl(s, wsum);
  if (above < K && K <= above + s) {
    unsigned acc = above;
#pragma unroll
    for (int k = Q - 1; k >= 0; --k) {
      if (acc < K && K <= acc + h[k]) {
        ctl[0] = threadIdx.x * Q + k;
        ctl[1] = K - acc;
      }
      acc += h[k];
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ kernel
struct SmemPtrs {
  float* acc;        // [kPW]
  unsigned* chart;   // [rp][kP]
  float* absv;       // [rp]
  unsigned* hist;    // [kBins0]
  uint2* cand;       // [kCandCap]
  unsigned char* lists;
  unsigned* ctl;     // control words and prefix tables
};

// control-area word offsets
enum : int {
  kCtlFlag = 0, kCtlCross = 2, kCtlWsum = 8,            // kCtlWsum: 32 words
  kCtlNd = 42, kCtlNs = 43, kCtlItem = 44, kCtlDone = 45, kCtlLast = 46,
  kCtlPanelTot = 64,                                    // [kMaxPanels]
  kCtlPC = 128,                                         // [kMaxPanels][nb + 1]
};

struct RoundLists {
  uint4* dense;      // {row, v bits, tau, 0}
  uint4* sparse;     // {first chunk, chunks, v bits, tau}
  unsigned* srow;    // row of each sparse entry
  unsigned* spre;    // prefix of chunk counts [ns + 1]
};
constexpr int kRoundRows = kThreads;

__device__ __forceinline__ RoundLists round_lists(unsigned char* base) {
  RoundLists L;
  L.dense = reinterpret_cast<uint4*>(base);
  L.sparse = L.dense + kRoundRows;
  L.srow = reinterpret_cast<unsigned*>(L.sparse + kRoundRows);
  L.spre = L.srow + kRoundRows;
  return L;
}

// Work bytes of a (row, panel) unit from its info word.
__device__ __forceinline__ unsigned unit_bytes(unsigned info, int stripes) {
  if (info & 0x80000000u) return (unsigned)stripes * (kStripe * 2);
  return info * (unsigned)(kCS * 3);
}

__global__ void __launch_bounds__(kThreads, 1) k_effort(const __grid_constant__ Job jb) {
  extern __shared__ __align__(16) unsigned char smem[];
  const HandleDesc& hd = jb.hd;
  const WsPtrs& ws = jb.ws;
  const int I = hd.I, O = hd.O, P = hd.P;
  const unsigned nb = gridDim.x;
  const unsigned bnb = jb.barrier_nb;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rp = rows_per_block(I, (int)nb);
  const int r0 = min(I, b * rp), r1 = min(I, r0 + rp), nr = r1 - r0;

  size_t o_chart, o_hist, o_cand, o_lists, o_ctl;
  smem_layout(I, (int)nb, &o_chart, &o_hist, &o_cand, &o_lists, &o_ctl);
  SmemPtrs S;
  S.acc = reinterpret_cast<float*>(smem);
  S.chart = reinterpret_cast<unsigned*>(smem + o_chart);
  S.absv = reinterpret_cast<float*>(S.chart + (size_t)rp * kP);
  S.hist = reinterpret_cast<unsigned*>(smem + o_hist);
  S.cand = reinterpret_cast<uint2*>(smem + o_cand);
  S.lists = smem + o_lists;
  S.ctl = reinterpret_cast<unsigned*>(smem + o_ctl);
  unsigned* wsum = S.ctl + kCtlWsum;
  unsigned* PC = S.ctl + kCtlPC;  // PC[p * (nb + 1) + b']: block totals, then their prefix

  // The next call may start its prologue as soon as SMs free up.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  EFFORT_MARK(0);

  // ---- prologue: prepared-matrix data and shared memory only
  for (int e = tid; e < nr * kP; e += kThreads) S.chart[e] = hd.probes[(size_t)r0 * kP + e];
  for (int e = tid; e < kBins0; e += kThreads) S.hist[e] = 0u;
  if (tid < 64) S.ctl[tid] = 0u;

  asm volatile("griddepcontrol.wait;" ::: "memory");
  EFFORT_MARK(1);

  const int mode = jb.mode;
  unsigned* status = ws.hdr + kHdrStatus;
  float c = 0.0f;
  const int oc0 = (int)((long long)O * b / nb), oc1 = (int)((long long)O * (b + 1) / nb);  // this block's columns

  // ---- nothing is used: zero outputs, no grid-wide work
  if (mode == kModeNone) {
    for (int j = oc0 + tid; j < oc1; j += kThreads) jb.out[j] = 0.0f;
    if (jb.rowlen_out)
      for (int i = r0 + tid; i < r1; i += kThreads) jb.rowlen_out[i] = 0u;
    if (b == 0 && tid == 0) {
      if (jb.cutoff_out) *jb.cutoff_out = __int_as_float(0x7F800000);
      if (jb.count_out) *jb.count_out = 0ull;
    }
    return;
  }

  // out is accumulated with reductions after the next grid barrier: clear
  // this block's columns now; |v| of the owned rows (non-finite entries are
  // flagged)
  for (int j = oc0 + tid; j < oc1; j += kThreads) jb.out[j] = 0.0f;
  const float* vf = reinterpret_cast<const float*>(jb.v);
  const __half* vh = reinterpret_cast<const __half*>(jb.v);
  for (int t = tid; t < nr; t += kThreads) {
    const float x = jb.vdtype ? __half2float(vh[r0 + t]) : vf[r0 + t];
    if (!isfinite(x)) atomicOr(status, kStatusNonfiniteV);
    S.absv[t] = fabsf(x);
    if (jb.rowlen_out) jb.rowlen_out[r0 + t] = (mode == kModeAll) ? (unsigned)hd.n : 0u;
  }
  __syncthreads();

  auto panel_stripes = [&](int p) -> int {
    const int w = min(kPW, O - p * kPW);
    return (w + kStripe - 1) / kStripe;
  };

  if (mode == kModeSelect) {
    // ---- phase 1: chart and first-digit histogram
    for (int e = tid; e < nr * kP; e += kThreads) {
      const int k = e & (kP - 1);
      const float x = __fmul_rn(S.absv[e >> 4], h2f(S.chart[e]));
      const unsigned xb = __float_as_uint(x);
      S.chart[e] = xb;
      const unsigned w = (unsigned)hd.pw[k];
      if (w) atomicAdd(&S.hist[xb >> 19], w);
    }
    __syncthreads();
    for (int e = tid; e < kBins0; e += kThreads) {
      const unsigned h = S.hist[e];
      if (h) atomicAdd(&ws.ghist0[e], h);
    }
    EFFORT_MARK(2);
    if (!grid_barrier(ws.bar, bnb, status, (int*)&S.ctl[kCtlFlag])) return;
    EFFORT_MARK(3);

    // ---- phase 2: crossing bin, candidates, dispatch bounds, prefetch
    unsigned h4[4];
    {
      const uint4 q = __ldcg(reinterpret_cast<const uint4*>(ws.ghist0) + tid);
      h4[0] = q.x;
      h4[1] = q.y;
      h4[2] = q.z;
      h4[3] = q.w;
    }
    find_crossing<4>(h4, (unsigned)jb.K, wsum, S.ctl + kCtlCross);
    const unsigned b1 = S.ctl[kCtlCross], K1 = S.ctl[kCtlCross + 1];
    const float lo = __uint_as_float(b1 << 19);
    // candidates: the owned chart entries of the crossing bin
    for (int e0 = 0; e0 < nr * kP; e0 += kThreads) {
      const int e = e0 + tid;
      bool in = false;
      unsigned xb = 0, w = 0;
      if (e < nr * kP) {
        xb = S.chart[e];
        w = (unsigned)hd.pw[e & (kP - 1)];
        in = w != 0 && (xb >> 19) == b1;
      }
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, in);
      if (bal) {
        unsigned basei = 0;
        if (lane == 0) basei = atomicAdd(ws.hdr + kHdrCand, (unsigned)__popc(bal));
        basei = __shfl_sync(0xFFFFFFFFu, basei, 0);
        const unsigned pos = basei + __popc(bal & ((1u << lane) - 1u));
        if (in && pos < (unsigned)kCandCap) ws.cand[pos] = make_uint2(xb, w);
      }
    }
    // dispatch bounds per (row, panel) with tau(lo), lo <= c: every load
    // first, the L2 prefetch of the units after all of them
    unsigned* wtmp = reinterpret_cast<unsigned*>(S.lists);  // [nr][kMaxPanels] unit bytes
    unsigned* lxs = wtmp + (size_t)rp * kMaxPanels;         // [nr][kMaxPanels] first chunk
    unsigned* infs = lxs + (size_t)rp * kMaxPanels;         // [nr][kMaxPanels] info
    unsigned* taul = infs + (size_t)rp * kMaxPanels;        // [nr]
    for (int t = tid; t < nr; t += kThreads) taul[t] = tau_of(S.absv[t], lo);
    __syncthreads();
    for (int e = tid; e < nr * P; e += kThreads) {
      const int t = e / P, p = e - t * P;
      const int i = r0 + t;
      const unsigned tau = taul[t];
      const uint4 L = hd.lst[(size_t)i * P + p];  // {first chunk, stored chunks, tail, kept}
      unsigned info = 0;
      if (L.w != 0u && tau < 0x7C00u) {
        // the stored chunks' first magnitudes, loaded together (a list of a
        // 2048-column panel has at most 14 stored chunks)
        unsigned short hv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          hv[k] = ((unsigned)k < L.y && EFFORT_IN_RANGE(L.x + k < hd.total_chunks, status)) ? hd.head[L.x + k]
                                                                                               : (unsigned short)0;
        unsigned m = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k) m += ((unsigned)k < L.y && hv[k] >= tau) ? 1u : 0u;
        for (unsigned k = 16; k < L.y; ++k)
          if (EFFORT_IN_RANGE(L.x + k < hd.total_chunks, status)) m += (hd.head[L.x + k] >= tau) ? 1u : 0u;
        if (L.z >= tau && L.z != 0u) info = 0x80000000u;  // the stored part does not reach tau
        else info = m;
      }
      ws.info[(size_t)i * P + p] = info;
      wtmp[t * kMaxPanels + p] = unit_bytes(info, panel_stripes(p));
      lxs[t * kMaxPanels + p] = L.x;
      infs[t * kMaxPanels + p] = info;
    }
    __syncthreads();
    // per-panel prefix over the owned rows (one warp per panel)
    for (int p = warp; p < P; p += kWarps) {
      unsigned run = 0;
      for (int t0 = 0; t0 < nr; t0 += 32) {
        const int t = t0 + lane;
        const unsigned x = (t < nr) ? wtmp[t * kMaxPanels + p] : 0u;
        unsigned y = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned z = __shfl_up_sync(0xFFFFFFFFu, y, o);
          if (lane >= o) y += z;
        }
        if (t < nr) ws.rowpre[(size_t)(r0 + t) * P + p] = run + y - x;
        run += __shfl_sync(0xFFFFFFFFu, y, 31);
      }
      if (lane == 0) ws.ctot[(size_t)b * P + p] = run;
    }
    // ask L2 for the units' bytes while the select finishes
    for (int e = tid; e < nr * P; e += kThreads) {
      const int t = e / P, p = e - t * P;
      const unsigned bytes = wtmp[t * kMaxPanels + p];
      if (!bytes) continue;
      const unsigned info = infs[t * kMaxPanels + p];
      if (info & 0x80000000u) {
        prefetch_l2_bulk(hd.wdense + (size_t)(r0 + t) * hd.dstride + (size_t)p * kPW, bytes);
      } else {
        const size_t x = lxs[t * kMaxPanels + p];
        prefetch_l2_bulk(hd.vals + x * kCS, info * (unsigned)(kCS * 2));
        prefetch_l2_bulk(hd.gaps + x * kCS, info * (unsigned)kCS);
      }
    }
    EFFORT_MARK(4);
    if (!grid_barrier(ws.bar, bnb, status, (int*)&S.ctl[kCtlFlag])) return;
    EFFORT_MARK(5);

    // ---- phase 3: resolve c over the candidates; block totals, in one round
    // the first-digit histogram is read by nobody any more: clear this block's share
    for (int e = b * (kBins0 / 4) / (int)nb * 4 + tid, e1 = (b + 1) * (kBins0 / 4) / (int)nb * 4; e < e1;
         e += kThreads)
      ws.ghist0[e] = 0u;
    const unsigned M = __ldcg(ws.hdr + kHdrCand);
    for (int e = tid; e < (int)nb * P; e += kThreads) {
      const int bb = e / P, p = e - bb * P;
      PC[(size_t)p * (nb + 1) + bb] = __ldcg(&ws.ctot[e]);
    }
    unsigned b2 = 0, b3 = 0;
    if (M <= (unsigned)kCandCap) {
      for (unsigned e = tid; e < M; e += kThreads) S.cand[e] = __ldcg(&ws.cand[e]);
      for (int e = tid; e < kBins1 + kBins2; e += kThreads) S.hist[e] = 0u;
      __syncthreads();
      for (unsigned e = tid; e < M; e += kThreads) atomicAdd(&S.hist[(S.cand[e].x >> 9) & (kBins1 - 1)], S.cand[e].y);
      __syncthreads();
      {
        unsigned h1[1] = {S.hist[tid]};
        find_crossing<1>(h1, K1, wsum, S.ctl + kCtlCross);
      }
      b2 = S.ctl[kCtlCross];
      const unsigned K2 = S.ctl[kCtlCross + 1];
      for (unsigned e = tid; e < M; e += kThreads) {
        const unsigned xb = S.cand[e].x;
        if (((xb >> 9) & (kBins1 - 1)) == b2) atomicAdd(&S.hist[kBins1 + (xb & (kBins2 - 1))], S.cand[e].y);
      }
      __syncthreads();
      {
        unsigned h1[1] = {tid < kBins2 ? S.hist[kBins1 + tid] : 0u};
        find_crossing<1>(h1, K2, wsum, S.ctl + kCtlCross);
      }
      b3 = S.ctl[kCtlCross];
    } else {
      // too many candidates for one block: two more grid-wide histogram passes
      for (int e = tid; e < kBins1 + kBins2; e += kThreads) S.hist[e] = 0u;
      __syncthreads();
      for (int e = tid; e < nr * kP; e += kThreads) {
        const unsigned xb = S.chart[e], w = (unsigned)hd.pw[e & (kP - 1)];
        if (w && (xb >> 19) == b1) atomicAdd(&S.hist[(xb >> 9) & (kBins1 - 1)], w);
      }
      __syncthreads();
      for (int e = tid; e < kBins1; e += kThreads)
        if (S.hist[e]) atomicAdd(&ws.ghist1[e], S.hist[e]);
      if (!grid_barrier(ws.bar, bnb, status, (int*)&S.ctl[kCtlFlag])) return;
      {
        unsigned h1[1] = {__ldcg(&ws.ghist1[tid])};
        find_crossing<1>(h1, K1, wsum, S.ctl + kCtlCross);
      }
      b2 = S.ctl[kCtlCross];
      const unsigned K2 = S.ctl[kCtlCross + 1];
      for (int e = tid; e < nr * kP; e += kThreads) {
        const unsigned xb = S.chart[e], w = (unsigned)hd.pw[e & (kP - 1)];
        if (w && (xb >> 19) == b1 && ((xb >> 9) & (kBins1 - 1)) == b2) atomicAdd(&S.hist[kBins1 + (xb & (kBins2 - 1))], w);
      }
      __syncthreads();
      for (int e = tid; e < kBins2; e += kThreads)
        if (S.hist[kBins1 + e]) atomicAdd(&ws.ghist2[e], S.hist[kBins1 + e]);
      if (!grid_barrier(ws.bar, bnb, status, (int*)&S.ctl[kCtlFlag])) return;
      // ghist1 is read by nobody any more
      if (b == 0)
        for (int e = tid; e < kBins1; e += kThreads) ws.ghist1[e] = 0u;
      {
        unsigned h1[1] = {tid < kBins2 ? __ldcg(&ws.ghist2[tid]) : 0u};
        find_crossing<1>(h1, K2, wsum, S.ctl + kCtlCross);
      }
      b3 = S.ctl[kCtlCross];
    }
    c = __uint_as_float((b1 << 19) | (b2 << 9) | b3);
    if (b == 0 && tid == 0 && jb.cutoff_out) *jb.cutoff_out = c;
    // c = 0: every kept product is used (fillers, pads and dropped weights add +0)
    if (c == 0.0f && jb.rowlen_out)
      for (int t = tid; t < nr; t += kThreads) jb.rowlen_out[r0 + t] = (unsigned)hd.n;
  } else {
    // every (row, panel) is a dense unit: the block totals are arithmetic
    for (int e = tid; e < (int)nb * P; e += kThreads) {
      const int bb = e / P, p = e - bb * P;
      const int ra = min(I, bb * rp), rb = min(I, ra + rp);
      PC[(size_t)p * (nb + 1) + bb] = (unsigned)(rb - ra) * ((unsigned)panel_stripes(p) * (kStripe * 2));
    }
    if (b == 0 && tid == 0 && jb.cutoff_out) *jb.cutoff_out = 0.0f;
    // the cleared out must be complete before any block adds to it
    if (!grid_barrier(ws.bar, bnb, status, (int*)&S.ctl[kCtlFlag])) return;
  }
  EFFORT_MARK(6);

  // ---- partition: per panel, the prefix of the owner blocks' totals (shared memory only)
  const bool all = (mode == kModeAll);
  const bool count_all = all || c == 0.0f;  // used set = every kept entry
  __syncthreads();
  for (int p = warp; p < P; p += kWarps) {
    unsigned* pc = PC + (size_t)p * (nb + 1);
    unsigned run = 0;
    for (int b0 = 0; b0 < (int)nb; b0 += 32) {
      const int bb = b0 + lane;
      const unsigned x = (bb < (int)nb) ? pc[bb] : 0u;
      unsigned y = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned z = __shfl_up_sync(0xFFFFFFFFu, y, o);
        if (lane >= o) y += z;
      }
      __syncwarp();
      if (bb < (int)nb) pc[bb] = run + y - x;
      run += __shfl_sync(0xFFFFFFFFu, y, 31);
    }
    if (lane == 0) {
      pc[nb] = run;
      S.ctl[kCtlPanelTot + p] = run;
    }
  }
  __syncthreads();
  unsigned long long Wtot = 0;
  for (int p = 0; p < P; ++p) Wtot += S.ctl[kCtlPanelTot + p];
  const unsigned long long x0 = Wtot * (unsigned long long)b / nb, x1 = Wtot * (unsigned long long)(b + 1) / nb;
  EFFORT_MARK(7);

  const unsigned long long pol = evict_first_policy();
  const RoundLists RL = round_lists(S.lists);
  unsigned long long my_count = 0;
  unsigned long long my_dense_bytes = 0, my_sparse_bytes = 0;  // summed over the block by thread 0
  unsigned* rowlen = jb.rowlen_out;
  const bool want_rowlen = (rowlen != nullptr) && !count_all;
  const bool out16 = ((uintptr_t)jb.out & 15u) == 0;

  bool first_round = true;
  unsigned long long pbase = 0;
  for (int p = 0; p < P; ++p) {
    const unsigned long long Wp = S.ctl[kCtlPanelTot + p];
    const unsigned long long pa = pbase, pe = pbase + Wp;
    pbase = pe;
    if (pe <= x0 || pa >= x1 || Wp == 0) continue;
    const unsigned y0 = (unsigned)((x0 > pa ? x0 : pa) - pa), y1 = (unsigned)((x1 < pe ? x1 : pe) - pa);
    const int stripes = panel_stripes(p);
    const unsigned* PCp = PC + (size_t)p * (nb + 1);
    for (int j = tid; j < kPW; j += kThreads) S.acc[j] = 0.0f;
    // rows from the first row of the owner block with the last prefix <= y0
    int cursor;
    {
      int lo_b = 0, hi_b = (int)nb - 1;
      while (lo_b < hi_b) {
        const int mid = (lo_b + hi_b + 1) >> 1;
        if (PCp[mid] <= y0) lo_b = mid;
        else hi_b = mid - 1;
      }
      cursor = min(I, lo_b * rp);
    }

    for (;;) {
      // ---- build the work lists of rows [cursor, cursor + kRoundRows)
      if (tid == 0) {
        S.ctl[kCtlNd] = 0u;
        S.ctl[kCtlNs] = 0u;
        S.ctl[kCtlDone] = 0u;
        S.ctl[kCtlItem] = 0u;
      }
      __syncthreads();
      {
        const int i = cursor + tid;
        bool isd = false, iss = false;
        unsigned vbits = 0, tau = 0, ch0 = 0, nch = 0;
        if (i < I) {
          const int owner = i / rp;
          // everything the row needs, loaded in one round
          unsigned info, pre, lx = 0;
          if (all) {
            info = 0x80000000u;
            pre = (unsigned)(i - owner * rp) * ((unsigned)stripes * (kStripe * 2));
          } else {
            info = __ldcg(&ws.info[(size_t)i * P + p]);
            pre = __ldcg(&ws.rowpre[(size_t)i * P + p]);
            lx = reinterpret_cast<const unsigned*>(hd.lst)[((size_t)i * P + p) * 4];
          }
          const float vi = jb.vdtype ? __half2float(vh[i]) : vf[i];
          const unsigned pos = PCp[owner] + pre;
          if (pos >= y1) {
            S.ctl[kCtlDone] = 1u;
          } else if (info != 0u) {
            vbits = __float_as_uint(vi);
            tau = all ? 0u : tau_of(fabsf(vi), c);
            if (info & 0x80000000u) {
              isd = pos >= y0;
            } else {
              // chunks whose start lies in [y0, y1)
              const unsigned cb = (unsigned)(kCS * 3);
              const unsigned klo = (pos >= y0) ? 0u : (y0 - pos + cb - 1) / cb;
              const unsigned khi = min(info, (y1 - pos + cb - 1) / cb);
              if (klo < khi) {
                iss = true;
                ch0 = lx + klo;
                nch = khi - klo;
              }
            }
          }
        } else {
          S.ctl[kCtlDone] = 1u;
        }
        const unsigned bd = __ballot_sync(0xFFFFFFFFu, isd), bs = __ballot_sync(0xFFFFFFFFu, iss);
        unsigned bd0 = 0, bs0 = 0;
        if (lane == 0) {
          if (bd) bd0 = atomicAdd(&S.ctl[kCtlNd], (unsigned)__popc(bd));
          if (bs) bs0 = atomicAdd(&S.ctl[kCtlNs], (unsigned)__popc(bs));
        }
        bd0 = __shfl_sync(0xFFFFFFFFu, bd0, 0);
        bs0 = __shfl_sync(0xFFFFFFFFu, bs0, 0);
        const unsigned below = (1u << lane) - 1u;
        if (isd) RL.dense[bd0 + __popc(bd & below)] = make_uint4((unsigned)i, vbits, tau, 0u);
        if (iss) {
          const unsigned q = bs0 + __popc(bs & below);
          RL.sparse[q] = make_uint4(ch0, nch, vbits, tau);
          RL.srow[q] = (unsigned)i;
        }
      }
      __syncthreads();
      const int nd = (int)S.ctl[kCtlNd], ns = (int)S.ctl[kCtlNs];
      const bool done = S.ctl[kCtlDone] != 0u;
      if (tid == 0) my_dense_bytes += (unsigned long long)nd * (unsigned)stripes * (kStripe * 2);
      // prefix of the sparse chunk counts
      unsigned total_chunks = 0;
      {
        const unsigned x = (tid < ns) ? RL.sparse[tid].y : 0u;
        const unsigned ex = block_prefix_excl(x, wsum, &total_chunks);
        if (tid < ns) RL.spre[tid] = ex;
        if (tid == 0) {
          RL.spre[ns] = total_chunks;
          my_sparse_bytes += (unsigned long long)total_chunks * (kCS * 3);
        }
      }
      __syncthreads();
      if (first_round) EFFORT_MARK(8);

      // ---- dense units: warp w owns stripe w % stripes over groups of 4 rows
      {
        const int step = kWarps / stripes;
        if (warp < step * stripes) {
          const int s = warp % stripes, g0 = warp / stripes;
          float2 a[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) a[m] = make_float2(0.0f, 0.0f);
          unsigned dcount = 0;
          const size_t colbase = (size_t)p * kPW + (size_t)s * kStripe + 8 * lane;
          for (int g = g0 * 4; g < nd; g += step * 4) {
            uint4 wv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (g + u < nd) {
                const unsigned r = RL.dense[g + u].x;
                if (EFFORT_IN_RANGE(r < (unsigned)I, status)) wv[u] = ld_stream_v4(hd.wdense + (size_t)r * hd.dstride + colbase, pol);
                else wv[u] = make_uint4(0u, 0u, 0u, 0u);
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (g + u < nd) {
                const uint4 rec = RL.dense[g + u];
                const unsigned tau2 = rec.z | (rec.z << 16);
                const float vi = __uint_as_float(rec.y);
                const float2 v2 = make_float2(vi, vi);
                const unsigned w4[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
                unsigned rc = 0;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                  const unsigned msk = ge_mask(w4[m], tau2);
                  rc += __popc(msk);
                  const unsigned wm = w4[m] & msk;
                  const float2 wf = __half22float2(*reinterpret_cast<const __half2*>(&wm));
                  a[m] = __ffma2_rn(v2, wf, a[m]);
                }
                dcount += rc >> 4;
                if (want_rowlen) {
                  unsigned r = rc >> 4;
#pragma unroll
                  for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
                  if (lane == 0 && r) atomicAdd(&rowlen[rec.x], r);
                }
              }
            }
          }
          my_count += dcount;
          // registers into the panel accumulator
          const int cl = s * kStripe + 8 * lane;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            if (a[m].x != 0.0f) atomicAdd(&S.acc[cl + 2 * m], a[m].x);
            if (a[m].y != 0.0f) atomicAdd(&S.acc[cl + 2 * m + 1], a[m].y);
          }
        }
      }
      if (first_round) EFFORT_MARK(9);

      // ---- sparse chunks: items of 8 chunks, taken dynamically by the warps
      {
        const int nitems = (int)((total_chunks + 7) / 8);
        const int grp = lane >> 3, sl = lane & 7;
        unsigned scount = 0;
        for (;;) {
          int item = 0;
          if (lane == 0) item = (int)atomicAdd(&S.ctl[kCtlItem], 1u);
          item = __shfl_sync(0xFFFFFFFFu, item, 0);
          if (item >= nitems) break;
          uint4 vv[2];
          uint2 gg[2];
          float vi[2];
          unsigned tau[2], row[2];
          bool ok[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const unsigned j = (unsigned)item * 8u + (unsigned)(h * 4 + grp);
            ok[h] = j < total_chunks;
            if (ok[h]) {
              // entry r with spre[r] <= j < spre[r + 1]
              int lo_r = 0, hi_r = ns - 1;
              while (lo_r < hi_r) {
                const int mid = (lo_r + hi_r + 1) >> 1;
                if (RL.spre[mid] <= j) lo_r = mid;
                else hi_r = mid - 1;
              }
              const uint4 e = RL.sparse[lo_r];
              const unsigned chunk = e.x + (j - RL.spre[lo_r]);
              ok[h] = EFFORT_IN_RANGE(chunk < hd.total_chunks, status);
              vi[h] = __uint_as_float(e.z);
              tau[h] = e.w;
              row[h] = RL.srow[lo_r];
              if (ok[h]) {
                vv[h] = ld_stream_v4(hd.vals + (size_t)chunk * kCS + 8 * sl, pol);
                gg[h] = ld_stream_v2(hd.gaps + (size_t)chunk * kCS + 8 * sl, pol);
              }
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // gaps to columns: inclusive sums inside the lane, exclusive across the 8 lanes
            const unsigned gl = ok[h] ? gg[h].x : 0u, gh = ok[h] ? gg[h].y : 0u;
            int cs[8];
            cs[0] = (int)(gl & 0xFFu);
            cs[1] = cs[0] + (int)((gl >> 8) & 0xFFu);
            cs[2] = cs[1] + (int)((gl >> 16) & 0xFFu);
            cs[3] = cs[2] + (int)(gl >> 24);
            cs[4] = cs[3] + (int)(gh & 0xFFu);
            cs[5] = cs[4] + (int)((gh >> 8) & 0xFFu);
            cs[6] = cs[5] + (int)((gh >> 16) & 0xFFu);
            cs[7] = cs[6] + (int)(gh >> 24);
            int ex = cs[7];
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
              const int y = __shfl_up_sync(0xFFFFFFFFu, ex, o, 8);
              if (sl >= o) ex += y;
            }
            ex -= cs[7];
            const int basecol = ex - 1;
            const unsigned w4[4] = {vv[h].x, vv[h].y, vv[h].z, vv[h].w};
            const unsigned tau2 = tau[h] | (tau[h] << 16);
            unsigned rc = 0;
            if (ok[h]) {
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                const unsigned msk = ge_mask(w4[m], tau2);
                const int ca = basecol + cs[2 * m], cb2 = basecol + cs[2 * m + 1];
                if ((msk & 0xFFFFu) && EFFORT_IN_RANGE((unsigned)ca < (unsigned)kPW, status)) {
                  atomicAdd(&S.acc[ca], __fmul_rn(vi[h], h2f(w4[m] & 0xFFFFu)));
                  ++rc;
                }
                if ((msk & 0xFFFF0000u) && EFFORT_IN_RANGE((unsigned)cb2 < (unsigned)kPW, status)) {
                  atomicAdd(&S.acc[cb2], __fmul_rn(vi[h], h2f(w4[m] >> 16)));
                  ++rc;
                }
              }
            }
            scount += rc;
            if (want_rowlen) {
              unsigned r = rc;
#pragma unroll
              for (int o = 4; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o, 8);
              if (ok[h] && sl == 0 && r) atomicAdd(&rowlen[row[h]], r);
            }
          }
        }
        my_count += scount;
      }
      __syncthreads();
      if (first_round) EFFORT_MARK(10);
      first_round = false;
      if (done) break;
      cursor += kRoundRows;
      if (cursor >= I) break;
    }
    // this block's share of panel p, added into out (float4 reductions)
    {
      const int pw = min(kPW, O - p * kPW);
      float* dst = jb.out + (size_t)p * kPW;
      if (out16) {
        for (int j = tid; j < pw / 4; j += kThreads) {
          const float4 a4 = reinterpret_cast<const float4*>(S.acc)[j];
          if (a4.x != 0.0f || a4.y != 0.0f || a4.z != 0.0f || a4.w != 0.0f)
            atomicAdd(reinterpret_cast<float4*>(dst) + j, a4);
        }
        for (int j = pw / 4 * 4 + tid; j < pw; j += kThreads)
          if (S.acc[j] != 0.0f) atomicAdd(dst + j, S.acc[j]);
      } else {
        for (int j = tid; j < pw; j += kThreads)
          if (S.acc[j] != 0.0f) atomicAdd(dst + j, S.acc[j]);
      }
    }
    __syncthreads();
  }
  EFFORT_MARK(11);

  // ---- used count and planned bytes; the last block to finish publishes them
  {
    unsigned long long x = my_count;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    if (lane == 0 && x && !count_all) atomicAdd(ws.count, x);
    if (tid == 0) {
      unsigned long long* run = reinterpret_cast<unsigned long long*>(ws.hdr + kHdrBytesRun);
      if (my_dense_bytes) atomicAdd(run, my_dense_bytes);
      if (my_sparse_bytes) atomicAdd(run + 1, my_sparse_bytes);
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned arrived = atomicAdd(ws.hdr + kHdrDone, 1u);
    S.ctl[kCtlLast] = (arrived == nb - 1u) ? 1u : 0u;
  }
  __syncthreads();
  if (S.ctl[kCtlLast]) {
    __threadfence();
    if (tid == 0) {
      const unsigned long long cnt = count_all ? hd.kept_total : __ldcg(ws.count);
      if (jb.count_out) *jb.count_out = cnt;
      *ws.count = 0ull;
      ws.hdr[kHdrCand] = 0u;
      ws.hdr[kHdrDone] = 0u;
      unsigned long long* run = reinterpret_cast<unsigned long long*>(ws.hdr + kHdrBytesRun);
      unsigned long long* last = reinterpret_cast<unsigned long long*>(ws.hdr + kHdrBytesLast);
      last[0] = __ldcg(run);
      last[1] = __ldcg(run + 1);
      run[0] = 0ull;
      run[1] = 0ull;
    }
    // the last digit's histogram of the many-candidates path is read by nobody any more
    if (mode == kModeSelect)
      for (int e = tid; e < kBins2; e += kThreads) ws.ghist2[e] = 0u;
  }
  EFFORT_MARK(13);
}

// ------------------------------------------------------------------ launch
cudaError_t effort_kernel_attributes(size_t smem) {
  return cudaFuncSetAttribute(k_effort, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

int effort_blocks_per_sm(size_t smem) {
  int nbk = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nbk, k_effort, kThreads, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return nbk;
}

cudaError_t launch_effort(const Job& job, int nb, size_t smem, cudaStream_t stream) {
  // (marks, when set, come with the job)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nb);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_effort, job);
}

}  // namespace effort
