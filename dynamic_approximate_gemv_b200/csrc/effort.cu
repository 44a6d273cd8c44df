// One approximate matvec in one kernel: the `approxMul` step of the pages'
// pseudo-code (Hacker News item 40067677, "Show HN: Speeding up LLM inference
// 2x times (possibly)": cutoff_chart = v * probes, cutoff = topK(chart,
// effort), then the multiply over the leading part of every sorted row), with
// the cost split the author gives in Hacker News item 40095016 (about
// O(inDim log inDim) for the cutoff, O(inDim) for the dispatch,
// O(effort inDim outDim) multiplications).
//
// Grid: one block per SM, all resident at once.  The blocks meet at grid-wide
// barriers over a monotonic counter in the scratch; every wait has a time
// limit, after which the kernel sets a status bit and leaves.
//
//   Cutoff (row a2).  Block b owns rows [b rp, b rp + rp) of the chart
//   x_ik = fl32(|v_i| p_ik).  The chart's fp32 patterns are non-negative and
//   order like unsigned integers, so c is found by a weighted radix select:
//   every block adds its entries' probe weights into a global histogram of
//   bits [30:19], writes its entries grouped by that digit into its own
//   segment of the scratch and, per digit it holds, a descriptor (first
//   slot, count) into a [digit][block] table (barrier B1).  Every block then
//   finds the bin where the weight counted from the top reaches K, reads
//   that bin's row of descriptors and, through them, the bin's entries from
//   all segments, and resolves bits [18:0] over them in shared memory (with
//   more candidates than fit, by two more grid-wide histogram passes).  One
//   grid barrier in the common case.
//
//   Work split.  Block b streams output panel p = b mod P for the rows
//   i = b / P + k nbp (nbp blocks share a panel; rows interleave so the
//   heavy rows of a vector spread over the blocks).  Each (row, panel) is a
//   work unit.  The units' list records and their stored chunks' first
//   magnitudes are loaded while B1 fills.
//
//   Dispatch (row a3).  Once c is known: for every unit the threshold
//   tau_i(c), the smallest fp16 magnitude m with fl32(|v_i| m) >= c (|w| >=
//   tau_i holds exactly when fl32(|v_i| |w|) >= c, because the product does
//   not decrease as |w| grows).  The unit is read from the dense copy when
//   the stored part of its list does not reach tau_i, else as the stored
//   chunks whose first magnitude reaches tau_i.  A block-wide prefix sum over
//   the units turns these counts into a dense-unit list and a sparse-chunk
//   list.
//
//   Multiply (row a4).  All 16 warps stream with plain 16-byte loads, a batch
//   in flight per lane (8 dense units, or 8 sparse chunks per lane group):
//     dense units: warp w owns 256-column stripe w mod 8 of every other unit;
//     packed fp16 magnitude mask, packed fp32 FMA into registers that stay
//     for the call;
//     sparse chunks: 8 lanes per chunk, 8 slots per lane, segmented scan of
//     the gaps to the columns, shared-memory integer atomic add of each used
//     product into the panel accumulator.
//   The panel accumulator is 32-bit fixed point (shared-memory integer
//   atomics cost a fraction of float ones): its unit 2^-s is set per call so
//   that sum |v_i| * max |w|, which bounds every partial sum, stays below 2^30
//   units; each fp32 product is rounded once to the unit.  Each block adds
//   its panel sums into out with float4 reductions (out was cleared by its
//   column owners before B1); the last block to finish (a counter, no wait)
//   publishes |S| and resets the scratch words.  The order of the fp32
//   additions into out varies from call to call, so out is reproducible to
//   rounding, c, |S| and the L_i bit for bit.
#include "effort_internal.cuh"

namespace effort {

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ unsigned smem_addr(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }

constexpr unsigned long long kWaitLimitNs = 200ull * 1000 * 1000;  // 0.2 s for any single wait

// mask with 0xFFFF in each half whose magnitude is >= tau (both halves hold tau)
__device__ __forceinline__ unsigned ge_mask(unsigned w2, unsigned tau2) {
  const unsigned mag = w2 & 0x7FFF7FFFu;
  return __hge2_mask(*reinterpret_cast<const __half2*>(&mag), *reinterpret_cast<const __half2*>(&tau2));
}
__device__ __forceinline__ float h2f(unsigned bits16) { return __half2float(__ushort_as_half((unsigned short)bits16)); }
__device__ __forceinline__ bool passes(float a, unsigned m, float x) { return __fmul_rn(a, h2f(m)) >= x; }

// Smallest binary16 magnitude m (0..0x7BFF) with fl32(a * m) >= x; 0x7C00 if
// none.  fl32(a * m) does not decrease as m grows, so the answer is the first
// pattern that passes.  A guess from x / a is corrected by exact product
// tests; a binary search over all patterns settles any guess the short
// correction does not.
__device__ __forceinline__ unsigned tau_of(float a, float x) {
  if (!(x > 0.0f)) return 0u;
  if (!passes(a, 0x7BFFu, x)) return 0x7C00u;
  unsigned m = __half_as_ushort(__float2half_rn(__fdividef(x, a))) & 0x7FFFu;  // a guess: the tests below decide
  if (m > 0x7BFFu) m = 0x7BFFu;
#pragma unroll 1
  for (int k = 0; k < 4 && m > 0 && passes(a, m - 1, x); ++k) --m;
#pragma unroll 1
  for (int k = 0; k < 4 && m < 0x7BFFu && !passes(a, m, x); ++k) ++m;
  if (passes(a, m, x) && (m == 0 || !passes(a, m - 1, x))) return m;
  unsigned lo = 0, hi = 0x7BFFu;
  while (lo < hi) {
    const unsigned mid = (lo + hi) >> 1;
    if (passes(a, mid, x)) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

// Q8: the smallest |q| m (0..128) with fl32(a * (s m)) >= x, as the binary16
// bits of m; 0x7C00 if none.  s m is exact in fp32 (11 + 8 significant
// bits), so the test is the oracle's fl32(|v_i| |w_ij|) >= c; it does not
// decrease as m grows, so a binary search finds the first m that passes.
__device__ __forceinline__ unsigned tau_q8(float a, float s, float x) {
  if (!(x > 0.0f)) return 0u;
  if (!(__fmul_rn(a, __fmul_rn(s, 128.0f)) >= x)) return 0x7C00u;
  int lo = 0, hi = 128;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__fmul_rn(a, __fmul_rn(s, (float)mid)) >= x) hi = mid;
    else lo = mid + 1;
  }
  return __half_as_ushort(__int2half_rn(lo));
}

// Q8: 8 int8 values (two words) as four words of two binary16 values each
// (every int8 is a binary16 value), in the order of the fp16 layout.  Each
// byte is biased to u = q + 128 (an xor of its top bit) and placed under the
// high byte 0x64: the binary16 with bits 0x64uu is 1024 + u, so one packed
// subtraction of 1152 gives q exactly.
__device__ __forceinline__ uint4 widen_q8(unsigned lo, unsigned hi) {
  const unsigned a = lo ^ 0x80808080u, b = hi ^ 0x80808080u;
  const __half2 bias = __halves2half2(__ushort_as_half((unsigned short)0x6480u),
                                      __ushort_as_half((unsigned short)0x6480u));  // 1152
  unsigned o[4] = {__byte_perm(a, 0x64646464u, 0x5140u), __byte_perm(a, 0x64646464u, 0x5342u),
                   __byte_perm(b, 0x64646464u, 0x5140u), __byte_perm(b, 0x64646464u, 0x5342u)};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&o[k]), bias);
    o[k] = *reinterpret_cast<const unsigned*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Debug builds (-DEFFORT_DEBUG) check every index a kernel takes from data
// (rows, chunks, decoded columns, stage offsets) before using it; a bad one
// sets kStatusInternal (effort_check then returns EFFORT_ERR_DEVICE) and the
// access is skipped.  Release builds rely on the prepared format, whose
// indices are in range by construction.
#ifdef EFFORT_DEBUG
#define EFFORT_IN_RANGE(cond, status) ((cond) ? true : (atomicOr((status), kStatusInternal), false))
#else
#define EFFORT_IN_RANGE(cond, status) true
#endif

// Phase marks (measurement entry point only): thread 0 of every block stores
// the global timer at fixed points of the call into marks[block][k].
#define EFFORT_MARK(k)                                                                     \
  do {                                                                                     \
    if (jb.marks && threadIdx.x == 0) jb.marks[(size_t)blockIdx.x * kMarks + (k)] = global_ns(); \
  } while (0)
#define EFFORT_MARK_LANE0(k)                                                               \
  do {                                                                                     \
    if (jb.marks && (threadIdx.x & 31) == 0) jb.marks[(size_t)blockIdx.x * kMarks + (k)] = global_ns(); \
  } while (0)

// Grid-wide barrier over a monotonic counter.  Every call starts with the
// counter at a multiple of nb (each of its barriers adds nb), so a block that
// read the call's base knows the k-th barrier of the call completes at base +
// (k + 1) nb: it arrives with a reduction (no round trip) and polls.  The
// calling thread's block must have ordered its writes before the call.
__device__ __forceinline__ void grid_arrive_thread(unsigned long long* bar) {
  __threadfence();
  asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(bar) : "memory");
}
__device__ __forceinline__ bool grid_wait_thread(unsigned long long* bar, unsigned long long target, unsigned* status) {
  const unsigned long long t0 = global_ns();
  for (;;) {
    unsigned long long cur;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(cur) : "l"(bar) : "memory");
    if (cur >= target) break;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
  __threadfence();
  return true;
}
// Whole-block form: returns the same value in every thread.
__device__ __forceinline__ bool grid_barrier_block(unsigned long long* bar, unsigned long long target, unsigned* status,
                                                   unsigned* flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    grid_arrive_thread(bar);
    *flag = grid_wait_thread(bar, target, status) ? 1u : 0u;
  }
  __syncthreads();
  return *flag != 0;
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
  if (warp == 0) {
    unsigned y = (lane < kWarps) ? wsum[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned z = __shfl_up_sync(0xFFFFFFFFu, y, o);
      if (lane >= o) y += z;
    }
    if (lane < kWarps) wsum[lane] = y;  // inclusive over warps
  }
  __syncthreads();
  const unsigned low = (warp > 0) ? wsum[warp - 1] : 0u;
  *total = wsum[kWarps - 1];
  __syncthreads();
  return low + x - s;
}

// Block-wide: the bin where the weight counted from the top reaches K.
// Thread t holds the weights of bins [t Q, t Q + Q) in h[0..Q).  Writes the
// bin and K minus the weight of all higher bins to out[0], out[1].
template <int Q>
__device__ __forceinline__ void block_crossing(const unsigned (&h)[Q], unsigned K, unsigned* wsum, unsigned* out) {
  unsigned s = 0;
#pragma unroll
  for (int k = 0; k < Q; ++k) s += h[k];
  unsigned total = 0;
  const unsigned ex = block_prefix_excl(s, wsum, &total);
  const unsigned above = total - ex - s;
  if (above < K && K <= above + s) {
    unsigned acc = above;
#pragma unroll
    for (int k = Q - 1; k >= 0; --k) {
      if (acc < K && K <= acc + h[k]) {
        out[0] = threadIdx.x * Q + k;
        out[1] = K - acc;
      }
      acc += h[k];
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ kernel
// control-area word offsets
enum : int {
  kCtlFlag = 0, kCtlCross = 2, kCtlWsum = 8,  // kCtlWsum: kWarps words
  kCtlC = 40, kCtlSc = 41, kCtlInvSc = 42, kCtlLast = 43, kCtlExtraDense = 44, kCtlChunks = 45,
  kCtlCounts = 48,  // 2 kWarps 64-bit words: per-warp used counts
};
// the call's 64-bit count word: |S| of vector 0 in bits [39:0], finished
// blocks above
constexpr int kArrivalShift = 40;

struct KSmem {
  int* iacc;
  unsigned* chart;
  float* absv;
  unsigned* hist;
  unsigned* hist2;
  uint2* cand;
  uint4* ulst;
  unsigned short* uhead;
  float* uv;
  unsigned* utau;
  unsigned short* dlist;
  unsigned* cidx;
  unsigned short* cunit;
  unsigned* ctl;
  float* us;      // Q8: scale of each unit's row
  float* cscale;  // Q8: |scale| of each cutoff row
};

// Stored chunks of a list whose first magnitude reaches tau: the first 16
// heads come from shared memory (two 16-byte reads, compared two at a time;
// the slots past the list's stored chunks hold 0 and are not counted), any
// further ones from the prepared matrix.
__device__ __forceinline__ unsigned chunks_reaching(const HandleDesc& hd, const uint4& Lr, const unsigned short* uh,
                                                    unsigned tau, unsigned* status) {
  const uint4 ha = reinterpret_cast<const uint4*>(uh)[0], hb = reinterpret_cast<const uint4*>(uh)[1];
  const unsigned t2 = tau | (tau << 16);
  const unsigned bits = __popc(__vcmpgeu2(ha.x, t2)) + __popc(__vcmpgeu2(ha.y, t2)) + __popc(__vcmpgeu2(ha.z, t2)) +
                        __popc(__vcmpgeu2(ha.w, t2)) + __popc(__vcmpgeu2(hb.x, t2)) + __popc(__vcmpgeu2(hb.y, t2)) +
                        __popc(__vcmpgeu2(hb.z, t2)) + __popc(__vcmpgeu2(hb.w, t2));
  unsigned m = min(bits >> 4, min(Lr.y, 16u));
  for (unsigned k = 16; k < Lr.y; ++k)
    if (EFFORT_IN_RANGE(Lr.x + k < hd.total_chunks, status)) m += (hd.head[Lr.x + k] >= tau) ? 1u : 0u;
  (void)status;
  return m;
}

// V vectors per launch (1, or 2 on one matrix: the union of their prefixes is
// read once and each vector's threshold applied to it).  Per-vector state is
// held in arrays of V.
// WK: kWeightF16, or kWeightQ8 (int8 values widened to binary16 as they are
// loaded, so the masks and products below serve both; the row scale enters
// the chart, the thresholds and the unit's v).
template <int V, int WK>
__global__ void __launch_bounds__(kThreads, 1) k_effort(const __grid_constant__ Job jb) {
  constexpr bool kQ8 = WK == kWeightQ8;
  extern __shared__ __align__(128) unsigned char smem[];
  const HandleDesc& hd = jb.hd;
  const WsPtrs& ws = jb.ws;  // vector 0's scratch holds the grid barrier and the call's counters
  const int I = hd.I, O = hd.O, P = hd.P;
  const unsigned nb = gridDim.x;
  const unsigned bnb = jb.barrier_nb;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rp = rows_per_block(I, (int)nb);
  const int r0 = min(I, b * rp), r1 = min(I, r0 + rp), nr = r1 - r0;
  // the block's streaming units: panel p, rows j0, j0 + nbp, ...
  const int p = b % P;
  const int nbp = ((int)nb - 1 - p) / P + 1;
  const int j0 = b / P;
  const int nu = (j0 < I) ? (I - 1 - j0) / nbp + 1 : 0;
  const int pwid = min(kPW, O - p * kPW);
  const int stripes = (pwid + kStripe - 1) / kStripe;
  const unsigned dense_bytes = (unsigned)stripes * (kStripe * (kQ8 ? 1 : 2));
  const int mode = jb.mode;

  // per-vector arguments
  const void* vptr[V];
  float* outp[V];
  float* cutp[V];
  unsigned long long* cntp[V];
  WsPtrs wsv[V];
  unsigned long long Kv[V];
  vptr[0] = jb.v;
  outp[0] = jb.out;
  cutp[0] = jb.cutoff_out;
  cntp[0] = jb.count_out;
  wsv[0] = jb.ws;
  Kv[0] = jb.K;
  if constexpr (V > 1) {
    vptr[1] = jb.v2;
    outp[1] = jb.out2;
    cutp[1] = jb.cutoff_out2;
    cntp[1] = jb.count_out2;
    wsv[1] = jb.ws2;
    Kv[1] = jb.K2;
  }

  const SmemLayout L = smem_layout(I, (int)nb, V);
  KSmem S;
  S.iacc = reinterpret_cast<int*>(smem + L.iacc);
  S.chart = reinterpret_cast<unsigned*>(smem + L.chart);
  S.absv = reinterpret_cast<float*>(smem + L.absv);
  S.hist = reinterpret_cast<unsigned*>(smem + L.hist);
  S.hist2 = reinterpret_cast<unsigned*>(smem + L.hist2);
  S.cand = reinterpret_cast<uint2*>(smem + L.cand);
  S.ulst = reinterpret_cast<uint4*>(smem + L.ulst);
  S.uhead = reinterpret_cast<unsigned short*>(smem + L.uhead);
  S.uv = reinterpret_cast<float*>(smem + L.uv);
  S.utau = reinterpret_cast<unsigned*>(smem + L.utau);
  S.dlist = reinterpret_cast<unsigned short*>(smem + L.dlist);
  S.cidx = reinterpret_cast<unsigned*>(smem + L.cidx);
  S.cunit = reinterpret_cast<unsigned short*>(smem + L.cunit);
  S.ctl = reinterpret_cast<unsigned*>(smem + L.ctl);
  S.us = reinterpret_cast<float*>(smem + L.us);
  S.cscale = reinterpret_cast<float*>(smem + L.cscale);
  unsigned* wsum = S.ctl + kCtlWsum;
  unsigned* status = ws.hdr + kHdrStatus;
  const int chs = nr * kP;  // chart entries of one vector (the chart of vector k at S.chart + k rp kP)

  // The next call may start its prologue as soon as SMs free up.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  EFFORT_MARK(0);

  // ---- prologue: prepared-matrix data and shared memory only
  for (int e = tid; e < chs; e += kThreads) S.chart[e] = hd.probes[(size_t)r0 * kP + e];
  for (int e = tid; e < V * kBins0; e += kThreads) {
    S.hist[e] = 0u;
    reinterpret_cast<unsigned*>(S.cand)[e] = 0u;
  }
  for (int e = tid; e < kBins1 + kBins2; e += kThreads) S.hist2[e] = 0u;
  for (int e = tid; e < V * kPW; e += kThreads) S.iacc[e] = 0;
  if (tid < 256) S.ctl[tid] = 0u;
  const int nu0 = min(nu, kUnitCap);  // units of the first round
  if (mode == kModeAll) {
    // every unit is read whole from the dense copy: ask L2 for them now
    for (int u = tid; u < nu0; u += kThreads)
      if constexpr (kQ8)
        prefetch_l2_bulk(hd.wdense8 + (size_t)(j0 + u * nbp) * hd.dstride + (size_t)p * kPW, dense_bytes);
      else
        prefetch_l2_bulk(hd.wdense + (size_t)(j0 + u * nbp) * hd.dstride + (size_t)p * kPW, dense_bytes);
  }
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  EFFORT_MARK(1);
  // the barrier counter stands at base (a multiple of nb) plus the arrivals of
  // blocks already at this call's first barrier (fewer than nb)
  const unsigned long long bar_base = (__ldcg(ws.bar) / nb) * nb;
  int nbar = 0;  // grid barriers of this call so far
  // the last-call byte words start over (the blocks add to them at the end,
  // after at least one grid barrier)
  if (b == 0 && tid == 0 && !jb.accumulate_bytes) {
    unsigned long long* last = reinterpret_cast<unsigned long long*>(ws.hdr + kHdrBytesLast);
    last[0] = 0ull;
    last[1] = 0ull;
  }

  const int oc0 = (int)((long long)O * b / nb), oc1 = (int)((long long)O * (b + 1) / nb);  // this block's columns

  // ---- nothing is used: zero outputs, no grid-wide work (one vector only)
  if (mode == kModeNone) {
    for (int j = oc0 + tid; j < oc1; j += kThreads) {
      jb.out[j] = 0.0f;
      if (jb.out_mirror) jb.out_mirror[j] = 0.0f;
    }
    if (jb.rowlen_out)
      for (int i = r0 + tid; i < r1; i += kThreads) jb.rowlen_out[i] = 0u;
    if (b == 0 && tid == 0) {
      if (jb.cutoff_out) *jb.cutoff_out = __int_as_float(0x7F800000);
      if (jb.count_out) *jb.count_out = 0ull;
    }
    return;
  }

  // out is accumulated with reductions after the next grid barrier: clear
  // this block's columns now.  |v| of the cutoff rows (non-finite entries
  // are flagged) and their sum over the grid, which with the largest |w|
  // bounds every partial sum of out; v of the streaming rows.
#pragma unroll
  for (int k = 0; k < V; ++k) {
    for (int j = oc0 + tid; j < oc1; j += kThreads) outp[k][j] = 0.0f;
    const float* vf = reinterpret_cast<const float*>(vptr[k]);
    const __half* vh = reinterpret_cast<const __half*>(vptr[k]);
    for (int u = tid; u < nu0; u += kThreads) {
      const int i = j0 + u * nbp;
      S.uv[k * kUnitCap + u] = jb.vdtype ? __half2float(vh[i]) : vf[i];
      if constexpr (kQ8)
        if (k == 0) S.us[u] = h2f(hd.scales[i]);
    }
    for (int t0 = 0; t0 < nr; t0 += kThreads) {
      const int t = t0 + tid;
      float ax = 0.0f;
      if (t < nr) {
        const float x = jb.vdtype ? __half2float(vh[r0 + t]) : vf[r0 + t];
        if (!isfinite(x)) atomicOr(status, kStatusNonfiniteV);
        ax = fabsf(x);
        S.absv[k * rp + t] = ax;
        if constexpr (kQ8)
          if (k == 0) S.cscale[t] = fabsf(h2f(hd.scales[r0 + t]));
        if (k == 0 && jb.rowlen_out) jb.rowlen_out[r0 + t] = (mode == kModeAll) ? (unsigned)hd.n : 0u;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ax += __shfl_xor_sync(0xFFFFFFFFu, ax, o);
      if (lane == 0 && ax != 0.0f) atomicAdd(reinterpret_cast<float*>(wsv[k].hdr + kHdrVsum), ax);
    }
  }
  __syncthreads();

  float c[V];
  unsigned vsum_bits[V], b1[V], K1[V];  // b1, K1: crossing bin of the first digit, rank left inside it
#pragma unroll
  for (int k = 0; k < V; ++k) {
    c[k] = 0.0f;
    vsum_bits[k] = b1[k] = K1[k] = 0u;
  }
  if (mode == kModeSelect) {
    // ---- phase 1: charts, first-digit histograms, entries grouped by bin
    unsigned* hcnt = reinterpret_cast<unsigned*>(S.cand);  // [V][kBins0] entries per bin, then (start << 16) | count
    unsigned short* rank = reinterpret_cast<unsigned short*>(S.cidx);  // [V][chs] entry's place inside its bin
    // entry e is probe e mod kP of its row, and kThreads is a multiple of kP:
    // every entry this thread visits has the same probe weight
    const unsigned w = (unsigned)hd.pw[tid & (kP - 1)];
    if (w)
      for (int e = tid; e < chs; e += kThreads) {
        const unsigned pb = S.chart[e];  // probe bits, replaced by vector 0's chart
#pragma unroll
        for (int k = V - 1; k >= 0; --k) {
          const float pm = kQ8 ? __fmul_rn(S.cscale[e >> 4], h2f(pb)) : h2f(pb);  // probe |w| (exact)
          const unsigned xb = __float_as_uint(__fmul_rn(S.absv[k * rp + (e >> 4)], pm));
          S.chart[k * rp * kP + e] = xb;
          atomicAdd(&S.hist[k * kBins0 + (xb >> 19)], w);
          rank[k * chs + e] = (unsigned short)atomicAdd(&hcnt[k * kBins0 + (xb >> 19)], 1u);
        }
      }
    else
      for (int e = tid; e < chs; e += kThreads) {
        const unsigned pb = S.chart[e];
#pragma unroll
        for (int k = V - 1; k >= 0; --k)
          S.chart[k * rp * kP + e] = __float_as_uint(
              __fmul_rn(S.absv[k * rp + (e >> 4)], kQ8 ? __fmul_rn(S.cscale[e >> 4], h2f(pb)) : h2f(pb)));
      }
    __syncthreads();
    // each bin's first slot in the block's segment (bins in ascending order)
#pragma unroll
    for (int k = 0; k < V; ++k) {
      constexpr int kQ0 = kBins0 / kThreads;
      unsigned cq[kQ0], sum = 0, total = 0;
#pragma unroll
      for (int q = 0; q < kQ0; ++q) {
        cq[q] = hcnt[k * kBins0 + tid * kQ0 + q];
        sum += cq[q];
      }
      unsigned at = block_prefix_excl(sum, wsum, &total);
#pragma unroll
      for (int q = 0; q < kQ0; ++q) {
        hcnt[k * kBins0 + tid * kQ0 + q] = (at << 16) | cq[q];
        at += cq[q];
      }
    }
    __syncthreads();
    // the weighted entries into the block's segment, grouped by bin (the
    // order inside a bin is the order of the counting atomics; it does not
    // matter), then the global histogram and this block's bin descriptors
    if (w)
      for (int e = tid; e < chs; e += kThreads)
#pragma unroll
        for (int k = 0; k < V; ++k) {
          const unsigned xb = S.chart[k * rp * kP + e];
          const unsigned slot = (hcnt[k * kBins0 + (xb >> 19)] >> 16) + rank[k * chs + e];
          wsv[k].seg[(size_t)b * rp * kP + slot] = make_uint2(xb, w);
        }
#pragma unroll
    for (int k = 0; k < V; ++k)
      for (int e = tid; e < kBins0; e += kThreads) {
        const unsigned h = S.hist[k * kBins0 + e];
        if (h) {
          atomicAdd(&wsv[k].ghist0[e], h);
          wsv[k].desc[(size_t)e * nb + b] = hcnt[k * kBins0 + e];
        }
      }
    EFFORT_MARK(2);
    __syncthreads();
    if (tid == 0) grid_arrive_thread(ws.bar);
    ++nbar;
    // while B1 fills (thread 0 waits): the first round's list records and the
    // first 16 stored chunks' first magnitudes of each
    if (warp > 0) {
      for (int u = tid - 32; u < nu0; u += kThreads - 32) S.ulst[u] = hd.lst[(size_t)(j0 + u * nbp) * P + p];
      // warps 1.. only (named barrier 1): 16 consecutive threads read one unit's heads
      asm volatile("bar.sync 1, %0;" ::"r"(kThreads - 32) : "memory");
      for (int e = tid - 32; e < nu0 * 16; e += kThreads - 32) {
        const uint4 Lr = S.ulst[e >> 4];
        const unsigned k = (unsigned)(e & 15);
        S.uhead[e] = (k < Lr.y && EFFORT_IN_RANGE(Lr.x + k < hd.total_chunks, status)) ? hd.head[Lr.x + k]
                                                                                        : (unsigned short)0;
      }
    }
    if (tid == 0)
      S.ctl[kCtlFlag] = grid_wait_thread(ws.bar, bar_base + (unsigned long long)nbar * bnb, status) ? 1u : 0u;
    __syncthreads();
    if (!S.ctl[kCtlFlag]) return;
    EFFORT_MARK(3);

    // ---- phase 2: crossing bins
#pragma unroll
    for (int k = 0; k < V; ++k) {
      constexpr int kQ0 = kBins0 / kThreads;
      unsigned h0[kQ0];
      vsum_bits[k] = __ldcg(wsv[k].hdr + kHdrVsum);
#pragma unroll
      for (int q = 0; q < kQ0; ++q) h0[q] = __ldcg(&wsv[k].ghist0[tid * kQ0 + q]);
      block_crossing<kQ0>(h0, (unsigned)Kv[k], wsum, S.ctl + kCtlCross);
      b1[k] = S.ctl[kCtlCross];
      K1[k] = S.ctl[kCtlCross + 1];
    }
    // every block's descriptor of the crossing bin (thread t: block t's)
    unsigned dsc[V];
#pragma unroll
    for (int k = 0; k < V; ++k) dsc[k] = ((unsigned)tid < nb) ? __ldcg(&wsv[k].desc[(size_t)b1[k] * nb + tid]) : 0u;
    // this block's descriptors of the other bins are read by nobody: clear
    // them for the next call (the crossing bin's row is cleared by the last
    // block)
#pragma unroll
    for (int k = 0; k < V; ++k)
      for (int e = tid; e < kBins0; e += kThreads)
        if (S.hist[k * kBins0 + e] && (unsigned)e != b1[k]) wsv[k].desc[(size_t)e * nb + b] = 0u;
    EFFORT_MARK(4);

    // ---- phase 3: bits [18:0] of each c
#pragma unroll
    for (int k = 0; k < V; ++k) {
      const WsPtrs& w_ = wsv[k];
      unsigned* h1 = S.hist2;           // [kBins1]
      unsigned* h2 = S.hist2 + kBins1;  // [kBins2]
      const unsigned* chart = S.chart + k * rp * kP;
      unsigned b2 = 0, b3 = 0;
      if (k > 0) {
        // the digit histograms of the previous vector start over
        __syncthreads();
        for (int e = tid; e < kBins1 + kBins2; e += kThreads) S.hist2[e] = 0u;
        __syncthreads();
      }
      // the crossing bin's entries, from the blocks' segments through their
      // descriptors
      unsigned* gpos = reinterpret_cast<unsigned*>(S.cunit);  // [nb + 1] first candidate of each block
      unsigned* gsrc = gpos + (nb + 1);                        // [nb] its first slot in the block's segment
      unsigned M = 0;
      const unsigned at = block_prefix_excl(dsc[k] & 0xFFFFu, wsum, &M);
      if ((unsigned)tid < nb) {
        gpos[tid] = at;
        gsrc[tid] = dsc[k] >> 16;
      }
      if (tid == 0) gpos[nb] = M;
      __syncthreads();
      if (M <= (unsigned)kCandCap) {
        for (unsigned e0 = 0; e0 < M; e0 += 4 * kThreads) {
          uint2 t4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const unsigned e = e0 + q * kThreads + tid;
            t4[q] = make_uint2(0u, 0u);
            if (e < M) {
              // the block holding candidate e: the last one whose first candidate is <= e
              unsigned lo = 0, hi = nb - 1;
              while (lo < hi) {
                const unsigned mid = (lo + hi + 1) >> 1;
                if (gpos[mid] <= e) lo = mid;
                else hi = mid - 1;
              }
              const unsigned slot = gsrc[lo] + (e - gpos[lo]);
              if (EFFORT_IN_RANGE(slot < (unsigned)(rp * kP), status))
                t4[q] = __ldcg(&w_.seg[(size_t)lo * rp * kP + slot]);
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const unsigned e = e0 + q * kThreads + tid;
            if (e < M) S.cand[e] = t4[q];
          }
        }
        EFFORT_MARK(5);
        __syncthreads();
        for (unsigned e = tid; e < M; e += kThreads) atomicAdd(&h1[(S.cand[e].x >> 9) & (kBins1 - 1)], S.cand[e].y);
        __syncthreads();
        {
          unsigned hq[kBins1 / kThreads];
#pragma unroll
          for (int q = 0; q < kBins1 / kThreads; ++q) hq[q] = h1[tid * (kBins1 / kThreads) + q];
          block_crossing<kBins1 / kThreads>(hq, K1[k], wsum, S.ctl + kCtlCross);
        }
        b2 = S.ctl[kCtlCross];
        const unsigned K2 = S.ctl[kCtlCross + 1];
        for (unsigned e = tid; e < M; e += kThreads) {
          const unsigned xb = S.cand[e].x;
          if (((xb >> 9) & (kBins1 - 1)) == b2) atomicAdd(&h2[xb & (kBins2 - 1)], S.cand[e].y);
        }
        __syncthreads();
        {
          unsigned hq[kBins2 / kThreads];
#pragma unroll
          for (int q = 0; q < kBins2 / kThreads; ++q) hq[q] = h2[tid * (kBins2 / kThreads) + q];
          block_crossing<kBins2 / kThreads>(hq, K2, wsum, S.ctl + kCtlCross);
        }
        b3 = S.ctl[kCtlCross];
      } else {
        // too many candidates for one block: two more grid-wide histogram passes
        for (int e = tid; e < chs; e += kThreads) {
          const unsigned xb = chart[e];
          if (w && (xb >> 19) == b1[k]) atomicAdd(&h1[(xb >> 9) & (kBins1 - 1)], w);
        }
        __syncthreads();
        for (int e = tid; e < kBins1; e += kThreads)
          if (h1[e]) atomicAdd(&w_.ghist1[e], h1[e]);
        if (!grid_barrier_block(ws.bar, bar_base + (unsigned long long)(++nbar) * bnb, status, &S.ctl[kCtlFlag]))
          return;
        {
          unsigned hq[kBins1 / kThreads];
#pragma unroll
          for (int q = 0; q < kBins1 / kThreads; ++q) hq[q] = __ldcg(&w_.ghist1[tid * (kBins1 / kThreads) + q]);
          block_crossing<kBins1 / kThreads>(hq, K1[k], wsum, S.ctl + kCtlCross);
        }
        b2 = S.ctl[kCtlCross];
        const unsigned K2 = S.ctl[kCtlCross + 1];
        for (int e = tid; e < chs; e += kThreads) {
          const unsigned xb = chart[e];
          if (w && (xb >> 19) == b1[k] && ((xb >> 9) & (kBins1 - 1)) == b2) atomicAdd(&h2[xb & (kBins2 - 1)], w);
        }
        __syncthreads();
        for (int e = tid; e < kBins2; e += kThreads)
          if (h2[e]) atomicAdd(&w_.ghist2[e], h2[e]);
        if (!grid_barrier_block(ws.bar, bar_base + (unsigned long long)(++nbar) * bnb, status, &S.ctl[kCtlFlag]))
          return;
        // ghist1 is read by nobody any more
        if (b == 0)
          for (int e = tid; e < kBins1; e += kThreads) w_.ghist1[e] = 0u;
        {
          unsigned hq[kBins2 / kThreads];
#pragma unroll
          for (int q = 0; q < kBins2 / kThreads; ++q) hq[q] = __ldcg(&w_.ghist2[tid * (kBins2 / kThreads) + q]);
          block_crossing<kBins2 / kThreads>(hq, K2, wsum, S.ctl + kCtlCross);
        }
        b3 = S.ctl[kCtlCross];
      }
      c[k] = __uint_as_float((b1[k] << 19) | (b2 << 9) | b3);
      if (b == 0 && tid == 0 && cutp[k]) *cutp[k] = c[k];
    }
    // c = 0: every kept product is used (fillers, pads and dropped weights add +0)
    if (c[0] == 0.0f && jb.rowlen_out)
      for (int t = tid; t < nr; t += kThreads) jb.rowlen_out[r0 + t] = (unsigned)hd.n;
  } else {
    // every (row, panel) is read whole: the cleared out must be complete
    // before any block adds to it
    if (!grid_barrier_block(ws.bar, bar_base + (unsigned long long)(++nbar) * bnb, status, &S.ctl[kCtlFlag])) return;
    vsum_bits[0] = __ldcg(ws.hdr + kHdrVsum);
    if (b == 0 && tid == 0 && jb.cutoff_out) *jb.cutoff_out = 0.0f;
  }
  EFFORT_MARK(6);

  // fixed-point unit of each accumulator: 2^-s with every partial sum below
  // 2^30 units (|sum| <= sum |v_i| max |w| < bound / 2)
  float sc[V], inv_sc[V];
  bool count_all[V];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    sc[k] = 1.0f;
    inv_sc[k] = 1.0f;
    const float wmax = kQ8 ? __uint_as_float(hd.wmax_bits) : h2f(hd.wmax_bits);  // largest kept |w|
    const float bound = 2.0f * __uint_as_float(vsum_bits[k]) * wmax;
    if (bound > 0.0f && isfinite(bound)) {
      int ex = 0;
      frexpf(bound, &ex);  // bound < 2^ex
      const int sh = max(-120, min(120, 30 - ex));
      sc[k] = ldexpf(1.0f, sh);
      inv_sc[k] = ldexpf(1.0f, -sh);
    }
    count_all[k] = mode == kModeAll || c[k] == 0.0f;
  }
  const bool want_rowlen = V == 1 && jb.rowlen_out != nullptr && !count_all[0];

  float2 acc[V][4];
#pragma unroll
  for (int k = 0; k < V; ++k)
#pragma unroll
    for (int m = 0; m < 4; ++m) acc[k][m] = make_float2(0.0f, 0.0f);
  unsigned long long my_count[V];
#pragma unroll
  for (int k = 0; k < V; ++k) my_count[k] = 0;
  unsigned long long planned_dense = 0, planned_sparse = 0;  // thread 0
  const int sj = warp & 7, half = warp >> 3;                 // dense: stripe, units k = half mod 2
  const int g8 = lane >> 3, sl = lane & 7;                   // sparse: lane group, slot octet

  for (int u0 = 0; u0 < nu; u0 += kUnitCap) {
    const int nuR = min(kUnitCap, nu - u0);
    if (u0 > 0) {
      // later rounds: this round's records and v
      __syncthreads();
      if (mode == kModeSelect) {
        for (int u = tid; u < nuR; u += kThreads) S.ulst[u] = hd.lst[(size_t)(j0 + (u0 + u) * nbp) * P + p];
        __syncthreads();
        for (int e = tid; e < nuR * 16; e += kThreads) {
          const uint4 Lr = S.ulst[e >> 4];
          const unsigned k = (unsigned)(e & 15);
          S.uhead[e] = (k < Lr.y && EFFORT_IN_RANGE(Lr.x + k < hd.total_chunks, status)) ? hd.head[Lr.x + k]
                                                                                            : (unsigned short)0;
        }
      }
#pragma unroll
      for (int k = 0; k < V; ++k) {
        const float* vf = reinterpret_cast<const float*>(vptr[k]);
        const __half* vh = reinterpret_cast<const __half*>(vptr[k]);
        for (int u = tid; u < nuR; u += kThreads) {
          const int i = j0 + (u0 + u) * nbp;
          S.uv[k * kUnitCap + u] = jb.vdtype ? __half2float(vh[i]) : vf[i];
          if constexpr (kQ8)
            if (k == 0) S.us[u] = h2f(hd.scales[i]);
        }
      }
      if (tid == 0) S.ctl[kCtlExtraDense] = 0u;
      __syncthreads();
    }
    // ---- dispatch (one unit per thread): each vector's threshold tau_i(c),
    // the smallest fp16 magnitude m with fl32(|v_i| m) >= c; the unit is
    // skipped (nothing reaches the lowest threshold), read dense (the stored
    // part of its list does not reach it) or read as the stored chunks whose
    // first magnitude reaches it: the union of the vectors' prefixes
    const int u = tid;
    unsigned kind = 0, m = 0, first = 0;  // kind: 0 none, 1 dense, 2 sparse
    if (u < nuR) {
      unsigned tmin = 0x7C00u;
      bool all = false;
#pragma unroll
      for (int k = 0; k < V; ++k) {
        unsigned tau = 0u;
        if (count_all[k]) {
          all = true;
        } else {
          if constexpr (kQ8)
            tau = tau_q8(fabsf(S.uv[k * kUnitCap + u]), fabsf(S.us[u]), c[k]);
          else
            tau = tau_of(fabsf(S.uv[k * kUnitCap + u]), c[k]);
          tmin = min(tmin, tau);
        }
        S.utau[k * kUnitCap + u] = tau;
        if constexpr (kQ8) S.uv[k * kUnitCap + u] = __fmul_rn(S.uv[k * kUnitCap + u], S.us[u]);  // v_i s_i
      }
      if (all) {
        kind = 1;
      } else {
        const uint4 Lr = S.ulst[u];  // {first chunk, stored chunks, tail, kept}
        first = Lr.x;
        if (Lr.w != 0u && tmin < 0x7C00u) {
          if (Lr.z >= tmin && Lr.z != 0u) {
            kind = 1;
          } else {
            m = chunks_reaching(hd, Lr, S.uhead + u * 16, tmin, status);
            kind = m ? 2u : 0u;
          }
        }
      }
    }
    unsigned tot = 0;
    const unsigned pos = block_prefix_excl((kind == 1 ? (1u << 16) : 0u) | (kind == 2 ? m : 0u), wsum, &tot);
    const unsigned nd0 = tot >> 16;
    if (tid == 0) S.ctl[kCtlChunks] = min(tot & 0xFFFFu, (unsigned)kChunkCap);
    __syncthreads();
    if (kind == 2) {
      const unsigned cp = pos & 0xFFFFu;
      if (cp + m <= (unsigned)kChunkCap) {
        for (unsigned t = 0; t < m; ++t) {
          S.cidx[cp + t] = first + t;
          S.cunit[cp + t] = (unsigned short)u;
        }
      } else {
        // past the round's chunk capacity: read this unit dense instead
        atomicMin(&S.ctl[kCtlChunks], cp);
        kind = 1;
        S.dlist[nd0 + atomicAdd(&S.ctl[kCtlExtraDense], 1u)] = (unsigned short)u;
      }
    }
    if (kind == 1 && (pos >> 16) < nd0 && m == 0) S.dlist[pos >> 16] = (unsigned short)u;
    __syncthreads();
    const unsigned nd = nd0 + S.ctl[kCtlExtraDense];
    const unsigned nch = S.ctl[kCtlChunks];
    if (tid == 0) {
      planned_dense += (unsigned long long)nd * dense_bytes;
      planned_sparse += (unsigned long long)nch * (unsigned)(kCS * (kQ8 ? 2 : 3));
    }
    EFFORT_MARK(7);

    // ---- multiply: dense units, warp (stripe sj, half) takes units k = half,
    // half + 2, ... of the dense list, kDenseBatch loads in flight per lane
    if constexpr (V == 1) {
      if (sj < stripes) {
        const size_t lane_off = (size_t)p * kPW + sj * kStripe + 8 * lane;
        const uint16_t* base = hd.wdense + lane_off;
        const int8_t* base8 = hd.wdense8 + lane_off;
        for (unsigned k0 = (unsigned)half; k0 < nd; k0 += 2 * kDenseBatch) {
          uint4 wv[kDenseBatch];
          unsigned tq[kDenseBatch];
          float vq[kDenseBatch];
          int iq[kDenseBatch];
#pragma unroll
          for (int q = 0; q < kDenseBatch; ++q) {
            const unsigned k = k0 + 2 * q;
            wv[q] = make_uint4(0u, 0u, 0u, 0u);
            tq[q] = 0x7C00u;
            vq[q] = 0.0f;
            iq[q] = 0;
            if (k < nd) {
              const unsigned uu = S.dlist[k];
              const int i = j0 + (u0 + (int)uu) * nbp;
              if constexpr (kQ8) {
                const uint2 r = __ldcs(reinterpret_cast<const uint2*>(base8 + (size_t)i * hd.dstride));
                wv[q].x = r.x;
                wv[q].y = r.y;
              } else {
                wv[q] = __ldcs(reinterpret_cast<const uint4*>(base + (size_t)i * hd.dstride));
              }
              tq[q] = S.utau[uu];
              vq[q] = S.uv[uu];
              iq[q] = i;
            }
          }
#pragma unroll
          for (int q = 0; q < kDenseBatch; ++q) {
            const unsigned tau2 = tq[q] | (tq[q] << 16);
            const float2 v2 = make_float2(vq[q], vq[q]);
            if constexpr (kQ8) wv[q] = widen_q8(wv[q].x, wv[q].y);
            const unsigned w4[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
            unsigned rc = 0;
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
              const unsigned msk = ge_mask(w4[mm], tau2);
              rc += __popc(msk);
              const unsigned wm = w4[mm] & msk;
              const float2 wf = __half22float2(*reinterpret_cast<const __half2*>(&wm));
              acc[0][mm] = __ffma2_rn(v2, wf, acc[0][mm]);
            }
            my_count[0] += rc >> 4;
            if (want_rowlen) {
              unsigned r = rc >> 4;
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
              if (lane == 0 && r) atomicAdd(&jb.rowlen_out[iq[q]], r);
            }
          }
        }
      }
    } else {
      // two vectors: one load of each unit, each vector's mask and FMA
    if (sj < stripes) {
      const size_t lane_off = (size_t)p * kPW + sj * kStripe + 8 * lane;
      const uint16_t* base = hd.wdense + lane_off;
      const int8_t* base8 = hd.wdense8 + lane_off;
      for (unsigned k0 = (unsigned)half; k0 < nd; k0 += 2 * kDenseBatch) {
        uint4 wv[kDenseBatch];
        unsigned uq[kDenseBatch];
#pragma unroll
        for (int q = 0; q < kDenseBatch; ++q) {
          const unsigned k = k0 + 2 * q;
          wv[q] = make_uint4(0u, 0u, 0u, 0u);
          uq[q] = 0xFFFFu;
          if (k < nd) {
            uq[q] = S.dlist[k];
            const size_t roff = (size_t)(j0 + (u0 + (int)uq[q]) * nbp) * hd.dstride;
            if constexpr (kQ8) {
              const uint2 r = __ldcs(reinterpret_cast<const uint2*>(base8 + roff));
              wv[q].x = r.x;
              wv[q].y = r.y;
            } else {
              wv[q] = __ldcs(reinterpret_cast<const uint4*>(base + roff));
            }
          }
        }
#pragma unroll
        for (int q = 0; q < kDenseBatch; ++q) {
          const bool okq = uq[q] != 0xFFFFu;
          if constexpr (kQ8) wv[q] = widen_q8(wv[q].x, wv[q].y);
          const unsigned w4[4] = {wv[q].x, wv[q].y, wv[q].z, wv[q].w};
#pragma unroll
          for (int k = 0; k < V; ++k) {
            const unsigned tau = okq ? S.utau[k * kUnitCap + uq[q]] : 0x7C00u;
            const float vi = okq ? S.uv[k * kUnitCap + uq[q]] : 0.0f;
            const unsigned tau2 = tau | (tau << 16);
            const float2 v2 = make_float2(vi, vi);
            unsigned rc = 0;
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
              const unsigned msk = ge_mask(w4[mm], tau2);
              rc += __popc(msk);
              const unsigned wm = w4[mm] & msk;
              const float2 wf = __half22float2(*reinterpret_cast<const __half2*>(&wm));
              acc[k][mm] = __ffma2_rn(v2, wf, acc[k][mm]);
            }
            my_count[k] += rc >> 4;
            if (want_rowlen) {
              unsigned r = rc >> 4;
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
              if (lane == 0 && r && okq) atomicAdd(&jb.rowlen_out[j0 + (u0 + (int)uq[q]) * nbp], r);
            }
          }
        }
      }
    }
    }
    EFFORT_MARK_LANE0(8);

    // ---- multiply: sparse chunks, lane group (warp, g8) takes chunks
    // 4 warp + g8 + 64 j; 8 lanes per chunk, 8 slots per lane
    for (unsigned t0 = (unsigned)(warp * 4); t0 < nch; t0 += 64u * kSparseBatch) {
      uint4 vv[kSparseBatch];
      uint2 gg[kSparseBatch];
      unsigned uq[kSparseBatch];
#pragma unroll
      for (int q = 0; q < kSparseBatch; ++q) {
        const unsigned t = t0 + (unsigned)g8 + 64u * q;
        vv[q] = make_uint4(0u, 0u, 0u, 0u);
        gg[q] = make_uint2(0u, 0u);
        uq[q] = 0xFFFFu;
        if (t < nch) {
          const unsigned ci = S.cidx[t];
          if (EFFORT_IN_RANGE(ci < hd.total_chunks, status)) {
            uq[q] = S.cunit[t];
            if constexpr (kQ8) {
              const uint2 r = __ldcs(reinterpret_cast<const uint2*>(hd.vals8 + (size_t)ci * kCS) + sl);
              vv[q].x = r.x;
              vv[q].y = r.y;
            } else {
              vv[q] = __ldcs(reinterpret_cast<const uint4*>(hd.vals + (size_t)ci * kCS) + sl);
            }
            gg[q] = __ldcs(reinterpret_cast<const uint2*>(hd.gaps + (size_t)ci * kCS) + sl);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kSparseBatch; ++q) {
        const bool ok = uq[q] != 0xFFFFu;
        // gaps to columns: inclusive sums inside the lane, exclusive across the 8 lanes
        int cs[8];
        cs[0] = (int)(gg[q].x & 0xFFu);
        cs[1] = cs[0] + (int)((gg[q].x >> 8) & 0xFFu);
        cs[2] = cs[1] + (int)((gg[q].x >> 16) & 0xFFu);
        cs[3] = cs[2] + (int)(gg[q].x >> 24);
        cs[4] = cs[3] + (int)(gg[q].y & 0xFFu);
        cs[5] = cs[4] + (int)((gg[q].y >> 8) & 0xFFu);
        cs[6] = cs[5] + (int)((gg[q].y >> 16) & 0xFFu);
        cs[7] = cs[6] + (int)(gg[q].y >> 24);
        int ex = cs[7];
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          const int y = __shfl_up_sync(0xFFFFFFFFu, ex, o, 8);
          if (sl >= o) ex += y;
        }
        const int basecol = ex - cs[7] - 1;
        if constexpr (kQ8) vv[q] = widen_q8(vv[q].x, vv[q].y);
        const unsigned w4[4] = {vv[q].x, vv[q].y, vv[q].z, vv[q].w};
#pragma unroll
        for (int k = 0; k < V; ++k) {
          const unsigned tau = ok ? S.utau[k * kUnitCap + uq[q]] : 0x7C00u;
          const float vi = ok ? S.uv[k * kUnitCap + uq[q]] : 0.0f;
          const unsigned tau2 = tau | (tau << 16);
          int* iacc = S.iacc + k * kPW;
          unsigned rc = 0;
          if (ok) {
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
              const unsigned msk = ge_mask(w4[mm], tau2);
              const int ca = basecol + cs[2 * mm], cb = basecol + cs[2 * mm + 1];
              if ((msk & 0xFFFFu) && EFFORT_IN_RANGE((unsigned)ca < (unsigned)kPW, status)) {
                atomicAdd(&iacc[ca], __float2int_rn(__fmul_rn(vi, h2f(w4[mm] & 0xFFFFu)) * sc[k]));
                ++rc;
              }
              if ((msk & 0xFFFF0000u) && EFFORT_IN_RANGE((unsigned)cb < (unsigned)kPW, status)) {
                atomicAdd(&iacc[cb], __float2int_rn(__fmul_rn(vi, h2f(w4[mm] >> 16)) * sc[k]));
                ++rc;
              }
            }
          }
          my_count[k] += rc;
          if (want_rowlen) {
            unsigned r = rc;
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o, 8);
            if (ok && sl == 0 && r) atomicAdd(&jb.rowlen_out[j0 + (u0 + (int)uq[q]) * nbp], r);
          }
        }
      }
    }
    EFFORT_MARK_LANE0(9);
    __syncthreads();
  }

  // dense registers into the panel accumulators (fixed point)
  if (sj < stripes) {
    const int cl = sj * kStripe + 8 * lane;
#pragma unroll
    for (int k = 0; k < V; ++k)
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {
        const int qx = __float2int_rn(acc[k][mm].x * sc[k]), qy = __float2int_rn(acc[k][mm].y * sc[k]);
        if (qx) atomicAdd(&S.iacc[k * kPW + cl + 2 * mm], qx);
        if (qy) atomicAdd(&S.iacc[k * kPW + cl + 2 * mm + 1], qy);
      }
  }
  __syncthreads();
  EFFORT_MARK(10);

  // this block's panel sums, added into out (float4 reductions)
  if (nu > 0) {
#pragma unroll
    for (int k = 0; k < V; ++k) {
      float* dst = outp[k] + (size_t)p * kPW;
      const int* ia = S.iacc + k * kPW;
      if (((uintptr_t)outp[k] & 15u) == 0) {
        for (int j = tid; j < pwid / 4; j += kThreads) {
          const int4 q = reinterpret_cast<const int4*>(ia)[j];
          if (q.x | q.y | q.z | q.w)
            atomicAdd(reinterpret_cast<float4*>(dst) + j,
                      make_float4((float)q.x * inv_sc[k], (float)q.y * inv_sc[k], (float)q.z * inv_sc[k],
                                  (float)q.w * inv_sc[k]));
        }
        for (int j = pwid / 4 * 4 + tid; j < pwid; j += kThreads)
          if (ia[j]) atomicAdd(dst + j, (float)ia[j] * inv_sc[k]);
      } else {
        for (int j = tid; j < pwid; j += kThreads)
          if (ia[j]) atomicAdd(dst + j, (float)ia[j] * inv_sc[k]);
      }
    }
  }
  EFFORT_MARK(11);

  // ---- used counts and planned bytes.  The block's count of vector 0 and
  // its arrival go into one 64-bit counter (arrivals in bits [63:40]), so
  // the block that arrives last gets the total with its own atomic; the
  // planned bytes go straight into the last-call words (cleared before the
  // first barrier unless the call accumulates them).
  unsigned long long* wcnt = reinterpret_cast<unsigned long long*>(S.ctl + kCtlCounts);  // [V][kWarps]
#pragma unroll
  for (int k = 0; k < V; ++k) {
    unsigned long long x = my_count[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    if (lane == 0) wcnt[k * kWarps + warp] = count_all[k] ? 0ull : x;
  }
  if (tid == 0) {
    unsigned long long* last = reinterpret_cast<unsigned long long*>(ws.hdr + kHdrBytesLast);
    if (planned_dense) atomicAdd(last, planned_dense);
    if (planned_sparse) atomicAdd(last + 1, planned_sparse);
  }
  __syncthreads();
  if (tid == 0) {
    unsigned long long mine[V];
#pragma unroll
    for (int k = 0; k < V; ++k) {
      mine[k] = 0ull;
      for (int q = 0; q < kWarps; ++q) mine[k] += wcnt[k * kWarps + q];
    }
#pragma unroll
    for (int k = 1; k < V; ++k)
      if (mine[k]) atomicAdd(wsv[k].count, mine[k]);
    __threadfence();
    const unsigned long long add = (1ull << kArrivalShift) | mine[0];
    const unsigned long long before = atomicAdd(ws.count, add);
    const bool is_last = (before >> kArrivalShift) == (unsigned long long)(nb - 1u);
    S.ctl[kCtlLast] = is_last ? 1u : 0u;
    if (is_last) {
      __threadfence();
      const unsigned long long total0 = (before + add) & ((1ull << kArrivalShift) - 1ull);
#pragma unroll
      for (int k = 0; k < V; ++k) {
        const unsigned long long cnt = count_all[k] ? hd.kept_total : (k == 0 ? total0 : __ldcg(wsv[k].count));
        if (cntp[k]) *cntp[k] = cnt;
        *wsv[k].count = 0ull;
        wsv[k].hdr[kHdrVsum] = 0u;
      }
    }
  }
  __syncthreads();
  if (S.ctl[kCtlLast]) {
    __threadfence();
    // the first-digit histograms, the crossing bins' descriptors and the last
    // digit's histograms of the many-candidates path are read by nobody any more
    if (mode == kModeSelect)
#pragma unroll
      for (int k = 0; k < V; ++k) {
        for (int e = tid; e < kBins0; e += kThreads) wsv[k].ghist0[e] = 0u;
        for (int e = tid; e < (int)nb; e += kThreads) wsv[k].desc[(size_t)b1[k] * nb + e] = 0u;
        for (int e = tid; e < kBins2; e += kThreads) wsv[k].ghist2[e] = 0u;
      }
    // every block has added its sums: the finished out to host memory
    if (jb.out_mirror)
      for (int j = tid; j < O; j += kThreads) jb.out_mirror[j] = __ldcg(jb.out + j);
  }
  EFFORT_MARK(13);
}

// ------------------------------------------------------------------ launch
size_t effort_smem_bytes(int I, int nb) { return smem_layout(I, nb, 2).total; }  // covers both forms

// The kernel may take up to the device's opt-in shared memory per block: the
// attribute is a per-function setting, so it must cover every prepared
// geometry at once (the one a later effort_prepare needs may be smaller).
cudaError_t effort_kernel_attributes(int I, size_t smem) {
  (void)I;
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  if ((size_t)optin < smem) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(k_effort<1, kWeightF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_effort<2, kWeightF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_effort<1, kWeightQ8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_effort<2, kWeightQ8>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  return e;
}

// Blocks of a launch that can all be resident at once: one per SM.
int effort_grid_size(int I, int sms, size_t smem) {
  (void)I;
  int nbk = 0;
  // every instantiation must fit one block per SM
  const void* fns[4] = {(const void*)k_effort<1, kWeightF16>, (const void*)k_effort<2, kWeightF16>,
                        (const void*)k_effort<1, kWeightQ8>, (const void*)k_effort<2, kWeightQ8>};
  for (const void* f : fns) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nbk, f, kThreads, smem) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    if (nbk < 1) return 0;
  }
  return sms;
}

// One matvec (nvec = 1) or two on one matrix (nvec = 2, job.v2 ...).  smem is
// the handle's size, which covers the two-vector layout.
cudaError_t launch_effort(const Job& job, int nb, size_t smem, cudaStream_t stream, int nvec) {
  (void)smem;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nb);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_layout(job.hd.I, nb, nvec).total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (job.hd.wk == kWeightQ8)
    return nvec == 2 ? cudaLaunchKernelEx(&cfg, k_effort<2, kWeightQ8>, job)
                     : cudaLaunchKernelEx(&cfg, k_effort<1, kWeightQ8>, job);
  return nvec == 2 ? cudaLaunchKernelEx(&cfg, k_effort<2, kWeightF16>, job)
                   : cudaLaunchKernelEx(&cfg, k_effort<1, kWeightF16>, job);
}

}  // namespace effort
