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
//           Weighted radix select over the bit patterns, 3 passes of
//           12 / 10 / 9 bits; each pass builds CTA-local weighted histograms,
//           merges them across the cluster through distributed shared memory
//           (each CTA sums one slice of bins and broadcasts it), and picks the
//           digit where the weight counted from the top first reaches K.
//   dispatch per row: the probes that pass c narrow the rank range of the
//           row's selection boundary; the checkpoint magnitudes inside that
//           range give k_i, the number of checkpoint blocks of H ranks that are
//           used entirely.  Rows with 2 * k_i * H >= n are "dense" (read from
//           the dense copy), other active rows are "sparse" (read from the
//           sorted buckets), rows whose largest product is below c are off.
//           Records go to fixed slots of their 32-row group.
#include <cooperative_groups.h>

#include "effort_internal.cuh"

namespace cg = cooperative_groups;

namespace effort {

__device__ __forceinline__ float load_v(const Job& jb, int i) {
  if (jb.vdtype == 1) return __half2float(reinterpret_cast<const __half*>(jb.v)[i]);
  return reinterpret_cast<const float*>(jb.v)[i];
}

// Inclusive prefix sum over the block (blockDim.x == kCutThreads).
__device__ __forceinline__ unsigned block_inclusive_scan(unsigned x, unsigned* warp_tot, unsigned& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const unsigned before = warp > 0 ? warp_tot[warp - 1] : 0u;
  total = warp_tot[31];
  __syncthreads();
  return x + before;
}

struct CutShared {
  unsigned warp_tot[32];
  unsigned sel_digit;
  unsigned sel_krem;
};

// One radix pass over `bits` bits starting at `shift`.
template <int B>
__device__ void radix_pass(cg::cluster_group& cluster, int cl, int crank, int shift, const unsigned* chart,
                           int nelem, const int* pw, unsigned* lh, unsigned* mg, unsigned& prefix,
                           unsigned& pmask, unsigned& krem, CutShared& cs) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) lh[b] = 0u;
  __syncthreads();
  for (int e = threadIdx.x; e < nelem; e += blockDim.x) {
    const unsigned x = chart[e];
    const int w = pw[e & (kP - 1)];
    if (w > 0 && (x & pmask) == prefix) atomicAdd(&lh[(x >> shift) & (B - 1)], (unsigned)w);
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
  // D = max{digit d : weight of digits >= d reaches krem}
  constexpr int q = (B + kCutThreads - 1) / kCutThreads;
  const int lo = threadIdx.x * q, hi = min(B, lo + q);
  unsigned local = 0;
  for (int b = lo; b < hi; ++b) local += mg[b];
  unsigned total;
  const unsigned incl = block_inclusive_scan(local, cs.warp_tot, total);
  unsigned cum = total - incl;  // weight of all digits above my range
  for (int b = hi - 1; b >= lo; --b) {
    const unsigned nb = mg[b];
    if (cum < krem && cum + nb >= krem) {
      cs.sel_digit = (unsigned)b;
      cs.sel_krem = krem - cum;
    }
    cum += nb;
  }
  __syncthreads();
  prefix |= cs.sel_digit << shift;
  pmask |= (unsigned)(B - 1) << shift;
  krem = cs.sel_krem;
  __syncthreads();
}

template <int NJ>
__global__ void __launch_bounds__(kCutThreads, 1) k_cutoff_dispatch(const __grid_constant__ Jobs<NJ> jobs, int cl) {
  // let the multiply kernel of this call get onto the idle SMs early; it waits
  // for this grid's completion before touching anything written here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const Job& jb = jobs.j[blockIdx.x / cl];

  __shared__ HandleDesc d;
  __shared__ CutShared cs;
  if (threadIdx.x < (int)(sizeof(HandleDesc) / 4))
    reinterpret_cast<int*>(&d)[threadIdx.x] = reinterpret_cast<const int*>(jb.hd)[threadIdx.x];
  __syncthreads();

  const int I = d.I, n = d.n, C = d.C, H = d.H;
  const int RP = cut_rows_per_cta(I, cl);
  const int i0 = crank * RP;
  const int nr = max(0, min(I, i0 + RP) - i0);
  const int G = (I + kGroupRows - 1) / kGroupRows;

  extern __shared__ unsigned smem[];
  unsigned* chart = smem;
  float* vs = reinterpret_cast<float*>(chart + (size_t)RP * kP);
  unsigned* h0 = reinterpret_cast<unsigned*>(vs + RP);
  unsigned* m0 = h0 + kBins0;
  unsigned* h1 = m0 + kBins0;
  unsigned* m1 = h1 + kBins1;
  unsigned* h2 = m1 + kBins1;
  unsigned* m2 = h2 + kBins2;

  int mode = jb.mode;
  bool bad = false;
  for (int r = threadIdx.x; r < nr; r += blockDim.x) {
    const float x = load_v(jb, i0 + r);
    if (!isfinite(x)) bad = true;
    vs[r] = x;
  }
  if (bad) atomicOr(jb.ws.status, kStatusNonfiniteV);
  __syncthreads();
  if (mode == kModeSelect) {
    for (int e = threadIdx.x; e < nr * kP; e += blockDim.x) {
      const int r = e >> 4, k = e & (kP - 1);
      const float p = __half2float(__ushort_as_half(d.probes[(size_t)(i0 + r) * kP + k]));
      chart[e] = __float_as_uint(__fmul_rn(fabsf(vs[r]), p));
    }
  }
  __syncthreads();

  unsigned prefix = 0u, pmask = 0u;
  unsigned krem = (unsigned)jb.K;
  if (mode == kModeSelect) {
    radix_pass<kBins0>(cluster, cl, crank, 19, chart, nr * kP, d.pw, h0, m0, prefix, pmask, krem, cs);
    radix_pass<kBins1>(cluster, cl, crank, 9, chart, nr * kP, d.pw, h1, m1, prefix, pmask, krem, cs);
    radix_pass<kBins2>(cluster, cl, crank, 0, chart, nr * kP, d.pw, h2, m2, prefix, pmask, krem, cs);
  }
  const float c = (mode == kModeAll) ? 0.0f : (mode == kModeNone) ? __int_as_float(0x7F800000) : __uint_as_float(prefix);
  const unsigned cbits = __float_as_uint(c);
  if (mode == kModeSelect && cbits == 0u) mode = kModeAll;  // every kept product passes c = 0

  if (crank == 0 && threadIdx.x == 0) {
    jb.ws.c[0] = c;
    jb.ws.count[0] = 0ull;
    if (jb.cutoff_out) jb.cutoff_out[0] = c;
  }

  // dispatch: one thread per row; a warp covers one 32-row group
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < RP; base += blockDim.x) {
    const int r = base + threadIdx.x;
    const int i = i0 + r;
    const bool valid = r < nr;
    int cls = kClassOff, ki = 0;
    float vi = 0.0f;
    if (valid) {
      vi = vs[r];
      if (mode == kModeAll) {
        cls = kClassDense;
        ki = C;
      } else if (mode == kModeSelect) {
        const float av = fabsf(vi);
        int last_sel = -1, first_unsel = n;
        for (int k = 0; k < kP; ++k) {
          const int rk = d.prank[k];
          if (rk < 0) continue;
          if (chart[r * kP + k] >= cbits) last_sel = rk;
          else if (first_unsel == n) first_unsel = rk;
        }
        const int known = min(C, (last_sel + 1) / H);
        const int kend = (first_unsel >= n) ? C : min(C - 1, (first_unsel + 1 + H - 1) / H - 1);
        ki = known;
        const uint16_t* ck = d.ckmag + (size_t)i * (C + 1);
        for (int k = known; k < kend; ++k) {
          const float m = __half2float(__ushort_as_half(ck[1 + k]));
          if (__fmul_rn(av, m) >= c) ki = k + 1;
          else break;
        }
        bool active = (ki > 0) || (last_sel >= 0);
        if (!active) active = __fmul_rn(av, __half2float(__ushort_as_half(ck[0]))) >= c;
        if (active) cls = (2 * ki * H >= n) ? kClassDense : kClassSparse;
      }
      if (jb.rowlen_out) jb.rowlen_out[i] = (mode == kModeAll) ? (unsigned)n : 0u;
    }
    const unsigned bs = __ballot_sync(0xFFFFFFFFu, cls == kClassSparse);
    const unsigned bd = __ballot_sync(0xFFFFFFFFu, cls == kClassDense);
    const int g = (i0 + base) / kGroupRows + warp;
    // a group is written only by the CTA whose row range holds it
    if (base + warp * kGroupRows < RP && g < G) {
      const unsigned lt = (1u << lane) - 1u;
      const uint4 rec = make_uint4((unsigned)i, __float_as_uint(vi), (unsigned)ki, (unsigned)cls);
      if (cls == kClassSparse) jb.ws.rec[(size_t)g * kRecPerGroup + __popc(bs & lt)] = rec;
      if (cls == kClassDense) jb.ws.rec[(size_t)g * kRecPerGroup + 32 + __popc(bd & lt)] = rec;
      if (lane == 0) jb.ws.gcnt[g] = (unsigned)__popc(bs) | ((unsigned)__popc(bd) << 8);
    }
  }
}

template <int NJ>
cudaError_t launch_cutoff_t(const Jobs<NJ>& jobs, int njobs, int I, int cl, cudaStream_t stream) {
  const size_t smem = cut_smem_bytes(I, cl);
  cudaError_t e = cudaFuncSetAttribute(k_cutoff_dispatch<NJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (cl > 8) {
    e = cudaFuncSetAttribute(k_cutoff_dispatch<NJ>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(cl * njobs), 1, 1);
  cfg.blockDim = dim3(kCutThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_cutoff_dispatch<NJ>, jobs, cl);
}

cudaError_t launch_cutoff(const Jobs<1>& jobs, int I, int cl, cudaStream_t stream) {
  return launch_cutoff_t<1>(jobs, 1, I, cl, stream);
}
cudaError_t launch_cutoff_batch(const Jobs<kMaxJobs>& jobs, int njobs, int I, int cl, cudaStream_t stream) {
  return launch_cutoff_t<kMaxJobs>(jobs, njobs, I, cl, stream);
}

}  // namespace effort
