// Host side of the C ABI declared in include/effort.h: argument checks,
// storage and scratch allocation, the host arithmetic of each call (the
// target count K, the call mode) and the kernel launches.  Every step of the
// matvec itself runs in the kernels of prep.cu, effort.cu and dense.cu.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <vector>
#include <new>

#include "../../include/effort.h"
#include "effort_internal.cuh"

namespace effort {
cudaError_t launch_prep(const void* W, const uint16_t* scales, int wk, int I, int O, int n, int P, int dstride,
                        const int* prank, void* wdense, uint16_t* probes, void* vals, uint8_t* gaps, uint16_t* head,
                        uint4* lst, unsigned* chunk_count, unsigned cap_chunks, unsigned* status, cudaStream_t stream);
unsigned long long prep_chunk_bound_per_row(int O, int n);
size_t effort_smem_bytes(int I, int nb);
cudaError_t effort_kernel_attributes(int I, size_t smem);
int effort_grid_size(int I, int sms, size_t smem);
cudaError_t launch_effort(const Job& job, int nb, size_t smem, cudaStream_t stream, int nvec = 1);
cudaError_t launch_dense(const uint16_t* W, int I, int O, const void* v, int vdtype, float* out, float* part,
                         unsigned* tilecnt, int T, int S, cudaStream_t stream);
int dense_ctas_per_sm();
}  // namespace effort

using namespace effort;

namespace {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- allocation
// Every device allocation of the library goes through dev_alloc.  An optional
// cap on the bytes the library holds at once (environment variable
// EFFORT_ALLOC_CAP_BYTES) turns larger requests into EFFORT_ERR_NOMEM before
// CUDA is asked, which lets allocation failure be exercised on purpose.
std::atomic<unsigned long long> g_live_bytes{0};

unsigned long long alloc_cap() {
  const char* e = getenv("EFFORT_ALLOC_CAP_BYTES");
  if (!e || !*e) return ~0ull;
  return strtoull(e, nullptr, 10);
}
bool within_cap(size_t bytes) { return g_live_bytes.load() + bytes <= alloc_cap(); }

effort_status_t dev_alloc(void** p, size_t bytes) {
  *p = nullptr;
  if (!within_cap(bytes)) return EFFORT_ERR_NOMEM;
  if (cudaMalloc(p, bytes) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return EFFORT_ERR_NOMEM;
  }
  g_live_bytes += bytes;
  return EFFORT_OK;
}
void dev_free(void* p, size_t bytes) {
  if (!p) return;
  cudaFree(p);
  g_live_bytes -= bytes;
}

struct DevBuf {
  void* p = nullptr;
  size_t bytes = 0;
  effort_status_t alloc(size_t b) {
    bytes = b;
    return dev_alloc(&p, b);
  }
  void release() {
    dev_free(p, bytes);
    p = nullptr;
    bytes = 0;
  }
};

// ---------------------------------------------------------------- geometry
struct Geometry {
  int I, O, n, P, dstride;
  int nb;       // blocks of the matvec kernel (one per SM)
  size_t smem;  // its dynamic shared memory
  int T;        // 256-column tiles (dense baseline)
  int S_dense;  // row slices of the dense baseline
};

effort_status_t make_geometry(int64_t I, int64_t O, int n, Geometry* g) {
  int dev = 0, sms = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  g->I = (int)I;
  g->O = (int)O;
  g->n = n;
  g->P = (int)((O + kPW - 1) / kPW);
  g->dstride = (int)((O + kStripe - 1) / kStripe * kStripe);
  g->T = (int)((O + 255) / 256);
  g->nb = sms;
  g->smem = effort_smem_bytes(g->I, sms);
  if (g->smem > (size_t)optin) return EFFORT_ERR_UNSUPPORTED;
  if (effort_kernel_attributes(g->I, g->smem) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  g->nb = effort_grid_size(g->I, sms, g->smem);  // every block must be resident at once
  if (g->nb < 1 || g->nb > kMaxGrid || (long long)rows_per_block(g->I, g->nb) * kP > kMaxSegEntries)
    return EFFORT_ERR_UNSUPPORTED;
  int Sd = (sms * dense_ctas_per_sm()) / g->T;
  if (Sd < 1) Sd = 1;
  if (Sd > (int)((I + 7) / 8)) Sd = (int)((I + 7) / 8);
  g->S_dense = Sd < 1 ? 1 : Sd;
  return EFFORT_OK;
}

// ---------------------------------------------------------------- scratch
// Bytes of one call's scratch, carved in this order.
static size_t desc_bytes(const Geometry& g) { return (size_t)kBins0 * g.nb * 4; }
static size_t seg_bytes(const Geometry& g) { return (size_t)g.nb * rows_per_block(g.I, g.nb) * kP * 8; }
size_t scratch_bytes(const Geometry& g) {
  return align_up((size_t)kHdrWords * 4 + 16, 256)                 // header, barrier, count
         + align_up((size_t)(kBins0 + kBins1 + kBins2) * 4, 256)   // histograms
         + align_up(desc_bytes(g), 256)                            // first-digit bin descriptors
         + align_up(seg_bytes(g), 256)                             // chart entries grouped by bin
         ;
}
// Bytes that must be zero before the first call (header, histograms, descriptors).
size_t scratch_zero_bytes(const Geometry& g) {
  return align_up((size_t)kHdrWords * 4 + 16, 256) + align_up((size_t)(kBins0 + kBins1 + kBins2) * 4, 256) +
         align_up(desc_bytes(g), 256);
}

WsPtrs carve(char* b, const Geometry& g) {
  WsPtrs w;
  w.hdr = (unsigned*)b;
  w.bar = (unsigned long long*)(b + kHdrWords * 4);
  w.count = w.bar + 1;
  b += align_up((size_t)kHdrWords * 4 + 16, 256);
  w.ghist0 = (unsigned*)b;
  w.ghist1 = w.ghist0 + kBins0;
  w.ghist2 = w.ghist1 + kBins1;
  b += align_up((size_t)(kBins0 + kBins1 + kBins2) * 4, 256);
  w.desc = (unsigned*)b;
  b += align_up(desc_bytes(g), 256);
  w.seg = (uint2*)b;
  return w;
}

unsigned long long target_count(float effort, long long N) {
  const double x = (double)effort * (double)N;  // one double rounding, then half away from zero
  return (unsigned long long)llround(x);
}

bool effort_ok(float e) { return e == e && e > 0.0f && e <= 1.0f; }

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
    else prev = -1;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

}  // namespace


// Offset of out inside effort_gemv_host's staging buffer (v first).
static size_t stage_out_offset(int I) { return ((size_t)I * 4 + 255) / 256 * 256; }

struct effort_handle_s {
  int dev = 0;
  Geometry g = {};
  float keep = 1.0f;
  HandleDesc hd = {};
  DevBuf chunks;   // vals, gaps, head
  DevBuf tables;   // lst, wdense, probes
  DevBuf ws;       // per-call scratch
  DevBuf stage;    // effort_gemv_host staging: v (in_dim x 4 B), then out (out_dim x 4 B)
  WsPtrs slot = {};
  size_t storage_bytes = 0;
  cudaStream_t last_stream = nullptr;
};

struct effort_workspace_s {
  int dev = 0;
  Geometry g = {};
  int max_pairs = 0;
  DevBuf ws;
  WsPtrs slot = {};
  DevBuf ws2;          // the second vector's scratch of a two-vector launch
  WsPtrs slot2 = {};
  DevBuf dense_part;  // dense baseline: partial tiles and arrival counters
  cudaStream_t last_stream = nullptr;
};

namespace effort {

// The scratch header words, barrier counter, histograms and bin descriptors
// start at zero (they are contiguous from the header).
cudaError_t clear_scratch(const WsPtrs& w, const Geometry& g, cudaStream_t s) {
  return cudaMemsetAsync(w.hdr, 0, scratch_zero_bytes(g), s);
}

size_t handle_scratch_bytes(effort_handle_t h) { return scratch_bytes(h->g); }
WsPtrs handle_carve(effort_handle_t h, char* base) { return carve(base, h->g); }
size_t handle_scratch_zero_bytes(effort_handle_t h) { return scratch_zero_bytes(h->g); }

static effort_status_t fill_job(effort_handle_t h, const WsPtrs& ws, const void* v, effort_dtype_t v_dtype,
                                float effort, float* out, float* cutoff_out, uint64_t* count_out,
                                uint32_t* rowlen_out, Job* j) {
  if (!v || !out) return EFFORT_ERR_ARG;
  if (v_dtype != EFFORT_F32 && v_dtype != EFFORT_F16) return EFFORT_ERR_ARG;
  if (!effort_ok(effort)) return EFFORT_ERR_ARG;
  const long long N = (long long)h->g.I * (long long)h->g.O;
  const unsigned long long K = target_count(effort, N);
  memset(j, 0, sizeof(*j));
  j->hd = h->hd;
  j->barrier_nb = (unsigned)h->g.nb;
  // test hook: a barrier count no grid reaches makes every grid-wide wait run
  // out (bounded) so that the timeout status and the recovery can be checked
  if (const char* t = getenv("EFFORT_TEST_UNREACHABLE_BARRIER"))
    if (t[0] == '1') j->barrier_nb = (unsigned)h->g.nb + 1u;
  j->v = v;
  j->out = out;
  j->cutoff_out = cutoff_out;
  j->count_out = (unsigned long long*)count_out;
  j->rowlen_out = rowlen_out;
  j->ws = ws;
  j->K = K;
  j->mode = (K >= h->hd.kept_total) ? kModeAll : (K == 0 ? kModeNone : kModeSelect);
  j->vdtype = (int)v_dtype;
  return EFFORT_OK;
}

effort_status_t handle_fill_job(effort_handle_t h, const WsPtrs& ws, const void* v, effort_dtype_t v_dtype,
                                float effort, float* out, float* cutoff_out, uint64_t* count_out, Job* j) {
  if (!h) return EFFORT_ERR_ARG;
  return fill_job(h, ws, v, v_dtype, effort, out, cutoff_out, count_out, nullptr, j);
}

cudaError_t handle_launch(effort_handle_t h, const Job& j, cudaStream_t s) {
  return launch_effort(j, h->g.nb, h->g.smem, s);
}
int handle_device(effort_handle_t h) { return h->dev; }

}  // namespace effort

extern "C" {

const char* effort_status_string(effort_status_t s) {
  switch (s) {
    case EFFORT_OK: return "ok";
    case EFFORT_ERR_ARG: return "invalid argument";
    case EFFORT_ERR_CUDA: return "CUDA error";
    case EFFORT_ERR_NOMEM: return "out of memory";
    case EFFORT_ERR_NONFINITE: return "non-finite input";
    case EFFORT_ERR_DEVICE: return "device-side inconsistency or timeout";
    case EFFORT_ERR_UNSUPPORTED: return "unsupported size";
  }
  return "unknown status";
}

// Both weight kinds: W is binary16 [in x out] (wk = kWeightF16), or int8
// [in x out] with one binary16 scale per row (kWeightQ8).  esz: bytes of one
// weight value.
static effort_status_t prepare_impl(const void* W, const uint16_t* scales, int wk, int64_t in_dim, int64_t out_dim,
                                    float keep_fraction, void* stream, effort_handle_t* out_handle) {
  if (!out_handle) return EFFORT_ERR_ARG;
  *out_handle = nullptr;
  if (!W || in_dim < 1 || out_dim < 1) return EFFORT_ERR_ARG;
  if (wk == kWeightF16 && ((uintptr_t)W & 1u) != 0) return EFFORT_ERR_ARG;
  if (wk == kWeightQ8 && (!scales || ((uintptr_t)scales & 1u) != 0)) return EFFORT_ERR_ARG;
  if (!(keep_fraction > 0.0f && keep_fraction <= 1.0f)) return EFFORT_ERR_ARG;
  if (out_dim > EFFORT_MAX_OUT_DIM || in_dim > EFFORT_MAX_IN_DIM) return EFFORT_ERR_UNSUPPORTED;
  if ((unsigned long long)in_dim * (unsigned long long)out_dim >= (1ull << 32)) return EFFORT_ERR_UNSUPPORTED;
  const int n = (int)floor((double)keep_fraction * (double)out_dim + 0.5);
  if (n < 1) return EFFORT_ERR_ARG;
  const size_t esz = (wk == kWeightQ8) ? 1 : 2;

  // storage sizes need no device: check them against the allocation cap first
  const int I = (int)in_dim, O = (int)out_dim;
  const int P = (O + kPW - 1) / kPW, dstride = (O + kStripe - 1) / kStripe * kStripe;
  const unsigned long long cap_chunks = prep_chunk_bound_per_row(O, n) * (unsigned long long)I;
  const size_t sz_lst = align_up((size_t)I * P * 16, 256);
  const size_t sz_dense = align_up((size_t)I * dstride * esz, 256);
  const size_t sz_probe = align_up((size_t)I * kP * 2, 256);
  const size_t sz_scale = (wk == kWeightQ8) ? align_up((size_t)I * 2, 256) : 0;
  const size_t sz_tables = sz_lst + sz_dense + sz_probe + sz_scale + 256;
  const size_t sz_tmp = align_up((size_t)cap_chunks * kCS * (esz + 1) + (size_t)cap_chunks * 2, 256);
  if (!within_cap(sz_tables + sz_tmp)) return EFFORT_ERR_NOMEM;
  if (cap_chunks >= (1ull << 31)) return EFFORT_ERR_UNSUPPORTED;

  effort_handle_s* h = new (std::nothrow) effort_handle_s();
  if (!h) return EFFORT_ERR_NOMEM;
  if (cudaGetDevice(&h->dev) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return EFFORT_ERR_CUDA;
  }
  effort_status_t st = make_geometry(in_dim, out_dim, n, &h->g);
  if (st != EFFORT_OK) {
    delete h;
    return st;
  }
  h->keep = keep_fraction;
  HandleDesc& d = h->hd;
  d.I = I;
  d.O = O;
  d.n = n;
  d.P = P;
  d.dstride = dstride;
  d.wk = wk;
  d.kept_total = (unsigned long long)I * (unsigned long long)n;
  int prank[kP];
  for (int k = 1; k <= kP; ++k) {
    const int b0 = (int)(((long long)(k - 1) * n) / kP), b1 = (int)(((long long)k * n) / kP);
    d.pw[k - 1] = b1 - b0;
    prank[k - 1] = (b1 > b0) ? (b0 + b1) / 2 : -1;
  }

  DevBuf tmp;
  auto fail = [&](effort_status_t s) {
    cudaGetLastError();
    tmp.release();
    h->tables.release();
    h->chunks.release();
    h->ws.release();
    h->stage.release();
    delete h;
    return s;
  };
  if ((st = h->tables.alloc(sz_tables)) != EFFORT_OK) return fail(st);
  if ((st = tmp.alloc(sz_tmp)) != EFFORT_OK) return fail(st);
  char* tb = (char*)h->tables.p;
  d.lst = (const uint4*)tb;
  void* dense = tb + sz_lst;
  if (wk == kWeightQ8) d.wdense8 = (const int8_t*)dense;
  else d.wdense = (const uint16_t*)dense;
  d.probes = (const uint16_t*)(tb + sz_lst + sz_dense);
  if (wk == kWeightQ8) d.scales = (const uint16_t*)(tb + sz_lst + sz_dense + sz_probe);
  unsigned* ctl = (unsigned*)(tb + sz_lst + sz_dense + sz_probe + sz_scale);  // [0] chunks, [1] max |w|, [2] status
  void* tvals = tmp.p;
  uint8_t* tgaps = (uint8_t*)tmp.p + (size_t)cap_chunks * kCS * esz;
  uint16_t* thead = (uint16_t*)(tgaps + (size_t)cap_chunks * kCS);

  cudaStream_t s = (cudaStream_t)stream;
  h->last_stream = s;
  cudaError_t e = cudaMemsetAsync(h->tables.p, 0, sz_tables, s);
  // the handle keeps its own copy of the row scales
  if (e == cudaSuccess && wk == kWeightQ8)
    e = cudaMemcpyAsync((void*)d.scales, scales, (size_t)I * 2, cudaMemcpyDefault, s);
  if (e == cudaSuccess)
    e = launch_prep(W, d.scales, wk, I, O, n, P, dstride, prank, dense, (uint16_t*)d.probes, tvals, tgaps, thead,
                    (uint4*)d.lst, ctl, (unsigned)cap_chunks, ctl + 2, s);
  unsigned ctl_h[3] = {0, 0, 0};
  if (e == cudaSuccess) e = cudaMemcpyAsync(ctl_h, ctl, 12, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(EFFORT_ERR_CUDA);
  if (ctl_h[2] & kStatusNonfiniteW) return fail(EFFORT_ERR_NONFINITE);
  if (ctl_h[2] & kStatusInternal) return fail(EFFORT_ERR_DEVICE);
  d.wmax_bits = ctl_h[1];

  // the used chunks into storage of the exact size
  const size_t nch = ctl_h[0];
  d.total_chunks = (unsigned)nch;
  const size_t cv = align_up(nch * kCS * esz, 256), cg = align_up(nch * kCS, 256), chd = align_up(nch * 2 + 2, 256);
  if ((st = h->chunks.alloc(cv + cg + chd)) != EFFORT_OK) return fail(st);
  char* cb = (char*)h->chunks.p;
  if (wk == kWeightQ8) d.vals8 = (const int8_t*)cb;
  else d.vals = (const uint16_t*)cb;
  d.gaps = (const uint8_t*)(cb + cv);
  d.head = (const uint16_t*)(cb + cv + cg);
  e = cudaMemcpyAsync(cb, tvals, nch * kCS * esz, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync((void*)d.gaps, tgaps, nch * kCS, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync((void*)d.head, thead, nch * 2, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(EFFORT_ERR_CUDA);
  tmp.release();
  h->storage_bytes = h->chunks.bytes + h->tables.bytes;

  // per-call scratch and the host-call staging buffer
  if ((st = h->ws.alloc(scratch_bytes(h->g))) != EFFORT_OK) return fail(st);
  h->slot = carve((char*)h->ws.p, h->g);
  if (clear_scratch(h->slot, h->g, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) return fail(EFFORT_ERR_CUDA);
  if ((st = h->stage.alloc(stage_out_offset(I) + (size_t)O * 4)) != EFFORT_OK) return fail(st);
  *out_handle = h;
  return EFFORT_OK;
}

effort_status_t effort_prepare(const void* W, int64_t in_dim, int64_t out_dim, float keep_fraction, void* stream,
                               effort_handle_t* out_handle) {
  return prepare_impl(W, nullptr, kWeightF16, in_dim, out_dim, keep_fraction, stream, out_handle);
}

effort_status_t effort_prepare_q8(const int8_t* q, const uint16_t* scales, int64_t in_dim, int64_t out_dim,
                                  float keep_fraction, void* stream, effort_handle_t* out_handle) {
  return prepare_impl(q, scales, kWeightQ8, in_dim, out_dim, keep_fraction, stream, out_handle);
}

effort_status_t effort_gemv_ex(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort, float* out,
                               float* cutoff_out, uint64_t* count_out, uint32_t* rowlen_out, void* stream) {
  if (!h) return EFFORT_ERR_ARG;
  Job job;
  effort_status_t st = fill_job(h, h->slot, v, v_dtype, effort, out, cutoff_out, count_out, rowlen_out, &job);
  if (st != EFFORT_OK) return st;
  DeviceGuard guard(h->dev);
  cudaStream_t s = (cudaStream_t)stream;
  h->last_stream = s;
  if (launch_effort(job, h->g.nb, h->g.smem, s) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}

effort_status_t effort_gemv_timed(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort, float* out,
                                  uint64_t* marks, void* stream) {
  if (!h || !marks) return EFFORT_ERR_ARG;
  Job job;
  effort_status_t st = fill_job(h, h->slot, v, v_dtype, effort, out, nullptr, nullptr, nullptr, &job);
  if (st != EFFORT_OK) return st;
  job.marks = (unsigned long long*)marks;
  DeviceGuard guard(h->dev);
  cudaStream_t s = (cudaStream_t)stream;
  h->last_stream = s;
  if (launch_effort(job, h->g.nb, h->g.smem, s) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}

effort_status_t effort_grid_blocks(effort_handle_t h, int32_t* blocks) {
  if (!h || !blocks) return EFFORT_ERR_ARG;
  *blocks = h->g.nb;
  return EFFORT_OK;
}

effort_status_t effort_gemv_host(effort_handle_t h, const void* v_host, effort_dtype_t v_dtype, float effort,
                                 float* out_host, void* stream) {
  if (!h || !v_host || !out_host) return EFFORT_ERR_ARG;
  if (v_dtype != EFFORT_F32 && v_dtype != EFFORT_F16) return EFFORT_ERR_ARG;
  if (!effort_ok(effort)) return EFFORT_ERR_ARG;
  DeviceGuard guard(h->dev);
  cudaStream_t s = (cudaStream_t)stream;
  // v is copied into the staging buffer (every block of the kernel reads
  // it, which in place across the host link would cost a round trip per
  // block); out is accumulated with device-memory reductions, so it goes
  // through the staging buffer and one copy back
  void* d_v = h->stage.p;
  float* d_out = reinterpret_cast<float*>(static_cast<char*>(h->stage.p) + stage_out_offset(h->g.I));
  const size_t vbytes = (size_t)h->g.I * (v_dtype == EFFORT_F16 ? 2 : 4);
  if (cudaMemcpyAsync(d_v, v_host, vbytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  // page-locked out mapped into the device's address space is written by the
  // kernel's last block; other host memory is copied back after the kernel
  void* mout = nullptr;
  {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, out_host) == cudaSuccess && a.type == cudaMemoryTypeHost) mout = a.devicePointer;
    cudaGetLastError();
  }
  Job job;
  effort_status_t st = fill_job(h, h->slot, d_v, v_dtype, effort, d_out, nullptr, nullptr, nullptr, &job);
  if (st != EFFORT_OK) return st;
  job.out_mirror = (float*)mout;
  h->last_stream = s;
  if (launch_effort(job, h->g.nb, h->g.smem, s) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  if (!mout && cudaMemcpyAsync(out_host, d_out, (size_t)h->g.O * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}

effort_status_t effort_gemv(effort_handle_t h, const float* v, float effort, float* out, void* stream) {
  return effort_gemv_ex(h, v, EFFORT_F32, effort, out, nullptr, nullptr, nullptr, stream);
}

effort_status_t effort_check(effort_handle_t h) {
  if (!h) return EFFORT_ERR_ARG;
  DeviceGuard guard(h->dev);
  unsigned int st = 0;
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return EFFORT_ERR_CUDA;
  if (cudaMemcpy(&st, h->slot.hdr + kHdrStatus, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return EFFORT_ERR_CUDA;
  if (st) {
    // a timed-out grid leaves the barrier counter and histograms mid-call:
    // start the scratch over (the status word with it)
    if (clear_scratch(h->slot, h->g, h->last_stream) != cudaSuccess || cudaStreamSynchronize(h->last_stream) != cudaSuccess)
      return EFFORT_ERR_CUDA;
  }
  if (st & (kStatusInternal | kStatusTimeout)) return EFFORT_ERR_DEVICE;
  if (st & kStatusNonfiniteV) return EFFORT_ERR_NONFINITE;
  return EFFORT_OK;
}

effort_status_t effort_workspace_create(int64_t in_dim, int64_t out_dim, int32_t max_pairs, effort_workspace_t* out_ws) {
  if (!out_ws) return EFFORT_ERR_ARG;
  *out_ws = nullptr;
  if (in_dim < 1 || out_dim < 1 || max_pairs < 1) return EFFORT_ERR_ARG;
  if (out_dim > EFFORT_MAX_OUT_DIM || in_dim > EFFORT_MAX_IN_DIM) return EFFORT_ERR_UNSUPPORTED;
  effort_workspace_s* w = new (std::nothrow) effort_workspace_s();
  if (!w) return EFFORT_ERR_NOMEM;
  if (cudaGetDevice(&w->dev) != cudaSuccess) {
    cudaGetLastError();
    delete w;
    return EFFORT_ERR_CUDA;
  }
  effort_status_t st = make_geometry(in_dim, out_dim, (int)out_dim, &w->g);
  if (st == EFFORT_OK) st = w->ws.alloc(scratch_bytes(w->g));
  if (st == EFFORT_OK) {
    w->slot = carve((char*)w->ws.p, w->g);
    if (clear_scratch(w->slot, w->g, nullptr) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) st = EFFORT_ERR_CUDA;
  }
  if (st == EFFORT_OK && max_pairs >= 2) {
    st = w->ws2.alloc(scratch_bytes(w->g));
    if (st == EFFORT_OK) {
      w->slot2 = carve((char*)w->ws2.p, w->g);
      if (clear_scratch(w->slot2, w->g, nullptr) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
        st = EFFORT_ERR_CUDA;
    }
  }
  const size_t dense_bytes = align_up((size_t)w->g.S_dense * w->g.T * 256 * 4, 256) + align_up((size_t)w->g.T * 4, 256);
  if (st == EFFORT_OK) st = w->dense_part.alloc(dense_bytes);
  if (st == EFFORT_OK && cudaMemset(w->dense_part.p, 0, dense_bytes) != cudaSuccess) st = EFFORT_ERR_CUDA;
  if (st != EFFORT_OK) {
    cudaGetLastError();
    w->ws.release();
    w->ws2.release();
    w->dense_part.release();
    delete w;
    return st;
  }
  w->max_pairs = max_pairs;
  *out_ws = w;
  return EFFORT_OK;
}

effort_status_t effort_workspace_destroy(effort_workspace_t w) {
  if (!w) return EFFORT_ERR_ARG;
  {
    DeviceGuard guard(w->dev);
    cudaStreamSynchronize(w->last_stream);
    w->ws.release();
    w->ws2.release();
    w->dense_part.release();
  }
  delete w;
  return EFFORT_OK;
}

effort_status_t effort_gemv_batched(effort_workspace_t ws, const effort_handle_t* handles, const int32_t* hidx,
                                    const int32_t* vidx, int32_t n_pairs, const void* V, effort_dtype_t v_dtype,
                                    const float* efforts, float* OUT, float* cutoffs_out, uint64_t* counts_out,
                                    void* stream) {
  if (!ws || !handles || !hidx || !vidx || !V || !efforts || !OUT) return EFFORT_ERR_ARG;
  if (n_pairs < 1 || n_pairs > ws->max_pairs) return EFFORT_ERR_ARG;
  if (v_dtype != EFFORT_F32 && v_dtype != EFFORT_F16) return EFFORT_ERR_ARG;
  const int I = ws->g.I, O = ws->g.O;
  const size_t vsz = (v_dtype == EFFORT_F16) ? 2 : 4;
  for (int p = 0; p < n_pairs; ++p) {
    if (hidx[p] < 0 || vidx[p] < 0) return EFFORT_ERR_ARG;
    effort_handle_t h = handles[hidx[p]];
    if (!h || h->g.I != I || h->g.O != O || !effort_ok(efforts[p])) return EFFORT_ERR_ARG;
  }
  DeviceGuard guard(ws->dev);
  cudaStream_t s = (cudaStream_t)stream;
  ws->last_stream = s;
  // Pairs on the same matrix whose cutoffs both select go two at a time into
  // one grid that reads the union of their prefixes once (each keeps its own
  // cutoff, thresholds and output); the rest run one grid per pair.  All
  // grids are on one stream, each waiting for the one before, so they share
  // the workspace's scratch.
  auto job_of = [&](int p, const WsPtrs& slot, Job* job) {
    effort_handle_t h = handles[hidx[p]];
    const effort_status_t st =
        fill_job(h, slot, (const char*)V + (size_t)vidx[p] * I * vsz, v_dtype, efforts[p], OUT + (size_t)p * O,
                 cutoffs_out ? cutoffs_out + p : nullptr, counts_out ? counts_out + p : nullptr, nullptr, job);
    job->accumulate_bytes = 1;  // the call's bytes are the sum over its grids
    return st;
  };
  // the call's planned bytes start over
  if (cudaMemsetAsync(ws->slot.hdr + kHdrBytesLast, 0, 16, s) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  auto launch_one = [&](int p) -> effort_status_t {
    Job job;
    effort_status_t st = job_of(p, ws->slot, &job);
    if (st != EFFORT_OK) return st;
    if (launch_effort(job, ws->g.nb, ws->g.smem, s, 1) != cudaSuccess) {
      cudaGetLastError();
      return EFFORT_ERR_CUDA;
    }
    return EFFORT_OK;
  };
  std::vector<int> waiting;  // per handle index: a selecting pair without a partner yet, or -1
  for (int p = 0; p < n_pairs; ++p) {
    Job a;
    effort_status_t st = job_of(p, ws->slot, &a);
    if (st != EFFORT_OK) return st;
    const int hx = hidx[p];
    if ((int)waiting.size() <= hx) waiting.resize(hx + 1, -1);
    if (a.mode != kModeSelect || !ws->ws2.p) {
      st = launch_one(p);
      if (st != EFFORT_OK) return st;
      continue;
    }
    if (waiting[hx] < 0) {
      waiting[hx] = p;
      continue;
    }
    Job first, second;
    st = job_of(waiting[hx], ws->slot, &first);
    if (st == EFFORT_OK) st = job_of(p, ws->slot2, &second);
    if (st != EFFORT_OK) return st;
    first.v2 = second.v;
    first.out2 = second.out;
    first.cutoff_out2 = second.cutoff_out;
    first.count_out2 = second.count_out;
    first.ws2 = second.ws;
    first.K2 = second.K;
    waiting[hx] = -1;
    if (launch_effort(first, ws->g.nb, ws->g.smem, s, 2) != cudaSuccess) {
      cudaGetLastError();
      return EFFORT_ERR_CUDA;
    }
  }
  for (int hx = 0; hx < (int)waiting.size(); ++hx)
    if (waiting[hx] >= 0) {
      const effort_status_t st = launch_one(waiting[hx]);
      if (st != EFFORT_OK) return st;
    }
  return EFFORT_OK;
}

effort_status_t effort_workspace_check(effort_workspace_t ws) {
  if (!ws) return EFFORT_ERR_ARG;
  DeviceGuard guard(ws->dev);
  unsigned int st = 0;
  if (cudaStreamSynchronize(ws->last_stream) != cudaSuccess) return EFFORT_ERR_CUDA;
  if (cudaMemcpy(&st, ws->slot.hdr + kHdrStatus, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return EFFORT_ERR_CUDA;
  if (st) {
    // a timed-out grid leaves the scratch mid-call: start both slots over
    if (clear_scratch(ws->slot, ws->g, ws->last_stream) != cudaSuccess) return EFFORT_ERR_CUDA;
    if (ws->ws2.p && clear_scratch(ws->slot2, ws->g, ws->last_stream) != cudaSuccess) return EFFORT_ERR_CUDA;
    if (cudaStreamSynchronize(ws->last_stream) != cudaSuccess) return EFFORT_ERR_CUDA;
  }
  if (st & (kStatusInternal | kStatusTimeout)) return EFFORT_ERR_DEVICE;
  if (st & kStatusNonfiniteV) return EFFORT_ERR_NONFINITE;
  return EFFORT_OK;
}

effort_status_t effort_workspace_last_call_bytes(effort_workspace_t ws, uint64_t* dense_bytes, uint64_t* sparse_bytes) {
  if (!ws || !dense_bytes || !sparse_bytes) return EFFORT_ERR_ARG;
  DeviceGuard guard(ws->dev);
  unsigned long long b[2] = {0, 0};
  if (cudaStreamSynchronize(ws->last_stream) != cudaSuccess ||
      cudaMemcpy(b, ws->slot.hdr + kHdrBytesLast, 16, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  *dense_bytes = b[0];
  *sparse_bytes = b[1];
  return EFFORT_OK;
}

effort_status_t effort_dense_gemv(effort_workspace_t ws, const void* W, int64_t in_dim, int64_t out_dim, const void* v,
                                  effort_dtype_t v_dtype, float* out, void* stream) {
  if (!ws || !W || !v || !out) return EFFORT_ERR_ARG;
  if (in_dim != ws->g.I || out_dim != ws->g.O) return EFFORT_ERR_ARG;
  if ((out_dim % 8) != 0 || ((uintptr_t)W & 15u) != 0) return EFFORT_ERR_ARG;
  if (v_dtype != EFFORT_F32 && v_dtype != EFFORT_F16) return EFFORT_ERR_ARG;
  DeviceGuard guard(ws->dev);
  cudaStream_t s = (cudaStream_t)stream;
  ws->last_stream = s;
  float* part = (float*)ws->dense_part.p;
  unsigned* tilecnt = (unsigned*)((char*)ws->dense_part.p + align_up((size_t)ws->g.S_dense * ws->g.T * 256 * 4, 256));
  cudaError_t e = launch_dense((const uint16_t*)W, ws->g.I, ws->g.O, v, (int)v_dtype, out, part, tilecnt, ws->g.T,
                               ws->g.S_dense, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}

effort_status_t effort_get_info(effort_handle_t h, int64_t* in_dim, int64_t* out_dim, float* keep_fraction,
                                size_t* device_bytes) {
  if (!h) return EFFORT_ERR_ARG;
  if (in_dim) *in_dim = h->g.I;
  if (out_dim) *out_dim = h->g.O;
  if (keep_fraction) *keep_fraction = h->keep;
  if (device_bytes) *device_bytes = h->storage_bytes;
  return EFFORT_OK;
}

effort_status_t effort_get_layout(effort_handle_t h, effort_layout_t* L) {
  if (!h || !L) return EFFORT_ERR_ARG;
  L->in_dim = h->g.I;
  L->out_dim = h->g.O;
  L->n_kept = h->hd.n;
  L->n_panels = h->hd.P;
  L->panel_width = kPW;
  L->chunk_slots = kCS;
  L->store_num = kStoreNum;
  L->store_den = kStoreDen;
  L->n_probes = kP;
  L->dense_stride = h->hd.dstride;
  L->total_chunks = h->hd.total_chunks;
  const bool q8 = h->hd.wk == kWeightQ8;
  L->vals = q8 ? (const void*)h->hd.vals8 : (const void*)h->hd.vals;
  L->gaps = h->hd.gaps;
  L->head = h->hd.head;
  L->lists = h->hd.lst;
  L->wdense = q8 ? (const void*)h->hd.wdense8 : (const void*)h->hd.wdense;
  L->probes = h->hd.probes;
  L->scratch_bytes = h->ws.bytes;
  L->weight_kind = h->hd.wk;
  L->scales = h->hd.scales;
  return EFFORT_OK;
}

effort_status_t effort_destroy(effort_handle_t h) {
  if (!h) return EFFORT_ERR_ARG;
  {
    DeviceGuard guard(h->dev);
    cudaStreamSynchronize(h->last_stream);
    h->stage.release();
    h->ws.release();
    h->chunks.release();
    h->tables.release();
  }
  delete h;
  return EFFORT_OK;
}

effort_status_t effort_last_call_bytes(effort_handle_t h, uint64_t* dense_bytes, uint64_t* sparse_bytes) {
  if (!h || !dense_bytes || !sparse_bytes) return EFFORT_ERR_ARG;
  DeviceGuard guard(h->dev);
  unsigned long long b[2] = {0, 0};
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess ||
      cudaMemcpy(b, h->slot.hdr + kHdrBytesLast, 16, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  *dense_bytes = b[0];
  *sparse_bytes = b[1];
  return EFFORT_OK;
}

effort_status_t effort_device_bytes_held(uint64_t* bytes) {
  if (!bytes) return EFFORT_ERR_ARG;
  *bytes = g_live_bytes.load();
  return EFFORT_OK;
}

}  // extern "C"
