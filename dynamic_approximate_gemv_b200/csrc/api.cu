// Host side of the C ABI declared in include/effort.h: argument checks,
// storage and scratch allocation, the host arithmetic of each call (the
// target count K, the call mode) and the kernel launches.  Every step of the
// matvec itself runs in the kernels of prep.cu, cutoff.cu, mac.cu, dense.cu.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "../../include/effort.h"
#include "effort_internal.cuh"

namespace effort {
cudaError_t launch_prep(const uint16_t* W, const HandleDesc* d_desc, int I, int O, uint16_t* vals, uint8_t* idx,
                        uint16_t* wdense, uint16_t* probes, uint16_t* ckmag, uint8_t* cnt, unsigned int* status,
                        cudaStream_t stream);
cudaError_t launch_cutoff(const Jobs<1>& jobs, int I, int cl, cudaStream_t stream);
cudaError_t launch_cutoff_batch(const Jobs<kMaxJobs>& jobs, int njobs, int I, int cl, cudaStream_t stream);
cudaError_t launch_mac(const Jobs<1>& jobs, int T, int S, cudaStream_t stream);
cudaError_t launch_mac_batch(const Jobs<kMaxJobs>& jobs, int njobs, int T, int S, cudaStream_t stream);
cudaError_t launch_dense(const uint16_t* W, int I, int O, const void* v, int vdtype, float* out, float* part,
                         unsigned* tilecnt, int T, int S, cudaStream_t stream);
int mac_ctas_per_sm();
int dense_ctas_per_sm();
cudaError_t init_kernel_attributes();
size_t cutoff_max_dynamic_smem();
int cutoff_max_clusters(int cl, size_t smem);
}  // namespace effort

using namespace effort;

namespace {

struct Geometry {
  int I, O, T, G;
  int S;        // row slices of the multiply kernel (grid T x S)
  int S_dense;  // row slices of the dense baseline
  int cl;       // CTAs in the cutoff cluster
  int dense_q16;  // dense-row threshold (share of the row surely used, x 65536)
};

struct WsBlock {
  void* base = nullptr;
  size_t bytes = 0;
  WsPtrs p = {};
};

int g_num_sms = 0;
int g_smem_optin = 0;

cudaError_t device_info() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  return cudaDeviceGetAttribute(&g_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Chooses the cutoff cluster size and the split-K slice counts.
effort_status_t make_geometry(int64_t I, int64_t O, Geometry* g) {
  if (device_info() != cudaSuccess) return EFFORT_ERR_CUDA;
  if (init_kernel_attributes() != cudaSuccess) return EFFORT_ERR_CUDA;
  g->I = (int)I;
  g->O = (int)O;
  g->T = (int)((O + kTW - 1) / kTW);
  g->G = (int)((I + kGroupRows - 1) / kGroupRows);
  g->cl = 0;
  const size_t dyn_max = cutoff_max_dynamic_smem();
  for (int cl : {16, 8}) {  // the wider cluster halves each CTA's share of the rows
    const size_t sm = cut_smem_bytes(g->I, cl);
    if (sm <= dyn_max && cutoff_max_clusters(cl, sm) >= 1) {
      g->cl = cl;
      break;
    }
  }
  if (g->cl == 0) return EFFORT_ERR_UNSUPPORTED;
  // T x S CTAs fill the SMs once (two resident per SM); every slice keeps at
  // least one 32-row group
  const int slots = g_num_sms * mac_ctas_per_sm();
  int S = slots / g->T;
  if (S < 1) S = 1;
  if (S > g->G) S = g->G;
  g->S = S;
  // rows whose surely-used share reaches this fraction are read from the dense
  // copy (2 B per weight, register accumulation) instead of their buckets.  A
  // sparse row-tile's short prefix rounds up to whole sectors twice (values,
  // columns), so a row read through its buckets costs more per used product
  // than its byte count suggests; measured step times are flat from 0.1 to
  // 0.2 and rise above that
  double frac = 0.2;
  if (const char* env = getenv("EFFORT_DENSE_FRACTION")) {
    const double f = atof(env);
    if (f > 0.0 && f <= 1.0) frac = f;
  }
  g->dense_q16 = (int)(frac * 65536.0 + 0.5);
  // the dense baseline's T x Sd CTAs fill the SMs once as well
  int Sd = (g_num_sms * dense_ctas_per_sm()) / g->T;
  if (Sd < 1) Sd = 1;
  if (Sd > (int)((I + 7) / 8)) Sd = (int)((I + 7) / 8);
  if (Sd < 1) Sd = 1;
  g->S_dense = Sd;
  return EFFORT_OK;
}

// One contiguous device block of scratch for `npairs` jobs.
effort_status_t alloc_ws(const Geometry& g, int npairs, WsBlock* out, WsPtrs* slots) {
  const int S = g.S > g.S_dense ? g.S : g.S_dense;
  const size_t per = align_up(256, 256)                                  // c, count, done, status
                     + align_up((size_t)g.T * 4, 256)                    // tilecnt
                     + align_up((size_t)g.G * 4, 256)                    // gcnt
                     + align_up((size_t)g.G * g.T * 32, 256)             // ut
                     + align_up((size_t)g.G * kRecPerGroup * 8, 256)     // rec
                     + align_up((size_t)S * g.T * kTW * 4, 256);         // part
  const size_t bytes = per * (size_t)npairs;
  void* base = nullptr;
  if (cudaMalloc(&base, bytes) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_NOMEM;
  }
  if (cudaMemset(base, 0, bytes) != cudaSuccess) {
    cudaFree(base);
    return EFFORT_ERR_CUDA;
  }
  for (int p = 0; p < npairs; ++p) {
    char* b = (char*)base + per * p;
    WsPtrs w;
    w.c = (float*)(b + 0);
    w.count = (unsigned long long*)(b + 8);
    w.done = (unsigned int*)(b + 16);
    w.status = (unsigned int*)(b + 20);
    b += 256;
    w.tilecnt = (unsigned int*)b;
    b += align_up((size_t)g.T * 4, 256);
    w.gcnt = (unsigned int*)b;
    b += align_up((size_t)g.G * 4, 256);
    w.ut = (unsigned char*)b;
    b += align_up((size_t)g.G * g.T * 32, 256);
    w.rec = (uint2*)b;
    b += align_up((size_t)g.G * kRecPerGroup * 8, 256);
    w.part = (float*)b;
    slots[p] = w;
  }
  out->base = base;
  out->bytes = bytes;
  out->p = slots[0];
  return EFFORT_OK;
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

// Device address of page-locked host memory mapped into the device's address
// space (cudaHostAlloc, cudaMallocHost, cudaHostRegister with mapping), else
// nullptr (pageable memory, device memory, unknown pointers).
static void* mapped_host_pointer(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return (a.type == cudaMemoryTypeHost) ? a.devicePointer : nullptr;
}

// Offset of out inside effort_gemv_host's staging buffer (v first).
static size_t stage_out_offset(int I) { return ((size_t)I * 4 + 255) / 256 * 256; }

struct effort_handle_s {
  int dev = 0;
  Geometry g = {};
  float keep = 1.0f;
  HandleDesc hd = {};
  HandleDesc* d_desc = nullptr;
  void* storage = nullptr;
  size_t storage_bytes = 0;
  WsBlock ws;
  WsPtrs slot = {};
  void* stage = nullptr;  // device staging of effort_gemv_host: v (in_dim x 4 B), then out (out_dim x 4 B)
  cudaStream_t last_stream = nullptr;
};

struct effort_workspace_s {
  int dev = 0;
  Geometry g = {};
  int max_pairs = 0;
  WsBlock ws;
  WsPtrs* slots = nullptr;
  cudaStream_t last_stream = nullptr;
};

extern "C" {

const char* effort_status_string(effort_status_t s) {
  switch (s) {
    case EFFORT_OK: return "ok";
    case EFFORT_ERR_ARG: return "invalid argument";
    case EFFORT_ERR_CUDA: return "CUDA error";
    case EFFORT_ERR_NOMEM: return "out of memory";
    case EFFORT_ERR_NONFINITE: return "non-finite input";
    case EFFORT_ERR_DEVICE: return "device-side inconsistency";
    case EFFORT_ERR_UNSUPPORTED: return "unsupported size";
  }
  return "unknown status";
}

effort_status_t effort_prepare(const void* W, int64_t in_dim, int64_t out_dim, float keep_fraction, void* stream,
                               effort_handle_t* out_handle) {
  if (!out_handle) return EFFORT_ERR_ARG;
  *out_handle = nullptr;
  if (!W || in_dim < 1 || out_dim < 1) return EFFORT_ERR_ARG;
  if (((uintptr_t)W & 1u) != 0) return EFFORT_ERR_ARG;
  if (!(keep_fraction > 0.0f && keep_fraction <= 1.0f)) return EFFORT_ERR_ARG;
  if (out_dim > EFFORT_MAX_OUT_DIM || in_dim > EFFORT_MAX_IN_DIM) return EFFORT_ERR_UNSUPPORTED;
  if ((unsigned long long)in_dim * (unsigned long long)out_dim >= (1ull << 32)) return EFFORT_ERR_UNSUPPORTED;
  const int n = (int)floor((double)keep_fraction * (double)out_dim + 0.5);
  if (n < 1) return EFFORT_ERR_ARG;

  effort_handle_s* h = new (std::nothrow) effort_handle_s();
  if (!h) return EFFORT_ERR_NOMEM;
  cudaGetDevice(&h->dev);
  effort_status_t st = make_geometry(in_dim, out_dim, &h->g);
  if (st != EFFORT_OK) {
    delete h;
    return st;
  }
  h->keep = keep_fraction;
  const Geometry& g = h->g;
  const int I = g.I, T = g.T;
  int H = 2 * T;
  H = (H + 31) / 32 * 32;
  if (H < 32) H = 32;
  const int C = (n + H - 1) / H;

  HandleDesc& d = h->hd;
  d.I = I;
  d.O = g.O;
  d.T = T;
  d.n = n;
  d.C = C;
  d.H = H;
  d.dstride = T * kTW;
  d.kept_total = (unsigned long long)I * (unsigned long long)n;
  for (int k = 1; k <= kP; ++k) {
    const int b0 = (int)(((long long)(k - 1) * n) / kP), b1 = (int)(((long long)k * n) / kP);
    d.pw[k - 1] = b1 - b0;
    d.prank[k - 1] = (b1 > b0) ? (b0 + b1) / 2 : -1;
  }

  const size_t nb = (size_t)T * I * kCap;
  const size_t sz_vals = align_up(nb * 2, 256), sz_idx = align_up(nb, 256);
  const size_t sz_dense = align_up((size_t)I * T * kTW * 2, 256);
  const size_t sz_probe = align_up((size_t)I * kP * 2, 256);
  const size_t sz_ck = align_up((size_t)I * (C + 1) * 2, 256);
  const size_t sz_cnt = align_up((size_t)I * C * T, 256);
  const size_t sz_desc = align_up(sizeof(HandleDesc), 256);
  const size_t sz_status = 256;
  const size_t total = sz_vals + sz_idx + sz_dense + sz_probe + sz_ck + sz_cnt + sz_desc + sz_status;
  if (cudaMalloc(&h->storage, total) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return EFFORT_ERR_NOMEM;
  }
  h->storage_bytes = total;
  char* b = (char*)h->storage;
  d.vals = (const uint16_t*)b;
  b += sz_vals;
  d.idx = (const uint8_t*)b;
  b += sz_idx;
  d.wdense = (const uint16_t*)b;
  b += sz_dense;
  d.probes = (const uint16_t*)b;
  b += sz_probe;
  d.ckmag = (const uint16_t*)b;
  b += sz_ck;
  d.cnt = (const uint8_t*)b;
  b += sz_cnt;
  h->d_desc = (HandleDesc*)b;
  b += sz_desc;
  unsigned int* prep_status = (unsigned int*)b;

  cudaStream_t s = (cudaStream_t)stream;
  h->last_stream = s;
  cudaError_t e = cudaMemsetAsync(h->storage, 0, total, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(h->d_desc, &d, sizeof(HandleDesc), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = launch_prep((const uint16_t*)W, h->d_desc, I, g.O, (uint16_t*)d.vals, (uint8_t*)d.idx, (uint16_t*)d.wdense,
                    (uint16_t*)d.probes, (uint16_t*)d.ckmag, (uint8_t*)d.cnt, prep_status, s);
  unsigned int status_h = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&status_h, prep_status, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cudaFree(h->storage);
    delete h;
    return EFFORT_ERR_CUDA;
  }
  if (status_h & kStatusNonfiniteW) {
    cudaFree(h->storage);
    delete h;
    return EFFORT_ERR_NONFINITE;
  }
  st = alloc_ws(g, 1, &h->ws, &h->slot);
  if (st != EFFORT_OK) {
    cudaFree(h->storage);
    delete h;
    return st;
  }
  if (cudaMalloc(&h->stage, stage_out_offset(g.I) + (size_t)g.O * 4) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(h->ws.base);
    cudaFree(h->storage);
    delete h;
    return EFFORT_ERR_NOMEM;
  }
  *out_handle = h;
  return EFFORT_OK;
}

static effort_status_t fill_job(effort_handle_t h, const WsPtrs& ws, const void* v, effort_dtype_t v_dtype,
                                float effort, float* out, float* cutoff_out, uint64_t* count_out,
                                uint32_t* rowlen_out, Job* j) {
  if (!v || !out) return EFFORT_ERR_ARG;
  if (v_dtype != EFFORT_F32 && v_dtype != EFFORT_F16) return EFFORT_ERR_ARG;
  if (!effort_ok(effort)) return EFFORT_ERR_ARG;
  const long long N = (long long)h->g.I * (long long)h->g.O;
  const unsigned long long K = target_count(effort, N);
  j->hd = h->hd;
  j->v = v;
  j->out = out;
  j->cutoff_out = cutoff_out;
  j->count_out = (unsigned long long*)count_out;
  j->rowlen_out = rowlen_out;
  j->ws = ws;
  j->K = K;
  j->mode = (K >= h->hd.kept_total) ? kModeAll : (K == 0 ? kModeNone : kModeSelect);
  j->vdtype = (int)v_dtype;
  j->dense_q16 = h->g.dense_q16;
  return EFFORT_OK;
}

effort_status_t effort_gemv_ex(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort, float* out,
                               float* cutoff_out, uint64_t* count_out, uint32_t* rowlen_out, void* stream) {
  if (!h) return EFFORT_ERR_ARG;
  Jobs<1> jobs;
  effort_status_t st = fill_job(h, h->slot, v, v_dtype, effort, out, cutoff_out, count_out, rowlen_out, &jobs.j[0]);
  if (st != EFFORT_OK) return st;
  DeviceGuard guard(h->dev);
  cudaStream_t s = (cudaStream_t)stream;
  h->last_stream = s;
  cudaError_t e = launch_cutoff(jobs, h->g.I, h->g.cl, s);
  if (e == cudaSuccess) e = launch_mac(jobs, h->g.T, h->g.S, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}

effort_status_t effort_gemv_split(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort, float* out,
                                  float* cutoff_out, uint64_t* count_out, void* mid_event, void* stream) {
  if (!h || !mid_event) return EFFORT_ERR_ARG;
  Jobs<1> jobs;
  effort_status_t st = fill_job(h, h->slot, v, v_dtype, effort, out, cutoff_out, count_out, nullptr, &jobs.j[0]);
  if (st != EFFORT_OK) return st;
  DeviceGuard guard(h->dev);
  cudaStream_t s = (cudaStream_t)stream;
  h->last_stream = s;
  cudaError_t e = launch_cutoff(jobs, h->g.I, h->g.cl, s);
  // under stream capture the event is recorded as an external event-record
  // node, so that the phases of a captured graph can be timed too
  if (e == cudaSuccess) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(s, &cap);
    if (e == cudaSuccess)
      e = (cap == cudaStreamCaptureStatusActive)
              ? cudaEventRecordWithFlags((cudaEvent_t)mid_event, s, cudaEventRecordExternal)
              : cudaEventRecord((cudaEvent_t)mid_event, s);
  }
  if (e == cudaSuccess) e = launch_mac(jobs, h->g.T, h->g.S, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}

effort_status_t effort_gemv_host(effort_handle_t h, const void* v_host, effort_dtype_t v_dtype, float effort,
                                 float* out_host, void* stream) {
  if (!h || !v_host || !out_host) return EFFORT_ERR_ARG;
  if (v_dtype != EFFORT_F32 && v_dtype != EFFORT_F16) return EFFORT_ERR_ARG;
  if (!effort_ok(effort)) return EFFORT_ERR_ARG;
  DeviceGuard guard(h->dev);
  cudaStream_t s = (cudaStream_t)stream;
  // page-locked memory mapped into the device's address space is read and
  // written in place by the kernels; other host memory goes through the
  // staging buffer with one copy each way
  void* mv = mapped_host_pointer(v_host);
  void* mo = mapped_host_pointer(out_host);
  void* d_v = mv ? mv : h->stage;
  float* d_out = mo ? static_cast<float*>(mo)
                    : reinterpret_cast<float*>(static_cast<char*>(h->stage) + stage_out_offset(h->g.I));
  const size_t vbytes = (size_t)h->g.I * (v_dtype == EFFORT_F16 ? 2 : 4);
  if (!mv && cudaMemcpyAsync(d_v, v_host, vbytes, cudaMemcpyHostToDevice, s) != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  const effort_status_t st = effort_gemv_ex(h, d_v, v_dtype, effort, d_out, nullptr, nullptr, nullptr, stream);
  if (st != EFFORT_OK) return st;
  if (!mo && cudaMemcpyAsync(out_host, d_out, (size_t)h->g.O * 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
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
  if (cudaMemcpy(&st, h->slot.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return EFFORT_ERR_CUDA;
  if (st && cudaMemset(h->slot.status, 0, 4) != cudaSuccess) return EFFORT_ERR_CUDA;
  if (st & kStatusNonfiniteV) return EFFORT_ERR_NONFINITE;
  if (st & kStatusInternal) return EFFORT_ERR_DEVICE;
  return EFFORT_OK;
}

effort_status_t effort_workspace_create(int64_t in_dim, int64_t out_dim, int32_t max_pairs, effort_workspace_t* out_ws) {
  if (!out_ws) return EFFORT_ERR_ARG;
  *out_ws = nullptr;
  if (in_dim < 1 || out_dim < 1 || max_pairs < 1) return EFFORT_ERR_ARG;
  if (out_dim > EFFORT_MAX_OUT_DIM || in_dim > EFFORT_MAX_IN_DIM) return EFFORT_ERR_UNSUPPORTED;
  effort_workspace_s* w = new (std::nothrow) effort_workspace_s();
  if (!w) return EFFORT_ERR_NOMEM;
  cudaGetDevice(&w->dev);
  effort_status_t st = make_geometry(in_dim, out_dim, &w->g);
  if (st != EFFORT_OK) {
    delete w;
    return st;
  }
  w->slots = new (std::nothrow) WsPtrs[max_pairs];
  if (!w->slots) {
    delete w;
    return EFFORT_ERR_NOMEM;
  }
  st = alloc_ws(w->g, max_pairs, &w->ws, w->slots);
  if (st != EFFORT_OK) {
    delete[] w->slots;
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
    cudaFree(w->ws.base);
  }
  delete[] w->slots;
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
  }
  DeviceGuard guard(ws->dev);
  cudaStream_t s = (cudaStream_t)stream;
  ws->last_stream = s;
  for (int p0 = 0; p0 < n_pairs; p0 += kMaxJobs) {
    const int nj = (n_pairs - p0 < kMaxJobs) ? n_pairs - p0 : kMaxJobs;
    Jobs<kMaxJobs> jobs;
    memset(&jobs, 0, sizeof(jobs));
    for (int q = 0; q < nj; ++q) {
      const int p = p0 + q;
      effort_handle_t h = handles[hidx[p]];
      if (!h || h->g.I != I || h->g.O != O) return EFFORT_ERR_ARG;
      effort_status_t st = fill_job(h, ws->slots[p], (const char*)V + (size_t)vidx[p] * I * vsz, v_dtype, efforts[p],
                                    OUT + (size_t)p * O, cutoffs_out ? cutoffs_out + p : nullptr,
                                    counts_out ? counts_out + p : nullptr, nullptr, &jobs.j[q]);
      if (st != EFFORT_OK) return st;
    }
    cudaError_t e = launch_cutoff_batch(jobs, nj, I, ws->g.cl, s);
    if (e == cudaSuccess) e = launch_mac_batch(jobs, nj, ws->g.T, ws->g.S, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return EFFORT_ERR_CUDA;
    }
  }
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
  cudaError_t e = launch_dense((const uint16_t*)W, ws->g.I, ws->g.O, v, (int)v_dtype, out, ws->slots[0].part,
                               ws->slots[0].tilecnt, ws->g.T, ws->g.S_dense, s);
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
  if (device_bytes) *device_bytes = h->storage_bytes + h->ws.bytes;
  return EFFORT_OK;
}

effort_status_t effort_get_layout(effort_handle_t h, effort_layout_t* L) {
  if (!h || !L) return EFFORT_ERR_ARG;
  L->in_dim = h->g.I;
  L->out_dim = h->g.O;
  L->n_kept = h->hd.n;
  L->n_tiles = h->hd.T;
  L->bucket_cap = kCap;
  L->ck_step = h->hd.H;
  L->n_ck = h->hd.C;
  L->n_probes = kP;
  L->vals = h->hd.vals;
  L->idx = h->hd.idx;
  L->probes = h->hd.probes;
  L->ckmag = h->hd.ckmag;
  L->cnt = h->hd.cnt;
  L->wdense = h->hd.wdense;
  L->rec = h->slot.rec;
  L->gcnt = h->slot.gcnt;
  L->n_groups = h->g.G;
  return EFFORT_OK;
}

effort_status_t effort_destroy(effort_handle_t h) {
  if (!h) return EFFORT_ERR_ARG;
  {
    DeviceGuard guard(h->dev);
    cudaStreamSynchronize(h->last_stream);
    cudaFree(h->stage);
    cudaFree(h->ws.base);
    cudaFree(h->storage);
  }
  delete h;
  return EFFORT_OK;
}

}  // extern "C"

namespace effort {

// For entry points that bring their own per-call scratch: the handle's device
// and the launch geometry of one call.
effort_status_t handle_call_geometry(effort_handle_t h, int* dev, int* I, int* T, int* G, int* S, int* cl) {
  if (!h) return EFFORT_ERR_ARG;
  *dev = h->dev;
  *I = h->g.I;
  *T = h->g.T;
  *G = h->g.G;
  *S = h->g.S;
  *cl = h->g.cl;
  return EFFORT_OK;
}

// The same argument checks and job description as effort_gemv_ex, with the
// caller's scratch in place of the handle's.
effort_status_t handle_fill_job(effort_handle_t h, const WsPtrs& ws, const void* v, effort_dtype_t v_dtype,
                                float effort, float* out, float* cutoff_out, uint64_t* count_out, Job* j) {
  if (!h) return EFFORT_ERR_ARG;
  return fill_job(h, ws, v, v_dtype, effort, out, cutoff_out, count_out, nullptr, j);
}

}  // namespace effort
