// effort_gemv_static: the single-pair matvec of effort_gemv_ex with its
// per-call scratch in a fixed device array of this module instead of memory
// the handle allocated.  It serves callers that must not allocate device
// memory on the call path: code that runs while another component owns the
// allocator (a caching allocator that must see every allocation, or a memory
// pool sized up front), and code that must keep its footprint fixed and known
// before the first call.
//
// The scratch is one static array per device (every module-scope __device__
// variable exists once per device context).  Its address is taken once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call that runs there.  Every call then clears the words that must start at
// zero with one cudaMemsetAsync on the call's stream and launches the same
// two kernels as effort_gemv_ex.
//
// All calls on one device share the array: calls that overlap on the GPU
// (different streams without ordering, or concurrent host threads) race and
// give wrong results.
#include <mutex>

#include "../../include/effort.h"
#include "effort_internal.cuh"

namespace effort {
cudaError_t launch_cutoff(const Jobs<1>& jobs, int I, int cl, cudaStream_t stream);
cudaError_t launch_mac(const Jobs<1>& jobs, int T, int S, cudaStream_t stream);
effort_status_t handle_call_geometry(effort_handle_t h, int* dev, int* I, int* T, int* G, int* S, int* cl);
effort_status_t handle_fill_job(effort_handle_t h, const WsPtrs& ws, const void* v, effort_dtype_t v_dtype,
                                float effort, float* out, float* cutoff_out, uint64_t* count_out, Job* j);
}  // namespace effort

using namespace effort;

namespace {

constexpr size_t kScratchBytes = EFFORT_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Bytes of scratch one call needs: header (c, count, done, status), the
// per-tile arrival counters, the dispatch tables and the split-K partials.
size_t scratch_bytes(int T, int G, int S) {
  return 256 + align256((size_t)T * 4) + align256((size_t)G * 4) + align256((size_t)G * T * 32) +
         align256((size_t)G * kRecPerGroup * 8) + align256((size_t)S * T * kTW * 4);
}

// Carves the scratch in the same order as the handle's own workspace.
WsPtrs carve(char* b, int T, int G) {
  WsPtrs w;
  w.c = (float*)(b + 0);
  w.count = (unsigned long long*)(b + 8);
  w.done = (unsigned int*)(b + 16);
  w.status = (unsigned int*)(b + 20);
  b += 256;
  w.tilecnt = (unsigned int*)b;
  b += align256((size_t)T * 4);
  w.gcnt = (unsigned int*)b;
  b += align256((size_t)G * 4);
  w.ut = (unsigned char*)b;
  b += align256((size_t)G * T * 32);
  w.rec = (uint2*)b;
  b += align256((size_t)G * kRecPerGroup * 8);
  w.part = (float*)b;
  return w;
}

// Address of this device's copy of the array; looked up once per device.
// The caller has made `dev` current.
effort_status_t scratch_for_device(int dev, char** out) {
  if (dev < 0 || dev >= kMaxDevices) return EFFORT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return EFFORT_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = (char*)g_scratch_ptr[dev];
  return EFFORT_OK;
}

struct CurrentDevice {
  int prev = -1;
  bool ok = true;
  explicit CurrentDevice(int dev) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) {
      ok = false;
    } else if (cur != dev) {
      ok = cudaSetDevice(dev) == cudaSuccess;
      prev = cur;
    }
  }
  ~CurrentDevice() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

}  // namespace

extern "C" effort_status_t effort_gemv_static(effort_handle_t h, const void* v, effort_dtype_t v_dtype,
                                              float effort, float* out, float* cutoff_out, uint64_t* count_out,
                                              uint32_t* status_out, void* stream) {
  int dev = 0, I = 0, T = 0, G = 0, S = 0, cl = 0;
  effort_status_t st = handle_call_geometry(h, &dev, &I, &T, &G, &S, &cl);
  if (st != EFFORT_OK) return st;
  const size_t need = scratch_bytes(T, G, S);
  if (need > kScratchBytes) return EFFORT_ERR_UNSUPPORTED;
  CurrentDevice guard(dev);
  if (!guard.ok) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  char* base = nullptr;
  st = scratch_for_device(dev, &base);
  if (st != EFFORT_OK) return st;
  const WsPtrs ws = carve(base, T, G);
  Jobs<1> jobs;
  st = handle_fill_job(h, ws, v, v_dtype, effort, out, cutoff_out, count_out, &jobs.j[0]);
  if (st != EFFORT_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // header and per-tile counters start at zero; everything else is written
  // before it is read within the call
  cudaError_t e = cudaMemsetAsync(base, 0, 256 + align256((size_t)T * 4), s);
  if (e == cudaSuccess) e = launch_cutoff(jobs, I, cl, s);
  if (e == cudaSuccess) e = launch_mac(jobs, T, S, s);
  if (e == cudaSuccess && status_out) e = cudaMemcpyAsync(status_out, ws.status, 4, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}
