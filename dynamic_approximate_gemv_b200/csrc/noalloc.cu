// effort_gemv_static: the single-pair matvec of effort_gemv_ex with its
// per-call scratch in a fixed device array of this module instead of memory
// the handle allocated.  It serves callers that must not allocate device
// memory on the call path: code that runs while another component owns the
// allocator (a caching allocator that must see every allocation, or a memory
// pool sized up front), and code that must keep its footprint fixed and known
// before the first call.
//
// The scratch is one static array per device (every module-scope __device__
// variable exists once per device context).  Its address is taken with
// cudaGetSymbolAddress, with that device current, on the first call that runs
// in a given context of that device, and taken again if the context changed
// since (a cudaDeviceReset creates a new primary context, in which the module
// and its array are loaded anew).  Every call then clears the words that must
// start at zero with one cudaMemsetAsync on the call's stream and launches
// the same kernel as effort_gemv_ex.
//
// All calls on one device share the array: calls that overlap on the GPU
// (different streams without ordering, or concurrent host threads) race and
// give wrong results.
#include <mutex>

#include "../../include/effort.h"
#include "effort_internal.cuh"

namespace effort {
size_t handle_scratch_bytes(effort_handle_t h);
size_t handle_scratch_zero_bytes(effort_handle_t h);
WsPtrs handle_carve(effort_handle_t h, char* base);
int handle_device(effort_handle_t h);
effort_status_t handle_fill_job(effort_handle_t h, const WsPtrs& ws, const void* v, effort_dtype_t v_dtype,
                                float effort, float* out, float* cutoff_out, uint64_t* count_out, Job* j);
cudaError_t handle_launch(effort_handle_t h, const Job& j, cudaStream_t s);
}  // namespace effort

using namespace effort;

namespace {

constexpr size_t kScratchBytes = EFFORT_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};

// The calling thread's current context, through the driver entry point the
// runtime hands out (no link-time dependency on the driver library).
typedef int (*CtxGetCurrentFn)(void**);
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static bool looked = false;
  if (!looked) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
    else
      cudaGetLastError();
    looked = true;
  }
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Address of this device's copy of the array, looked up once per device and
// context.  The caller has made `dev` current.
effort_status_t scratch_for_device(int dev, char** out) {
  if (dev < 0 || dev >= kMaxDevices) return EFFORT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  void* ctx = current_context();
  if (!g_scratch_ptr[dev] || ctx != g_scratch_ctx[dev] || ctx == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return EFFORT_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
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
  if (!h) return EFFORT_ERR_ARG;
  Job probe;
  effort_status_t st = handle_fill_job(h, WsPtrs{}, v, v_dtype, effort, out, cutoff_out, count_out, &probe);
  if (st != EFFORT_OK) return st;
  if (handle_scratch_bytes(h) > kScratchBytes) return EFFORT_ERR_UNSUPPORTED;
  const int dev = handle_device(h);
  CurrentDevice guard(dev);
  if (!guard.ok) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  char* base = nullptr;
  st = scratch_for_device(dev, &base);
  if (st != EFFORT_OK) return st;
  const WsPtrs ws = handle_carve(h, base);
  Job job;
  st = handle_fill_job(h, ws, v, v_dtype, effort, out, cutoff_out, count_out, &job);
  if (st != EFFORT_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // header, barrier counter, histograms and bin descriptors start at zero
  // (whatever an earlier call on this device left, a timed-out one
  // included); everything else is written before it is read within the call
  cudaError_t e = cudaMemsetAsync(base, 0, handle_scratch_zero_bytes(h), s);
  if (e == cudaSuccess) e = handle_launch(h, job, s);
  if (e == cudaSuccess && status_out)
    e = cudaMemcpyAsync(status_out, ws.hdr + kHdrStatus, 4, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EFFORT_ERR_CUDA;
  }
  return EFFORT_OK;
}
