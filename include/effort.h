/*
 * effort.h -- C ABI of the B200 (sm_100a) library for the "Effort"
 * approximate matrix-vector multiply.
 *
 * The method (Hacker News item 40067677, "Show HN: Speeding up LLM inference
 * 2x times (possibly)", the pseudo-code quoted in a commenter's question and
 * the author's replies): every row of the weight matrix is stored sorted by
 * |w| descending; per call, an input vector v and an effort in (0, 1] pick a
 * cutoff c from per-row probes (cutoff_chart = v * probes, cutoff =
 * topK(chart, effort)), and only the products with |v_i| * |w_ij| >= c are
 * multiplied and added.  The author's complexity reply (Hacker News item
 * 40095016) gives O(effort * inDim * outDim) multiplications, O(inDim) for the
 * dispatch and about O(inDim log inDim) for the cutoff.
 *
 * Conventions (all entry points):
 *  - W is [in_dim x out_dim] binary16, row-major: row i holds the weights that
 *    multiply v[i], and out[j] = sum_i v[i] * W[i][j] (the matrix is already
 *    "flipped" in the sense of the pages).
 *  - Pointers named W, v, V, out, OUT, *_out are DEVICE pointers unless stated.
 *    The caller owns them; the library never frees them.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Every call returns an effort_status_t.  Argument errors are detected on
 *    the host before anything is launched.  No exception or abort crosses the
 *    ABI.  Device faults are never used to signal errors.
 *  - Selection rule: a kept pair (i, j) is used iff the single-precision
 *    product fl32(|v_i| * |w_ij|) (round to nearest even, no FMA, no flush to
 *    zero) is >= c.  Ties at c are used.  Outputs are accumulated in fp32.
 */
#ifndef EFFORT_H
#define EFFORT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct effort_handle_s* effort_handle_t;        /* prepared matrix, library-owned */
typedef struct effort_workspace_s* effort_workspace_t;  /* per-call scratch, library-owned */

typedef enum {
  EFFORT_OK = 0,
  EFFORT_ERR_ARG = 1,          /* bad pointer, size, effort, keep fraction or dtype */
  EFFORT_ERR_CUDA = 2,         /* a CUDA runtime call or kernel launch failed */
  EFFORT_ERR_NOMEM = 3,        /* device or host allocation failed */
  EFFORT_ERR_NONFINITE = 4,    /* W (prepare) or v (reported by effort_check) held inf/NaN */
  EFFORT_ERR_DEVICE = 5,       /* a kernel reported an internal inconsistency */
  EFFORT_ERR_UNSUPPORTED = 6   /* sizes outside the limits stated below */
} effort_status_t;

typedef enum { EFFORT_F32 = 0, EFFORT_F16 = 1 } effort_dtype_t;

/* Size limits of this build. */
#define EFFORT_MAX_OUT_DIM 32768      /* a row is sorted inside one thread block */
#define EFFORT_MAX_IN_DIM 40960       /* the cutoff's chart lives in one cluster's shared memory */
#define EFFORT_MAX_PAIRS_PER_LAUNCH 16
#define EFFORT_STATIC_SCRATCH_BYTES (2u << 20) /* per-device scratch of effort_gemv_static */

/*
 * effort_prepare -- the offline pass: `precompute(W)` of the pages.
 *   Sorts every row of W by |w| descending (ties: lower column first), keeps
 *   the first n = floor(keep_fraction * out_dim + 1/2) entries of each row
 *   (the post text: the format lets the loader skip the least important
 *   weights), takes 16 midpoint-rank probes per row, and stores the kept
 *   entries in output-tile buckets of 256 columns (fp16 value + 8-bit local
 *   index, bucket-sorted by |w|), a dense copy of the kept weights, and the
 *   checkpoint tables the dispatch uses.
 *   W: device, binary16 [in_dim x out_dim], 2-byte aligned; read only during
 *      the call (the stream is synchronised before returning; the caller may
 *      free W afterwards).
 *   keep_fraction: (0, 1].  Must keep at least one weight per row.
 *   Limits: 1 <= out_dim <= EFFORT_MAX_OUT_DIM, 1 <= in_dim <= EFFORT_MAX_IN_DIM,
 *           in_dim * out_dim < 2^32.
 *   Returns EFFORT_ERR_NONFINITE (and no handle) if W holds inf or NaN.
 *   On success *out_handle owns all device storage; free it with effort_destroy.
 */
effort_status_t effort_prepare(const void* W, int64_t in_dim, int64_t out_dim, float keep_fraction,
                               void* stream, effort_handle_t* out_handle);

/*
 * effort_gemv -- one approximate matvec: `approxMul(v, ...)` of the pages.
 *   v: device fp32 [in_dim]; out: device fp32 [out_dim], fully overwritten.
 *   effort in (0, 1]: K = llround(effort * in_dim * out_dim) products are
 *   targeted; the cutoff c is the weighted K-th largest entry of the chart
 *   fl32(|v_i| * probe_ik) (c = 0 if K >= the kept count, c = +inf if K = 0).
 *   Asynchronous and stream-ordered: no host synchronisation and no
 *   allocation; two kernels (cutoff+dispatch, then multiply-accumulate).
 *   A handle holds one call's scratch: calls on the same handle must be
 *   ordered (same stream, or synchronised); concurrent calls on one handle race.
 */
effort_status_t effort_gemv(effort_handle_t h, const float* v, float effort, float* out, void* stream);

/*
 * effort_gemv_ex -- effort_gemv with a v dtype and optional device outputs.
 *   v: device, EFFORT_F32 or EFFORT_F16, [in_dim].
 *   cutoff_out: nullable device float, receives c.
 *   count_out: nullable device uint64, receives |S|, the number of used products.
 *   rowlen_out: nullable device uint32 [in_dim], receives L_i, the number of
 *     used products of row i (always a leading part of row i's sorted order).
 */
effort_status_t effort_gemv_ex(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort,
                               float* out, float* cutoff_out, uint64_t* count_out, uint32_t* rowlen_out,
                               void* stream);

/*
 * effort_gemv_host -- effort_gemv_ex on HOST buffers, for callers that hold v
 *   and want out in host memory.  The pages have no counterpart: this is a
 *   library service around the same matvec.  On `stream`, in order, the same
 *   two kernels as effort_gemv_ex, with v (in_dim elements of v_dtype) and
 *   out (out_dim fp32) moved across the host link as follows:
 *   - page-locked memory mapped into the device's address space (cudaHostAlloc,
 *     cudaMallocHost, cudaHostRegister with mapping; cudaPointerGetAttributes
 *     decides) is read (v) and written (out) in place by the kernels, with no
 *     copy operation;
 *   - other host memory goes through the handle's device staging buffer, with
 *     one cudaMemcpyAsync before the kernels (v) and one after (out); CUDA
 *     stages pageable copies, which may block the host.
 *   v_host, out_host: host memory, non-NULL.
 *   The call does not synchronise: out_host holds the result once the stream
 *   has passed this call (cudaStreamSynchronize, an event).  The caller must
 *   not modify v_host or read out_host before then.
 *   The staging buffer (in_dim x 4 + out_dim x 4 bytes) is allocated by
 *   effort_prepare and belongs to the handle: calls on one handle must be
 *   ordered (one stream), like the handle's workspace.
 */
effort_status_t effort_gemv_host(effort_handle_t h, const void* v_host, effort_dtype_t v_dtype, float effort,
                                 float* out_host, void* stream);

/*
 * effort_gemv_split -- effort_gemv_ex that also records `mid_event` (a
 *   cudaEvent_t passed as void*, created by the caller) on the stream between
 *   the cutoff/dispatch kernel and the multiply kernel, so that each phase can
 *   be timed with events.  The multiply kernel then starts after the event
 *   instead of launching early against the first kernel.  mid_event non-NULL.
 *   Under stream capture the event is recorded with cudaEventRecordExternal,
 *   so that it becomes an event-record node of the CUDA graph.
 */
effort_status_t effort_gemv_split(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort,
                                  float* out, float* cutoff_out, uint64_t* count_out, void* mid_event,
                                  void* stream);

/*
 * effort_gemv_static -- effort_gemv_ex (without rowlen_out) whose per-call
 *   scratch is a fixed array of EFFORT_STATIC_SCRATCH_BYTES (2 MiB) per device,
 *   compiled into the library, instead of the handle's workspace.  The pages
 *   have no counterpart: this is a library service, not part of the method.
 *   It is for callers that must not allocate device memory on the call path,
 *   e.g. code running under another component's allocator (a caching
 *   allocator that must account for every byte, a memory pool sized up
 *   front), or that needs its device footprint fixed before the first call.
 *   The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *   library routine.  It issues one cudaMemsetAsync that clears the scratch
 *   words that must start at zero, the same two kernels as effort_gemv_ex,
 *   and, if status_out is given, one 4-byte device-to-device copy.
 *   v, v_dtype, effort, out, cutoff_out, count_out: as for effort_gemv_ex.
 *   status_out: nullable device uint32; receives 0 if the call saw only
 *     finite entries of v and no internal inconsistency, nonzero otherwise
 *     (the output is then unspecified).  effort_check does not see this call.
 *   Set-up: the first call on a device looks up that device's copy of the
 *     array (cudaGetSymbolAddress, with the handle's device made current);
 *     make that first call before any stream capture on the device.
 *   Every call on one device shares the array: calls that may overlap on the
 *     GPU (unordered streams, concurrent host threads) race and give wrong
 *     results; order them on one stream.
 *   Returns EFFORT_ERR_UNSUPPORTED when the handle's geometry needs more than
 *     EFFORT_STATIC_SCRATCH_BYTES of scratch (4096 x 14336 needs about 0.5 MiB,
 *     14336 x 4096 about 0.6 MiB), and when the device ordinal is 64 or above.
 */
effort_status_t effort_gemv_static(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort,
                                   float* out, float* cutoff_out, uint64_t* count_out, uint32_t* status_out,
                                   void* stream);

/*
 * effort_check -- synchronises the handle's last stream and reports whether a
 *   call since the previous check saw a non-finite entry of v
 *   (EFFORT_ERR_NONFINITE; those calls' outputs are unspecified) or an internal
 *   device inconsistency (EFFORT_ERR_DEVICE).  Clears the flags.
 */
effort_status_t effort_check(effort_handle_t h);

/*
 * Workspaces: scratch for effort_gemv_batched and effort_dense_gemv.
 *   Sized for matrices of in_dim x out_dim and up to max_pairs concurrent pairs
 *   per call (max_pairs >= 1).  Allocates device memory (not stream-ordered).
 */
effort_status_t effort_workspace_create(int64_t in_dim, int64_t out_dim, int32_t max_pairs,
                                        effort_workspace_t* out_ws);
effort_status_t effort_workspace_destroy(effort_workspace_t ws);

/*
 * effort_gemv_batched -- n_pairs independent matvecs (MoE-style routing: each
 *   vector meets the experts it was routed to; the author's complexity reply
 *   likens the per-multiplication choice of buckets to expert routing).
 *   Pair p uses handles[hidx[p]], vector V + vidx[p] * in_dim (dtype v_dtype),
 *   efforts[p], and writes OUT + p * out_dim (fp32).  hidx, vidx, efforts:
 *   HOST arrays of n_pairs entries.  All handles must share in_dim/out_dim
 *   with the workspace.  cutoffs_out [n_pairs] float and counts_out
 *   [n_pairs] uint64 are nullable device arrays.  One cutoff per pair.
 *   Launches two kernels per group of up to EFFORT_MAX_PAIRS_PER_LAUNCH pairs.
 *   n_pairs <= the workspace's max_pairs.
 */
effort_status_t effort_gemv_batched(effort_workspace_t ws, const effort_handle_t* handles, const int32_t* hidx,
                                    const int32_t* vidx, int32_t n_pairs, const void* V, effort_dtype_t v_dtype,
                                    const float* efforts, float* OUT, float* cutoffs_out, uint64_t* counts_out,
                                    void* stream);

/*
 * effort_dense_gemv -- the dense baseline out = W^T v (every weight, fp32
 *   accumulation), hand-written streaming kernel.  W: device binary16
 *   [in_dim x out_dim], out_dim a multiple of 8, 16-byte aligned.  v: fp32 or
 *   fp16 [in_dim].  Uses the workspace's first pair slot.
 */
effort_status_t effort_dense_gemv(effort_workspace_t ws, const void* W, int64_t in_dim, int64_t out_dim,
                                  const void* v, effort_dtype_t v_dtype, float* out, void* stream);

/* Sizes and footprint of a prepared matrix. */
effort_status_t effort_get_info(effort_handle_t h, int64_t* in_dim, int64_t* out_dim, float* keep_fraction,
                                size_t* device_bytes);

/*
 * effort_layout_t -- read-only view of a handle's device storage, for format
 * checks.  Bucket (i, t) holds the kept entries of row i with columns in
 * [256 t, 256 t + 256), sorted by |w| descending (ties: lower column), at
 * entry offset (t * in_dim + i) * bucket_cap of `vals` (binary16 bits) and
 * `idx` (column - 256 t); unused slots hold +0.0 / 0.
 * probes: [in_dim][16] |w| binary16 bits at the probe ranks (0 for empty segments).
 * ckmag: [in_dim][n_ck + 1]: [0] = |w| at rank 0; [1 + k] = |w| at rank
 *   min((k + 1) * ck_step, n) - 1.
 * cnt: [in_dim][n_ck][n_tiles] uint8: entries of tile t among the first
 *   min((k + 1) * ck_step, n) ranks of row i, saturated at 255.
 * wdense: [in_dim][n_tiles * 256] binary16: kept weights at their columns, 0 elsewhere.
 * rec / gcnt: the last call's dispatch records (see the library source).
 */
typedef struct {
  int64_t in_dim, out_dim;
  int32_t n_kept, n_tiles, bucket_cap, ck_step, n_ck, n_probes;
  const void* vals;
  const void* idx;
  const void* probes;
  const void* ckmag;
  const void* cnt;
  const void* wdense;
  const void* rec;
  const void* gcnt;
  int32_t n_groups;
} effort_layout_t;

effort_status_t effort_get_layout(effort_handle_t h, effort_layout_t* layout);

/* Frees the handle's device storage after synchronising its last stream. */
effort_status_t effort_destroy(effort_handle_t h);

/* Static string naming a status code. */
const char* effort_status_string(effort_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* EFFORT_H */
