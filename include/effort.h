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
 *  - W is [in_dim x out_dim] binary16 (or, for effort_prepare_q8, int8 with one
 *    binary16 scale per row), row-major: row i holds the weights that
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
  EFFORT_ERR_DEVICE = 5,       /* a kernel reported an internal inconsistency or a wait timed out */
  EFFORT_ERR_UNSUPPORTED = 6   /* sizes outside the limits stated below */
} effort_status_t;

typedef enum { EFFORT_F32 = 0, EFFORT_F16 = 1 } effort_dtype_t;

/* Size limits of this build. */
#define EFFORT_MAX_OUT_DIM 32768      /* a row is sorted inside one thread block */
#define EFFORT_MAX_IN_DIM 40960       /* a block's share of the chart lives in its shared memory */
#define EFFORT_STATIC_SCRATCH_BYTES (8u << 20) /* per-device scratch of effort_gemv_static */

/*
 * effort_prepare -- the offline pass: `precompute(W)` of the pages.
 *   Sorts every row of W by |w| descending (ties: lower column first), keeps
 *   the first n = floor(keep_fraction * out_dim + 1/2) entries of each row
 *   (the post text: the format lets the loader skip the least important
 *   weights), takes 16 midpoint-rank probes per row, and stores, for every row
 *   and every panel of 2048 output columns, the leading 3/8 of the row's kept
 *   entries in that panel in rank order, cut into chunks of 64 slots (each
 *   chunk sorted by column: fp16 value + 8-bit column gap); plus a dense copy
 *   of the kept weights for rows a call uses beyond that share.
 *   W: device, binary16 [in_dim x out_dim], 2-byte aligned; read only during
 *      the call (the stream is synchronised before returning; the caller may
 *      free W afterwards).
 *   keep_fraction: (0, 1].  Must keep at least one weight per row.
 *   Limits: 1 <= out_dim <= EFFORT_MAX_OUT_DIM, 1 <= in_dim <= EFFORT_MAX_IN_DIM,
 *           in_dim * out_dim < 2^32.
 *   Returns EFFORT_ERR_NONFINITE (and no handle) if W holds inf or NaN, and
 *   EFFORT_ERR_NOMEM if a device allocation fails or would take the library's
 *   device memory past the cap set by the environment variable
 *   EFFORT_ALLOC_CAP_BYTES (read at each allocation; unset = no cap).
 *   On success *out_handle owns all device storage; free it with effort_destroy.
 */
effort_status_t effort_prepare(const void* W, int64_t in_dim, int64_t out_dim, float keep_fraction,
                               void* stream, effort_handle_t* out_handle);

/*
 * effort_prepare_q8 -- effort_prepare for Q8 weights: int8 values q and one
 *   binary16 scale per row, the weight being w_ij = s_i * q_ij, taken exactly
 *   (the post says Q8 is in the works and the author that the algorithm
 *   should work on top of Q8: Hacker News item 40067677, "Show HN: Speeding
 *   up LLM inference 2x times (possibly)", the post text and the author's
 *   replies).  Everything the matvec computes follows from those weights as
 *   for effort_prepare: row order |w| descending with ties to the lower
 *   column, keep, probes, the cutoff c, the used set fl32(|v_i| |w_ij|) >= c
 *   and out.  The stored matrix holds q as int8: 2 bytes per chunk slot
 *   (value and gap) and 1 byte per column of the dense copy.
 *   q: device int8 [in_dim x out_dim], row-major (row i multiplies v[i]);
 *   scales: device binary16 bits [in_dim], 2-byte aligned, finite (zero and
 *   negative scales are allowed); both are read during the call only (the
 *   handle keeps its own copy of the scales).
 *   keep_fraction, stream, out_handle and the limits: as for effort_prepare.
 *   Returns EFFORT_ERR_NONFINITE if a scale is inf or NaN, EFFORT_ERR_ARG for
 *   a null or misaligned pointer or a bad keep_fraction.  Every matvec entry
 *   point accepts the handle (the dense baseline is for binary16 only).
 */
effort_status_t effort_prepare_q8(const int8_t* q, const uint16_t* scales, int64_t in_dim, int64_t out_dim,
                                  float keep_fraction, void* stream, effort_handle_t* out_handle);

/*
 * effort_gemv -- one approximate matvec: `approxMul(v, ...)` of the pages.
 *   v: device fp32 [in_dim]; out: device fp32 [out_dim], fully overwritten.
 *   effort in (0, 1]: K = llround(effort * in_dim * out_dim) products are
 *   targeted; the cutoff c is the weighted K-th largest entry of the chart
 *   fl32(|v_i| * probe_ik) (c = 0 if K >= the kept count, c = +inf if K = 0).
 *   Asynchronous and stream-ordered: no host synchronisation and no
 *   allocation; one kernel whose blocks (one per SM) compute the cutoff,
 *   the dispatch and the multiply-accumulate, meeting at grid-wide barriers.
 *   out is accumulated in fp32 with reductions whose order varies from call
 *   to call: c, |S| and the L_i are reproducible bit for bit, out to rounding.
 *   Each barrier wait has a time limit (0.2 s); a wait that runs out sets a
 *   status bit that effort_check reports as EFFORT_ERR_DEVICE.
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
 *   kernel as effort_gemv_ex, with v (in_dim elements of v_dtype) and out
 *   (out_dim fp32) moved across the host link as follows:
 *   - v is copied into the handle's device staging buffer with one
 *     cudaMemcpyAsync before the kernel (every block of the kernel reads v,
 *     so reading it in place across the host link would cost a host-link
 *     round trip per block);
 *   - out is accumulated in the staging buffer (the kernel adds partial sums
 *     into it with device-memory reductions).  When out_host is page-locked
 *     memory mapped into the device's address space (cudaHostAlloc,
 *     cudaMallocHost, cudaHostRegister with mapping; cudaPointerGetAttributes
 *     decides), the kernel's last block writes the finished out into it;
 *     otherwise it is copied back with one cudaMemcpyAsync after the kernel
 *     (CUDA stages copies to pageable memory, which may block the host).
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
 * effort_gemv_timed -- effort_gemv_ex (no optional outputs) that also stores
 *   the GPU global timer (ns) at fixed points of the call, for per-phase
 *   timing: marks is a device uint64 array [blocks][16] (blocks from
 *   effort_grid_blocks); entry k of block b is written by that block when it
 *   reaches point k: 0 start, 1 after waiting for the preceding grid, 2 chart
 *   histogram, entries and bin descriptors written, 3 after the first grid
 *   barrier, 4 crossing bin found, 5 the crossing bin's entries gathered
 *   (not reached with more than 4096 of them), 6 cutoff resolved, 7 work
 *   lists built,
 *   8 dense units streamed, 9 sparse chunks streamed, 10 registers added into
 *   the panel accumulator, 11 the block's sums added into out, 13 the block is
 *   done (12, 14 and 15 are not used); 8 and 9 are written by lane 0 of every
 *   warp (the last write stays).  Points a call does not reach (effort 1
 *   skips 2..5, a tiny effort returns after 1) keep their old
 *   contents.  The pages have no counterpart: a measurement service.
 */
effort_status_t effort_gemv_timed(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort,
                                  float* out, uint64_t* marks, void* stream);

/* Blocks of the grid a matvec on this handle launches (one per SM). */
effort_status_t effort_grid_blocks(effort_handle_t h, int32_t* blocks);

/*
 * effort_gemv_static -- effort_gemv_ex (without rowlen_out) whose per-call
 *   scratch is a fixed array of EFFORT_STATIC_SCRATCH_BYTES (8 MiB) per device,
 *   compiled into the library, instead of the handle's workspace.  The pages
 *   have no counterpart: this is a library service, not part of the method.
 *   It is for callers that must not allocate device memory on the call path,
 *   e.g. code running under another component's allocator (a caching
 *   allocator that must account for every byte, a memory pool sized up
 *   front), or that needs its device footprint fixed before the first call.
 *   The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *   library routine.  It issues one cudaMemsetAsync that clears the scratch
 *   words that must start at zero, the same kernel as effort_gemv_ex, and,
 *   if status_out is given, one 4-byte device-to-device copy.
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
 *     EFFORT_STATIC_SCRATCH_BYTES of scratch (a geometry needs about 2.4 MiB
 *     of histograms and bin descriptors on a 148-SM device plus 128 bytes per
 *     input row for the chart entries: 3.0 MiB at in_dim 4096, 7.7 MiB at
 *     EFFORT_MAX_IN_DIM), and when the device ordinal is 64 or above.
 *   The array's address is looked up again whenever the device's primary
 *     context has changed (after cudaDeviceReset), never kept across it.
 */
effort_status_t effort_gemv_static(effort_handle_t h, const void* v, effort_dtype_t v_dtype, float effort,
                                   float* out, float* cutoff_out, uint64_t* count_out, uint32_t* status_out,
                                   void* stream);

/*
 * effort_check -- synchronises the handle's last stream and reports whether a
 *   call since the previous check saw a non-finite entry of v
 *   (EFFORT_ERR_NONFINITE; those calls' outputs are unspecified) or a device
 *   inconsistency: a grid-wide wait that ran out of time, or, in a library
 *   built with -DEFFORT_DEBUG, an index a kernel found out of range
 *   (EFFORT_ERR_DEVICE; outputs of the calls since the previous check are
 *   unspecified).  Clears the flags; after an error it also resets the
 *   handle's scratch, so that later calls start clean.
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
 *   Two pairs on the same handle whose cutoffs both select (0 < K < the kept
 *   count) run as one kernel that reads the union of their prefixes once:
 *   each (row, panel) of the matrix is read as far as the lower of the two
 *   thresholds needs, and each vector's own threshold is applied to it, so
 *   each pair's cutoff, count and output are those of its own call (outputs
 *   to rounding).  Every other pair runs as one kernel of its own.  All
 *   kernels run in order on `stream` and share the workspace's scratch (two
 *   slots, the second allocated when max_pairs >= 2).  n_pairs <= the
 *   workspace's max_pairs.
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

/* Sizes and footprint of a prepared matrix (device_bytes: its stored format,
 * not counting the per-call scratch and staging buffer). */
effort_status_t effort_get_info(effort_handle_t h, int64_t* in_dim, int64_t* out_dim, float* keep_fraction,
                                size_t* device_bytes);

/*
 * effort_layout_t -- read-only view of a handle's device storage, for format
 * checks.  Panel p covers columns [panel_width p, panel_width (p + 1)).
 * lists: [in_dim][n_panels] of {first chunk, stored chunks, tail, kept}: list
 *   (i, p) holds the kept entries of row i in panel p in row i's order (|w|
 *   descending, ties: lower column); its leading ceil(kept * store_num /
 *   store_den) entries are stored in chunks [first, first + stored chunks);
 *   tail is the |w| binary16 bits of the first entry not stored (0 if none).
 * vals / gaps: chunk c occupies slots [chunk_slots c, chunk_slots (c + 1)):
 *   binary16 value bits and 8-bit column gaps.  The slots of a chunk are in
 *   column order; the column of a slot is -1 + the sum of the gaps up to and
 *   including it (panel-local).  Filler slots (value +0, gap 255) bridge gaps
 *   above 255; pad slots (value +0, gap 0) fill the chunk.
 * head: [total_chunks] |w| bits of each chunk's first (largest) rank.
 * wdense: [in_dim][dense_stride] binary16: kept weights at their columns, +0
 *   elsewhere.  probes: [in_dim][16] |w| bits at the probe ranks (0 for empty
 *   segments).  scratch_bytes: the handle's per-call scratch.
 * weight_kind: 0 for a matrix from effort_prepare, 1 for one from
 *   effort_prepare_q8.  For Q8, vals and wdense hold int8 q (1 byte per slot
 *   or column), tail, head and probes hold the binary16 bits of |q| (0 on a
 *   row whose scale is 0), and scales is the handle's copy of the row
 *   scales [in_dim] (binary16); null for fp16.
 */
typedef struct {
  int64_t in_dim, out_dim;
  int32_t n_kept, n_panels, panel_width, chunk_slots, store_num, store_den, n_probes, dense_stride;
  uint32_t total_chunks;
  const void* vals;
  const void* gaps;
  const void* head;
  const void* lists;
  const void* wdense;
  const void* probes;
  size_t scratch_bytes;
  int32_t weight_kind;
  const void* scales;
} effort_layout_t;

effort_status_t effort_get_layout(effort_handle_t h, effort_layout_t* layout);

/* Frees the handle's device storage after synchronising its last stream. */
effort_status_t effort_destroy(effort_handle_t h);

/*
 * effort_last_call_bytes -- the bytes of the prepared matrix that the handle's
 *   last finished call (effort_gemv, _ex, _host) planned to read: dense_bytes
 *   for the (row, panel) units it read from the dense copy (512 bytes per
 *   256-column stripe; 256 for Q8), sparse_bytes for the chunks (3 bytes per
 *   slot, 2 for Q8; 64 slots per chunk).  Synchronises the handle's last stream.  The pages have
 *   no counterpart: a measurement service.  dense_bytes, sparse_bytes: host
 *   pointers, non-NULL.
 */
effort_status_t effort_last_call_bytes(effort_handle_t h, uint64_t* dense_bytes, uint64_t* sparse_bytes);

/*
 * effort_workspace_check -- effort_check for the workspace's calls
 *   (effort_gemv_batched, effort_dense_gemv): synchronises its last stream,
 *   reports EFFORT_ERR_NONFINITE if a pair's v held inf or NaN and
 *   EFFORT_ERR_DEVICE after a timed-out wait or an out-of-range index (debug
 *   build), clears the flags and, after an error, the workspace's scratch.
 */
effort_status_t effort_workspace_check(effort_workspace_t ws);

/*
 * effort_workspace_last_call_bytes -- the same for the workspace's last
 *   effort_gemv_batched call: the bytes its grids planned to read, summed
 *   over the grids (a grid serving two pairs on one matrix reads the union of
 *   their prefixes once, and counts it once).  Synchronises the workspace's
 *   last stream.  A measurement service.
 */
effort_status_t effort_workspace_last_call_bytes(effort_workspace_t ws, uint64_t* dense_bytes,
                                                 uint64_t* sparse_bytes);

/* Device memory the library holds at this moment, over all handles and
 * workspaces of the process (the figure EFFORT_ALLOC_CAP_BYTES is checked
 * against).  bytes: host pointer, non-NULL. */
effort_status_t effort_device_bytes_held(uint64_t* bytes);

/* Static string naming a status code. */
const char* effort_status_string(effort_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* EFFORT_H */
