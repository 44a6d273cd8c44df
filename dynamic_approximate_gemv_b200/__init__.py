"""Python binding of libeffort, the B200 library for the Effort approximate matvec.

Argument marshalling only: tensors are passed to the C ABI of
``include/effort.h`` as raw device pointers with torch's current CUDA stream;
every step of the computation runs in the library's CUDA kernels.  There is no
fallback: if ``libeffort.so`` is missing or a call fails, an exception is
raised.

Method: Hacker News item 40067677, "Show HN: Speeding up LLM inference 2x times
(possibly)" -- rows sorted by |w|, probes, cutoff = topK(v * probes, effort),
multiply over the used leading part of every row.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libeffort.so")
# EFFORT_DEBUG_LIB=1 loads the bounds-checking build (kernels compiled with
# -DEFFORT_DEBUG report bad indices through effort_check instead of using them)
LIB_DEBUG_PATH = os.path.join(_HERE, "libeffort_debug.so")

F32, F16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "CUDA error", 3: "out of memory",
          4: "non-finite input", 5: "device-side inconsistency", 6: "unsupported size"}
MAX_OUT_DIM = 32768
MAX_IN_DIM = 40960

_lib = None


class EffortError(RuntimeError):
    def __init__(self, status, what):
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class Layout(ctypes.Structure):
    _fields_ = [("in_dim", ctypes.c_int64), ("out_dim", ctypes.c_int64),
                ("n_kept", ctypes.c_int32), ("n_panels", ctypes.c_int32), ("panel_width", ctypes.c_int32),
                ("chunk_slots", ctypes.c_int32), ("store_num", ctypes.c_int32), ("store_den", ctypes.c_int32),
                ("n_probes", ctypes.c_int32), ("dense_stride", ctypes.c_int32), ("total_chunks", ctypes.c_uint32),
                ("vals", ctypes.c_void_p), ("gaps", ctypes.c_void_p), ("head", ctypes.c_void_p),
                ("lists", ctypes.c_void_p), ("wdense", ctypes.c_void_p), ("probes", ctypes.c_void_p),
                ("scratch_bytes", ctypes.c_size_t), ("weight_kind", ctypes.c_int32), ("scales", ctypes.c_void_p)]


def lib():
    """Load libeffort.so (built in-tree by dynamic_approximate_gemv_b200.build)."""
    global _lib
    if _lib is None:
        path = LIB_DEBUG_PATH if os.environ.get("EFFORT_DEBUG_LIB") == "1" else LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run `python -m dynamic_approximate_gemv_b200.build`")
        L = ctypes.CDLL(path)
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
        sig = {
            "effort_prepare": [vp, i64, i64, f32, vp, ctypes.POINTER(vp)],
            "effort_prepare_q8": [vp, vp, i64, i64, f32, vp, ctypes.POINTER(vp)],
            "effort_gemv": [vp, vp, f32, vp, vp],
            "effort_gemv_ex": [vp, vp, ctypes.c_int, f32, vp, vp, vp, vp, vp],
            "effort_gemv_host": [vp, vp, ctypes.c_int, f32, vp, vp],
            "effort_gemv_timed": [vp, vp, ctypes.c_int, f32, vp, vp, vp],
            "effort_grid_blocks": [vp, ctypes.POINTER(i32)],
            "effort_gemv_static": [vp, vp, ctypes.c_int, f32, vp, vp, vp, vp, vp],
            "effort_check": [vp],
            "effort_workspace_create": [i64, i64, i32, ctypes.POINTER(vp)],
            "effort_workspace_destroy": [vp],
            "effort_gemv_batched": [vp, vp, vp, vp, i32, vp, ctypes.c_int, vp, vp, vp, vp, vp],
            "effort_dense_gemv": [vp, vp, i64, i64, vp, ctypes.c_int, vp, vp],
            "effort_get_info": [vp, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(f32),
                                ctypes.POINTER(ctypes.c_size_t)],
            "effort_get_layout": [vp, ctypes.POINTER(Layout)],
            "effort_destroy": [vp],
            "effort_device_bytes_held": [ctypes.POINTER(ctypes.c_uint64)],
            "effort_last_call_bytes": [vp, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64)],
            "effort_workspace_last_call_bytes": [vp, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64)],
            "effort_workspace_check": [vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.effort_status_string.argtypes = [ctypes.c_int]
        L.effort_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status, what):
    if status != 0:
        raise EffortError(status, what)


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _vdtype(v):
    if v.dtype == torch.float32:
        return F32
    if v.dtype == torch.float16:
        return F16
    raise TypeError("v must be float32 or float16")


def _need_cuda(t, name):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


class _CudaView:
    """Zero-copy torch view of library-owned device memory (read-only use)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


class PreparedMatrix:
    """A weight matrix W [in_dim x out_dim] (fp16) prepared for effort_gemv."""

    def __init__(self, W, keep_fraction=1.0):
        _need_cuda(W, "W")
        if W.dtype != torch.float16 or W.dim() != 2:
            raise ValueError("W must be a 2-D float16 tensor")
        self.in_dim, self.out_dim = W.shape
        self.device = W.device
        self.keep_fraction = float(keep_fraction)
        h = ctypes.c_void_p()
        with torch.cuda.device(W.device):
            _check(lib().effort_prepare(_ptr(W), self.in_dim, self.out_dim, ctypes.c_float(keep_fraction),
                                        _stream(W.device), ctypes.byref(h)), "effort_prepare")
        self._h = h

    @classmethod
    def from_q8(cls, q, scales, keep_fraction=1.0):
        """A Q8 matrix: int8 q [in_dim x out_dim] and float16 row scales
        [in_dim] (w = scales[i] * q[i, j], exact), prepared for effort_gemv."""
        _need_cuda(q, "q")
        _need_cuda(scales, "scales")
        if q.dtype != torch.int8 or q.dim() != 2:
            raise ValueError("q must be a 2-D int8 tensor")
        if scales.dtype != torch.float16 or tuple(scales.shape) != (q.shape[0],):
            raise ValueError("scales must be float16 [in_dim]")
        self = cls.__new__(cls)
        self.in_dim, self.out_dim = q.shape
        self.device = q.device
        self.keep_fraction = float(keep_fraction)
        h = ctypes.c_void_p()
        with torch.cuda.device(q.device):
            _check(lib().effort_prepare_q8(_ptr(q), _ptr(scales), self.in_dim, self.out_dim,
                                           ctypes.c_float(keep_fraction), _stream(q.device), ctypes.byref(h)),
                   "effort_prepare_q8")
        self._h = h
        return self

    def gemv(self, v, effort, out=None, cutoff=None, count=None, rowlen=None):
        """out[j] = sum over used (i, j) of v[i] * W[i, j]; returns out (fp32)."""
        _need_cuda(v, "v")
        if v.shape != (self.in_dim,):
            raise ValueError("v has the wrong shape")
        if out is None:
            out = torch.empty(self.out_dim, device=v.device, dtype=torch.float32)
        _need_cuda(out, "out")
        if out.dtype != torch.float32 or out.shape != (self.out_dim,):
            raise ValueError("out must be float32 [out_dim]")
        for t, dt, shp, nm in ((cutoff, torch.float32, (1,), "cutoff"), (count, torch.int64, (1,), "count"),
                               (rowlen, torch.int32, (self.in_dim,), "rowlen")):
            if t is not None:
                _need_cuda(t, nm)
                if t.dtype != dt or tuple(t.shape) != shp:
                    raise ValueError(f"{nm} must be {dt} of shape {shp}")
        _check(lib().effort_gemv_ex(self._h, _ptr(v), _vdtype(v), ctypes.c_float(effort), _ptr(out), _ptr(cutoff),
                                    _ptr(count), _ptr(rowlen), _stream(v.device)), "effort_gemv")
        return out

    def gemv_host(self, v, effort, out=None):
        """gemv on host tensors: v (float32 or float16 [in_dim]) is copied to the
        device, the matvec runs, and out (float32 [out_dim], host) is copied
        back, all on the current stream of the handle's device.  Pinned
        (page-locked) tensors keep the copies asynchronous.  out is valid once
        that stream has passed the call (e.g. torch.cuda.synchronize())."""
        if not (isinstance(v, torch.Tensor) and v.device.type == "cpu" and v.is_contiguous()):
            raise ValueError("v must be a contiguous host tensor")
        if v.shape != (self.in_dim,):
            raise ValueError("v has the wrong shape")
        if out is None:
            out = torch.empty(self.out_dim, dtype=torch.float32, pin_memory=True)
        if not (isinstance(out, torch.Tensor) and out.device.type == "cpu" and out.is_contiguous()):
            raise ValueError("out must be a contiguous host tensor")
        if out.dtype != torch.float32 or out.shape != (self.out_dim,):
            raise ValueError("out must be float32 [out_dim]")
        _check(lib().effort_gemv_host(self._h, _ptr(v), _vdtype(v), ctypes.c_float(effort), _ptr(out),
                                      _stream(self.device)), "effort_gemv_host")
        return out

    def gemv_static(self, v, effort, out=None, cutoff=None, count=None, status=None):
        """gemv whose scratch is the library's fixed per-device array (no device
        allocation by the library; calls on one device must not overlap).
        status: optional int32 [1] tensor, set nonzero if v held inf/NaN."""
        _need_cuda(v, "v")
        if v.shape != (self.in_dim,):
            raise ValueError("v has the wrong shape")
        if out is None:
            out = torch.empty(self.out_dim, device=v.device, dtype=torch.float32)
        _need_cuda(out, "out")
        if out.dtype != torch.float32 or out.shape != (self.out_dim,):
            raise ValueError("out must be float32 [out_dim]")
        for t, dt, nm in ((cutoff, torch.float32, "cutoff"), (count, torch.int64, "count"),
                          (status, torch.int32, "status")):
            if t is not None:
                _need_cuda(t, nm)
                if t.dtype != dt or tuple(t.shape) != (1,):
                    raise ValueError(f"{nm} must be {dt} of shape (1,)")
        _check(lib().effort_gemv_static(self._h, _ptr(v), _vdtype(v), ctypes.c_float(effort), _ptr(out),
                                        _ptr(cutoff), _ptr(count), _ptr(status), _stream(v.device)),
               "effort_gemv_static")
        return out

    def grid_blocks(self):
        n = ctypes.c_int32()
        _check(lib().effort_grid_blocks(self._h, ctypes.byref(n)), "effort_grid_blocks")
        return n.value

    def gemv_timed(self, v, effort, out, marks):
        """gemv that stores per-phase global-timer marks into `marks`
        (int64 [grid_blocks(), 16] on the device)."""
        _need_cuda(v, "v")
        _need_cuda(out, "out")
        _need_cuda(marks, "marks")
        if marks.dtype != torch.int64 or tuple(marks.shape) != (self.grid_blocks(), 16):
            raise ValueError("marks must be int64 [grid_blocks(), 16]")
        _check(lib().effort_gemv_timed(self._h, _ptr(v), _vdtype(v), ctypes.c_float(effort), _ptr(out), _ptr(marks),
                                       _stream(v.device)), "effort_gemv_timed")
        return out

    def last_call_bytes(self):
        """(dense, sparse) bytes of the prepared matrix the last finished call
        planned to read (synchronises the handle's stream)."""
        d, sp = ctypes.c_uint64(), ctypes.c_uint64()
        _check(lib().effort_last_call_bytes(self._h, ctypes.byref(d), ctypes.byref(sp)), "effort_last_call_bytes")
        return d.value, sp.value

    def check(self):
        _check(lib().effort_check(self._h), "effort_check")

    def info(self):
        i, o = ctypes.c_int64(), ctypes.c_int64()
        k, b = ctypes.c_float(), ctypes.c_size_t()
        _check(lib().effort_get_info(self._h, ctypes.byref(i), ctypes.byref(o), ctypes.byref(k), ctypes.byref(b)),
               "effort_get_info")
        return {"in_dim": i.value, "out_dim": o.value, "keep_fraction": k.value, "device_bytes": b.value}

    def layout(self):
        """Device storage as read-only torch views (for format checks)."""
        L = Layout()
        _check(lib().effort_get_layout(self._h, ctypes.byref(L)), "effort_get_layout")
        I, P, nc, cs = L.in_dim, L.n_panels, L.total_chunks, L.chunk_slots

        def view(ptr, shape, typestr):
            return torch.as_tensor(_CudaView(ptr, shape, typestr), device=self.device)

        vt = "|i1" if L.weight_kind == 1 else "<i2"  # int8 values of a Q8 matrix
        out = {
            "n_kept": L.n_kept, "n_panels": P, "panel_width": L.panel_width, "chunk_slots": cs,
            "store_num": L.store_num, "store_den": L.store_den, "total_chunks": nc,
            "dense_stride": L.dense_stride, "scratch_bytes": L.scratch_bytes, "weight_kind": L.weight_kind,
            "vals": view(L.vals, (max(nc, 1) * cs,), vt), "gaps": view(L.gaps, (max(nc, 1) * cs,), "|u1"),
            "head": view(L.head, (max(nc, 1),), "<i2"), "lists": view(L.lists, (I, P, 4), "<u4"),
            "wdense": view(L.wdense, (I, L.dense_stride), vt), "probes": view(L.probes, (I, L.n_probes), "<i2"),
        }
        if L.weight_kind == 1:
            out["scales"] = view(L.scales, (I,), "<i2")
        return out

    def close(self):
        if getattr(self, "_h", None):
            lib().effort_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Workspace:
    """Scratch for batched and dense calls on in_dim x out_dim matrices."""

    def __init__(self, in_dim, out_dim, max_pairs=1, device=None):
        self.in_dim, self.out_dim, self.max_pairs = int(in_dim), int(out_dim), int(max_pairs)
        h = ctypes.c_void_p()
        with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
            _check(lib().effort_workspace_create(self.in_dim, self.out_dim, self.max_pairs, ctypes.byref(h)),
                   "effort_workspace_create")
        self._h = h

    def check(self):
        _check(lib().effort_workspace_check(self._h), "effort_workspace_check")

    def last_call_bytes(self):
        """(dense, sparse) bytes the last batched call's grids planned to read,
        summed over the grids (synchronises the workspace's stream)."""
        d, sp = ctypes.c_uint64(), ctypes.c_uint64()
        _check(lib().effort_workspace_last_call_bytes(self._h, ctypes.byref(d), ctypes.byref(sp)),
               "effort_workspace_last_call_bytes")
        return d.value, sp.value

    def close(self):
        if getattr(self, "_h", None):
            lib().effort_workspace_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def device_bytes_held():
    """Device memory the library holds now (all handles and workspaces)."""
    x = ctypes.c_uint64()
    _check(lib().effort_device_bytes_held(ctypes.byref(x)), "effort_device_bytes_held")
    return x.value


def gemv_batched(ws, mats, hidx, vidx, V, efforts, OUT=None, cutoffs=None, counts=None):
    """Independent matvecs: pair p uses mats[hidx[p]] on V[vidx[p]] at efforts[p] -> OUT[p]."""
    _need_cuda(V, "V")
    n = len(hidx)
    if not (len(vidx) == n and len(efforts) == n):
        raise ValueError("hidx, vidx and efforts must have the same length")
    if OUT is None:
        OUT = torch.empty(n, ws.out_dim, device=V.device, dtype=torch.float32)
    handles = (ctypes.c_void_p * len(mats))(*[m._h.value for m in mats])
    hi = (ctypes.c_int32 * n)(*[int(x) for x in hidx])
    vi = (ctypes.c_int32 * n)(*[int(x) for x in vidx])
    ef = (ctypes.c_float * n)(*[float(x) for x in efforts])
    if any(not (0 <= int(x) < len(mats)) for x in hidx) or any(not (0 <= int(x) < V.shape[0]) for x in vidx):
        raise ValueError("hidx / vidx out of range")
    _check(lib().effort_gemv_batched(ws._h, handles, hi, vi, n, _ptr(V), _vdtype(V), ef, _ptr(OUT), _ptr(cutoffs),
                                     _ptr(counts), _stream(V.device)), "effort_gemv_batched")
    return OUT


def dense_gemv(ws, W, v, out=None):
    """Dense baseline out = W^T v with the library's streaming kernel."""
    _need_cuda(W, "W")
    _need_cuda(v, "v")
    if out is None:
        out = torch.empty(W.shape[1], device=W.device, dtype=torch.float32)
    _check(lib().effort_dense_gemv(ws._h, _ptr(W), W.shape[0], W.shape[1], _ptr(v), _vdtype(v), _ptr(out),
                                   _stream(W.device)), "effort_dense_gemv")
    return out
