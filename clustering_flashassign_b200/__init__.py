"""Python binding of libfk.so (include/fk.h): exact batched Lloyd's K-Means on B200.

Argument marshalling only -- every step of the computation runs in the CUDA
library.  The functions mirror the C ABI names; they take torch tensors
(contiguous, row-major), pass their data pointers and sizes, and raise
``FkError`` when the library returns a status other than FK_OK.  There is no
fallback: when libfk.so is missing, importing this package raises.

    fk_assign(x, c, ids)                        FlashAssign      (B,N,d),(B,K,d) -> ids (B,N) int32
    fk_update(x, ids, centers, counts=None)     sort-inverse update, centers (B,K,d) fp32 in/out
    fk_sort(ids, K, perm, counts=None, offsets=None)
    fk_lloyd(x, init_centers, max_iter, tol, ids, centers) -> iterations run

Per-rank pieces of a data-parallel run (points of a batch split over ranks;
the loop that joins them with an all-reduce is clustering_flashassign_b200.dist):

    fk_point_norms(x, xn)                       ||x_i||^2 for the tensor-core assign
    fk_init_centers(init, centers)              fp32 master copy of the initial centroids
    fk_lloyd_step_partial(x, xn, centers_dt, ids, sums, counts)   assign + unnormalised update
    fk_update_finalize(sums, counts, centers, centers_dt, max_shift)
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfk.so")

FK_F32, FK_F16, FK_BF16 = 0, 1, 2
FK_OK, FK_EINVAL, FK_ENOMEM, FK_ECUDA, FK_ETIMEOUT, FK_EUNSUPPORTED = range(6)
FK_HOST_AUTO, FK_HOST_RESIDENT, FK_HOST_STREAM = 0, 1, 2
FK_FAULT_NONE, FK_FAULT_ALLOC, FK_FAULT_H2D, FK_FAULT_LAUNCH = 0, 1, 2, 3

DTYPES = {torch.float32: FK_F32, torch.float16: FK_F16, torch.bfloat16: FK_BF16}

EXPORTS = ["fk_assign", "fk_update", "fk_sort", "fk_lloyd", "fk_assign_noalloc", "fk_noalloc_device_error",
           "fk_status_string",
           "fk_last_error", "fk_device_error", "fk_release", "fk_profile_enable", "fk_profile_read", "fk_profile_timeline",
           "fk_launch_count", "fk_version", "fk_selftest_bounded_wait", "fk_point_norms",
           "fk_init_centers", "fk_lloyd_step_partial", "fk_update_finalize", "fk_inject_fault"]


class FkError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


class FkShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_longlong), ("K", ctypes.c_int),
                ("d", ctypes.c_int), ("dtype", ctypes.c_int)]


class FkOptions(ctypes.Structure):
    _fields_ = [("host_mode", ctypes.c_int), ("chunk_points", ctypes.c_longlong),
                ("verbose", ctypes.c_int)]


class FkProfile(ctypes.Structure):
    _fields_ = [("assign_ms", ctypes.c_double), ("assign_launches", ctypes.c_longlong),
                ("sort_ms", ctypes.c_double), ("reduce_ms", ctypes.c_double),
                ("finalize_ms", ctypes.c_double), ("update_calls", ctypes.c_longlong),
                ("kernel_launches", ctypes.c_longlong), ("update_ms", ctypes.c_double)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libfk.so not built at {LIB_PATH}; run python clustering_flashassign_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, LL, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
    sig = {
        "fk_assign": (I, [P, P, I, LL, I, I, I, P, P]),
        "fk_update": (I, [P, P, I, LL, I, I, P, P, P, I, P]),
        "fk_sort": (I, [P, I, LL, I, P, P, P, P]),
        "fk_assign_noalloc": (I, [P, P, I, LL, I, I, I, P, P]),
        "fk_noalloc_device_error": (I, [P]),
        "fk_lloyd": (I, [ctypes.POINTER(FkShape), P, P, I, F, P, P, P, ctypes.POINTER(I),
                         ctypes.POINTER(FkOptions)]),
        "fk_status_string": (ctypes.c_char_p, [I]),
        "fk_last_error": (ctypes.c_char_p, []),
        "fk_device_error": (I, [P]),
        "fk_release": (I, []),
        "fk_profile_enable": (I, [I]),
        "fk_profile_read": (I, [ctypes.POINTER(FkProfile), I]),
        "fk_profile_timeline": (I, [P, I, ctypes.POINTER(I)]),
        "fk_launch_count": (LL, []),
        "fk_version": (I, []),
        "fk_selftest_bounded_wait": (I, [LL, P]),
        "fk_point_norms": (I, [P, I, LL, I, I, P, P]),
        "fk_init_centers": (I, [P, I, I, I, I, P, P]),
        "fk_lloyd_step_partial": (I, [ctypes.POINTER(FkShape), P, P, P, P, P, P, P,
                                      ctypes.POINTER(FkOptions)]),
        "fk_update_finalize": (I, [P, P, I, I, I, I, P, P, P, P]),
        "fk_inject_fault": (I, [I, LL]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def _check(status: int, where: str) -> None:
    if status != FK_OK:
        detail = lib.fk_last_error().decode(errors="replace") or lib.fk_status_string(status).decode()
        raise FkError(status, where, detail)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _on(*tensors):
    """Make the device of the first CUDA tensor current for the call (the library
    works on the current device, and the default stream is that device's)."""
    for t in tensors:
        if t is not None and t.is_cuda:
            return torch.cuda.device(t.device)
    return contextlib.nullcontext()


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return DTYPES[t.dtype]


def fk_assign(x: torch.Tensor, c: torch.Tensor, ids: torch.Tensor, stream=None) -> torch.Tensor:
    """ids[b,i] = argmin_k ||c_k||^2 - 2 x_i.c_k (lowest k on ties)."""
    B, N, d = x.shape
    K = c.shape[1]
    with _on(x, c, ids):
        _check(lib.fk_assign(_ptr(x), _ptr(c), B, N, K, d, _dtype_code(x), _ptr(ids), _stream(stream)),
               "fk_assign")
    return ids


def fk_assign_noalloc(x: torch.Tensor, c: torch.Tensor, ids: torch.Tensor, stream=None) -> torch.Tensor:
    """fk_assign that allocates no device memory (static scratch; see include/fk.h).

    The C entry point makes no pointer query (so that it can run where the
    runtime refuses one), so the placement of the tensors is checked here:
    all three on one CUDA device, ids int32 of shape (B, N)."""
    B, N, d = x.shape
    K = c.shape[1]
    for name, t in (("x", x), ("c", c), ("ids", ids)):
        if not t.is_cuda:
            raise ValueError(f"fk_assign_noalloc: {name} must be a CUDA tensor")
        if t.device != x.device:
            raise ValueError(f"fk_assign_noalloc: {name} is on {t.device}, x on {x.device}")
    if ids.dtype != torch.int32 or tuple(ids.shape) != (B, N):
        raise ValueError(f"fk_assign_noalloc: ids must be int32 of shape {(B, N)}")
    if c.dtype != x.dtype or c.dim() != 3 or c.shape[0] != B or c.shape[2] != d:
        raise ValueError("fk_assign_noalloc: c must be (B, K, d) in x's dtype")
    with _on(x, c, ids):
        _check(lib.fk_assign_noalloc(_ptr(x), _ptr(c), B, N, K, d, _dtype_code(x), _ptr(ids),
                                     _stream(stream)), "fk_assign_noalloc")
    return ids


def fk_update(x: torch.Tensor, ids: torch.Tensor, centers: torch.Tensor, counts=None,
              max_shift=None, stream=None) -> torch.Tensor:
    """Sort-inverse update: centers (B,K,d) fp32 in/out, counts (B,K) int32 out."""
    B, N, d = x.shape
    K = centers.shape[1]
    with _on(x, ids, centers):
        _check(lib.fk_update(_ptr(x), _ptr(ids), B, N, K, d, _ptr(centers), _ptr(counts),
                             _stream(stream), _dtype_code(x), _ptr(max_shift)), "fk_update")
    return centers


def fk_sort(ids: torch.Tensor, K: int, perm: torch.Tensor, counts=None, offsets=None,
            stream=None) -> torch.Tensor:
    """Stable counting sort of ids: perm lists point indices ordered by (id, index)."""
    B, N = ids.shape
    with _on(ids, perm):
        _check(lib.fk_sort(_ptr(ids), B, N, K, _ptr(counts), _ptr(offsets), _ptr(perm), _stream(stream)),
               "fk_sort")
    return perm


def fk_lloyd(x: torch.Tensor, init_centers: torch.Tensor, max_iter: int, tol: float,
             ids: torch.Tensor, centers: torch.Tensor, stream=None, host_mode: int = FK_HOST_AUTO,
             chunk_points: int = 0, verbose: bool = False) -> int:
    """Lloyd loop; x / init / outputs may be device or host tensors. Returns iterations run."""
    B, N, d = x.shape
    K = init_centers.shape[1]
    shape = FkShape(B, N, K, d, _dtype_code(x))
    opts = FkOptions(host_mode, chunk_points, 1 if verbose else 0)
    iters = ctypes.c_int(0)
    with _on(x, init_centers, ids, centers):
        _check(lib.fk_lloyd(ctypes.byref(shape), _ptr(x), _ptr(init_centers), int(max_iter), float(tol),
                            _ptr(ids), _ptr(centers), _stream(stream), ctypes.byref(iters),
                            ctypes.byref(opts)), "fk_lloyd")
    return iters.value


def fk_point_norms(x: torch.Tensor, xn: torch.Tensor, stream=None) -> torch.Tensor:
    """xn (B, N) fp32 = ||x[b, i]||^2 of fp16 / bf16 points (B, N, d)."""
    B, N, d = x.shape
    with _on(x, xn):
        _check(lib.fk_point_norms(_ptr(x), B, N, d, _dtype_code(x), _ptr(xn), _stream(stream)),
               "fk_point_norms")
    return xn


def fk_init_centers(init: torch.Tensor, centers: torch.Tensor, stream=None) -> torch.Tensor:
    """centers (B, K, d) fp32 = init (B, K, d) in the points' dtype, widened exactly."""
    B, K, d = init.shape
    with _on(init, centers):
        _check(lib.fk_init_centers(_ptr(init), B, K, d, _dtype_code(init), _ptr(centers), _stream(stream)),
               "fk_init_centers")
    return centers


def fk_lloyd_step_partial(x: torch.Tensor, xn, centers_dt: torch.Tensor, ids: torch.Tensor,
                          sums: torch.Tensor, counts: torch.Tensor, stream=None,
                          chunk_points: int = 0) -> None:
    """Assign this block of points (device or pinned host) and write its per-cluster
    sums (B, K, d) fp32 and counts (B, K) int32 (no division)."""
    B, N, d = x.shape
    K = centers_dt.shape[1]
    shape = FkShape(B, N, K, d, _dtype_code(x))
    opts = FkOptions(FK_HOST_AUTO, chunk_points, 0)
    with _on(x, centers_dt, ids, sums):
        _check(lib.fk_lloyd_step_partial(ctypes.byref(shape), _ptr(x), _ptr(xn), _ptr(centers_dt), _ptr(ids),
                                         _ptr(sums), _ptr(counts), _stream(stream), ctypes.byref(opts)),
               "fk_lloyd_step_partial")


def fk_update_finalize(sums: torch.Tensor, counts: torch.Tensor, centers: torch.Tensor,
                       centers_dt=None, max_shift=None, dtype=None, stream=None) -> torch.Tensor:
    """centers = sums / counts where counts > 0 (else unchanged); centers_dt = rounded copy."""
    B, K, d = centers.shape
    code = _dtype_code(centers_dt) if centers_dt is not None else DTYPES[dtype or torch.float32]
    with _on(sums, counts, centers):
        _check(lib.fk_update_finalize(_ptr(sums), _ptr(counts), B, K, d, code, _ptr(centers), _ptr(centers_dt),
                                      _ptr(max_shift), _stream(stream)), "fk_update_finalize")
    return centers


def fk_device_error(stream=None) -> int:
    return int(lib.fk_device_error(_stream(stream)))


def fk_noalloc_device_error(stream=None) -> int:
    """Status recorded by the fk_assign_noalloc kernels (read and cleared)."""
    return int(lib.fk_noalloc_device_error(_stream(stream)))


def fk_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    """Status of a kernel whose mbarrier wait can never complete (FK_ETIMEOUT expected)."""
    return int(lib.fk_selftest_bounded_wait(ctypes.c_longlong(int(limit_ns)), _stream(stream)))


def fk_inject_fault(kind: int, nth: int = 1) -> None:
    """Arm one host-side failure (FK_FAULT_ALLOC / _H2D / _LAUNCH) at its nth occurrence;
    FK_FAULT_NONE disarms.  For tests of the error paths; no GPU is faulted."""
    _check(lib.fk_inject_fault(int(kind), int(nth)), "fk_inject_fault")


def fk_release() -> None:
    _check(lib.fk_release(), "fk_release")


def fk_profile_enable(on=True) -> None:
    """0 / False: off; 1 / True: every phase; 2: assign and whole update only;
    3: as 2, plus the streamed pipeline's per-chunk timeline (fk_profile_timeline)."""
    _check(lib.fk_profile_enable(int(on)), "fk_profile_enable")


def fk_profile_read(reset: bool = False) -> dict:
    p = FkProfile()
    _check(lib.fk_profile_read(ctypes.byref(p), 1 if reset else 0), "fk_profile_read")
    return {f: getattr(p, f) for f, _ in FkProfile._fields_}


def fk_profile_timeline(max_chunks: int = 4096):
    """Per-chunk events of the streamed pipeline recorded at profile level 3:
    a list of dicts {chunk, buf, copy_begin, copy_end, compute_begin,
    compute_end} in ms from the first copy (clears the record)."""
    import numpy as np
    out = np.zeros((max_chunks, 6), np.float64)
    n = ctypes.c_int(0)
    _check(lib.fk_profile_timeline(ctypes.c_void_p(out.ctypes.data), max_chunks, ctypes.byref(n)),
           "fk_profile_timeline")
    keys = ("chunk", "buf", "copy_begin", "copy_end", "compute_begin", "compute_end")
    return [dict(zip(keys, (int(r[0]), int(r[1]), *map(float, r[2:])))) for r in out[: n.value]]


def fk_launch_count() -> int:
    return int(lib.fk_launch_count())


def fk_version() -> int:
    return int(lib.fk_version())


def fk_status_string(status: int) -> str:
    return lib.fk_status_string(int(status)).decode()


def fk_last_error() -> str:
    return lib.fk_last_error().decode(errors="replace")
