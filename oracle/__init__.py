"""fp64 reference for batched Lloyd's K-Means -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never uses it.

Thin ctypes wrappers over ``fk_oracle.c``; every function there states the
definition it computes and the passage it follows.  Arrays are numpy; points
stay in their storage dtype ("f32" / "f16" / "bf16" with bf16 as raw uint16
bit patterns) and are widened exactly inside the C code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2, None: -1}
P = ctypes.c_void_p
I = ctypes.c_int
LL = ctypes.c_longlong
D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile fk_oracle.c into liboracle.so (gcc -O2, no fast-math, OpenMP over points)."""
    src = os.path.join(_HERE, "fk_oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
                               "-fPIC", "-shared", "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        sig = {
            "or_set_mutation": (None, [I]),
            "or_get_mutation": (I, []),
            "or_max_threads": (I, []),
            "or_widen": (I, [P, I, LL, P]),
            "or_round_value": (D, [D, I]),
            "or_round": (I, [P, LL, I, P]),
            "or_assign": (I, [P, I, P, I, LL, I, I, P, P, P, I]),
            "or_sort": (I, [P, I, LL, I, P, P]),
            "or_update": (I, [P, I, P, I, LL, I, I, P, P, P, P, P]),
            "or_objective": (D, [P, I, P, P, I, LL, I, I]),
            "or_lloyd": (I, [P, I, I, LL, I, I, I, I, D, P, P, P, P, P, P, I]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed ({rc})")


def set_mutation(m: int) -> None:
    """Plant a known mistake (test use only); 0 restores the plain definition."""
    _load().or_set_mutation(int(m))


def max_threads() -> int:
    return int(_load().or_max_threads())


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.ascontiguousarray(x)
    out = np.empty(x.shape, dtype=np.float64)
    _check(_load().or_widen(x.ctypes.data, DTYPE_CODE[dtype], x.size, out.ctypes.data), "widen")
    return out


def round_to(c: np.ndarray, dtype: str | None) -> np.ndarray:
    """Round fp64 values to ``dtype`` (nearest even) and return them as fp64."""
    c = _c(c, np.float64)
    out = np.empty_like(c)
    _check(_load().or_round(c.ctypes.data, c.size, DTYPE_CODE[dtype], out.ctypes.data), "round")
    return out


def assign(x: np.ndarray, dtype: str, chat: np.ndarray, nthreads: int = 0):
    """(ids int32 (B,N), gap fp64 (B,N), dmin fp64 (B,N)) against centroids chat (B,K,d) fp64."""
    x = np.ascontiguousarray(x)
    B, N, d = x.shape
    chat = _c(chat, np.float64)
    K = chat.shape[1]
    ids = np.empty((B, N), np.int32)
    gap = np.empty((B, N), np.float64)
    dmin = np.empty((B, N), np.float64)
    _check(_load().or_assign(x.ctypes.data, DTYPE_CODE[dtype], chat.ctypes.data, B, N, K, d,
                             ids.ctypes.data, gap.ctypes.data, dmin.ctypes.data, nthreads), "assign")
    return ids, gap, dmin


def sort(ids: np.ndarray, K: int):
    """(counts int64 (B,K), perm int64 (B,N)): point indices ordered by (id, index)."""
    ids = _c(ids, np.int32)
    B, N = ids.shape
    counts = np.empty((B, K), np.int64)
    perm = np.empty((B, N), np.int64)
    _check(_load().or_sort(ids.ctypes.data, B, N, K, counts.ctypes.data, perm.ctypes.data), "sort")
    return counts, perm


def update(x: np.ndarray, dtype: str, ids: np.ndarray, old: np.ndarray):
    """(new fp64 (B,K,d), counts int64 (B,K), shift fp64 (B,K), maxshift float)."""
    x = np.ascontiguousarray(x)
    B, N, d = x.shape
    ids = _c(ids, np.int32)
    old = _c(old, np.float64)
    K = old.shape[1]
    new = np.empty_like(old)
    counts = np.empty((B, K), np.int64)
    shift = np.empty((B, K), np.float64)
    ms = ctypes.c_double(0.0)
    _check(_load().or_update(x.ctypes.data, DTYPE_CODE[dtype], ids.ctypes.data, B, N, K, d,
                             old.ctypes.data, new.ctypes.data, counts.ctypes.data,
                             shift.ctypes.data, ctypes.addressof(ms)), "update")
    return new, counts, shift, ms.value


def objective(x: np.ndarray, dtype: str, c: np.ndarray, ids: np.ndarray) -> float:
    x = np.ascontiguousarray(x)
    B, N, d = x.shape
    c = _c(c, np.float64)
    ids = _c(ids, np.int32)
    return float(_load().or_objective(x.ctypes.data, DTYPE_CODE[dtype], c.ctypes.data, ids.ctypes.data,
                                      B, N, c.shape[1], d))


def lloyd(x: np.ndarray, dtype: str, init: np.ndarray, max_iter: int, tol: float,
          round_dtype: str | None = "same", nthreads: int = 0):
    """Run the Lloyd loop.  round_dtype="same" rounds centroids to x's dtype before
    each assign; None keeps them exact.  Returns a dict with ids, centers,
    counts, iters, maxshift and the per-iteration objective."""
    x = np.ascontiguousarray(x)
    B, N, d = x.shape
    centers = _c(init, np.float64).copy()
    K = centers.shape[1]
    rd = dtype if round_dtype == "same" else round_dtype
    ids = np.empty((B, N), np.int32)
    counts = np.empty((B, K), np.int64)
    iters = ctypes.c_int(0)
    ms = ctypes.c_double(0.0)
    trace = np.zeros(max(max_iter, 1), np.float64)
    _check(_load().or_lloyd(x.ctypes.data, DTYPE_CODE[dtype], B, N, K, d, DTYPE_CODE[rd], max_iter,
                            float(tol), ids.ctypes.data, centers.ctypes.data, counts.ctypes.data,
                            ctypes.addressof(iters), ctypes.addressof(ms), trace.ctypes.data,
                            nthreads), "lloyd")
    return {"ids": ids, "centers": centers, "counts": counts, "iters": iters.value,
            "maxshift": ms.value, "objective": trace[: iters.value]}
