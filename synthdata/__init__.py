"""Seeded synthetic inputs for batched K-Means (points and initial index sets).

The generator is plain C (``gen.c``) driven through ctypes.  It produces the
inputs only; no clustering arithmetic lives here.  Both the fp64 checker
(``oracle``) and the CUDA path consume these arrays.

Storage: fp32 arrays are ``np.float32``; fp16 arrays are ``np.float16``;
bf16 arrays are raw ``np.uint16`` bit patterns (numpy has no bfloat16).

The workload recipes mirror the five benchmark shapes of the flash-kmeans
material (the API example on the project page "flash-kmeans and the return of
exact K-Means on the GPU", the naive-assign breakdown shape in the paper
summary's "two bottlenecks" section, and the out-of-core billion-point case in
its "benchmarks" section).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None

DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2}
ELEM_SIZE = {"f32": 4, "f16": 2, "bf16": 2}


def build(force: bool = False) -> str:
    """Compile gen.c into libsynth.so next to it (gcc, OpenMP)."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_mixture.restype = ctypes.c_int
        lib.synth_mixture.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                      ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
        lib.synth_init_indices.restype = ctypes.c_int
        lib.synth_init_indices.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong,
                                           ctypes.c_int, ctypes.c_uint64]
        lib.synth_gather_rows.restype = ctypes.c_int
        lib.synth_gather_rows.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                          ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
        _lib = lib
    return _lib


def empty_points(B: int, N: int, d: int, dtype: str, out=None) -> np.ndarray:
    npdt = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}[dtype]
    if out is not None:
        assert out.dtype == npdt and out.size == B * N * d
        return out.reshape(B, N, d)
    return np.empty((B, N, d), dtype=npdt)


def mixture(B: int, N: int, d: int, dtype: str, n_comp: int, mean_std: float, zipf_s: float,
            seed: int, nthreads: int = 0, out: np.ndarray | None = None,
            with_components: bool = False):
    """Gaussian-mixture points (B, N, d) in ``dtype``; see gen.c for the recipe."""
    x = empty_points(B, N, d, dtype, out)
    comp = np.empty((B, N), dtype=np.int32) if with_components else None
    rc = _load().synth_mixture(x.ctypes.data, DTYPE_CODE[dtype], B, N, d, n_comp, float(mean_std),
                               float(zipf_s), seed & 0xFFFFFFFFFFFFFFFF, nthreads,
                               comp.ctypes.data if comp is not None else None)
    if rc != 0:
        raise RuntimeError(f"synth_mixture failed ({rc})")
    return (x, comp) if with_components else x


def init_indices(B: int, N: int, K: int, seed_base: int) -> np.ndarray:
    """(B, K) int64: K distinct indices per batch; batch b uses seed seed_base + b."""
    idx = np.empty((B, K), dtype=np.int64)
    rc = _load().synth_init_indices(idx.ctypes.data, B, N, K, seed_base)
    if rc != 0:
        raise RuntimeError(f"synth_init_indices failed ({rc})")
    return idx


def gather_rows(x: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """x[b, idx[b, k], :] for every b, k, keeping x's storage dtype."""
    x = np.ascontiguousarray(x)
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    B, N, d = x.shape
    K = idx.shape[1]
    out = np.empty((B, K, d), dtype=x.dtype)
    rc = _load().synth_gather_rows(x.ctypes.data, x.itemsize, B, N, d, idx.ctypes.data, K, out.ctypes.data)
    if rc != 0:
        raise RuntimeError("synth_gather_rows failed")
    return out


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to float64 (bf16 bit patterns included)."""
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def from_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to the storage dtype (round to nearest even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return a.copy()
    if dtype == "f16":
        return a.astype(np.float16)
    bits = a.view(np.uint32).astype(np.uint64)
    nan = (bits & 0x7F800000) == 0x7F800000
    nan &= (bits & 0x7FFFFF) != 0
    r = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = ((bits[nan] >> 16) | 0x40).astype(np.uint16)
    return r


@dataclass(frozen=True)
class Workload:
    """One benchmark shape and its data recipe."""
    name: str
    B: int
    N: int
    K: int
    d: int
    dtype: str
    n_comp: int
    mean_std: float
    zipf_s: float
    iters: int
    tol: float
    seed: int        # data seed
    init_seed: int   # batch b draws its initial index set with init_seed + b

    @property
    def esz(self) -> int:
        return ELEM_SIZE[self.dtype]


# Recipes: equal-weight isotropic mixtures unless stated; unit variance around each mean.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 8192, 64, 32, "f32", 64, 4.0, 0.0, 10, 0.0, 101, 1000),
    "api": Workload("api", 32, 75600, 1000, 128, "f16", 1, 0.0, 0.0, 20, 1e-4, 102, 2000),
    "zipf": Workload("zipf", 32, 65536, 1024, 128, "f16", 1024, 3.0, 1.2, 20, 0.0, 103, 3000),
    "splitd": Workload("splitd", 8, 32768, 4096, 1024, "bf16", 4096, 2.0, 0.0, 10, 0.0, 104, 4000),
    "largen": Workload("largen", 1, 1 << 28, 32768, 128, "f16", 32768, 4.0, 0.0, 3, 0.0, 105, 5000),
    # the large-D fp32 shape of the pages' FlashKMeans example (d = 2048, k = 1024)
    "f32large": Workload("f32large", 1, 1 << 19, 1024, 2048, "f32", 1024, 4.0, 0.0, 5, 0.0, 106, 6000),
}


def scaled(w: Workload, **kw) -> Workload:
    """The same recipe at other sizes (for checker-sized parity cases)."""
    return replace(w, **kw)


def make(w: Workload, nthreads: int = 0, out: np.ndarray | None = None):
    """(x, init_idx, init_centers) for a workload; init_centers keeps x's dtype."""
    x = mixture(w.B, w.N, w.d, w.dtype, w.n_comp, w.mean_std, w.zipf_s, w.seed, nthreads, out)
    idx = init_indices(w.B, w.N, w.K, w.init_seed)
    return x, idx, gather_rows(x, idx)
