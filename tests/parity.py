"""Parity rules between the CUDA library and the fp64 oracle.

- ids: equal, except for points whose oracle top-2 squared-distance gap is
  below 1e-3 * ||x||^2; where they differ, the GPU's choice must itself be
  within that margin of the oracle minimum (so it is a valid near-tie pick).
- counts, offsets, perm: bit-exact given identical ids.
- centroids: per centroid ||gpu - ref||_2 <= tol * max(||ref_k||, rms_k' ||ref_k'||),
  tol = 2e-3 for fp16 / bf16 inputs and 1e-5 for fp32 inputs.
"""
from __future__ import annotations

import numpy as np

import oracle
import synthdata

ID_GAP_REL = 1e-3
CENTER_TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 2e-3}


def xnorm2(x: np.ndarray, dtype: str) -> np.ndarray:
    xf = synthdata.to_f64(x, dtype)
    return (xf * xf).sum(-1)


def check_ids(gpu_ids, x, dtype, chat, ids_ref=None, gap=None, rows=None):
    """gpu_ids (B, n) for x (B, n, d) against centroids chat (B, K, d) fp64.
    Returns the number of tolerated near-tie differences."""
    gpu_ids = np.asarray(gpu_ids)
    if ids_ref is None:
        ids_ref, gap, _ = oracle.assign(x, dtype, chat)
    xn = xnorm2(x, dtype)
    diff = gpu_ids != ids_ref
    if not diff.any():
        return 0
    assert gpu_ids.min() >= 0 and gpu_ids.max() < chat.shape[1], "id out of range"
    allowed = gap < ID_GAP_REL * xn
    bad = diff & ~allowed
    assert not bad.any(), f"{int(bad.sum())} ids differ outside the near-tie rule (first at {np.argwhere(bad)[0]})"
    # the GPU's pick must be a near-minimum itself
    xf = synthdata.to_f64(x, dtype)
    for b, i in np.argwhere(diff):
        dg = ((xf[b, i] - chat[b, gpu_ids[b, i]]) ** 2).sum()
        dr = ((xf[b, i] - chat[b, ids_ref[b, i]]) ** 2).sum()
        assert dg - dr <= ID_GAP_REL * xn[b, i], f"GPU id at {(b, i)} is not a near-tie choice"
    return int(diff.sum())


def check_centers(gpu, ref, dtype, tol=None):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    tol = CENTER_TOL[dtype] if tol is None else tol
    nrm = np.sqrt((ref * ref).sum(-1))  # (B, K)
    rms = np.sqrt((nrm ** 2).mean(axis=-1, keepdims=True))
    scale = np.maximum(nrm, rms)
    err = np.sqrt(((gpu - ref) ** 2).sum(-1))
    worst = float((err / scale).max())
    assert (err <= tol * scale).all(), f"centroid error {worst:.3e} relative exceeds {tol}"
    return worst
