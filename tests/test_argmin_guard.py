"""FlashAssign's exact re-rank of far points (GPU, through the C ABI).

The resident-tile assign (16-bit points, d <= 128) ranks by an fp32 value
whose low byte carries the centroid column, so values within 2^-15 of each
other (relative to the squared distance) count as tied.  That is far inside
the near-tie band 1e-3 ||x||^2 while the nearest squared distance is a small
multiple of ||x||^2; for a point far from every centroid compared with its
own norm the merge could pick the wrong one of two centroids whose distances
differ by more than the band.  The kernel flags such points and re-ranks them
in fp64.  These inputs put every point there:

- points 0.05 * N(0, 1) (small norms) and centroids about 8 away, in pairs
  (2m, 2m + 1) identical but for one coordinate one fp16 / bf16 step closer
  to the origin in the odd one, so the higher index is nearer by a gap
  between the band and 2^-15 of the distance (a plain packed-key argmin ties
  them and keeps the lower, wrong index for most points);
- points exactly at the origin (band 0: only the exact argmin passes) with
  centroids of equal norm (the lowest index must win) and one of a norm one
  step smaller at a higher index.

The split-d assign (16-bit points, d > 128) ranks by the exact value
v = x.c - ||c||^2 / 2 in fp32, whose rounding is set by ||c||^2: with points
near the origin and centroids of norm ~16, pairs one step apart give v gaps
of about one fp32 step of v, above the near-tie band 1e-3 ||x||^2.  The
kernel re-ranks rows whose nearest distance exceeds 64 ||x||^2 in fp64; K is
chosen to span several 256-centroid chunks, so both the per-chunk work items
(fk_assign, fk_lloyd_step_partial) and the whole-tile items
(fk_assign_noalloc) are covered.

Each case runs through fk_assign (point norms from the shared tile),
fk_lloyd_step_partial with precomputed norms, and fk_assign_noalloc.
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import ID_GAP_REL, check_ids, xnorm2
from test_parity_kernels import to_dev

pytestmark = pytest.mark.gpu


def _round16(a: np.ndarray, dtype: str) -> np.ndarray:
    return a.astype(np.float16) if dtype == "f16" else synthdata.from_f32(a.astype(np.float32), "bf16")


def _step(v: np.ndarray, dtype: str) -> np.ndarray:
    """v moved one representable step toward zero (v > 0)."""
    if dtype == "f16":
        return np.nextafter(v.astype(np.float16), np.float16(0))
    return (v.view(np.uint16) - np.uint16(1)).astype(np.uint16)


def far_pairs(B, N, d, dtype, seed):
    rng = np.random.default_rng(seed)
    K = 64
    x = _round16(0.05 * rng.standard_normal((B, N, d)), dtype)
    # fp16: one step at 0.75 is 2^-11, a gap of about 7e-4; bf16 (8-bit
    # significand): one step at 0.375 is 2^-9, a gap of about 1.5e-3; the band
    # is 1e-3 ||x||^2 ~ 2e-4 and 2^-15 of the distance 1e-3 or more
    scale, c0 = (1.0, 0.75) if dtype == "f16" else (2.0, 0.375)
    v = _round16(scale * rng.standard_normal((B, K // 2, d)), dtype)
    v[..., 0] = _round16(np.full((B, K // 2), c0), dtype)
    c = np.repeat(v, 2, axis=1)
    c[:, 1::2, 0] = _step(c[:, 1::2, 0], dtype)
    return x, c


def far_pairs_splitd(B, N, K, d, dtype, seed):
    rng = np.random.default_rng(seed)
    # fp16: a step at 0.125 is 2^-14, a v gap of about 2^-15 next to v ~ -128
    # (fp32 step 2^-16 there); bf16: a step at 2^-5 is 2^-13, a v gap of
    # about 2^-18; the band is 1e-3 ||x||^2 ~ 6e-6 (x scale 0.005 / 0.004)
    xs, c0 = (0.005, 0.125) if dtype == "f16" else (0.004, 0.03125)
    x = _round16(xs * rng.standard_normal((B, N, d)), dtype)
    v = _round16(rng.standard_normal((B, K // 2, d)), dtype)
    v[..., 0] = _round16(np.full((B, K // 2), c0), dtype)
    c = np.repeat(v, 2, axis=1)
    c[:, 1::2, 0] = _step(c[:, 1::2, 0], dtype)
    return x, c


def zero_points(dtype, seed):
    rng = np.random.default_rng(seed)
    B, N, K, d = 1, 300, 40, 64
    x = _round16(0.3 * rng.standard_normal((B, N, d)), dtype)
    x[0, ::3] = 0                      # every third point at the origin
    c = _round16(1.0 + 0.5 * rng.random((B, K, d)), dtype)
    # the smallest norms: base (index 30) and its permutations; the squares
    # and their sums are exact in fp64, so the permutations tie exactly
    base = _round16(0.75 + 0.25 * rng.random(d), dtype)
    c[0, 30] = base
    c[0, 5] = base[::-1]               # equal norm, lower index: must beat 30 and 33
    c[0, 33] = np.roll(base, 7)        # equal norm, higher index
    c[0, 37] = base
    c[0, 37, 3] = _step(base[3:4], dtype)[0]   # one step smaller norm: nearest to the origin
    return x, c


def _run_all(x, c, dtype):
    """ids from fk_assign, from fk_lloyd_step_partial (precomputed norms) and
    from fk_assign_noalloc."""
    import clustering_flashassign_b200 as fk
    B, N, d = x.shape
    K = c.shape[1]
    xd, cd = to_dev(x, dtype), to_dev(c, dtype)
    out = {}
    ids = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, ids)
    out["fk_assign"] = ids.cpu().numpy()
    xn = torch.empty((B, N), dtype=torch.float32, device="cuda")
    fk.fk_point_norms(xd, xn)
    ids2 = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
    sums = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    fk.fk_lloyd_step_partial(xd, xn, cd, ids2, sums, counts)
    out["fk_lloyd_step_partial"] = ids2.cpu().numpy()
    ids3 = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
    fk.fk_assign_noalloc(xd, cd, ids3)
    out["fk_assign_noalloc"] = ids3.cpu().numpy()
    torch.cuda.synchronize()
    assert fk.fk_device_error() == 0
    counts_ref = np.stack([np.bincount(out["fk_lloyd_step_partial"][b], minlength=K) for b in range(B)])
    assert np.array_equal(counts.cpu().numpy(), counts_ref), "fused histogram does not match the re-ranked ids"
    return out


@pytest.mark.parametrize("B,N,d,dtype", [(2, 3000, 64, "f16"), (1, 1500, 128, "f16"), (2, 1000, 64, "bf16")])
def test_far_points_with_close_pairs_take_the_nearer_centroid(B, N, d, dtype):
    x, c = far_pairs(B, N, d, dtype, seed=17 + d)
    chat = synthdata.to_f64(c, dtype)
    ref, gap, dmin = oracle.assign(x, dtype, chat)
    xn = xnorm2(x, dtype)
    # the inputs test what they mean to: most points are far (> 16 ||x||^2),
    # their top-2 gap lies above the band but below 2^-15 of the distance, and
    # the nearer centroid is the higher (odd) index of its pair
    window = (gap > ID_GAP_REL * xn) & (gap < 2.0 ** -15 * dmin) & (dmin > 16 * xn)
    assert window.mean() > 0.9
    assert (ref[window] % 2 == 1).all()
    for name, g in _run_all(x, c, dtype).items():
        assert check_ids(g, x, dtype, chat, ref, gap) == 0, name
        assert np.array_equal(g, ref), name


@pytest.mark.parametrize("B,N,K,d,dtype", [(2, 1500, 600, 256, "f16"), (2, 1500, 600, 256, "bf16"),
                                           (1, 900, 64, 320, "f16")])
def test_splitd_far_points_with_close_pairs_take_the_nearer_centroid(B, N, K, d, dtype):
    x, c = far_pairs_splitd(B, N, K, d, dtype, seed=5 + d)
    chat = synthdata.to_f64(c, dtype)
    ref, gap, dmin = oracle.assign(x, dtype, chat)
    xn = xnorm2(x, dtype)
    # every point is far (> 64 ||x||^2), its top-2 gap lies above the band,
    # half of it (the v gap) within two fp32 steps of v ~ -dmin / 2, and the
    # nearer centroid is the odd one of its pair
    ulp_v = np.spacing((dmin / 2).astype(np.float32)).astype(np.float64)
    window = (gap > ID_GAP_REL * xn) & (gap / 2 < 2 * ulp_v) & (dmin > 64 * xn)
    assert window.mean() > 0.9
    assert (ref[window] % 2 == 1).all()
    for name, g in _run_all(x, c, dtype).items():
        assert check_ids(g, x, dtype, chat, ref, gap) == 0, name
        assert np.array_equal(g, ref), name


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_points_at_the_origin_are_ranked_exactly(dtype):
    x, c = zero_points(dtype, seed=3)
    chat = synthdata.to_f64(c, dtype)
    ref, gap, _ = oracle.assign(x, dtype, chat)
    assert (ref[0, ::3] == 37).all()
    for name, g in _run_all(x, c, dtype).items():
        assert (g[0, ::3] == 37).all(), name
        check_ids(g, x, dtype, chat, ref, gap)
    # without the one-step-smaller centroid the origin ties between 5, 30, 33:
    # the lowest index wins
    c2 = c.copy()
    c2[0, 37] = c2[0, 36]
    ref2, _, _ = oracle.assign(x, dtype, synthdata.to_f64(c2, dtype))
    assert (ref2[0, ::3] == 5).all()
    for name, g in _run_all(x, c2, dtype).items():
        assert (g[0, ::3] == 5).all(), name
