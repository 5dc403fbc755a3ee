"""Edge cases of the tensor-core assign and the update (GPU, through the C ABI).

- zero points and zero centroids (the packed-key path ranks by a strictly
  negative value: its bias must keep exact ties going to the lowest index),
- very small and very large norms (the 16-bit norm digits: precision near
  zero, the fp16 range limit reported through the device error word, bf16's
  fp32 range),
- the smallest tensor-core row (d = 8), a split-d shape with a ragged
  K-block, N = 1,
- K = N = 2^20 (the two-pass sort, one point per cluster on average).
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_centers, check_ids
from test_parity_kernels import case, to_dev

pytestmark = pytest.mark.gpu


def _assign(x, c, dtype):
    import clustering_flashassign_b200 as fk
    B, N, _ = x.shape
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(to_dev(x, dtype), to_dev(c, dtype), ids)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), fk.fk_device_error()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_zero_points_and_duplicate_zero_centroids_take_lowest_index(dtype):
    B, N, K, d = 1, 600, 300, 128
    x, _, c = case(B, N, K, d, dtype, seed=11)
    zero = np.zeros((d,), dtype=x.dtype)
    x[0, :50] = zero                  # points at the origin
    for k in (7, 131, 260, 299):      # the same zero centroid four times, across chunk halves
        c[0, k] = zero
    g, err = _assign(x, c, dtype)
    assert err == 0
    assert (g[0, :50] == 7).all()
    check_ids(g, x, dtype, synthdata.to_f64(c, dtype))


@pytest.mark.parametrize("scale", [1e-3, 3e-2, 60.0])
def test_small_and_large_norms_f16(scale):
    B, N, K, d = 2, 700, 260, 128
    x, _, c = case(B, N, K, d, "f32", seed=5)
    xs = (x * (scale / 3.0)).astype(np.float16)
    cs = (c * (scale / 3.0)).astype(np.float16)
    g, err = _assign(xs, cs, "f16")
    assert err == 0
    check_ids(g, xs, "f16", cs.astype(np.float64))


def test_norm_beyond_fp16_digit_range_is_reported():
    import clustering_flashassign_b200 as fk
    B, N, K, d = 1, 300, 40, 128
    x, _, c = case(B, N, K, d, "f16", seed=9)
    c[0, 5] = np.float16(6000.0)   # ||c||^2 = 128 * 3.6e7 = 4.6e9 > 2^32
    _, err = _assign(x, c, "f16")
    assert err == fk.FK_EUNSUPPORTED
    assert fk.fk_device_error() == 0   # read and cleared
    c[0, 5] = np.float16(4000.0)   # ||c||^2 = 2.05e9 < 2^32: fine
    g, err = _assign(x, c, "f16")
    assert err == 0
    check_ids(g, x, "f16", synthdata.to_f64(c, "f16"))


def test_bf16_has_the_fp32_range():
    B, N, K, d = 1, 500, 100, 64
    x, _, c = case(B, N, K, d, "f32", seed=13)
    xb = synthdata.from_f32((x * 3000.0).astype(np.float32), "bf16")
    cb = synthdata.from_f32((c * 3000.0).astype(np.float32), "bf16")
    g, err = _assign(xb, cb, "bf16")
    assert err == 0
    check_ids(g, xb, "bf16", synthdata.to_f64(cb, "bf16"))


@pytest.mark.parametrize("B,N,K,d,dtype", [
    (2, 333, 100, 8, "f16"),      # one 16-byte row
    (1, 300, 270, 136, "bf16"),   # split-d, last K-block 8 wide
    (3, 1, 1, 64, "f16"),         # a single point
])
def test_assign_shapes(B, N, K, d, dtype):
    x, _, c = case(B, N, K, d, dtype, seed=17)
    g, err = _assign(x, c, dtype)
    assert err == 0
    check_ids(g, x, dtype, synthdata.to_f64(c, dtype))


def test_k_equals_n_two_pass_sort_and_update():
    import clustering_flashassign_b200 as fk
    B, N, K, d = 1, 1 << 20, 1 << 20, 8
    w = synthdata.Workload("kn", B, N, K, d, "f16", 4096, 3.0, 0.0, 1, 0.0, 21, 210)
    x, idx, c = synthdata.make(w)
    xd, cd = to_dev(x, "f16"), to_dev(c, "f16")
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, ids)
    g = ids.cpu().numpy()
    rng = np.random.default_rng(3)
    sample = np.sort(rng.choice(N, size=256, replace=False))
    check_ids(g[:, sample], np.ascontiguousarray(x[:, sample]), "f16", synthdata.to_f64(c, "f16"))
    # every point is its own initial centroid's nearest candidate or a tie of it
    cen = torch.from_numpy(synthdata.to_f64(c, "f16").astype(np.float32)).cuda()
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    fk.fk_update(xd, ids, cen, counts)
    new, rc, _, _ = oracle.update(x, "f16", g, synthdata.to_f64(c, "f16"))
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    check_centers(cen.cpu().numpy(), new, "f16")
    assert fk.fk_device_error() == 0


def test_bounded_wait_expires_and_the_context_survives():
    """A kernel whose mbarrier wait can never complete gives up after its
    limit and reports FK_ETIMEOUT; later calls on the same context work."""
    import time

    import clustering_flashassign_b200 as fk
    t0 = time.perf_counter()
    st = fk.fk_selftest_bounded_wait(20_000_000)  # 20 ms
    dt = time.perf_counter() - t0
    assert st == fk.FK_ETIMEOUT
    assert 0.015 < dt < 5.0
    assert fk.fk_device_error() == 0  # the word was read and cleared
    x, _, c = case(1, 500, 40, 64, "f16", seed=23)
    g, err = _assign(x, c, "f16")
    assert err == 0
    check_ids(g, x, "f16", synthdata.to_f64(c, "f16"))


def test_host_memory_where_device_memory_is_required_is_refused():
    """Host buffers (pageable or pinned) passed where the ABI wants device
    memory return FK_EINVAL from the host-side check, before any launch; the
    device error word stays clean and the next valid call runs."""
    import clustering_flashassign_b200 as fk
    L = fk.lib
    B, N, K, d = 1, 512, 16, 64
    x, _, c = case(B, N, K, d, "f16", seed=61)
    xd, cd = to_dev(x, "f16"), to_dev(c, "f16")
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for xh in (torch.from_numpy(x).clone(), torch.from_numpy(x).pin_memory()):
        st = L.fk_assign(xh.data_ptr(), cd.data_ptr(), B, N, K, d, fk.FK_F16, ids.data_ptr(), s)
        assert st == fk.FK_EINVAL and "x must be device memory" in fk.fk_last_error()
    ids_h = torch.zeros((B, N), dtype=torch.int32)
    cen = torch.zeros((B, K, d), dtype=torch.float32, device="cuda")
    st = L.fk_update(xd.data_ptr(), ids_h.data_ptr(), B, N, K, d, cen.data_ptr(), None, s, fk.FK_F16, None)
    assert st == fk.FK_EINVAL and "ids must be device memory" in fk.fk_last_error()
    perm_h = torch.empty((B, N), dtype=torch.int32)
    st = L.fk_sort(ids.data_ptr(), B, N, K, None, None, perm_h.data_ptr(), s)
    assert st == fk.FK_EINVAL and "perm must be device memory" in fk.fk_last_error()
    torch.cuda.synchronize()
    assert fk.fk_device_error() == 0
    got, err = _assign(x, c, "f16")
    assert err == 0
    check_ids(got, x, "f16", synthdata.to_f64(c, "f16"))
