"""fp32 on the tensor cores (3xTF32, kind::tf32): edge cases through the C ABI.

- The switch between the CUDA-core and the tensor-core fp32 kernels (K * d
  at 16384) gives ids within the parity rules on both sides.
- K = N with one point per centroid; an empty cluster keeps its centroid.
- Streamed points (pinned host, chunks): the per-chunk widened rows assign
  exactly as the resident run, and the update agrees to rounding.
- The per-rank partial step rejects pageable host points.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_centers, check_ids
from test_parity_kernels import case, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K,d", [(511, 32), (512, 32), (128, 128), (127, 128)])
def test_both_sides_of_the_tensor_core_switch(K, d):
    import clustering_flashassign_b200 as fk
    B, N = 2, 2000
    x, _, c = case(B, N, K, d, "f32", mean_std=4.0, seed=61)
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(to_dev(x, "f32"), to_dev(c, "f32"), ids)
    torch.cuda.synchronize()
    assert fk.fk_device_error() == 0
    check_ids(ids.cpu().numpy(), x, "f32", c.astype(np.float64))


def test_k_equals_n_and_an_empty_cluster():
    import clustering_flashassign_b200 as fk
    B, N, K, d = 1, 1024, 1024, 64            # K * d = 65536: tensor cores
    x, _, _ = case(B, N, 64, d, "f32", mean_std=4.0, seed=63)
    c = x.copy()                              # every point is a centroid
    c[0, 5] = 1.0e4                           # ... except one far away: its cluster stays empty
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    xd, cd = to_dev(x, "f32"), to_dev(c, "f32")
    fk.fk_assign(xd, cd, ids)
    g = ids.cpu().numpy()
    check_ids(g, x, "f32", c.astype(np.float64))
    assert not (g == 5).any()
    cen = cd.clone()
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    fk.fk_update(xd, ids, cen, counts)
    new, rc, _, _ = oracle.update(x, "f32", g, c.astype(np.float64))
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    check_centers(cen.cpu().numpy(), new, "f32")
    assert torch.equal(cen[0, 5], cd[0, 5])


def test_streamed_fp32_matches_resident():
    import clustering_flashassign_b200 as fk
    B, N, K, d = 2, 6000, 256, 128
    x, _, c = case(B, N, K, d, "f32", n_comp=K // 2, mean_std=3.0, seed=67)
    cd = to_dev(c, "f32")
    res = []
    for mode, xin in [(fk.FK_HOST_RESIDENT, torch.from_numpy(x).pin_memory()),
                      (fk.FK_HOST_STREAM, torch.from_numpy(x).pin_memory())]:
        ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
        cen = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
        assert fk.fk_lloyd(xin, cd, 1, 0.0, ids, cen, host_mode=mode, chunk_points=2500) == 1
        res.append((ids.cpu().numpy(), cen.cpu().numpy()))
    np.testing.assert_array_equal(res[0][0], res[1][0])
    np.testing.assert_allclose(res[1][1], res[0][1], rtol=1e-5, atol=1e-5)
    new, _, _, _ = oracle.update(x, "f32", res[0][0], c.astype(np.float64))
    check_centers(res[1][1], new, "f32")


def test_partial_step_rejects_pageable_host_points():
    import clustering_flashassign_b200 as fk
    B, N, K, d = 1, 500, 32, 64
    x, _, c = case(B, N, K, d, "f16", seed=69)
    xh = torch.from_numpy(x)                  # pageable
    cd = to_dev(c, "f16")
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    sums = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    with pytest.raises(fk.FkError) as e:
        fk.fk_lloyd_step_partial(xh, None, cd, ids, sums, counts)
    assert e.value.status == fk.FK_EINVAL
    assert "pinned" in str(e.value)
