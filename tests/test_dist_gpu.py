"""Data-parallel Lloyd pieces on one GPU, through the C ABI.

- The per-rank partial step over three point blocks: the blocks' ids equal
  fk_assign over all the points bit for bit, and the blocks' sums and counts,
  added by the test in place of the all-reduce and finalized, match the
  oracle's update on those ids (counts exact, centroids within the parity
  tolerance).
- lloyd_data_parallel as one rank equals fk_lloyd bit for bit, with the
  points resident on the device and streamed from pinned host memory: the
  partial sums followed by the finalize from sums do the same fp32 arithmetic
  in the same order as fk_lloyd's update.
- The same loop through a real NCCL process group of one rank.
Several ranks on several GPUs are not run here (one GPU); their orchestration
is covered with gloo ranks on CPU (tests/test_dist_lloyd.py).
"""
import datetime
import os

import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_centers
from test_parity_kernels import case, to_dev

pytestmark = pytest.mark.gpu

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@pytest.mark.parametrize("dtype,d", [("f16", 128), ("bf16", 64), ("f32", 32)])
def test_partial_blocks_sum_to_the_update(dtype, d):
    import clustering_flashassign_b200 as fk
    from clustering_flashassign_b200.dist import block_of
    B, N, K, world = 2, 3001, 300, 3
    x, _, c = case(B, N, K, d, dtype, seed=31)
    xd, cd = to_dev(x, dtype), to_dev(c, dtype)
    full = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, full)
    ids_parts, sums, counts = [], None, None
    for r in range(world):
        n0, n1 = block_of(N, r, world)
        xb = xd[:, n0:n1].contiguous()
        xn = None
        if dtype != "f32":
            xn = torch.empty((B, n1 - n0), dtype=torch.float32, device="cuda")
            fk.fk_point_norms(xb, xn)
        ids_r = torch.empty((B, n1 - n0), dtype=torch.int32, device="cuda")
        s_r = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
        c_r = torch.empty((B, K), dtype=torch.int32, device="cuda")
        fk.fk_lloyd_step_partial(xb, xn, cd, ids_r, s_r, c_r)
        ids_parts.append(ids_r)
        sums = s_r if sums is None else sums + s_r
        counts = c_r if counts is None else counts + c_r
    ids = torch.cat(ids_parts, dim=1)
    assert torch.equal(ids, full)
    centers = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    fk.fk_init_centers(cd, centers)
    cdt = torch.empty_like(cd) if dtype != "f32" else None
    shift = torch.zeros((1,), dtype=torch.float32, device="cuda")
    fk.fk_update_finalize(sums, counts, centers, cdt, shift, dtype=TORCH_DT[dtype])
    torch.cuda.synchronize()
    assert fk.fk_device_error() == 0
    g = ids.cpu().numpy()
    new, rc, _, ms = oracle.update(x, dtype, g, synthdata.to_f64(c, dtype))
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    check_centers(centers.cpu().numpy(), new, dtype)
    assert abs(float(shift.item()) - ms) <= 1e-3 * ms + 1e-6
    if cdt is not None:  # the rounded copy for the next assign
        assert torch.equal(cdt, centers.to(TORCH_DT[dtype]))


@pytest.mark.parametrize("dtype,d", [("f16", 128), ("f32", 32)])
def test_blocks_below_k_and_an_empty_block(dtype, d):
    """Blocks of fewer points than clusters, and an empty block, still add up
    to the whole update: only the whole problem needs K <= N.  Every output of
    the partial step is written (the buffers start as 7s), an empty cluster of
    a block gets zeros and the empty block contributes zero sums and counts."""
    import clustering_flashassign_b200 as fk
    from clustering_flashassign_b200.dist import block_of
    B, N, K, world = 2, 600, 300, 5      # blocks of 120 points, K = 300
    x, _, c = case(B, N, K, d, dtype, seed=47)
    xd, cd = to_dev(x, dtype), to_dev(c, dtype)
    full = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, full)
    ids_parts, sums, counts = [], None, None
    for n0, n1 in [block_of(N, r, world) for r in range(world)] + [(N, N)]:
        xb = xd[:, n0:n1].contiguous()
        ids_r = torch.empty((B, n1 - n0), dtype=torch.int32, device="cuda")
        s_r = torch.full((B, K, d), 7.0, dtype=torch.float32, device="cuda")
        c_r = torch.full((B, K), 7, dtype=torch.int32, device="cuda")
        fk.fk_lloyd_step_partial(xb, None, cd, ids_r, s_r, c_r)
        if n1 == n0:
            torch.cuda.synchronize()
            assert int(c_r.abs().sum()) == 0 and float(s_r.abs().sum()) == 0.0
        ids_parts.append(ids_r)
        sums = s_r if sums is None else sums + s_r
        counts = c_r if counts is None else counts + c_r
    ids = torch.cat(ids_parts, dim=1)
    assert torch.equal(ids, full)
    centers = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    fk.fk_init_centers(cd, centers)
    cdt = torch.empty_like(cd) if dtype != "f32" else None
    fk.fk_update_finalize(sums, counts, centers, cdt, dtype=TORCH_DT[dtype])
    torch.cuda.synchronize()
    assert fk.fk_device_error() == 0
    new, rc, _, _ = oracle.update(x, dtype, ids.cpu().numpy(), synthdata.to_f64(c, dtype))
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    check_centers(centers.cpu().numpy(), new, dtype)


def _fk_lloyd(xd, cd, iters, **kw):
    import clustering_flashassign_b200 as fk
    B, N, _ = xd.shape
    K, d = cd.shape[1], cd.shape[2]
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    n = fk.fk_lloyd(xd, cd, iters, 0.0, ids, cen, **kw)
    assert n == iters
    return ids, cen


def _dp(xd, cd, iters, steps=None):
    from clustering_flashassign_b200.dist import lloyd_data_parallel
    B, N, _ = xd.shape
    K, d = cd.shape[1], cd.shape[2]
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    n = lloyd_data_parallel(xd, cd, iters, 0.0, ids, cen, steps=steps)
    torch.cuda.synchronize()
    assert n == iters
    return ids, cen


@pytest.mark.parametrize("dtype,d", [("f16", 128), ("bf16", 64), ("f32", 32), ("f16", 256),
                                     ("f32", 128)])   # fp32 on the tensor cores (K * d >= 16384)
def test_one_rank_is_fk_lloyd(dtype, d):
    B, N, K = 2, 4000, 200
    x, _, c = case(B, N, K, d, dtype, seed=37)
    xd, cd = to_dev(x, dtype), to_dev(c, dtype)
    ids_a, cen_a = _fk_lloyd(xd, cd, 4)
    ids_b, cen_b = _dp(xd, cd, 4)
    assert torch.equal(ids_a, ids_b)
    assert torch.equal(cen_a, cen_b)


def test_one_rank_streamed_is_fk_lloyd_streamed():
    import clustering_flashassign_b200 as fk
    from clustering_flashassign_b200.dist import CudaSteps
    B, N, K, d, chunk = 2, 5000, 100, 64, 1536
    x, _, c = case(B, N, K, d, "f16", seed=41)
    xh = torch.from_numpy(x).pin_memory()
    cd = to_dev(c, "f16")
    ids_a, cen_a = _fk_lloyd(xh, cd, 3, host_mode=fk.FK_HOST_STREAM, chunk_points=chunk)
    ids_b, cen_b = _dp(xh, cd, 3, steps=CudaSteps(chunk_points=chunk))
    assert torch.equal(ids_a, ids_b)
    assert torch.equal(cen_a, cen_b)


def test_nccl_group_of_one_rank():
    import socket

    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, N, K, d = 1, 3000, 64, 128
        x, _, c = case(B, N, K, d, "f16", seed=43)
        xd, cd = to_dev(x, "f16"), to_dev(c, "f16")
        ids_a, cen_a = _fk_lloyd(xd, cd, 3)
        ids_b, cen_b = _dp(xd, cd, 3)
        assert torch.equal(ids_a, ids_b)
        assert torch.equal(cen_a, cen_b)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype,d", [("f16", 128), ("bf16", 256), ("f32", 32)])
def test_batch_shares_are_fk_lloyd_on_all_batches(dtype, d):
    """lloyd_batch_split over the shares of three ranks, run one after another
    in this process (no exchange is needed with tol = 0), concatenates to
    fk_lloyd over all the batches bit for bit: the batches never interact."""
    from clustering_flashassign_b200.dist import block_of, lloyd_batch_split
    B, N, K, world = 5, 1500, 120, 3
    x, _, c = case(B, N, K, d, dtype, seed=47)
    xd, cd = to_dev(x, dtype), to_dev(c, dtype)
    ids_a, cen_a = _fk_lloyd(xd, cd, 3)
    ids_b, cen_b = [], []
    for r in range(world):
        b0, b1 = block_of(B, r, world)
        ids = torch.empty((b1 - b0, N), dtype=torch.int32, device="cuda")
        cen = torch.empty((b1 - b0, K, d), dtype=torch.float32, device="cuda")
        assert lloyd_batch_split(xd[b0:b1].contiguous(), cd[b0:b1].contiguous(), 3, 0.0, ids, cen) == 3
        ids_b.append(ids)
        cen_b.append(cen)
    assert torch.equal(ids_a, torch.cat(ids_b))
    assert torch.equal(cen_a, torch.cat(cen_b))
