"""Data-parallel Lloyd over point blocks (clustering_flashassign_b200.dist) on CPU.

Ranks are gloo processes; the per-rank steps (assign of the block, its
per-cluster sums and counts, the division) are done by the fp64 oracle, so
these tests check the orchestration on its own: the contiguous block split,
the all-reduce of sums and counts, the identical finalize on every rank and
the common tol stop.  The reference is the oracle's own single-process Lloyd
over all the points.  The CUDA steps are covered by tests/test_dist_gpu.py.
"""
import datetime
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from clustering_flashassign_b200.dist import block_of, gather_batches, lloyd_batch_split, lloyd_data_parallel


class OracleSteps:
    """Per-rank steps in fp64 with the oracle (CPU tensors)."""

    def point_norms(self, x):
        return None

    def init_centers(self, init, centers):
        centers.copy_(init.to(torch.float64))

    def partial(self, x, xn, centers_dt, ids, sums, counts):
        xb = x.numpy()
        B, n, d = xb.shape
        if n == 0:  # an empty block contributes zero totals (as fk_lloyd_step_partial)
            sums.zero_()
            counts.zero_()
            return
        g, _, _ = oracle.assign(xb, "f32", centers_dt.to(torch.float64).numpy())
        ids.copy_(torch.from_numpy(g))
        K = sums.shape[1]
        s = np.zeros((B, K, d), np.float64)
        c = np.zeros((B, K), np.int64)
        for b in range(B):
            np.add.at(s[b], g[b], xb[b].astype(np.float64))
            c[b] = np.bincount(g[b], minlength=K)
        sums.copy_(torch.from_numpy(s))
        counts.copy_(torch.from_numpy(c.astype(np.int32)))

    def finalize(self, sums, counts, centers, centers_dt, shift, dtype):
        s, c, old = sums.numpy(), counts.numpy(), centers.numpy()
        new = np.where(c[..., None] > 0, s / np.maximum(c, 1)[..., None], old)
        shift[0] = float(np.sqrt(((new - old) ** 2).sum(-1)).max())
        centers.copy_(torch.from_numpy(new))


def _data(seed, B, N, K, d):
    rng = np.random.default_rng(seed)
    means = rng.normal(0.0, 6.0, size=(B, K, d))
    lab = rng.integers(0, K, size=(B, N))
    x = (means[np.arange(B)[:, None], lab] + rng.normal(size=(B, N, d))).astype(np.float32)
    idx = np.stack([rng.choice(N, size=K, replace=False) for _ in range(B)])
    init = np.stack([x[b, idx[b]] for b in range(B)])
    init[:, K - 1] = 1.0e3  # far from every point: its cluster stays empty in every iteration
    return x, init


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        seed, B, N, K, d, max_iter, tol = case
        x, init = _data(seed, B, N, K, d)
        n0, n1 = block_of(N, rank, world)
        xb = torch.from_numpy(np.ascontiguousarray(x[:, n0:n1]))
        ids = torch.empty((B, n1 - n0), dtype=torch.int32)
        centers = torch.empty((B, K, d), dtype=torch.float64)
        it = lloyd_data_parallel(xb, torch.from_numpy(init), max_iter, tol, ids, centers,
                                 steps=OracleSteps())
        out[rank] = (it, n0, n1, ids.numpy().copy(), centers.numpy().copy())
    finally:
        dist.destroy_process_group()


def _run(world, case):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, case, out), nprocs=world, join=True)
        return dict(out)


def test_block_of_covers_every_point_once():
    for N in (1, 7, 1000, 1001):
        for world in (1, 2, 3, 8):
            blocks = [block_of(N, r, world) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == N
            for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("world,case", [
    (2, (3, 2, 1001, 9, 4, 6, 0.0)),     # fixed count, uneven blocks, an empty cluster
    (3, (4, 1, 900, 6, 3, 50, 1e-9)),    # tol stop: every rank stops at the same iteration
    (4, (5, 1, 3, 2, 3, 3, 0.0)),        # more ranks than points: blocks below K, one empty block
])
def test_data_parallel_matches_single_process_lloyd(world, case):
    seed, B, N, K, d, max_iter, tol = case
    res = _run(world, case)
    x, init = _data(seed, B, N, K, d)
    ref = oracle.lloyd(x, "f32", init, max_iter, tol, round_dtype=None)
    its = {res[r][0] for r in range(world)}
    assert its == {ref["iters"]}, (its, ref["iters"])
    if tol > 0:
        assert ref["iters"] < max_iter, "the tol case should stop early"
    ids = np.concatenate([res[r][3] for r in range(world)], axis=1)
    assert [res[r][1:3] for r in range(world)] == [block_of(N, r, world) for r in range(world)]
    np.testing.assert_array_equal(ids, ref["ids"])
    for r in range(1, world):
        np.testing.assert_array_equal(res[r][4], res[0][4])   # identical on every rank
    np.testing.assert_allclose(res[0][4], ref["centers"], rtol=1e-12, atol=1e-12)
    # the far initial centroid kept its value (its cluster is empty)
    assert (ref["counts"][:, K - 1] == 0).all()
    np.testing.assert_array_equal(res[0][4][:, K - 1], init[:, K - 1].astype(np.float64))


def _x_for_init(seed, B, N, d, dtype):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, N, d), generator=g).to(dtype)
    x[:, :, 0] = -0.0  # a sum with zeros in floating point would turn these into +0.0
    return x


def _init_worker(rank, world, port, case, out):
    from clustering_flashassign_b200.dist import initial_centers_over_blocks
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        seed, B, N, K, d, dtype = case
        x = _x_for_init(seed, B, N, d, dtype)
        n0, n1 = block_of(N, rank, world)
        got = initial_centers_over_blocks(x[:, n0:n1].contiguous(), K, seed)
        out[rank] = (str(got.dtype), tuple(got.shape), got.view(torch.int16 if got.element_size() == 2
                                                                 else torch.int32).numpy().copy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, (7, 2, 1001, 9, 8, torch.float16)),
    (3, (8, 1, 900, 50, 3, torch.float32)),
    (4, (9, 2, 3, 2, 8, torch.bfloat16)),   # more ranks than points: blocks below K, an empty block
])
def test_initial_centers_over_blocks_are_one_process_choice(world, case):
    """Every rank gets, bit for bit, the initial centroids a single process with
    all the points picks (the facade's data-parallel training starts there)."""
    from clustering_flashassign_b200.kmeans import _initial_centers
    seed, B, N, K, d, dtype = case
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_init_worker, args=(world, port, case, out), nprocs=world, join=True)
        res = dict(out)
    ref = _initial_centers(_x_for_init(seed, B, N, d, dtype), K, seed, "cpu")
    bits = ref.view(torch.int16 if ref.element_size() == 2 else torch.int32).numpy()
    for r in range(world):
        assert res[r][0] == str(ref.dtype) and res[r][1] == tuple(ref.shape)
        np.testing.assert_array_equal(res[r][2], bits)


def _too_few_worker(rank, world, port, out):
    from clustering_flashassign_b200.dist import initial_centers_over_blocks
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        try:
            initial_centers_over_blocks(torch.zeros((1, 2, 4)), 5)   # 2 points per rank, K = 5
            out[rank] = "returned"
        except ValueError as e:
            out[rank] = str(e)
    finally:
        dist.destroy_process_group()


def test_initial_centers_over_blocks_fail_on_every_rank_together():
    """K above the whole problem's point count raises on every rank after the
    size exchange, so no rank is left waiting in a collective."""
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_too_few_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    assert all("only 4 points" in v for v in res.values()), res


def _split_worker(rank, world, port, case, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        seed, B, N, K, d, max_iter, tol = case
        x, init = _data(seed, B, N, K, d)
        b0, b1 = block_of(B, rank, world)
        xs = torch.from_numpy(np.ascontiguousarray(x[b0:b1]))
        ids = torch.empty((b1 - b0, N), dtype=torch.int32)
        centers = torch.empty((b1 - b0, K, d), dtype=torch.float64)
        it = lloyd_batch_split(xs, torch.from_numpy(np.ascontiguousarray(init[b0:b1])), max_iter, tol, ids,
                               centers, steps=OracleSteps())
        all_ids = gather_batches(ids, B)
        all_c = gather_batches(centers, B)
        out[rank] = (it, all_ids.numpy().copy(), all_c.numpy().copy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, (6, 5, 400, 7, 4, 5, 0.0)),      # fixed count, 3 + 2 batches
    (3, (7, 4, 300, 5, 3, 60, 1e-9)),    # tol stop decided over all batches
    (3, (8, 2, 200, 4, 2, 4, 0.0)),      # more ranks than batches: one rank holds none
])
def test_batch_split_matches_single_process_lloyd(world, case):
    """Each rank runs its share of the batches; after the gather every rank
    holds the single-process result, and with tol every rank stopped after the
    same iteration as the single process (the global max-shift rule)."""
    seed, B, N, K, d, max_iter, tol = case
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_split_worker, args=(world, port, case, out), nprocs=world, join=True)
        res = dict(out)
    x, init = _data(seed, B, N, K, d)
    ref = oracle.lloyd(x, "f32", init, max_iter, tol, round_dtype=None)
    assert {res[r][0] for r in range(world)} == {ref["iters"]}
    if tol > 0:
        assert ref["iters"] < max_iter, "the tol case should stop early"
    for r in range(world):
        np.testing.assert_array_equal(res[r][1], ref["ids"])
        np.testing.assert_allclose(res[r][2], ref["centers"], rtol=1e-12, atol=1e-12)
