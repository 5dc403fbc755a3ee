"""GPU parity of whole Lloyd runs (fk_lloyd) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import CENTER_TOL, check_centers, check_ids
from test_parity_kernels import case, from_dev16, to_dev

pytestmark = pytest.mark.gpu


def round_dtype(c32: np.ndarray, dtype: str) -> np.ndarray:
    return synthdata.from_f32(c32, dtype).reshape(c32.shape)


@pytest.mark.parametrize("B,N,K,d,dtype", [(2, 3000, 200, 128, "f16"), (2, 2500, 150, 64, "bf16"),
                                           (1, 4000, 64, 32, "f32"), (1, 1500, 300, 256, "bf16"),
                                           (1, 3000, 256, 128, "f32")])   # fp32 on the tensor cores
def test_lockstep_iterations(B, N, K, d, dtype):
    """Each iteration: oracle assign with the GPU's dtype centroids, oracle
    update with the GPU's ids; the GPU continues from its own centroids."""
    import clustering_flashassign_b200 as fk
    x, idx, c0 = case(B, N, K, d, dtype, n_comp=K // 2, mean_std=2.0)
    xd = to_dev(x, dtype)
    centers = torch.from_numpy(synthdata.to_f64(c0, dtype).astype(np.float32)).cuda()
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    flips = 0
    for it in range(5):
        c32 = centers.cpu().numpy()
        ch = round_dtype(c32, dtype)
        fk.fk_assign(xd, to_dev(ch, dtype), ids)
        g = ids.cpu().numpy()
        flips += check_ids(g, x, dtype, synthdata.to_f64(ch, dtype))
        fk.fk_update(xd, ids, centers, counts)
        new, rc, _, _ = oracle.update(x, dtype, g, c32.astype(np.float64))
        np.testing.assert_array_equal(counts.cpu().numpy(), rc)
        check_centers(centers.cpu().numpy(), new, dtype)
    assert flips <= B * N * 1e-3


@pytest.mark.parametrize("dtype,K", [("f16", 100), ("bf16", 100), ("f32", 100), ("f32", 300)])
def test_lloyd_equals_its_steps(dtype, K):
    """fk_lloyd == fk_assign / fk_update with centroids rounded to dtype in between
    (fp32 with K = 300 runs on the tensor cores: fk_lloyd splits the points once,
    fk_assign on every call)."""
    import clustering_flashassign_b200 as fk
    B, N, d = 2, 2000, 64
    x, idx, c0 = case(B, N, K, d, dtype, n_comp=60, mean_std=3.0)
    xd, cd = to_dev(x, dtype), to_dev(c0, dtype)
    ids_l = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen_l = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    n = fk.fk_lloyd(xd, cd, 4, 0.0, ids_l, cen_l)
    assert n == 4
    centers = cd.float().contiguous()
    ids = torch.empty_like(ids_l)
    for _ in range(4):
        ch = centers.to(cd.dtype).contiguous()  # round to nearest even
        fk.fk_assign(xd, ch, ids)
        fk.fk_update(xd, ids, centers)
    # the update is deterministic (no float atomics), so the two runs are bit-identical
    assert torch.equal(ids_l, ids)
    assert torch.equal(cen_l, centers)


def test_tiny_config_free_running():
    """Tiny workload (B=1, N=8192, K=64, d=32, fp32, 10 iterations, tol=0) run
    whole on both sides from the same seed-chosen initial centroids."""
    import clustering_flashassign_b200 as fk
    w = synthdata.WORKLOADS["tiny"]
    x, idx, init = synthdata.make(w)
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
    cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device="cuda")
    n = fk.fk_lloyd(torch.from_numpy(x).cuda(), torch.from_numpy(init).cuda(), w.iters, w.tol, ids, cen)
    assert n == w.iters
    r = oracle.lloyd(x, "f32", init.astype(np.float64), w.iters, w.tol)
    g = ids.cpu().numpy()
    flips = int((g != r["ids"]).sum())
    obj_gpu = oracle.objective(x, "f32", cen.cpu().numpy().astype(np.float64), g)
    obj_ref = oracle.objective(x, "f32", r["centers"], r["ids"])
    assert flips == 0, f"{flips} ids differ; objectives gpu {obj_gpu} ref {obj_ref}"
    check_centers(cen.cpu().numpy(), r["centers"], "f32")


def test_tol_semantics():
    import clustering_flashassign_b200 as fk
    # separated blobs converge in a few iterations
    B, N, K, d = 1, 4000, 8, 16
    x, idx, c0 = case(B, N, K, d, "f16", n_comp=8, mean_std=40.0)
    xd, cd = to_dev(x, "f16"), to_dev(c0, "f16")
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    assert fk.fk_lloyd(xd, cd, 7, 1e9, ids, cen) == 1          # first shift is below a huge tol
    assert fk.fk_lloyd(xd, cd, 7, 0.0, ids, cen) == 7          # tol <= 0 never stops early
    n = fk.fk_lloyd(xd, cd, 30, 1e-3, ids, cen)
    r = oracle.lloyd(x, "f16", synthdata.to_f64(c0, "f16"), 30, 1e-3)
    assert n < 30 and n == r["iters"]
    assert fk.fk_lloyd(xd, cd, 0, 0.0, ids, cen) == 0


def test_empty_clusters_keep_their_centroid():
    import clustering_flashassign_b200 as fk
    B, N, K, d = 1, 2000, 40, 32
    x, idx, c0 = case(B, N, K, d, "f16", n_comp=4, mean_std=30.0)
    c0 = c0.copy()
    c0[0, 30:] = (np.float16(500.0))  # far away: these ten never win a point
    xd, cd = to_dev(x, "f16"), to_dev(c0, "f16")
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    fk.fk_lloyd(xd, cd, 5, 0.0, ids, cen)
    assert (ids.cpu().numpy() < 30).all()
    np.testing.assert_array_equal(cen.cpu().numpy()[0, 30:], np.full((10, d), 500.0, np.float32))
    r = oracle.lloyd(x, "f16", synthdata.to_f64(c0, "f16"), 5, 0.0)
    check_centers(cen.cpu().numpy(), r["centers"], "f16")


def test_host_buffers_resident_and_streamed():
    """x in pinned host memory: resident copy and chunked streaming (ragged
    chunks, several per batch) give the oracle's result."""
    import clustering_flashassign_b200 as fk
    B, N, K, d = 2, 3000, 50, 64
    x, idx, c0 = case(B, N, K, d, "f16", n_comp=50, mean_std=6.0)
    xh = torch.from_numpy(x).pin_memory()
    ch = torch.from_numpy(c0).pin_memory()
    r = oracle.lloyd(x, "f16", synthdata.to_f64(c0, "f16"), 4, 0.0)
    for mode, chunk in [(fk.FK_HOST_RESIDENT, 0), (fk.FK_HOST_STREAM, 700), (fk.FK_HOST_STREAM, 0)]:
        ids = torch.empty((B, N), dtype=torch.int32).pin_memory()      # host outputs too
        cen = torch.empty((B, K, d), dtype=torch.float32)               # pageable host output
        n = fk.fk_lloyd(xh, ch, 4, 0.0, ids, cen, host_mode=mode, chunk_points=chunk)
        assert n == 4
        g = ids.numpy()
        assert (g != r["ids"]).mean() <= 1e-3, f"mode {mode} chunk {chunk}"
        check_centers(cen.numpy(), r["centers"], "f16")


@pytest.mark.parametrize("K", [20, 5000])   # one counting pass; two passes (K > 4096)
def test_out_of_range_ids_are_counted_nowhere(K):
    """Two ids outside [0, K), after a valid call has left full sort buffers
    behind: the error is reported, not faulted, and every other point's result
    is the oracle's over the valid points alone -- counts, centroids and the
    stable permutation -- with -1 in perm past the counted points."""
    import clustering_flashassign_b200 as fk
    B, N, d = 1, 12000, 16
    x, _, c0 = case(B, N, K, d, "f16", seed=53)
    xd = to_dev(x, "f16")
    c64 = synthdata.to_f64(c0, "f16")
    rng = np.random.default_rng(53)
    ok = torch.from_numpy(rng.integers(0, K, (B, N)).astype(np.int32)).cuda()
    fk.fk_update(xd, ok, torch.from_numpy(c64.astype(np.float32)).cuda())
    fk.fk_sort(ok, K, torch.empty((B, N), dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert fk.fk_device_error() == fk.FK_OK
    g = rng.integers(0, K, (B, N)).astype(np.int32)
    g[0, 7] = K
    g[0, 9] = -1
    ids = torch.from_numpy(g).cuda()
    cen = torch.from_numpy(c64.astype(np.float32)).cuda()
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    fk.fk_update(xd, ids, cen, counts)
    perm = torch.full((B, N), 12345, dtype=torch.int32, device="cuda")
    fk.fk_sort(ids, K, perm)
    torch.cuda.synchronize()
    assert fk.fk_device_error() == fk.FK_EINVAL
    assert fk.fk_device_error() == fk.FK_OK  # reading clears it
    keep = (g[0] >= 0) & (g[0] < K)
    new, rc, _, _ = oracle.update(x[:, keep], "f16", g[:, keep], c64)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    check_centers(cen.cpu().numpy(), new, "f16")
    _, operm = oracle.sort(g[:, keep], K)
    nv = int(keep.sum())
    p = perm.cpu().numpy()[0]
    np.testing.assert_array_equal(p[:nv], np.flatnonzero(keep)[operm[0]])
    assert (p[nv:] == -1).all()


def test_repeated_runs_are_bit_identical():
    """No float atomics anywhere in the update: two runs give identical bits."""
    import clustering_flashassign_b200 as fk
    B, N, K, d = 4, 20000, 500, 128
    x, idx, c0 = case(B, N, K, d, "f16", n_comp=40, zipf=1.2, mean_std=2.0)
    xd, cd = to_dev(x, "f16"), to_dev(c0, "f16")
    outs = []
    for _ in range(2):
        ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
        cen = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
        fk.fk_lloyd(xd, cd, 6, 0.0, ids, cen)
        outs.append((ids, cen))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("tol_iters", [2, 3])
def test_tol_stop_returns_the_same_state_as_a_fixed_run(tol_iters):
    """The assign of the next iteration is queued before the host reads the
    shift; when the shift stops the loop that assign must not leak: ids and
    centroids equal those of a run with exactly that many iterations."""
    import clustering_flashassign_b200 as fk
    B, N, K, d = 2, 3000, 12, 32
    x, idx, c0 = case(B, N, K, d, "f16", n_comp=12, mean_std=25.0)
    xd, cd = to_dev(x, "f16"), to_dev(c0, "f16")
    ids_f = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen_f = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    # max centroid shift of iteration n (n >= 2) from fixed runs of n - 1 and n iterations
    cens = []
    for n in range(1, tol_iters + 1):
        fk.fk_lloyd(xd, cd, n, 0.0, ids_f, cen_f)
        cens.append(cen_f.clone())
    s_stop = float((cens[-1] - cens[-2]).norm(dim=-1).max())
    tol = s_stop * 1.0001  # the run stops at iteration tol_iters, or earlier
    ids_t = torch.empty_like(ids_f)
    cen_t = torch.empty_like(cen_f)
    n = fk.fk_lloyd(xd, cd, 20, tol, ids_t, cen_t)
    fk.fk_lloyd(xd, cd, n, 0.0, ids_f, cen_f)
    assert n <= tol_iters
    assert torch.equal(ids_t, ids_f)
    assert torch.equal(cen_t, cen_f)
