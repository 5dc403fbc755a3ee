"""The user-level entry points (clustering_flashassign_b200.kmeans).

batch_kmeans_Euclid and FlashKMeans are thin: they choose the initial
centroids (seeded, K distinct points per batch), convert the input to the
compute dtype and call fk_lloyd / fk_assign.  The GPU tests check that they
return exactly what those calls return for the same initial centroids, and
that predict follows the parity rules against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_ids
from test_parity_kernels import case, from_dev16, to_dev


def test_init_indices_are_distinct_and_seeded():
    from clustering_flashassign_b200.kmeans import init_indices
    a = init_indices(3, 1000, 64, seed=5)
    b = init_indices(3, 1000, 64, seed=5)
    c = init_indices(3, 1000, 64, seed=6)
    assert a.shape == (3, 64)
    assert torch.equal(a, b) and not torch.equal(a, c)
    for row in a:
        assert len(set(row.tolist())) == 64 and int(row.min()) >= 0 and int(row.max()) < 1000


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_batch_kmeans_euclid_is_fk_lloyd(dtype):
    import clustering_flashassign_b200 as fk
    from clustering_flashassign_b200.kmeans import batch_kmeans_Euclid, init_indices
    B, N, K, d = 2, 3000, 50, 64
    x, _, _ = case(B, N, K, d, dtype, seed=51)
    xd = to_dev(x, dtype)
    ids, centers, iters = batch_kmeans_Euclid(xd, K, tol=0.0, max_iter=5, seed=3)
    assert iters == 5
    idx = init_indices(B, N, K, seed=3).cuda()
    init = torch.stack([xd[b].index_select(0, idx[b]) for b in range(B)]).contiguous()
    ids_r = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen_r = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    assert fk.fk_lloyd(xd, init, 5, 0.0, ids_r, cen_r) == 5
    assert torch.equal(ids, ids_r) and torch.equal(centers, cen_r)


@pytest.mark.gpu
def test_flashkmeans_2d_host_input_fit_predict_and_predict():
    from clustering_flashassign_b200.kmeans import FlashKMeans, batch_kmeans_Euclid
    N, K, d = 4000, 40, 32
    x, _, _ = case(1, N, K, d, "f32", seed=53)
    data = torch.from_numpy(x[0])                       # (N, d) fp32 on the host
    km = FlashKMeans(d=d, k=K, niter=6, dtype=torch.float16, seed=9)
    labels = km.fit_predict(data)
    assert labels.shape == (N,) and labels.dtype == torch.int32 and labels.is_cuda
    assert km.centroids.shape == (K, d) and km.iters == 6
    ids, centers, _ = batch_kmeans_Euclid(data.unsqueeze(0).to(torch.float16).cuda(), K, tol=0.0,
                                          max_iter=6, seed=9)
    assert torch.equal(labels, ids[0]) and torch.equal(km.centroids, centers[0])
    # predict: one more assignment against the trained centroids, rounded to fp16
    p = km.predict(data)
    x16 = x.astype(np.float16)
    chat = km.centroids.to(torch.float16).float().cpu().numpy().astype(np.float64)[None]
    check_ids(p.cpu().numpy()[None], x16, "f16", chat)


@pytest.mark.gpu
def test_flashkmeans_tol_stops_early():
    from clustering_flashassign_b200.kmeans import FlashKMeans
    B, N, K, d = 2, 6000, 16, 32
    x, _, _ = case(B, N, K, d, "bf16", n_comp=K, mean_std=20.0, seed=57)   # well separated
    km = FlashKMeans(d=d, k=K, niter=100, tol=1e-3, dtype=torch.bfloat16, seed=1)
    km.train(to_dev(x, "bf16"))
    assert 1 <= km.iters < 100
    assert km.centroids.shape == (B, K, d)
