"""The pages' two user-level entry points over libfk.

    ids, centers, iters = batch_kmeans_Euclid(x, n_clusters, tol=1e-4, verbose=False)
    km = FlashKMeans(d=128, k=8192, niter=100); labels = km.fit_predict(x)

"flash-kmeans and the return of exact K-Means on the GPU", section "Exact
K-Means, with the assignment step written in Triton" (batch_kmeans_Euclid on
a (B, N, d) tensor returning cluster ids and centers, and the FlashKMeans
class with d, k, dtype and train); "Flash-KMeans: Implementação Exata de
K-Means Roda 200× Mais Rápido que FAISS em GPUs", the usage listing
(FlashKMeans(d, k, niter) and fit_predict on a CPU tensor).  Every step of
the clustering runs in libfk (fk_lloyd, or fk_lloyd_step_partial /
fk_update_finalize across ranks); this module picks the initial centroids,
converts the input to the compute dtype and allocates the outputs.

Readings where the pages are silent: the initial centroids are K distinct
points per batch chosen by a seeded random permutation; batch_kmeans_Euclid
runs at most max_iter = 100 iterations; its third return value is the number
of iterations run.
"""
from __future__ import annotations

import torch

from . import FK_HOST_AUTO, fk_assign, fk_lloyd

_COMPUTE = (torch.float16, torch.bfloat16, torch.float32)


def init_indices(B: int, N: int, K: int, seed: int = 0) -> torch.Tensor:
    """(B, K) int64: K distinct point indices per batch, from a seeded permutation."""
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randperm(N, generator=g)[:K] for _ in range(B)])


def _initial_centers(x: torch.Tensor, K: int, seed: int, device) -> torch.Tensor:
    B, N, _ = x.shape
    idx = init_indices(B, N, K, seed)
    rows = torch.stack([x[b].index_select(0, idx[b].to(x.device)) for b in range(B)])
    return rows.to(device).contiguous()


def batch_kmeans_Euclid(x: torch.Tensor, n_clusters: int, tol: float = 1e-4, verbose: bool = False,
                        max_iter: int = 100, seed: int = 0, init_centers: torch.Tensor | None = None,
                        chunk_points: int = 0):
    """Exact batched Lloyd's K-Means.

    x (B, N, d) fp16 / bf16 / fp32 on a CUDA device or in host memory (pinned host
    memory is streamed in chunks when it does not fit).  Returns (ids (B, N) int32,
    centers (B, K, d) fp32, iterations run), on x's device (CUDA when x is on the host).
    """
    if x.dim() != 3:
        raise ValueError("x must be (B, N, d)")
    if x.dtype not in _COMPUTE:
        raise ValueError(f"unsupported dtype {x.dtype}")
    x = x.contiguous()
    B, N, d = x.shape
    dev = x.device if x.is_cuda else torch.device("cuda", torch.cuda.current_device())
    init = init_centers if init_centers is not None else _initial_centers(x, n_clusters, seed, dev)
    init = init.to(device=dev, dtype=x.dtype).contiguous()
    ids = torch.empty((B, N), dtype=torch.int32, device=dev)
    centers = torch.empty((B, n_clusters, d), dtype=torch.float32, device=dev)
    iters = fk_lloyd(x, init, max_iter, tol, ids, centers, host_mode=FK_HOST_AUTO,
                     chunk_points=chunk_points, verbose=verbose)
    return ids, centers, iters


class FlashKMeans:
    """scikit-learn-style K-Means over libfk.

    FlashKMeans(d, k, niter=20, tol=0.0, dtype=torch.float16, device=None, seed=0)
      train(data)        fit on data (N, d) or (B, N, d); sets self.centroids
      predict(data)      ids against the trained centroids (fk_assign)
      fit_predict(data)  train, then the ids of the last assignment
    device None: the current CUDA device.  When a torch.distributed process group
    is initialised, every rank passes its own contiguous block of the points (the
    blocks in rank order make up the data) and the ranks fit one model together
    (clustering_flashassign_b200.dist), starting from the centroids one process
    with all the points would pick; predict and fit_predict then return the
    labels of the caller's block.
    """

    def __init__(self, d: int, k: int, niter: int = 20, tol: float = 0.0,
                 dtype: torch.dtype = torch.float16, device=None, seed: int = 0, verbose: bool = False):
        if dtype not in _COMPUTE:
            raise ValueError(f"unsupported dtype {dtype}")
        self.d, self.k, self.niter, self.tol = d, k, niter, tol
        self.dtype, self.seed, self.verbose = dtype, seed, verbose
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.centroids: torch.Tensor | None = None   # (B, k, d) fp32, or (k, d) for 2-D input
        self.iters = 0
        self._labels: torch.Tensor | None = None

    def _prep(self, data: torch.Tensor):
        squeeze = data.dim() == 2
        x = data.unsqueeze(0) if squeeze else data
        if x.dim() != 3 or x.shape[-1] != self.d:
            raise ValueError(f"data must be (N, {self.d}) or (B, N, {self.d})")
        if x.dtype != self.dtype:
            x = x.to(self.dtype)
        if x.is_cuda and x.device != self.device:
            x = x.to(self.device)
        return x.contiguous(), squeeze

    def train(self, data: torch.Tensor) -> "FlashKMeans":
        import torch.distributed as dist
        x, squeeze = self._prep(data)
        B, n, d = x.shape
        if dist.is_available() and dist.is_initialized():
            from .dist import initial_centers_over_blocks, lloyd_data_parallel
            # the whole problem's initial centroids, assembled from the ranks' blocks
            init = initial_centers_over_blocks(x, self.k, self.seed).to(self.device)
            xb = x if x.is_cuda or x.is_pinned() else x.to(self.device)
            ids = torch.empty((B, n), dtype=torch.int32, device=self.device)
            centers = torch.empty((B, self.k, d), dtype=torch.float32, device=self.device)
            self.iters = lloyd_data_parallel(xb, init, self.niter, self.tol, ids, centers)
        else:
            ids, centers, self.iters = batch_kmeans_Euclid(
                x, self.k, tol=self.tol, verbose=self.verbose, max_iter=self.niter, seed=self.seed)
        self.centroids = centers[0] if squeeze else centers
        self._labels = ids[0] if squeeze else ids
        return self

    def predict(self, data: torch.Tensor) -> torch.Tensor:
        if self.centroids is None:
            raise RuntimeError("train the model first")
        x, squeeze = self._prep(data)
        if not x.is_cuda:
            x = x.to(self.device)
        c = self.centroids.unsqueeze(0) if squeeze else self.centroids
        ids = torch.empty(x.shape[:2], dtype=torch.int32, device=self.device)
        fk_assign(x, c.to(self.dtype).contiguous(), ids)
        return ids[0] if squeeze else ids

    def fit_predict(self, data: torch.Tensor) -> torch.Tensor:
        self.train(data)
        return self._labels
