"""The pages' two comparison kernels, rebuilt on B200 (bench.py reports their
times next to libfk's): they must compute what the method computes.

- Materialised-distance assign (one batched GEMM writes the (B, N, K)
  distances in fp32, argmin reads them): ids within the near-tie rule of the
  fp64 oracle.
- Scatter-atomic update (index_add_ of every point row, bincount, divide,
  empty clusters kept): counts exact and centroids within the parity
  tolerance of the oracle's update given the same ids.
"""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_centers, check_ids
from test_parity_kernels import case, to_dev

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_baselines_compute_the_method(dtype):
    B, N, K, d = 2, 3000, 300, 128
    x, _, c = case(B, N, K, d, dtype, seed=53)
    c[1, K - 1] = synthdata.from_f32(np.full(d, 60.0, np.float32), dtype) if dtype == "bf16" else 60.0
    # centroid K-1 of batch 1 is far from every point: its cluster stays empty
    xd, cd = to_dev(x, dtype), to_dev(c, dtype)
    chat = synthdata.to_f64(c, dtype)
    ids = bench.baseline_assign_materialised(xd, cd)
    torch.cuda.synchronize()
    g = ids.cpu().numpy().astype(np.int32)
    check_ids(g, x, dtype, chat)

    new, counts = bench.baseline_update_scatter(xd, ids.to(torch.int32), cd.float())
    ref_new, ref_counts, _, _ = oracle.update(x, dtype, g, chat)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref_counts)
    assert ref_counts[1, K - 1] == 0
    check_centers(new.cpu().numpy(), ref_new, dtype)
