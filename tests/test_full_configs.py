"""Full-size workloads in the launch configuration the benchmark times.

For each shape, fk_lloyd runs all but the last iteration; the last iteration
then runs step by step through the C ABI so that every output can be checked:
- every id of the first and the last batch against the oracle's assign with
  the GPU's dtype centroids (near-tie rule) where that costs the oracle a few
  seconds (the first batch's tiles are each CTA's first tiles, the last
  batch's its last ones, so the persistent schedule's tile-ahead buffers and
  barrier phases are checked over many tiles per CTA), else a random sample
  of their points; 256 random points of every other batch,
- counts and perm of the counting sort bit-exact against the oracle,
- the updated centroids against the oracle's fp64 means of the GPU's ids,
- and the one-call fk_lloyd result against that stepwise result.
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_centers, check_ids
from test_parity_kernels import to_dev

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
FULL_TERMS = 1.5e11   # a few seconds of the fp64 oracle on the host's cores


@pytest.mark.parametrize("name", ["tiny", "api", "zipf", "splitd", "f32large"])
def test_full_size_workload(name):
    import clustering_flashassign_b200 as fk
    w = synthdata.WORKLOADS[name]
    x, idx, init = synthdata.make(w)
    xd, initd = to_dev(x, w.dtype), to_dev(init, w.dtype)
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
    cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device="cuda")
    n = fk.fk_lloyd(xd, initd, w.iters - 1, 0.0, ids, cen)
    assert n == w.iters - 1

    # last iteration, step by step
    ch = cen.to(TORCH_DT[w.dtype]).contiguous()
    chat = synthdata.to_f64(from_dev(ch, w.dtype), w.dtype)
    fk.fk_assign(xd, ch, ids)
    g = ids.cpu().numpy()
    rng = np.random.default_rng(17)
    ends = sorted({0, w.B - 1})
    # about FULL_TERMS point-centroid-dimension terms of oracle work per batch
    n_full = min(w.N, max(4096, int(FULL_TERMS / (w.K * w.d))))
    for b in ends:
        pts = np.arange(w.N) if n_full == w.N else np.sort(rng.choice(w.N, size=n_full, replace=False))
        check_ids(g[b:b + 1, pts], np.ascontiguousarray(x[b:b + 1, pts]), w.dtype, chat[b:b + 1])
    rest = [b for b in range(w.B) if b not in ends]
    if rest:
        sample = np.sort(rng.choice(w.N, size=min(w.N, 256), replace=False))
        xs = np.ascontiguousarray(x[rest][:, sample])
        check_ids(g[rest][:, sample], xs, w.dtype, chat[rest])

    perm = torch.empty_like(ids)
    counts = torch.empty((w.B, w.K), dtype=torch.int32, device="cuda")
    fk.fk_sort(ids, w.K, perm, counts)
    rc, rp = oracle.sort(g, w.K)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(perm.cpu().numpy(), rp)

    old = cen.cpu().numpy().astype(np.float64)
    counts2 = torch.empty_like(counts)
    fk.fk_update(xd, ids, cen, counts2)
    np.testing.assert_array_equal(counts2.cpu().numpy(), rc)
    new, _, _, _ = oracle.update(x, w.dtype, g, old)
    check_centers(cen.cpu().numpy(), new, w.dtype)

    # the one-call Lloyd run is bit-identical to the stepwise one (deterministic update)
    ids_l = torch.empty_like(ids)
    cen_l = torch.empty_like(cen)
    n = fk.fk_lloyd(xd, initd, w.iters, 0.0, ids_l, cen_l)
    assert n == w.iters
    assert np.array_equal(ids_l.cpu().numpy(), g)
    assert torch.equal(cen_l, cen)
    assert fk.fk_device_error() == 0


def from_dev(t, dtype):
    if dtype == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def test_api_workload_with_tol_reports_iterations():
    import clustering_flashassign_b200 as fk
    w = synthdata.WORKLOADS["api"]
    x, idx, init = synthdata.make(w)
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
    cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device="cuda")
    n = fk.fk_lloyd(to_dev(x, "f16"), to_dev(init, "f16"), w.iters, w.tol, ids, cen)
    assert 1 <= n <= w.iters
