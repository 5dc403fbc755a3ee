"""Large-N streamed Lloyd: points in pinned host memory, chunked host-to-device
copies overlapped with assign / sort / segment reduce, finalize once per
iteration (the large-N workload: B=1, d=128, K=32768, fp16 mixture of 32768
components).

The workload runs at N = 2^24 in chunks of 2^20 points (4 GiB of points, 16
chunks, so the double-buffered pipeline and the per-chunk accumulation are
exercised many times), at N = 2^25 with the library's default 2^24-point
chunks (8 GiB: two full 4 GiB chunks alternate the two device buffers), and
at the full N = 2^28 (64 GiB of pinned host memory, 16 default chunks) when
the host has the memory for it (it is skipped, saying so, on a smaller host).

Lockstep parity after one iteration: sampled ids against the checker's assign
with the initial centroids; every centroid against the checker's update given
the GPU's ids (counts bit-exact, centroids within the fp16 tolerance).
"""

import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_centers, check_ids

pytestmark = pytest.mark.gpu


def _available_bytes():
    try:
        with open("/proc/meminfo") as f:
            for ln in f:
                if ln.startswith("MemAvailable:"):
                    return int(ln.split()[1]) * 1024
    except OSError:
        pass
    return 0


@pytest.mark.parametrize("points,chunk", [(1 << 24, 1 << 20), (1 << 25, 0), (1 << 28, 0)])
def test_largen_streamed_from_pinned_host(points, chunk):
    import clustering_flashassign_b200 as fk
    w = synthdata.scaled(synthdata.WORKLOADS["largen"], N=points)
    need = w.B * w.N * w.d * 2
    if need + (24 << 30) > _available_bytes():
        pytest.skip(f"needs {need / 2**30:.0f} GiB of pinned host memory plus headroom; "
                    f"{_available_bytes() / 2**30:.0f} GiB available")
    xt = torch.empty((w.B, w.N, w.d), dtype=torch.float16, pin_memory=True)
    x = xt.numpy()
    x_, idx, init = synthdata.make(w, out=x)
    assert x_ is x or np.shares_memory(x_, x)
    initd = torch.from_numpy(init).cuda()
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
    cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device="cuda")

    n = fk.fk_lloyd(xt, initd, 1, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM, chunk_points=chunk)
    torch.cuda.synchronize()
    assert n == 1
    assert fk.fk_device_error() == 0
    g = ids.cpu().numpy()
    assert g.min() >= 0 and g.max() < w.K

    # ids: the assign of the only iteration used the initial centroids (already in fp16)
    c0 = synthdata.to_f64(init, w.dtype)
    rng = np.random.default_rng(29)
    sample = np.sort(rng.choice(w.N, size=512, replace=False))
    check_ids(g[:, sample], np.ascontiguousarray(x[:, sample]), w.dtype, c0)

    # update given the GPU's ids: counts and every centroid
    new, counts, _, _ = oracle.update(x, w.dtype, g, c0)
    got = cen.cpu().numpy()
    check_centers(got, new, w.dtype)
    gcounts = np.bincount(g[0], minlength=w.K)
    np.testing.assert_array_equal(gcounts, counts[0])
    assert int(counts.sum()) == w.N


def test_largen_streamed_matches_device_resident_run():
    """The same problem with the points on the device gives the same ids and
    bit-identical centroids: the streamed pipeline only moves data."""
    import clustering_flashassign_b200 as fk
    w = synthdata.scaled(synthdata.WORKLOADS["largen"], N=1 << 21)
    xt = torch.empty((w.B, w.N, w.d), dtype=torch.float16, pin_memory=True)
    _, _, init = synthdata.make(w, out=xt.numpy())
    initd = torch.from_numpy(init).cuda()
    out = []
    for mode in ("stream", "device"):
        ids = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
        cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device="cuda")
        if mode == "stream":
            # the chunk boundary splits every batch into 4 chunks
            n = fk.fk_lloyd(xt, initd, 2, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM, chunk_points=1 << 19)
        else:
            n = fk.fk_lloyd(xt.cuda(), initd, 2, 0.0, ids, cen)
        assert n == 2
        out.append((ids.cpu(), cen.cpu()))
    assert torch.equal(out[0][0], out[1][0])
    # sums are folded chunk by chunk in the streamed run: equal up to fp32 rounding
    torch.testing.assert_close(out[0][1], out[1][1], rtol=1e-5, atol=1e-5)


def test_streamed_timeline_shows_copies_before_their_compute_and_overlap():
    """Profile level 3 records, per streamed chunk, the copy (copy stream) and
    the compute (compute stream): each copy ends before its chunk's compute
    begins, and the copy of chunk j + 1 starts before chunk j's compute ends
    (the double buffer overlaps them)."""
    import clustering_flashassign_b200 as fk
    w = synthdata.scaled(synthdata.WORKLOADS["largen"], N=1 << 21, K=4096)
    xt = torch.empty((w.B, w.N, w.d), dtype=torch.float16, pin_memory=True)
    _, _, init = synthdata.make(w, out=xt.numpy())
    initd = torch.from_numpy(init).cuda()
    ids = torch.empty((w.B, w.N), dtype=torch.int32, device="cuda")
    cen = torch.empty((w.B, w.K, w.d), dtype=torch.float32, device="cuda")
    fk.fk_lloyd(xt, initd, 1, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM, chunk_points=1 << 18)  # warm-up
    fk.fk_profile_timeline()  # nothing recorded at level 0
    fk.fk_profile_enable(3)
    try:
        fk.fk_lloyd(xt, initd, 2, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM, chunk_points=1 << 18)
        torch.cuda.synchronize()
    finally:
        fk.fk_profile_enable(False)
        fk.fk_profile_read(reset=True)
    tl = fk.fk_profile_timeline()
    assert len(tl) == 2 * 8
    assert [c["buf"] for c in tl] == [c["chunk"] & 1 for c in tl]
    for c in tl:
        assert c["copy_begin"] <= c["copy_end"] <= c["compute_begin"] + 1e-3 <= c["compute_end"] + 1e-3
    overlapped = sum(1 for a, b in zip(tl, tl[1:]) if b["copy_begin"] < a["compute_end"])
    assert overlapped >= len(tl) // 2
    assert fk.fk_profile_timeline() == []  # read once, then cleared
