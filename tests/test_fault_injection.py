"""Error paths through the C ABI, driven by host-side fault injection.

Each armed failure (workspace allocation, host-to-device copy, kernel launch)
makes the call report its status -- FK_ENOMEM or FK_ECUDA -- without faulting
the GPU; the next call works and gives the right result, and a failed call
followed by fk_release() leaves no library memory behind.  The FK_FAULT
environment variable arms the same failures in a fresh process.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_ids
from test_parity_kernels import case, to_dev

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(autouse=True)
def _disarm():
    import clustering_flashassign_b200 as fk
    yield
    fk.fk_inject_fault(fk.FK_FAULT_NONE)


def _assign_case():
    B, N, K, d = 2, 1000, 300, 128
    x, _, c = case(B, N, K, d, "f16", seed=71)
    return x, c, to_dev(x, "f16"), to_dev(c, "f16")


def test_allocation_failure_then_recovery():
    import clustering_flashassign_b200 as fk
    x, c, xd, cd = _assign_case()
    ids = torch.empty(x.shape[:2], dtype=torch.int32, device="cuda")
    fk.fk_release()
    fk.fk_inject_fault(fk.FK_FAULT_ALLOC, 1)
    with pytest.raises(fk.FkError) as e:
        fk.fk_assign(xd, cd, ids)
    assert e.value.status == fk.FK_ENOMEM and "injected allocation" in str(e.value)
    fk.fk_assign(xd, cd, ids)   # the fault fired once
    torch.cuda.synchronize()
    check_ids(ids.cpu().numpy(), x, "f16", synthdata.to_f64(c, "f16"))


def test_failed_calls_leave_no_library_memory():
    import clustering_flashassign_b200 as fk
    x, c, xd, cd = _assign_case()
    ids = torch.empty(x.shape[:2], dtype=torch.int32, device="cuda")
    cen = torch.empty((x.shape[0], c.shape[1], x.shape[2]), dtype=torch.float32, device="cuda")
    fk.fk_lloyd(xd, cd, 3, 0.0, ids, cen)   # every kernel's module loaded once
    torch.cuda.synchronize()
    fk.fk_release()
    free0 = torch.cuda.mem_get_info()[0]
    for kind, nth in [(fk.FK_FAULT_ALLOC, 4), (fk.FK_FAULT_LAUNCH, 5)]:
        fk.fk_inject_fault(kind, nth)
        with pytest.raises(fk.FkError):
            fk.fk_lloyd(xd, cd, 3, 0.0, ids, cen)
        torch.cuda.synchronize()
        fk.fk_release()
        assert torch.cuda.mem_get_info()[0] == free0


def test_launch_failure_is_reported_and_the_next_update_is_right():
    import clustering_flashassign_b200 as fk
    x, c, xd, cd = _assign_case()
    ids = torch.empty(x.shape[:2], dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, ids)
    cen = cd.float().contiguous()
    counts = torch.empty((x.shape[0], c.shape[1]), dtype=torch.int32, device="cuda")
    fk.fk_inject_fault(fk.FK_FAULT_LAUNCH, 2)   # the update's second kernel
    with pytest.raises(fk.FkError) as e:
        fk.fk_update(xd, ids, cen, counts)
    assert e.value.status == fk.FK_ECUDA and "injected launch" in str(e.value)
    torch.cuda.synchronize()
    cen = cd.float().contiguous()
    fk.fk_update(xd, ids, cen, counts)
    new, rc, _, _ = oracle.update(x, "f16", ids.cpu().numpy(), synthdata.to_f64(c, "f16"))
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    assert fk.fk_device_error() == 0


@pytest.mark.parametrize("mode,nth", [("resident", 1), ("stream", 3)])
def test_host_to_device_copy_failure(mode, nth):
    import clustering_flashassign_b200 as fk
    B, N, K, d = 2, 5000, 64, 64
    x, _, c = case(B, N, K, d, "f16", seed=73)
    xh = torch.from_numpy(x).pin_memory()
    cd = to_dev(c, "f16")
    hm = fk.FK_HOST_RESIDENT if mode == "resident" else fk.FK_HOST_STREAM
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    cen = torch.empty((B, K, d), dtype=torch.float32, device="cuda")
    fk.fk_inject_fault(fk.FK_FAULT_H2D, nth)   # streamed: the third chunk copy
    with pytest.raises(fk.FkError) as e:
        fk.fk_lloyd(xh, cd, 2, 0.0, ids, cen, host_mode=hm, chunk_points=1500)
    assert e.value.status == fk.FK_ECUDA and "injected host-to-device" in str(e.value)
    torch.cuda.synchronize()
    ids2, cen2 = torch.empty_like(ids), torch.empty_like(cen)
    assert fk.fk_lloyd(xh, cd, 2, 0.0, ids, cen, host_mode=hm, chunk_points=1500) == 2
    assert fk.fk_lloyd(xh, cd, 2, 0.0, ids2, cen2, host_mode=hm, chunk_points=1500) == 2
    assert torch.equal(ids, ids2) and torch.equal(cen, cen2)


def test_fault_from_the_environment():
    code = ("import torch, clustering_flashassign_b200 as fk\n"
            "x = torch.randn(1, 500, 64, device='cuda').half(); c = x[:, :32].contiguous()\n"
            "ids = torch.empty((1, 500), dtype=torch.int32, device='cuda')\n"
            "try:\n    fk.fk_assign(x, c, ids)\n    print('no failure')\n"
            "except fk.FkError as e:\n    print('status', e.status)\n"
            "fk.fk_assign(x, c, ids); torch.cuda.synchronize(); print('recovered')\n")
    env = dict(os.environ, FK_FAULT="alloc:1", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert "status 2" in out.stdout and "recovered" in out.stdout   # FK_ENOMEM == 2


def test_fp32_tensor_core_assign_recovers_after_a_stop_between_its_launches():
    """The fp32 tensor-core assign merges chunks through per-point keys that the
    next kernel turns into ids and clears.  A call stopped right after the assign
    kernel (its fourth launch: two row splits, the norm rows, the assign) leaves
    keys behind; the next call must clear them and give the right ids."""
    import clustering_flashassign_b200 as fk
    B, N, K, d = 1, 2000, 600, 64            # K * d >= 16384: tensor cores, 3 chunks
    x, _, c = case(B, N, K, d, "f32", mean_std=4.0, seed=83)
    xd, cd = to_dev(x, "f32"), to_dev(c, "f32")
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_inject_fault(fk.FK_FAULT_LAUNCH, 4)
    with pytest.raises(fk.FkError):
        fk.fk_assign(xd, cd, ids)
    torch.cuda.synchronize()
    # other centroids: a stale key of the stopped call (a value under the old
    # centroids) would win the merge and leave a wrong id
    c2 = (c[:, ::-1] * 0.5 + 1.0).astype(np.float32)
    ids.fill_(-1)
    fk.fk_assign(xd, to_dev(np.ascontiguousarray(c2), "f32"), ids)
    torch.cuda.synchronize()
    assert fk.fk_device_error() == 0
    check_ids(ids.cpu().numpy(), x, "f32", c2.astype(np.float64))
