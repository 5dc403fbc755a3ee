"""fk_assign_noalloc: the assign entry point for callers that cannot allocate.

Callers that run under an allocator owning all device memory, or inside loops
where cudaMalloc / cudaFree are not allowed, use this variant; its scratch is a
static device array.  The test drives it through the C ABI and checks that it
returns exactly what fk_assign returns, on two calls in a row with different
shapes (the shared scratch must not leak state from one call into the next),
and that the second call leaves free device memory unchanged.  This file is
collected last so that a failure here comes after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import check_ids

pytestmark = pytest.mark.gpu


def _inputs(B, N, K, d, dtype, seed):
    w = synthdata.Workload("na", B, N, K, d, dtype, K, 3.0, 0.0, 1, 0.0, seed, seed + 1)
    x, idx, c = synthdata.make(w)
    if dtype == "bf16":
        to = lambda a: torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    else:
        to = lambda a: torch.from_numpy(a).cuda()
    return to(x), to(c)


def _raw_noalloc(fk, x, c, ids):
    B, N, d = x.shape
    K = c.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fk.lib.fk_assign_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(c.data_ptr()), B, N, K,
                                    d, fk.DTYPES[x.dtype], ctypes.c_void_p(ids.data_ptr()), stream)


def test_noalloc_assign_matches_fk_assign_on_consecutive_calls():
    import clustering_flashassign_b200 as fk
    cases = [(4, 3000, 1000, 128, "f16", 5), (2, 2000, 300, 192, "bf16", 6), (1, 500, 70, 24, "f32", 7)]
    free_after_first = None
    for n, (B, N, K, d, dtype, seed) in enumerate(cases + cases[:1]):
        x, c = _inputs(B, N, K, d, dtype, seed)
        ref = torch.empty((B, N), dtype=torch.int32, device="cuda")
        fk.fk_assign(x, c, ref)
        got = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        st = _raw_noalloc(fk, x, c, got)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert st == fk.FK_OK, fk.fk_last_error()
        assert torch.equal(got, ref), f"call {n}: ids differ from fk_assign"
        if n > 0:  # the first call may load the module that holds the static array
            assert free1 == free0, "fk_assign_noalloc changed free device memory"
        free_after_first = free1
    assert free_after_first is not None


def test_noalloc_assign_rejects_shapes_beyond_its_scratch():
    import clustering_flashassign_b200 as fk
    d = ctypes.c_void_p(0x1000)
    # B * Kpad = 5 * 32768 > 2^17 norm rows of scratch
    st = fk.lib.fk_assign_noalloc(d, d, 5, 300000, 32768, 128, fk.FK_F16, d, None)
    assert st == fk.FK_EUNSUPPORTED
    assert "exceeds" in fk.fk_last_error()


def test_noalloc_fp32_on_cuda_cores_matches_the_oracle_where_fk_assign_uses_tf32():
    """fp32 with K * d >= 16384: fk_assign takes the 3xTF32 tensor-core path,
    this call the CUDA-core kernel (it cannot hold the widened points).  Both
    must satisfy the near-tie rule against the fp64 oracle; they may differ
    from each other only on near ties."""
    import clustering_flashassign_b200 as fk
    B, N, K, d = 2, 1500, 300, 64   # K * d = 19200
    x, c = _inputs(B, N, K, d, "f32", 8)
    chat = c.cpu().numpy().astype(np.float64)
    xn = x.cpu().numpy()
    ref, gap, _ = oracle.assign(xn, "f32", chat)
    for n in range(2):
        got = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
        assert _raw_noalloc(fk, x, c, got) == fk.FK_OK, fk.fk_last_error()
        torch.cuda.synchronize()
        check_ids(got.cpu().numpy(), xn, "f32", chat, ref, gap)
        tc = torch.empty((B, N), dtype=torch.int32, device="cuda")
        fk.fk_assign(x, c, tc)
        check_ids(tc.cpu().numpy(), xn, "f32", chat, ref, gap)


def test_noalloc_reports_a_norm_beyond_the_fp16_digit_range():
    """What the kernels record in the static error word is read (and cleared)
    by fk_noalloc_device_error, which allocates nothing either."""
    import clustering_flashassign_b200 as fk
    B, N, K, d = 1, 300, 40, 128
    x, c = _inputs(B, N, K, d, "f16", 9)
    assert fk.fk_noalloc_device_error() == fk.FK_OK
    c[0, 5] = 6000.0   # ||c||^2 = 128 * 3.6e7 = 4.6e9 > 2^32
    got = torch.full((B, N), -1, dtype=torch.int32, device="cuda")
    assert _raw_noalloc(fk, x, c, got) == fk.FK_OK   # asynchronous: nothing read yet
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert fk.fk_noalloc_device_error() == fk.FK_EUNSUPPORTED
    assert "2^32" in fk.fk_last_error()
    assert fk.fk_noalloc_device_error() == fk.FK_OK   # cleared
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, "fk_noalloc_device_error changed free device memory"
    c[0, 5] = 4000.0   # ||c||^2 = 2.05e9 < 2^32: fine
    ref = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(x, c, ref)
    assert _raw_noalloc(fk, x, c, got) == fk.FK_OK
    assert fk.fk_noalloc_device_error() == fk.FK_OK
    assert torch.equal(got, ref)
