"""CPU checks of the C ABI: the library loads, exports every symbol that
include/fk.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "fk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fk_[a-z_]+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    names = _declared()
    for n in ["fk_assign", "fk_update", "fk_lloyd", "fk_sort", "fk_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    import clustering_flashassign_b200 as fk
    for name in _declared():
        assert hasattr(fk.lib, name), f"libfk.so does not export {name}"
    assert sorted(fk.EXPORTS) == _declared()


def test_status_strings_and_version():
    import clustering_flashassign_b200 as fk
    assert fk.fk_status_string(fk.FK_OK) == "ok"
    assert fk.fk_status_string(fk.FK_EINVAL) == "invalid argument"
    assert fk.fk_status_string(fk.FK_ETIMEOUT) == "kernel wait timed out"
    assert fk.fk_status_string(99) == "unknown status"
    assert fk.fk_version() >= 100


@pytest.mark.parametrize("B,N,K,d,dtype,why", [
    (0, 10, 2, 8, 1, "positive"),
    (1, 0, 2, 8, 1, "positive"),
    (1, 10, 0, 8, 1, "positive"),
    (1, 10, 11, 8, 1, "K must not exceed N"),
    (1, 10, 2, 12, 1, "multiple of 16 bytes"),
    (1, 10, 2, 8, 7, "unknown dtype"),
    (1, 1 << 31, 2, 8, 1, "below 2^31"),
])
def test_argument_validation_happens_on_the_host(B, N, K, d, dtype, why):
    import clustering_flashassign_b200 as fk
    L = fk.lib
    dummy = ctypes.c_void_p(0x1000)
    st = L.fk_assign(dummy, dummy, B, N, K, d, dtype, dummy, None)
    assert st == fk.FK_EINVAL
    assert why in fk.fk_last_error()
    st = L.fk_update(dummy, dummy, B, N, K, d, dummy, None, None, dtype, None)
    assert st == fk.FK_EINVAL


def test_null_and_misaligned_pointers_are_rejected():
    import clustering_flashassign_b200 as fk
    L = fk.lib
    st = L.fk_assign(None, ctypes.c_void_p(0x1000), 1, 10, 2, 8, 1, ctypes.c_void_p(0x1000), None)
    assert st == fk.FK_EINVAL and "x is NULL" in fk.fk_last_error()
    st = L.fk_assign(ctypes.c_void_p(0x1008), ctypes.c_void_p(0x1000), 1, 10, 2, 8, 1,
                     ctypes.c_void_p(0x1000), None)
    assert st == fk.FK_EINVAL and "16-byte aligned" in fk.fk_last_error()
    shape = fk.FkShape(1, 10, 2, 8, 1)
    st = L.fk_lloyd(ctypes.byref(shape), ctypes.c_void_p(0x1000), None, 3, 0.0,
                    ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), None, None, None)
    assert st == fk.FK_EINVAL and "init_centers" in fk.fk_last_error()
    st = L.fk_lloyd(None, None, None, 3, 0.0, None, None, None, None, None)
    assert st == fk.FK_EINVAL


def test_unsupported_shapes():
    import clustering_flashassign_b200 as fk
    L = fk.lib
    d = ctypes.c_void_p(0x1000)
    assert L.fk_assign(d, d, 70000, 10, 2, 8, 1, d, None) == fk.FK_EUNSUPPORTED
    assert L.fk_sort(d, 1, 1 << 26, (1 << 24) + 1, None, None, d, None) == fk.FK_EUNSUPPORTED


def test_binding_rejects_noncontiguous_tensors():
    import torch
    import clustering_flashassign_b200 as fk
    x = torch.zeros(2, 16, 8, dtype=torch.float16).transpose(0, 1)
    with pytest.raises(ValueError):
        fk.fk_assign(x, torch.zeros(16, 2, 8, dtype=torch.float16), torch.zeros(16, 2, dtype=torch.int32))


def test_data_parallel_pieces_validate_on_the_host():
    """fk_point_norms, fk_init_centers, fk_lloyd_step_partial and fk_update_finalize
    reject bad shapes and pointers before any device work."""
    import clustering_flashassign_b200 as fk
    L = fk.lib
    p = ctypes.c_void_p(0x1000)
    assert L.fk_point_norms(p, 1, 10, 8, fk.FK_F32, p, None) == fk.FK_EUNSUPPORTED
    assert L.fk_point_norms(None, 1, 10, 8, fk.FK_F16, p, None) == fk.FK_EINVAL
    assert "x is NULL" in fk.fk_last_error()
    assert L.fk_point_norms(p, 1, 10, 12, fk.FK_F16, p, None) == fk.FK_EINVAL
    assert L.fk_init_centers(p, 1, 0, 8, fk.FK_F16, p, None) == fk.FK_EINVAL
    assert L.fk_init_centers(p, 1, 4, 8, fk.FK_F16, None, None) == fk.FK_EINVAL
    shape = fk.FkShape(1, 10, 2, 8, fk.FK_F16)
    assert L.fk_lloyd_step_partial(None, p, None, p, p, p, p, None, None) == fk.FK_EINVAL
    assert "shape is NULL" in fk.fk_last_error()
    assert L.fk_lloyd_step_partial(ctypes.byref(shape), p, None, p, p, None, p, None, None) == fk.FK_EINVAL
    assert "sums is NULL" in fk.fk_last_error()
    for bad in (fk.FkShape(1, -1, 4, 8, fk.FK_F16), fk.FkShape(1, 10, 4, 12, fk.FK_F16),
                fk.FkShape(0, 10, 4, 8, fk.FK_F16)):
        assert L.fk_lloyd_step_partial(ctypes.byref(bad), p, None, p, p, p, p, None, None) == fk.FK_EINVAL
    # a block may hold fewer points than clusters, or none: the shape passes and
    # the first failure is a pointer check (none of these fakes is device memory)
    for block in (fk.FkShape(1, 10, 11, 8, fk.FK_F16), fk.FkShape(1, 0, 4, 8, fk.FK_F16)):
        assert L.fk_lloyd_step_partial(ctypes.byref(block), None, None, p, None, p, p, None,
                                       None) == fk.FK_EINVAL
        assert "must be device memory" in fk.fk_last_error() or "is NULL" in fk.fk_last_error()
    assert L.fk_update_finalize(p, None, 1, 4, 8, fk.FK_F16, p, p, None, None) == fk.FK_EINVAL
    assert "counts is NULL" in fk.fk_last_error()
    assert L.fk_update_finalize(p, p, 1, 4, 8, 9, p, p, None, None) == fk.FK_EINVAL
    assert "unknown dtype" in fk.fk_last_error()


def test_fault_injection_arguments():
    import clustering_flashassign_b200 as fk
    L = fk.lib
    assert L.fk_inject_fault(7, 1) == fk.FK_EINVAL
    assert L.fk_inject_fault(fk.FK_FAULT_ALLOC, 0) == fk.FK_EINVAL
    assert L.fk_inject_fault(fk.FK_FAULT_ALLOC, 3) == fk.FK_OK
    assert L.fk_inject_fault(fk.FK_FAULT_NONE, 1) == fk.FK_OK   # disarmed again


def test_binding_runs_each_call_on_its_first_cuda_tensors_device(monkeypatch):
    """The wrappers enter torch.cuda.device(...) of the first CUDA tensor among
    their arguments (the library works on the current device); host-only
    arguments switch nothing."""
    import clustering_flashassign_b200 as fk
    seen = []

    class Recorder:
        def __init__(self, dev):
            seen.append(dev)

        def __enter__(self):
            return self

        def __exit__(self, *exc):
            return False

    class Tensor:  # stands in for a torch tensor on `dev` (None: host memory)
        def __init__(self, dev):
            self.is_cuda = dev is not None
            self.device = dev

    monkeypatch.setattr(fk.torch.cuda, "device", Recorder)
    with fk._on(Tensor(None), None, Tensor("cuda:1"), Tensor("cuda:0")):
        pass
    assert seen == ["cuda:1"]
    with fk._on(Tensor(None), None):
        pass
    assert seen == ["cuda:1"]


def test_noalloc_binding_rejects_host_tensors_before_any_launch(monkeypatch):
    """fk_assign_noalloc's C entry point makes no pointer query, so the binding
    checks the tensors' placement itself: host tensors, or ids of the wrong
    type or shape, raise ValueError and the library is never called."""
    import torch
    import clustering_flashassign_b200 as fk

    calls = []

    class Lib:
        def __getattr__(self, name):
            calls.append(name)
            raise AssertionError(f"library called: {name}")

    monkeypatch.setattr(fk, "lib", Lib())
    x = torch.zeros(1, 16, 8, dtype=torch.float16)
    c = torch.zeros(1, 4, 8, dtype=torch.float16)
    ids = torch.zeros(1, 16, dtype=torch.int32)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fk.fk_assign_noalloc(x, c, ids)
    assert calls == []
    assert fk.FK_OK == 0  # the module itself is intact


def test_noalloc_entry_point_shares_fk_assign_shape_rules():
    import clustering_flashassign_b200 as fk
    L = fk.lib
    d = ctypes.c_void_p(0x1000)
    for B, N, K, dd, dt in [(1, 10, 11, 8, 1), (1, 10, 2, 12, 1), (1, 10, 2, 8, 7), (0, 10, 2, 8, 1)]:
        assert L.fk_assign_noalloc(d, d, B, N, K, dd, dt, d, None) == fk.FK_EINVAL
    # K above 2^24 is refused by both (fp32 needs no scratch, so only the shape rule applies)
    assert L.fk_assign(d, d, 1, 1 << 26, (1 << 24) + 1, 8, fk.FK_F32, d, None) == fk.FK_EUNSUPPORTED
    assert L.fk_assign_noalloc(d, d, 1, 1 << 26, (1 << 24) + 1, 8, fk.FK_F32, d, None) == fk.FK_EUNSUPPORTED
