"""GPU parity of the individual steps against the fp64 oracle (lockstep).

Sizes span several point tiles (128), centroid chunks (256) and sort tiles
(4096) with ragged tails; every case runs through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
import synthdata
from parity import CENTER_TOL, check_centers, check_ids

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def from_dev16(t: torch.Tensor, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def case(B, N, K, d, dtype, n_comp=None, mean_std=3.0, zipf=0.0, seed=7):
    w = synthdata.Workload("case", B, N, K, d, dtype, n_comp or K, mean_std, zipf, 1, 0.0, seed, seed * 10)
    return synthdata.make(w)


ASSIGN_CASES = [
    # B, N, K, d, dtype
    (2, 1000, 300, 128, "f16"),    # resident-X variant, ragged tiles and chunks
    (2, 1000, 300, 128, "bf16"),
    (1, 777, 513, 64, "f16"),      # one K-block
    (3, 300, 40, 8, "f16"),        # d < 64: zero-filled K-block
    (2, 520, 260, 72, "bf16"),     # non-power-of-two d, two K-blocks
    (2, 400, 260, 192, "f16"),     # split-d variant
    (1, 700, 600, 1024, "bf16"),   # split-d, many K-blocks
    (4, 129, 129, 128, "f16"),     # one row past a point tile
    (2, 300, 257, 128, "f16"),     # one centroid past a chunk
    (1, 64, 1, 16, "f16"),         # K = 1, N below one tile
    (1, 256, 256, 32, "f16"),      # K = N
    (3, 40000, 700, 128, "f16"),   # 939 point tiles: several tiles per CTA
    (2, 45000, 520, 64, "bf16"),   # the same with one K-block, ragged last tile of each batch
]


@pytest.mark.parametrize("B,N,K,d,dtype", ASSIGN_CASES)
def test_flash_assign_matches_oracle(B, N, K, d, dtype):
    import clustering_flashassign_b200 as fk
    x, idx, c0 = case(B, N, K, d, dtype)
    xd, cd = to_dev(x, dtype), to_dev(c0, dtype)
    ids = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, ids)
    torch.cuda.synchronize()
    assert fk.fk_device_error() == 0
    chat = synthdata.to_f64(c0, dtype)
    check_ids(ids.cpu().numpy(), x, dtype, chat)


def test_flash_assign_exact_ties_take_lowest_index():
    import clustering_flashassign_b200 as fk
    B, N, K, d = 2, 700, 600, 128
    x, idx, c0 = case(B, N, K, d, "f16", seed=3)
    # duplicate centroids across chunks and across the two column halves
    for dst, src in [(599, 3), (300, 3), (130, 3), (257, 100), (511, 100), (555, 0)]:
        c0[:, dst] = c0[:, src]
    xd, cd = to_dev(x, "f16"), to_dev(c0, "f16")
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, cd, ids)
    g = ids.cpu().numpy()
    assert not np.isin(g, [599, 300, 130, 257, 511, 555]).any()
    # points equal to a centroid row pick the lowest duplicate
    xd2 = torch.cat([cd[:, [3, 100, 0], :], xd], dim=1).contiguous()
    ids2 = torch.empty((B, N + 3), dtype=torch.int32, device="cuda")
    fk.fk_assign(xd2, cd, ids2)
    assert ids2[:, :3].cpu().numpy().tolist() == [[3, 100, 0]] * B


@pytest.mark.parametrize("B,N,K,d", [
    (1, 8192, 64, 32), (2, 1000, 37, 5), (1, 300, 70, 100),   # CUDA cores (K * d < 16384 or d % 4)
    (2, 3000, 300, 64),      # tensor cores, 3xTF32: 192-wide extended rows, six K-blocks
    (1, 1000, 600, 100),     # ragged last K-block (300 = 9 x 32 + 12), ragged chunk
    (3, 300, 257, 128),      # ragged point tile, one centroid past a chunk
    (1, 2048, 1024, 2048),   # the large-D fp32 shape of the pages' FlashKMeans example
])
def test_fp32_assign_matches_oracle(B, N, K, d):
    import clustering_flashassign_b200 as fk
    x, idx, c0 = case(B, N, K, d, "f32", mean_std=4.0)
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(to_dev(x, "f32"), to_dev(c0, "f32"), ids)
    check_ids(ids.cpu().numpy(), x, "f32", c0.astype(np.float64))


SORT_CASES = [(2, 10000, 300), (1, 4096, 4096), (3, 5000, 1), (1, 9000, 5000), (2, 20000, 70000 // 10),
              (1, 300000, 33000)]


@pytest.mark.parametrize("B,N,K", SORT_CASES)
def test_counting_sort_is_bit_exact(B, N, K):
    import clustering_flashassign_b200 as fk
    rng = np.random.default_rng(B * 31 + K)
    # skewed ids: a few hot clusters plus a uniform tail, some clusters empty
    hot = rng.integers(0, K, size=(B, N)) % max(1, K // 7)
    uni = rng.integers(0, K, size=(B, N))
    ids = np.where(rng.random((B, N)) < 0.6, hot, uni).astype(np.int32)
    idt = torch.from_numpy(ids).cuda()
    perm = torch.empty((B, N), dtype=torch.int32, device="cuda")
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    offsets = torch.empty((B, K), dtype=torch.int32, device="cuda")
    fk.fk_sort(idt, K, perm, counts, offsets)
    rc, rp = oracle.sort(ids, K)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), np.cumsum(rc, axis=1) - rc)
    np.testing.assert_array_equal(perm.cpu().numpy(), rp)
    assert fk.fk_device_error() == 0


UPDATE_CASES = [
    (2, 1000, 300, 128, "f16"),
    (2, 1000, 300, 128, "bf16"),
    (1, 8192, 64, 32, "f32"),
    (2, 3000, 50, 30, "f32"),       # fp32 with d % 4 != 0 (scalar flush path)
    (1, 5000, 5000, 16, "f16"),     # many empty clusters, 2-pass sort
    (2, 600, 400, 1024, "bf16"),    # several column blocks
]


@pytest.mark.parametrize("B,N,K,d,dtype", UPDATE_CASES)
def test_update_matches_oracle_given_gpu_ids(B, N, K, d, dtype):
    import clustering_flashassign_b200 as fk
    x, idx, c0 = case(B, N, K, d, dtype, n_comp=max(2, K // 3), zipf=1.2)
    xd = to_dev(x, dtype)
    ids = torch.empty((B, N), dtype=torch.int32, device="cuda")
    fk.fk_assign(xd, to_dev(c0, dtype), ids)
    old = synthdata.to_f64(c0, dtype)
    centers = torch.from_numpy(old.astype(np.float32)).cuda()
    counts = torch.empty((B, K), dtype=torch.int32, device="cuda")
    ms = torch.zeros(1, dtype=torch.float32, device="cuda")
    fk.fk_update(xd, ids, centers, counts, ms)
    g_ids = ids.cpu().numpy()
    new, rc, shift, rms = oracle.update(x, dtype, g_ids, old)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    check_centers(centers.cpu().numpy(), new, dtype)
    empty = rc == 0
    if empty.any():  # empty clusters keep their previous value exactly
        np.testing.assert_array_equal(centers.cpu().numpy()[empty], old.astype(np.float32)[empty])
    # |shift_gpu - shift_ref| <= ||c_gpu - c_ref||, which the centroid rule bounds
    scale = float(np.sqrt((new ** 2).sum(-1)).max())
    assert abs(ms.item() - rms) <= 2 * CENTER_TOL[dtype] * max(scale, 1.0)
    # a second update from the new centers reuses the (cleared) workspace sums
    fk.fk_update(xd, ids, centers, counts, ms)
    new2, _, _, _ = oracle.update(x, dtype, g_ids, centers.cpu().numpy().astype(np.float64))
    check_centers(centers.cpu().numpy(), new2, dtype)
    assert ms.item() <= 1e-3 * max(1.0, float(np.abs(new).max()))
