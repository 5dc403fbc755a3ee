"""Pins for the fp64 oracle: it is checked against things other than itself.

- hand-derived worked examples (tests/golden/*.json, each citing its source),
- brute force on tiny inputs through an independent library argmin (numpy),
- closed forms (K = 1 gives the global mean; separated blobs give their sample
  means; a 3-4-5 shift),
- invariants (counts sum to N, perm is the (id, index) order, each centroid is
  the mean of its points, the objective does not increase without rounding),
- the dtype rounding against numpy's float16 / float32 conversions.

``test_planted_mistakes_are_caught`` plants each of a list of plausible bugs in
the oracle (on the CPU) and checks that at least one pin fails for each.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synthdata

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- pins


def pin_golden_lloyd_1d():
    g = _gold("lloyd_1d_worked.json")
    x = np.array(g["x"], np.float32)
    init = np.array(g["init"], np.float64)
    c = init.copy()
    for it in g["iters"]:
        ids, _, _ = oracle.assign(x, "f32", c)
        assert ids.tolist()[0] == it["ids"]
        obj = oracle.objective(x, "f32", c, ids)
        assert obj == pytest.approx(it["objective"], rel=1e-12)
        new, counts, _, ms = oracle.update(x, "f32", ids, c)
        np.testing.assert_allclose(new, np.array(it["centers"]), rtol=1e-12, atol=0)
        assert counts.tolist()[0] == it["counts"]
        assert ms == pytest.approx(it["maxshift"], rel=1e-12, abs=1e-15)
        c = new
    r = oracle.lloyd(x, "f32", init, 5, 0.0, round_dtype=None)
    assert r["iters"] == g["stop"]["tol0_max_iter5_iters"]
    np.testing.assert_allclose(r["centers"], np.array(g["iters"][-1]["centers"]), rtol=1e-12)
    assert r["ids"].tolist()[0] == g["iters"][-1]["ids"]
    np.testing.assert_allclose(r["objective"][:3], [i["objective"] for i in g["iters"]], rtol=1e-12)
    r = oracle.lloyd(x, "f32", init, 5, 1e-9, round_dtype=None)
    assert r["iters"] == g["stop"]["tol1e-9_iters"]


def pin_golden_update():
    g = _gold("update_empty_and_shift.json")
    x = np.array(g["x"], np.float32)
    ids = np.array(g["ids"], np.int32)
    old = np.array(g["old"], np.float64)
    new, counts, shift, ms = oracle.update(x, "f32", ids, old)
    np.testing.assert_allclose(new, np.array(g["new"]), rtol=1e-15, atol=0)
    assert counts.tolist() == g["counts"]
    np.testing.assert_allclose(shift, np.array(g["shift"]), rtol=1e-14, atol=0)
    assert ms == pytest.approx(g["maxshift"], rel=1e-14)
    cnt, perm = oracle.sort(ids, old.shape[1])
    assert cnt.tolist() == g["counts"]
    assert perm.tolist() == g["perm"]


def pin_golden_ties():
    g = _gold("assign_ties.json")
    for case in g["cases"]:
        x = np.array(case["x"], np.float32)
        c = np.array(case["c"], np.float64)
        ids, gap, _ = oracle.assign(x, "f32", c)
        assert ids.tolist() == case["ids"]
        np.testing.assert_allclose(gap, np.array(case["gap"]), rtol=0, atol=0)
        # the tie rule does not depend on where the tied pair sits
        ids2, _, _ = oracle.assign(x, "f32", c[:, ::-1].copy())
        K = c.shape[1]
        dist = ((x[0, 0].astype(np.float64)[None, :] - c[0][::-1]) ** 2).sum(-1)
        assert ids2[0, 0] == int(np.flatnonzero(dist == dist.min())[0])
        assert K >= 2


def pin_brute_force_tiny():
    rng = np.random.default_rng(11)
    for trial in range(40):
        B = int(rng.integers(1, 3))
        N = int(rng.integers(1, 65))
        K = int(rng.integers(1, 9))
        d = int(rng.integers(1, 7))
        # small integers make exact ties common; duplicate a centroid now and then
        x = rng.integers(-3, 4, size=(B, N, d)).astype(np.float32)
        c = rng.integers(-3, 4, size=(B, K, d)).astype(np.float64)
        if K >= 2 and trial % 3 == 0:
            c[:, K - 1] = c[:, 0]
        ids, gap, dmin = oracle.assign(x, "f32", c)
        D = ((x.astype(np.float64)[:, :, None, :] - c[:, None, :, :]) ** 2).sum(-1)  # (B,N,K)
        ref = np.argmin(D, axis=-1)  # first occurrence = lowest k
        np.testing.assert_array_equal(ids, ref)
        np.testing.assert_array_equal(dmin, D.min(-1))
        if K >= 2:
            s = np.sort(D, axis=-1)
            np.testing.assert_array_equal(gap, s[..., 1] - s[..., 0])
        # a second independent argmin: python min over (value, index) pairs
        for b in range(B):
            for i in range(N):
                assert ids[b, i] == min(range(K), key=lambda k: (D[b, i, k], k))
    # fp16 / bf16 inputs widen exactly
    xh = rng.standard_normal((1, 50, 8)).astype(np.float16)
    ch = rng.standard_normal((1, 5, 8))
    ids, _, _ = oracle.assign(xh, "f16", ch)
    D = ((xh.astype(np.float64)[:, :, None, :] - ch[:, None]) ** 2).sum(-1)
    np.testing.assert_array_equal(ids, np.argmin(D, -1))
    xb = synthdata.from_f32(rng.standard_normal((1, 50, 8)).astype(np.float32), "bf16").reshape(1, 50, 8)
    ids, _, _ = oracle.assign(xb, "bf16", ch)
    D = ((synthdata.to_f64(xb, "bf16")[:, :, None, :] - ch[:, None]) ** 2).sum(-1)
    np.testing.assert_array_equal(ids, np.argmin(D, -1))


def pin_k1_global_mean():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 300, 5)).astype(np.float32)
    init = x[:, :1, :].astype(np.float64)
    r = oracle.lloyd(x, "f32", init, 2, 0.0, round_dtype=None)
    assert (r["ids"] == 0).all()
    np.testing.assert_allclose(r["centers"][:, 0, :], x.astype(np.float64).mean(axis=1), rtol=1e-12, atol=1e-14)
    assert r["counts"].tolist() == [[300], [300]]


def pin_separated_blobs():
    # four blobs 1000 apart with unit noise: one Lloyd step from one point per
    # blob lands every centroid on its blob's sample mean, and it then stays.
    x, comp = synthdata.mixture(1, 2000, 6, "f32", 1, 0.0, 0.0, 21, with_components=True)
    offs = np.array([[0, 0, 0, 0, 0, 0], [1000, 0, 0, 0, 0, 0], [0, 1000, 0, 0, 0, 0], [0, 0, 0, 1000, 1000, 0]], np.float32)
    lab = np.arange(2000) % 4
    x = (x[0] + offs[lab])[None].astype(np.float32)
    init = np.stack([x[0, np.flatnonzero(lab == k)[0]] for k in range(4)])[None].astype(np.float64)
    true_means = np.stack([x[0, lab == k].astype(np.float64).mean(0) for k in range(4)])
    r = oracle.lloyd(x, "f32", init, 3, 0.0, round_dtype=None)
    np.testing.assert_array_equal(r["ids"][0], lab)
    np.testing.assert_allclose(r["centers"][0], true_means, rtol=1e-12, atol=1e-12)
    assert r["maxshift"] == 0.0


def pin_invariants():
    w = synthdata.scaled(synthdata.WORKLOADS["zipf"], B=2, N=3000, K=40, d=16, n_comp=40)
    x, idx, c0 = synthdata.make(w)
    c = synthdata.to_f64(c0, "f16")
    prev_obj = None
    for it in range(6):
        ids, gap, _ = oracle.assign(x, "f16", c)
        obj = oracle.objective(x, "f16", c, ids)
        if prev_obj is not None:  # exact centroids: Lloyd never increases the objective
            assert obj <= prev_obj * (1 + 1e-12)
        new, counts, shift, ms = oracle.update(x, "f16", ids, c)
        assert counts.sum(axis=1).tolist() == [w.N] * w.B
        cnt2, perm = oracle.sort(ids, w.K)
        np.testing.assert_array_equal(cnt2, counts)
        xf = synthdata.to_f64(x, "f16")
        for b in range(w.B):
            p = perm[b]
            assert np.array_equal(np.sort(p), np.arange(w.N))
            key = ids[b][p].astype(np.int64) * w.N + p
            assert (np.diff(key) > 0).all()  # sorted by id, then by index
            for k in range(w.K):
                m = ids[b] == k
                if m.any():
                    np.testing.assert_allclose(new[b, k], xf[b][m].mean(0), rtol=1e-12, atol=1e-12)
                else:
                    np.testing.assert_array_equal(new[b, k], c[b, k])
        assert ms == pytest.approx(float(np.sqrt(((new - c) ** 2).sum(-1)).max()), rel=1e-12)
        prev_obj = oracle.objective(x, "f16", new, ids)
        assert prev_obj <= obj * (1 + 1e-12)  # the update step never increases it either
        c = new


def pin_rounding():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-9, 5, 5000),
                        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e-8, 2.0 ** -24, 3 * 2.0 ** -26, 2.0 ** -25]])
    h = oracle.round_to(v, "f16")
    with np.errstate(over="ignore"):
        ref16 = v.astype(np.float16).astype(np.float64)  # numpy rounds from double
    np.testing.assert_array_equal(h, ref16)
    f = oracle.round_to(v, "f32")
    np.testing.assert_array_equal(f, v.astype(np.float32).astype(np.float64))
    # bf16: values exactly representable in fp32 round the same through fp32
    v32 = v.astype(np.float32).astype(np.float64)
    bb = oracle.round_to(v32, "bf16")
    ref = synthdata.to_f64(synthdata.from_f32(v32.astype(np.float32), "bf16"), "bf16")
    np.testing.assert_array_equal(bb, ref)
    # hand-checked bf16 ties: 1 + 2^-8 -> 1 (even), 1 + 3*2^-8 -> 1 + 2^-6 (even)
    assert oracle.round_to(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8]), "bf16").tolist() == [1.0, 1 + 2.0 ** -6]


PINS = [pin_golden_lloyd_1d, pin_golden_update, pin_golden_ties, pin_brute_force_tiny, pin_k1_global_mean,
        pin_separated_blobs, pin_invariants, pin_rounding]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    oracle.set_mutation(0)
    pin()


# Planted mistakes (see fk_oracle.c): 1 ties->highest k, 2 empty cluster zeroed,
# 3 mean divides by count+1, 4 last dimension dropped, 5 perm descending within
# a cluster, 6 L1-style shift, 7 wrong sign in the distance, 8 transposed
# centroid operand, 9 cluster 0 miscounted.
@pytest.mark.parametrize("mutation", range(1, 10))
def test_planted_mistakes_are_caught(mutation):
    caught = []
    try:
        oracle.set_mutation(mutation)
        for pin in PINS:
            try:
                pin()
            except (AssertionError, RuntimeError):
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert caught, f"planted mistake {mutation} passed every pin"
