"""The multi-rank (N > 1) path of bench.py on CPU: two gloo ranks.

bench.py shards by whole problems (weak scaling): every rank runs its own
B-batch workload with its own seeds and there is no data-path collective.  The
only collectives are the timing reductions (max of the step time, sum of the
iterations over ranks), which these tests run with the gloo backend.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthdata  # noqa: E402


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reduce_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: step time 10 + r ms, 20 + r iterations, a second pair for the e2e leg
        mx, sm = bench.reduce_over_ranks(dist, torch.device("cpu"), [10.0 + rank, 3.0 * rank],
                                         [20 + rank, 1])
        out[rank] = (tuple(mx), tuple(sm))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_reduce_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        mx, sm = res[r]
        assert mx == (11.0, 3.0), "every rank sees the slowest rank's time"
        assert sm == (41.0, 2.0), "every rank sees the total iteration count"


def test_reduce_over_ranks_single_process_is_identity():
    mx, sm = bench.reduce_over_ranks(None, torch.device("cpu"), [5.0, 1.5], [7, 2])
    assert mx == [5.0, 1.5] and sm == [7.0, 2.0]


def test_rank_workloads_are_independent_problems_of_one_shape():
    w0, w1 = bench.rank_workload(0), bench.rank_workload(1)
    assert (w0.B, w0.N, w0.K, w0.d, w0.dtype) == (w1.B, w1.N, w1.K, w1.d, w1.dtype)
    assert w0.seed != w1.seed and w0.init_seed != w1.init_seed
    # at a checker size the two ranks' points and initial index sets differ
    s0, s1 = bench.rank_workload(0, B=2, N=512, K=8), bench.rank_workload(1, B=2, N=512, K=8)
    x0, i0, _ = synthdata.make(s0)
    x1, i1, _ = synthdata.make(s1)
    assert x0.shape == x1.shape and not np.array_equal(x0, x1)
    assert not np.array_equal(i0, i1)
    # and rank 0 of the bench is the single-GPU workload itself
    assert bench.rank_workload(0) == synthdata.WORKLOADS[bench.WORKLOAD]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("world", [2])
def test_ranks_take_whole_problems(world):
    # weak scaling: the units one rank processes do not depend on the world size
    per_rank = [bench.rank_workload(r) for r in range(world)]
    assert all(w.B == synthdata.WORKLOADS[bench.WORKLOAD].B for w in per_rank)


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle timed on the host cores) prints
    exactly one JSON line with the keys the driver reads."""
    import json
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["n_gpus"] == 1
    assert {"value", "unit", "cores", "kind", "sample"} <= set(d["cpu_baseline"])
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
