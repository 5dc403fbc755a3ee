"""Environment defaults of fk_lloyd's options, each in a fresh process:
FK_VERBOSE=1 prints one line per iteration on stderr; FK_CHUNK_POINTS sets the
streamed chunk size when the caller passes 0, with the same result as passing
it explicitly."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CODE = """
import sys, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import clustering_flashassign_b200 as fk
from test_parity_kernels import case, to_dev
x, _, c = case(2, 5000, 64, 64, "f16", seed=79)
xh = torch.from_numpy(x).pin_memory(); cd = to_dev(c, "f16")
ids = torch.empty((2, 5000), dtype=torch.int32, device="cuda")
cen = torch.empty((2, 64, 64), dtype=torch.float32, device="cuda")
fk.fk_lloyd(xh, cd, 3, 0.0, ids, cen, host_mode=fk.FK_HOST_STREAM, chunk_points={chunk})
torch.save((ids.cpu(), cen.cpu()), {out!r})
"""


def _run(tmp_path, name, chunk, env_extra):
    out = str(tmp_path / f"{name}.pt")
    code = CODE.format(root=ROOT, tests=os.path.join(ROOT, "tests"), chunk=chunk, out=out)
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    return r, out


def test_verbose_and_chunk_size_from_the_environment(tmp_path):
    import torch
    r_env, out_env = _run(tmp_path, "env", 0, {"FK_VERBOSE": "1", "FK_CHUNK_POINTS": "1300"})
    r_arg, out_arg = _run(tmp_path, "arg", 1300, {})
    lines = [ln for ln in r_env.stderr.splitlines() if "iter" in ln and "max_shift" in ln]
    assert len(lines) == 3, r_env.stderr
    assert not [ln for ln in r_arg.stderr.splitlines() if "max_shift" in ln]
    a, b = torch.load(out_env), torch.load(out_arg)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
