"""The oracle's results do not depend on how many OpenMP threads it runs
with: every output is one fp64 sum taken in its natural order by one thread,
so runs with 1 and with 4 threads must agree bit for bit."""
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
import numpy as np
sys.path.insert(0, {root!r})
import oracle
r = np.random.default_rng(5)
u = r.standard_normal((3, 4, 300)); k = r.standard_normal((4, 300)); D = r.standard_normal(4)
w = r.standard_normal((3, 4, 300)); v = r.standard_normal((3, 4, 300))
u2 = r.standard_normal((2, 3, 24, 20)); k2 = r.standard_normal((3, 24, 20))
u3 = r.standard_normal((2, 2, 8, 12, 10)); k3 = r.standard_normal((2, 8, 12, 10))
bi, hi, ti = r.integers(0, 3, 50), r.integers(0, 4, 50), r.integers(0, 300, 50)
np.savez({out!r},
         y1=oracle.causal_conv1d(u, k, D=D, w=w, v=v),
         p1=oracle.causal_conv1d_points(u, k, bi, hi, ti, D=D),
         y2=oracle.causal_conv2d(u2, k2),
         y3=oracle.causal_conv3d(u3, k3),
         nt=oracle.num_threads())
"""


def _run(tmp_path, threads):
    out = str(tmp_path / f"oracle_{threads}.npz")
    env = dict(os.environ, OMP_NUM_THREADS=str(threads))
    r = subprocess.run([sys.executable, "-c", SCRIPT.format(root=ROOT, out=out)], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    return np.load(out)


def test_oracle_is_independent_of_thread_count(tmp_path):
    one, four = _run(tmp_path, 1), _run(tmp_path, 4)
    assert int(one["nt"]) == 1 and int(four["nt"]) == 4
    for name in ("y1", "p1", "y2", "y3"):
        assert np.array_equal(one[name], four[name]), name
