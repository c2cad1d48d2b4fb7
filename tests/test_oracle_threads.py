"""The oracle's results do not depend on how many host threads run it (it is also the timed CPU
baseline, run multi-threaded): one thread and the default give bitwise equal outputs."""
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = r"""
import sys
import numpy as np
sys.path.insert(0, sys.argv[1])
from oracle import oracle as orc
rng = np.random.default_rng(41)
n_h, d_h, d_c, d_r, s_q, lens = 6, 16, 32, 8, 2, (3, 70, 129)
T = len(lens) * s_q
q_c = rng.standard_normal((T, n_h, d_h)); q_r = rng.standard_normal((T, n_h, d_r))
q_pos = np.array([L - s_q + i for L in lens for i in range(s_q)], dtype=np.int64)
c = [rng.standard_normal((L, d_c)) for L in lens]; k = [rng.standard_normal((L, d_r)) for L in lens]
w_uk = rng.standard_normal((n_h * d_h, d_c)) / 6; w_uv = rng.standard_normal((n_h * d_h, d_c)) / 6
a = orc.decode_absorbed(q_c, q_r, q_pos, c, k, w_uk, w_uv, s_q=s_q)
n = orc.decode_naive(q_c, q_r, q_pos, c, k, w_uk, w_uv, s_q=s_q)
np.savez(sys.argv[2], ao=a.o, alat=a.o_lat, alse=a.lse, no=n.o, threads=orc.num_threads())
"""


def _run(tmp_path, name, threads):
    env = dict(os.environ)
    if threads is None:
        env.pop("OMP_NUM_THREADS", None)
    else:
        env["OMP_NUM_THREADS"] = str(threads)
    out = str(tmp_path / name)
    subprocess.run([sys.executable, "-c", _SCRIPT, ROOT, out], check=True, env=env, timeout=300)
    return np.load(out + ".npz")


def test_oracle_is_bitwise_independent_of_thread_count(oracle_mod, tmp_path):
    one = _run(tmp_path, "one", 1)
    many = _run(tmp_path, "many", 4)
    assert int(one["threads"]) == 1 and int(many["threads"]) == 4
    for key in ("ao", "alat", "alse", "no"):
        assert np.array_equal(one[key], many[key]), key
