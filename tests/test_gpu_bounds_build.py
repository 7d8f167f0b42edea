"""The bounds-checked device build on small ragged cases of every path.

libtq_bounds.so is libtq.so compiled with -DTQ_DEBUG_BOUNDS: each kernel checks
every address it computes from cache geometry, token positions or split ranges
against the buffer it belongs to, records a failed check in a device flag and
skips the access (nothing traps).  The same cases run in two child processes,
one per library: no check may fire, and both builds must produce the same
packed caches, outputs and logits bit for bit (the checks change no
arithmetic)."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _run(tmp_path, bounds):
    from compressed_attention_turboquantprod_b200 import build
    build.build(bounds=bounds)
    out = tmp_path / ("bounds.npz" if bounds else "plain.npz")
    env = dict(os.environ)
    env.pop("TQ_LIBRARY", None)
    if bounds:
        env["TQ_LIBRARY"] = "bounds"
    r = subprocess.run([sys.executable, os.path.join(HERE, "bounds_cases.py"), str(out)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    return np.load(out)


def test_bounds_checked_build_no_check_fires_and_results_identical(tmp_path):
    plain = _run(tmp_path, False)
    checked = _run(tmp_path, True)
    assert int(checked["bounds_enabled"][0]) == 1 and int(plain["bounds_enabled"][0]) == 0
    assert set(plain.files) == set(checked.files)
    for k in plain.files:
        if k == "bounds_enabled":
            continue
        a, b = plain[k], checked[k]
        assert a.shape == b.shape, k
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), f"{k} differs between the builds"
