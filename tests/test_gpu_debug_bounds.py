"""The bounds-checked build (libaut_debug.so: every kernel that computes its
own global addresses checks them and reports AUT_ERR_BOUNDS instead of
trapping) on real workloads: it must raise no false alarm, and the tiny
encoder's output must stay within the acceptance bound element by element.
Runs in a child process, which loads the debug library (AUT_LIB=debug)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_bounds_build_runs_clean():
    lib = os.path.join(os.path.dirname(HERE), "audio_encoder_aut_b200", "libaut_debug.so")
    if not os.path.exists(lib):
        from audio_encoder_aut_b200.build import build
        build(debug_bounds=True)
    env = dict(os.environ, AUT_LIB="debug")
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_run.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert d["lib"] == "libaut_debug.so"
    assert all(v == 0 for v in d["status"].values()), d["status"]
    assert d["tiny_max_err_over_rms"] <= 2e-2
