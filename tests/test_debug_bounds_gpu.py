"""The debug build (libpdn_debug.so: every kernel's computed workspace,
checkpoint, partial-sum and state-item indices checked, a failure recorded as
PDN_ERR_BOUNDS in the device error word and the access skipped or redirected)
runs a cross-section of the GPU parity suites in a subprocess. Those tests
assert a clean device error word after every call, so any index check that
fails, fails them; the results must still match the oracle."""
import os
import subprocess
import sys

import pytest

from linear_recurrence_sequence_chunked_b200 import build as pdn_build
from linear_recurrence_sequence_chunked_b200 import pdn

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suites_under_the_debug_build():
    lib = pdn_build.build(debug_bounds=True)
    assert os.path.basename(lib) == os.path.basename(pdn.DEBUG_LIB_PATH)
    env = dict(os.environ, PDN_LIBRARY=lib)
    sel = ("test_backward_lengths or test_backward_head_dims or test_backward_variants or "
           "test_backward_many_chains or test_backward_prologue or test_backward_training_mode or "
           "test_tc_variants or time_segments or test_decode or test_variants_small")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "-k", sel, "tests/test_backward_gpu.py", "tests/test_tc_gpu.py",
           "tests/test_decode_gpu.py", "tests/test_parity_gpu.py"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_debug_library_is_the_one_loaded():
    lib = pdn_build.build(debug_bounds=True)
    code = ("from linear_recurrence_sequence_chunked_b200 import pdn; pdn.load(); "
            "print(pdn._LIB_PATH)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       env=dict(os.environ, PDN_LIBRARY=lib), timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == lib
