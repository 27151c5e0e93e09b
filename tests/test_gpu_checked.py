"""The bounds-checked build (libgq4_checked.so, compiled with GQ4_CHECKED).

Its kernels test every weight, scale and activation-row index against the extent of its
array before the access and raise GQ4_ERR_BOUNDS in a library-wide status word instead of
reading outside (the pages' bug class: a scale read with a row index on an O*ng scale
array).  These tests run the parity cases of ragged shapes through the checked library
in a child process (the autouse fixture of conftest.py asserts a clear status word after
each), check that the reporting path works with an index test that touches no memory,
and that the ordinary build reports nothing."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.path.join(ROOT, "weight_only_int4_gq4_b200", "libgq4_checked.so")


def _child(args, timeout):
    env = dict(os.environ, GQ4_LIBRARY=CHECKED)
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_checked_library_reports_an_out_of_range_index():
    assert os.path.exists(CHECKED), "build it with `python -m weight_only_int4_gq4_b200.build --checked`"
    code = ("from weight_only_int4_gq4_b200 import gq4\n"
            "assert gq4.build_checked()\n"
            "gq4.selftest_bounds(2, 3); assert gq4.bounds_status() == 0\n"
            "gq4.selftest_bounds(3, 3); assert gq4.bounds_status() == gq4.ERR_BOUNDS\n"
            "gq4.selftest_bounds(-1, 3); assert gq4.bounds_status() == gq4.ERR_BOUNDS\n"
            "assert gq4.bounds_status() == 0\n"  # cleared by the read before
            "print('ok')\n")
    r = _child(["-c", code], 300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


def test_ordinary_library_reports_nothing():
    from weight_only_int4_gq4_b200 import gq4
    assert not gq4.build_checked()
    gq4.selftest_bounds(3, 3)
    torch.cuda.synchronize()
    assert gq4.bounds_status() == 0


def test_checked_library_parity_on_ragged_shapes():
    """The ragged-shape parity cases of every kernel family through the checked library:
    results within the tolerances, and no index outside its array."""
    sel = ("matvec_small or extremes or offset_binary or single_expert or gate_up_silu or route or rowmap or "
           "moe_small_full or tensor_core or nonfinite or stays_in_bounds or stay_in_bounds or quantize or "
           "dequant or matvec_rows or general_group or mla")
    r = _child(["-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "gpu", "-k", sel,
                "tests/test_gpu_parity.py", "tests/test_gpu_next.py", "tests/test_gpu_guards.py"], 1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout
