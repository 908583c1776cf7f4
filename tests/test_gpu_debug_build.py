"""The HEAL_DEBUG build (libheal_debug.so): the same kernels with every global store index
they compute checked on the device -- the stand-in for a memory checker, which is not
available on this pool.  A violation would be reported by heal_get_device_status() as
HEAL_ERR_INVALID_ARGUMENT instead of faulting.

The cases (tests/debug_build_cases.py, run in a process of its own because the library is
chosen per process) cover every GEMM tile configuration on ragged shapes, the split, the
KV writer at a cache offset and decode and prefill attention with the exact-S_int hook.
Each must leave the device status clean and match the oracle: GEMM within 1e-6 normwise
and bit-identical across configurations, split and KV codes bit-exact, S_int exact.
"""
import json
import os
import subprocess
import sys

import pytest

import error_compensated_gemm_b200._binding as B

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_build_runs_clean_and_matches_the_oracle():
    assert os.path.exists(B.DEBUG_LIB_PATH), "build libheal_debug.so first (build(debug=True))"
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_build_cases.py")], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    bad = {k: v for k, v in res.items() if not v["ok"]}
    assert not bad, bad
    assert len(res) >= 30
