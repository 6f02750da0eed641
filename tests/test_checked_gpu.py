"""The checked build on a B200.  libgqadecode_checked.so tests the element
index of every global access the kernels derive (query rows, triplet slots,
merged rows, tickets, appended rows, prefill output rows) against the
extent the call's arguments give it, records a failure in the status word
and skips the access.  Its self-test makes one check fail on purpose (the
guarded store is skipped, nothing else runs); then the GPU parity suites
run under it and must record no failed check (the autouse fixture in
conftest.py reads the report after every test).  Each runs in its own
process, with GQA_DECODE_CHECKED=1 selecting the library."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, timeout):
    env = dict(os.environ, GQA_DECODE_CHECKED="1")
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=timeout)


def test_selftest_reports_a_failed_check():
    code = "\n".join([
        "import torch",
        "import gqa_split_kv_decode_b200 as gk",
        "assert torch.cuda.is_available() and gk.checked_build()",
        "assert gk.get_status() == 0 and gk.bounds_report() is None",
        "gk.selftest_bounds()",
        "assert gk.get_status() == gk.ERR_DEVICE_BOUNDS",
        "assert gk.bounds_report() == (7, 1)",   # site 7 (self-test), index 1 of extent 1
        "assert gk.bounds_report() is None and gk.get_status() == 0",
        "print('checked build self-test ok')",
    ])
    r = _run(["-c", code], 300)
    assert r.returncode == 0 and "self-test ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


def test_parity_suites_record_no_failed_check():
    suites = ["tests/test_parity_gpu.py", "tests/test_plans_gpu.py", "tests/test_append_gpu.py",
              "tests/test_prefill_gpu.py", "tests/test_sharded_gpu.py"]
    r = _run(["-m", "pytest", *suites, "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider"], 1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
