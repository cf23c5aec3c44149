"""Failure detection on the GPU without a GPU fault, through the bounds-checked
build of the library (libwkv4_checked.so: every global index checked against
its buffer, an index outside it skipped and recorded in the device error
word; fault switches read from the environment), each case in a child
process of its own (tests/failure_child.py):

* the checked build on valid shapes of every entry point records nothing and
  matches the oracle;
* host-side fault injection (WKV4_FAULT=launch:N): the N-th launch is made
  with an empty grid, which the runtime rejects without running anything; the
  call returns WKV4_ERR_CUDA and every other call succeeds;
* the forward from host buffers whose second chunk's launch is made to fail
  returns WKV4_ERR_CUDA with its queued copies joined into the caller's
  stream, and the same call repeated is correct;
* a bounded device wait that runs out (WKV4_FAULT=exchange, a short limit):
  no scan CTA pushes its segment aggregate, on a shape of one channel tile and
  one round, so that no copy and no DSMEM store is in flight when the waits
  give up; the kernel records WKV4_ERR_TIMEOUT and returns, and the next call
  runs correctly in the same context.
"""

import os
import subprocess
import sys

import pytest

from rwkv_wkv_linear_b200 import _build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _child(*args, **env):
    e = dict(os.environ)
    e.pop("WKV4_FAULT", None)
    e.pop("WKV4_WAIT_ROUNDS", None)
    e["WKV4_LIB"] = _build.CHECKED_LIB
    e.update(env)
    r = subprocess.run([sys.executable, "-m", "tests.failure_child", *args], cwd=ROOT, env=e,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-3000:] + r.stderr[-3000:]


@pytest.fixture(scope="module")
def checked_lib(cuda_device):
    if not os.path.exists(_build.CHECKED_LIB):
        pytest.fail(f"{_build.CHECKED_LIB} is missing: run __graft_entry__.build()")
    return _build.CHECKED_LIB


def test_checked_build_records_nothing_on_valid_shapes(checked_lib):
    _child("clean")


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 6])
def test_injected_launch_failure(checked_lib, n):
    _child("launch", str(n), WKV4_FAULT=f"launch:{n}")


def test_host_forward_launch_failure(checked_lib):
    _child("host", WKV4_FAULT="launch:2")


def test_exchange_wait_runs_out(checked_lib):
    _child("exchange", WKV4_FAULT="exchange", WKV4_WAIT_ROUNDS="20")
