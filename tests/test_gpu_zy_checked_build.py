"""The checked build: libck_checked.so is the library compiled with its
device-side index checks (global stores and loads inside their tensor's rows
and columns, shared-memory accesses and bulk copies inside the CTA's
allocation, TMEM columns inside the allocation). A failed check skips the
access and sets a class bit instead of trapping. The quick parity suite must
pass against the oracle under it with no check failing (the conftest fixture
reads the bits after every test). compute-sanitizer is not available, so
this build and the guard bands of the parity tests stand in for it."""
import os
import re
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.path.join(ROOT, "int8_quantized_linear_convrot256_b200", "libck_checked.so")


@pytest.mark.gpu
def test_quick_parity_suite_under_the_checked_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert os.path.exists(CHECKED), "libck_checked.so is missing (build.py --checked)"
    env = dict(os.environ, CK_LIBRARY="libck_checked.so")
    cmd = [sys.executable, "-m", "pytest", "tests/test_gpu_parity.py", "tests/test_gpu_norm.py",
           "tests/test_gpu_nvfp4.py", "tests/test_zz_no_alloc.py", "-m", "gpu and not slow", "-x",
           "-q", "-p", "no:cacheprovider"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    m = re.search(r"(\d+) passed", r.stdout)
    assert m and int(m.group(1)) >= 100, r.stdout[-2000:]
    print(f"checked build: {m.group(1)} parity tests passed, no failed index check")


_FIRE = """
import int8_quantized_linear_convrot256_b200 as ck, torch
assert ck.is_checked_build()
assert ck.checked_violations() == 0
ck.test_checked_fire()
assert ck.checked_violations() == 4, "the failed check was not recorded"
assert ck.checked_violations() == 0, "the word was not cleared"
print("fire ok")
"""


@pytest.mark.gpu
def test_a_failed_check_is_recorded_and_cleared():
    """The mechanism itself: a check that fails on purpose (no access behind
    it) sets its class bit, which the next read returns and clears; the
    normal library ignores it."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert os.path.exists(CHECKED), "libck_checked.so is missing (build.py --checked)"
    env = dict(os.environ, CK_LIBRARY="libck_checked.so")
    r = subprocess.run([sys.executable, "-c", _FIRE], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "fire ok" in r.stdout, r.stdout + r.stderr
    import int8_quantized_linear_convrot256_b200 as ck

    if not ck.is_checked_build():
        ck.test_checked_fire()
        assert ck.checked_violations() == 0
