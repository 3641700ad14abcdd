"""The checked build (libqt2_checked.so, QT2_CHECKED): every kernel store is first checked
against the output array the call was given.  Its self-test records QT2_ERR_BOUNDS (one store
against a stated extent shorter than its array: the store is skipped, nothing leaves the
array), the product build's self-test records nothing (it has no checks), and the parity suites
of every producer and of the GEMMs pass bit for bit with the checked library loaded -- no
store of theirs leaves its array, and every status word stays clear."""
import os
import subprocess
import sys

import pytest

from nvfp4_quantized_b200 import build as qbuild
from nvfp4_quantized_b200 import qt2

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _checked_env():
    qbuild.build(checked=True)
    env = dict(os.environ)
    env["QT2_LIBRARY"] = "checked"
    return env


def test_product_build_has_no_checks():
    assert not qt2.qt2_build_checked()
    qt2.qt2_selftest_bounds()
    assert qt2.qt2_device_status() == 0


def test_checked_self_test_reports_a_skipped_store():
    code = (
        "from nvfp4_quantized_b200 import qt2\n"
        "assert qt2.LIB_PATH.endswith('libqt2_checked.so') and qt2.qt2_build_checked()\n"
        "assert qt2.qt2_device_status() == 0\n"
        "qt2.qt2_selftest_bounds()\n"
        "assert qt2.qt2_device_status() == qt2.QT2_ERR_BOUNDS\n"
        "assert qt2.qt2_device_status() == 0\n"
        "print('ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=_checked_env(), capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


def test_parity_suites_pass_under_the_checked_build():
    files = ["tests/test_gpu_quant.py", "tests/test_gpu_gemm.py", "tests/test_gpu_sr.py", "tests/test_gpu_fused.py",
             "tests/test_gpu_sq.py", "tests/test_gpu_local.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=_checked_env(), capture_output=True, text=True, timeout=3000)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
