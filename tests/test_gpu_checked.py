"""The checked build (libstrata_moe_checked.so, compiled with -DSTRATA_CHECKED):
every index the kernels take from data is bounds-checked into the device
status word. Its layer calls must give the normal build's parity on the tiny
layer, a full-size decode layer and the prefill path at 300 tokens, with
strata_moe_check_status reporting no failed check (any failed check raises
in those tests); its bounds self-test must report the recorded index. The
library is chosen at import time, so the checked build runs in a child
process."""
import os
import subprocess
import sys

import pytest

from gpu_harness import S

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECKED = os.path.join(ROOT, "bit_quantized_moe_warp_b200", "libstrata_moe_checked.so")


def _child_env():
    env = dict(os.environ)
    env["STRATA_MOE_LIB"] = CHECKED
    return env


def test_checked_build_parity():
    assert os.path.exists(CHECKED), "build the checked library first (__graft_entry__.build())"
    sel = ("test_tiny_layer or test_decode_layer_full_size or test_prefill_path_full_size_small_T "
           "or test_verify_layer_full_size or test_generated_ties")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_layer.py"), "-k", sel],
                       cwd=ROOT, env=_child_env(), capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout


def test_bounds_selftest_normal_and_checked():
    lib = S()
    assert lib.strata_is_checked_build() == 0
    assert lib.strata_selftest_bounds_check() == lib.STRATA_OK
    code = ("import bit_quantized_moe_warp_b200 as S, torch; torch.cuda.set_device(0); "
            "print(S.strata_is_checked_build(), S.strata_selftest_bounds_check(), S.LIB_PATH)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=_child_env(), capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    checked, status, path = r.stdout.split()
    assert path == CHECKED
    assert int(checked) == 1 and int(status) == lib.STRATA_ERR_BOUNDS
