"""The bounds-checking build (libw4a8_debug.so, W4A8_LIBRARY=debug) on the GPU.

Its kernels check every routing-derived index before use (the expert
offsets and tile tables the grouped GEMM decodes, segment rows, token ids);
one out of range raises W4A8_ERR_DEVICE_INDEX at the next
w4a8_check_device_error and the access is skipped.  The forward,
expert-parallel and shared-expert parity cases run on it in a child process:
they must pass with no check firing (each test ends with
w4a8_check_device_error), and an
expert id outside [-1, E) given to w4a8_moe_forward_experts must be reported,
as must bad indices given to the all-to-all row gather and combine.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_parity_cases_on_the_bounds_checking_build():
    from w4a8_quantized_moe_b200 import build as b
    b.build(debug_bounds=True)
    env = dict(os.environ, W4A8_LIBRARY="debug")
    check = ("import w4a8_quantized_moe_b200 as w; "
             "assert w.LIB_PATH.endswith('libw4a8_debug.so'); "
             "assert w.w4a8_build_flags() == 1")
    r = subprocess.run([sys.executable, "-c", check], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p",
                        "no:cacheprovider", os.path.join(HERE, "test_gpu_forward.py"),
                        os.path.join(HERE, "test_gpu_ep.py"),
                        os.path.join(HERE, "test_gpu_shared.py"), "-k",
                        "tiny_workload or ragged or multi_block or zipf_empty or zero_token_row "
                        "or padding or route_topk or dispatch_plan or gather_and_combine "
                        "or bad_send_rows or shared_gemms_inside"],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
