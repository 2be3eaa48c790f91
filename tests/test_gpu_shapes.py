"""Every grouped-GEMM shape against the oracle, not only the default ones.

The library picks its decode and prefill shapes once per process (from
W4A8_GEMM_DECODE_SHAPE / W4A8_GEMM_PREFILL_SHAPE / W4A8_SPLIT_TILES), so each
forced choice runs the forward parity cases of test_gpu_forward.py in a child
process.  The
cases mix both regimes (few and many tokens per expert), ragged tiles, empty
experts and several K groups per tile.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CASES = ("tiny_workload or ragged or multi_block_segments or zipf_empty or outliers_wide "
         "or decode_shape_multi_block or zero_token_row")


@pytest.mark.parametrize("var,shape", [
    ("W4A8_GEMM_DECODE_SHAPE", 1), ("W4A8_GEMM_DECODE_SHAPE", 2),
    ("W4A8_GEMM_DECODE_SHAPE", 3), ("W4A8_GEMM_DECODE_SHAPE", 4),
    ("W4A8_GEMM_DECODE_SHAPE", 5), ("W4A8_GEMM_DECODE_SHAPE", 6),
    ("W4A8_GEMM_PREFILL_SHAPE", 1), ("W4A8_GEMM_PREFILL_SHAPE", 2),
    ("W4A8_GEMM_PREFILL_SHAPE", 3), ("W4A8_GEMM_PREFILL_SHAPE", 4),
    # split tiling forced on for every batch (32-row tiles for experts with up
    # to 32 rows, 128-row tiles above) and off for every batch
    ("W4A8_SPLIT_TILES", 1), ("W4A8_SPLIT_TILES", 0),
], ids=lambda v: str(v))
def test_forward_parity_with_forced_shape(var, shape):
    env = dict(os.environ, **{var: str(shape)})
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p",
                        "no:cacheprovider", os.path.join(HERE, "test_gpu_forward.py"),
                        "-k", CASES],
                       env=env, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-15:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
