"""Host checks of the GPU tests' sampling helpers (no GPU)."""
import numpy as np

from gpu_helpers import boundary_rows


def test_boundary_rows_cover_partial_and_full_tiles():
    # host check of the sampler: a 300-row segment has 128-row tiles [0, 128),
    # [128, 256) and the partial [256, 300); 32-row tiles up to [288, 300)
    offsets = np.array([0, 5, 305, 310], dtype=np.int32)
    r = set(boundary_rows(offsets, n_segments=1).tolist())
    for lo, hi in ((0, 127), (128, 255), (256, 299), (0, 31), (288, 299), (256, 287)):
        assert 5 + lo in r and 5 + hi in r, (lo, hi)
