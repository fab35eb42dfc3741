"""The index-checked build (libtra_check.so, compiled with TRA_CHECK) on the
parity tests of the kernels whose indices it checks: the permutes (up to the
largest accepted N), the radius kernels, the mask kernels and the whole chain
on ragged and degenerate grids.  The kernels compare every index they derive
from the tile-major layout or from data they read with its extent, record an
index outside it in the device error word and skip the access; the tests
assert that the error word stays clear and that every result still matches
the oracle.  They run in a child process that loads the checked build."""
import os
import subprocess
import sys

import pytest

from entropy_adaptive_radius_b200 import build as tra_build
from entropy_adaptive_radius_b200 import tra
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUBSET = [
    "tests/test_gpu_a_layout.py",
    "tests/test_gpu_b_mask.py",
    "tests/test_gpu_d_variants.py",
    "tests/test_gpu_j_max_size.py::test_permute_at_the_largest_size",
    "tests/test_gpu_k_chain.py::test_chain_mid_size_every_element",
    "tests/test_gpu_n_edges.py",
]


def test_checked_build_passes_the_index_heavy_parity_tests():
    need_gpu()
    if not os.path.exists(tra.CHECK_LIB_PATH):
        tra_build.build(quiet=True, check=True)
    env = dict(os.environ, TRA_LIBRARY=tra.CHECK_LIB_PATH)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider"] + SUBSET,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
