"""The contractions at both N-tile widths (256 and 128 columns), on one CTA per tile
and on CTA pairs (256-row tiles), on the ragged parity shapes: the library picks the
width per launch from a wave-count model and the tile shape from a default, so each
combination is forced here once through EQAT_GEMM_BN / EQAT_GEMM_PAIR in a fresh
process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("pair", ["0", "1"])
@pytest.mark.parametrize("bn", ["256", "128"])
def test_parity_at_forced_tile_width(bn, pair):
    env = dict(os.environ, EQAT_GEMM_BN=bn, EQAT_GEMM_PAIR=pair)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_parity.py"), "-m", "gpu",
                        "-k", "fq_linear_bf16 or dq_linear_bf16 or reuses or single_contraction or wrap"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
