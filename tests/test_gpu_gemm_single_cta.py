"""The GEMM parity tests again with the one-CTA-per-tile kernel
(TP_GEMM_CTA_PAIR=1) instead of the default CTA-pair (cta_group::2) kernel,
in a subprocess so the choice is made before the library's first launch."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_gemm_suite_with_single_cta_tiles():
    env = dict(os.environ, TP_GEMM_CTA_PAIR="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_gemm.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
