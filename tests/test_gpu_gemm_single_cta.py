"""The GEMM parity tests again under each forced tile layout: one CTA per
128-row tile (TP_GEMM_CTA_PAIR=1) instead of CTA pairs, and 128-column tiles
everywhere (TP_GEMM_NARROW=1) with either pairing; under the static tile
schedule; and with every epilogue on the direct (row-per-thread) stores
instead of the TMA-staged ones (TP_GEMM_TMA_EPI=0); and with the backward
calls on one stream (TP_BWD_CONCURRENT=0). Each runs in a subprocess
so the choice is made before the library's first launch. The default run of
test_gpu_gemm.py lets the library choose per launch."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("pair,narrow,sched,tma,conc", [
    ("1", "0", "dynamic", "1", "1"), ("2", "0", "dynamic", "1", "1"), ("2", "1", "dynamic", "1", "1"),
    ("1", "1", "dynamic", "1", "1"), ("2", "0", "static", "1", "1"), ("2", "0", "dynamic", "0", "1"),
    ("1", "1", "dynamic", "0", "1"), ("2", "0", "dynamic", "1", "0")])
def test_gemm_suite_under_forced_layouts(pair, narrow, sched, tma, conc):
    """sched: tiles drawn from the launch's atomic counter (dynamic) or taken
    by a fixed stride per CTA pair (static); tma: TMA-staged epilogue where it
    applies (1) or direct stores everywhere (0); conc: the backward calls' dX /
    dH GEMM on the side stream beside small weight gradients (1) or every
    GEMM on the caller's stream (0)."""
    env = dict(os.environ, TP_GEMM_CTA_PAIR=pair, TP_GEMM_NARROW=narrow, TP_GEMM_SCHED=sched,
               TP_GEMM_TMA_EPI=tma, TP_BWD_CONCURRENT=conc)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_gemm.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
