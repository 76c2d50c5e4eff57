"""The prefill indexer's first pass on the linear lower bound, at every size.

By default the first pass uses the linear bound u_t . Kp[j] - c_t only for
query tiles with at least a few hundred pooled-key tiles (long contexts), and
the exact score below that, so the small parity cases would not reach the
bound.  QSA_INDEX_LB_MIN_KT=0 makes every query tile take the bound; this
re-runs the small-shape parity tests (all rows, exact ties, head weights of
any sign, chunked prefill) and the wait-timeout test in that mode, in a child
process so the setting does not leak into other tests."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    "tests/test_gpu_parity.py::test_prefill_all_rows",
    "tests/test_gpu_parity.py::test_full_budget_is_dense_attention",
    "tests/test_gpu_parity.py::test_chunked_prefill_with_q_pos0",
    "tests/test_gpu_edge.py::test_exact_ties",
    "tests/test_gpu_edge.py::test_head_weights_of_any_sign",
    "tests/test_gpu_edge.py::test_chunked_prefill_equals_one_shot",
    "tests/test_gpu_failure.py",
]


def test_small_cases_with_the_bound_forced():
    env = dict(os.environ, QSA_INDEX_LB_MIN_KT="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *CASES], env=env, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout, r.stdout[-2000:]
