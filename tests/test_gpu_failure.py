"""Failure detection on the GPU without a GPU fault.

Every wait inside the warp-specialised indexer is bounded in wall-clock time;
QSA_DEBUG_WAIT_NS shrinks the bound so a test can make the waits run out on
purpose.  The kernel must then stop early, record QSA_ERR_TIMEOUT in the
workspace status word, free its tensor memory and leave the context usable.
Runs in a child process so the debug bound does not leak into other tests."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import torch
import block_sparse_long_10_b200 as qsa
from block_sparse_long_10_b200 import synth
w = synth.Workload("t", "prefill", 1, 4096, 16, 2, 128, 4, 64, 4, 2048, 3, 0)
x = synth.make_prefill(w, "cuda")
kp = torch.empty(1, 1024, 64, dtype=torch.bfloat16, device="cuda")
qsa.qsa_pool(x["k_idx"], kp, 4)
sel = torch.empty(1, 4096, 512, dtype=torch.int32, device="cuda")
ws = qsa.workspace(qsa.qsa_index_topk_workspace_size(1, 4096, 1024, 4, 64, 4, 2048))
qsa.qsa_index_topk(x["q_idx"], x["w"], kp, sel, ws, 4, 2048)
print("STATUS", qsa.qsa_check_device_status(ws), flush=True)
qsa.qsa_index_topk(x["q_idx"], x["w"], kp, sel, ws, 4, 2048)
torch.cuda.synchronize()
print("CONTEXT OK", flush=True)
'''


def _run(extra_env):
    env = dict(os.environ, **extra_env)
    return subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True,
                          text=True, timeout=300, cwd=ROOT)


def test_wait_bound_runs_out_and_is_reported():
    r = _run({"QSA_DEBUG_WAIT_NS": "0"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert "STATUS 6" in r.stdout, r.stdout
    assert "CONTEXT OK" in r.stdout


def test_default_bound_does_not_trigger():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    assert "STATUS 0" in r.stdout, r.stdout
