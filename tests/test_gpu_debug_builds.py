"""The debugging aids: EP_CHECKED and EP_DEBUG.

EP_CHECKED=1 loads libep_b200_checked.so, the same kernels with device-side
invariant checks that set EP_DEVERR_CHECK instead of trapping.  On correct
inputs no check may fire and every output must still equal the oracle's.
EP_DEBUG=1 prints every launch's configuration to stderr.  Both run in a
child process, since the library is chosen when it is first loaded."""

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import numpy as np, torch
import oracle, workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import assert_parity, run_cuda, run_cuda_one_call, run_oracle
print("LIB", ep.library_path())
for name, one in (("mid", False), ("mid", True), ("decode", True), ("tiny", False)):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=41)
    y = W.make_y(w, seed=41)
    mode = ep.EP_X_BF16 if w.x_mode == "bf16" else ep.EP_X_BF16_TO_FP8
    g = run_cuda_one_call(inp, w, mode) if one else run_cuda(inp, w, y, mode)
    o = run_oracle(inp, w, None if one else y, mode)
    assert_parity(g, o, mode)
    assert g["handle"].check_error() == 0
print("CHILD_OK")
'''


def _child(env_extra):
    env = dict(os.environ, PYTHONPATH=ROOT, **env_extra)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=900)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_checked_build_matches_oracle_and_no_check_fires():
    r = _child({"EP_CHECKED": "1"})
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "libep_b200_checked.so" in r.stdout and "CHILD_OK" in r.stdout


def test_debug_prints_each_launch():
    r = _child({"EP_DEBUG": "1"})
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    # mid: the layout grids and the warp-unit dispatch; decode one-call: the
    # one-kernel layout + dispatch; tiny two-call: the one-CTA layout and
    # the row-path dispatch
    for kernel in ("layout_count_kernel", "layout_assign_kernel", "layout_single_kernel", "dispatch_kernel",
                   "dispatch_row_kernel(layout)", "dispatch_row_kernel", "combine_kernel"):
        assert f"[ep] {kernel}<" in r.stderr, kernel
