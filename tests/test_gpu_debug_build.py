"""The bounds-checked debug build on the GPU.

libulysses_debug.so is the same library compiled with ULY_DEBUG_BOUNDS:
every global index and TMA tile coordinate of the kernels is checked before
the access; one outside its buffer is recorded (ULY_ERR_BOUNDS in the
attention workspaces' status word, or the re-layout kernels' own word read by
ulysses_debug_status) and the access skipped.  This test runs the parity
files of the re-layouts, the attention forward and backward and the block
kernels in a fresh process with ULYSSES_DEBUG=1: every comparison must pass
and no check may fire (the attention tests assert a clean status word, and
an autouse fixture reads the re-layout word after every test).
"""
import os
import subprocess
import sys

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu

FILES = ["tests/test_gpu_relayout.py", "tests/test_gpu_attn_fwd.py", "tests/test_gpu_attn_bwd.py",
         "tests/test_gpu_ring_blocks.py"]


def test_parity_suites_pass_under_the_debug_build(cuda_device):
    lib = os.path.join(ROOT, "ulysses_head_attention_b200", "libulysses_debug.so")
    assert os.path.exists(lib), "build it with `python ulysses_head_attention_b200/build.py --debug`"
    env = dict(os.environ, ULYSSES_DEBUG="1")
    r = subprocess.run([sys.executable, "-m", "pytest", *FILES, "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
