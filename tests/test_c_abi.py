"""The C ABI from a C program: include/ulysses.h must compile as C11 with
-Wall -Wextra -pedantic -Werror and libulysses.so must link; the program
(tests/c/abi_from_c.c) then checks the host-side calls.  The refusal checks
pass null or fake device addresses, so they run only where no GPU is present
(a check that wrongly let one through must not reach a real device)."""
import os
import shutil
import subprocess

import pytest
import torch

from conftest import ROOT

LIB_DIR = os.path.join(ROOT, "ulysses_head_attention_b200")
SRC = os.path.join(ROOT, "tests", "c", "abi_from_c.c")


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler on this host")
    if not os.path.exists(os.path.join(LIB_DIR, "libulysses.so")):
        pytest.fail("libulysses.so is missing: build it with `python ulysses_head_attention_b200/build.py`")
    exe = str(tmp_path_factory.mktemp("c_abi") / "abi_from_c")
    cmd = [cc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"), SRC,
           "-L", LIB_DIR, "-lulysses", f"-Wl,-rpath,{LIB_DIR}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_header_compiles_as_c_and_queries_answer(program):
    r = subprocess.run([program], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"


@pytest.mark.skipif(torch.cuda.is_available(), reason="fake-pointer checks run only without a GPU")
def test_bad_arguments_are_refused_from_c(program):
    r = subprocess.run([program, "--refusals"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
