import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "large: full-size workload parity (slow)")
    config.addinivalue_line("markers", "oracle_heavy: minutes of fp64 oracle work on the host (n = 131072 in full)")


def read_golden(name):
    """Parse a golden fixture: non-comment lines split into whitespace tokens."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device on this host")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """Every parity comparison's measured error, beside its bound."""
    mod = sys.modules.get("gpu_util")
    recs = getattr(mod, "RECORDS", None) if mod else None
    if not recs:
        return
    tr = terminalreporter
    tr.section("measured errors (max-abs <= bound, mean-rel <= bound)")
    for what, ma, mr, bma, bmr in recs:
        rel = "" if mr != mr else f"  mean-rel {mr:.2e} (<= {bmr:g})"
        tr.write_line(f"{what}: max-abs {ma:.2e} (<= {bma:g}){rel}")


@pytest.fixture(autouse=True)
def _debug_build_bounds_record(request):
    """Under the bounds-checked debug build (ULYSSES_DEBUG=1), every GPU test
    must also leave the re-layout kernels' bounds record clean."""
    yield
    mod = sys.modules.get("ulysses_head_attention_b200")
    if mod is None or not getattr(mod, "DEBUG_BUILD", False) or request.node.get_closest_marker("gpu") is None:
        return
    assert mod.ulysses_debug_status() == 0, "an index fell outside its buffer (debug build)"
