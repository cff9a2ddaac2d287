import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))
for _p in (ROOT, TESTS):
    if _p not in sys.path:
        sys.path.insert(0, _p)


def pytest_sessionstart(session):
    # Bring the CUDA library and the CPU oracle up to date with their sources
    # (make does nothing when they are current).  nvcc cross-compiles for
    # sm_100a without a GPU, so this works on CPU-only machines too.
    import shutil
    import subprocess
    if shutil.which("make") is None:
        return
    for d in (os.path.join(ROOT, "engram_conditional_memory_hash_b200", "csrc"), os.path.join(ROOT, "oracle")):
        r = subprocess.run(["make", "-s", "-C", d], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"building {d} failed:\n{r.stdout}\n{r.stderr}")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case, minutes of CPU time")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.default()


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="needs a CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
