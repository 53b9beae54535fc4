import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def read_golden(name):
    """Non-comment lines of a golden fixture, split into tokens."""
    rows = []
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session", autouse=True)
def _built_cpu_libs():
    import oracle
    import synthgen
    oracle.build()
    synthgen.build()
    yield


def pytest_sessionfinish(session, exitstatus):
    """When the session ran against the bounds-checked build (NTX_LIB naming
    libntx_check.so), every index check of every kernel the tests launched
    must have passed: a recorded failure fails the session."""
    ntx = sys.modules.get("quantized_weight_gemv_dequant_b200")
    if ntx is None or getattr(ntx, "_lib", None) is None:
        return
    try:
        import torch
        if not torch.cuda.is_available() or ntx.ntx_check_enabled() != 1:
            return
        site, index = ntx.ntx_check_report()
    except Exception as e:  # pragma: no cover
        print(f"\nbounds-check report unavailable: {e}")
        session.exitstatus = 1
        return
    if site != 0:
        print(f"\nbounds check failed: site {site}, index {index}")
        session.exitstatus = 1
    else:
        print("\nbounds-checked build: every index check passed")
