import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RUN_OUTPUT_DIR = "gpurun_out"   # the folder a GPU run brings back
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


@pytest.fixture(scope="session")
def tpa():
    """The CUDA binding; GPU tests only.  Fails loudly if the library is missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test collected on a machine without a CUDA device")
    from tensor_product_attention_b200 import binding
    return binding


def pytest_sessionfinish(session, exitstatus):
    """Write the parity errors the GPU tests measured (max|gpu - oracle| / max|oracle| per
    output tensor) as JSON: to $TPA_PARITY_LOG, else to parity_errors.json in the run-output
    folder at the repository root when that folder exists.  The worst error per test shows
    the headroom against 1e-2 / 1e-5."""
    import json
    from helpers import RECORDED
    if not RECORDED:
        return
    path = os.environ.get("TPA_PARITY_LOG")
    if not path:
        out = os.path.join(ROOT, RUN_OUTPUT_DIR)
        if not os.path.isdir(out):
            return
        path = os.path.join(out, "parity_errors.json")
    worst = {}
    for r in RECORDED:
        w = worst.setdefault(r["test"], {"worst_err": 0.0, "checks": 0})
        w["worst_err"] = max(w["worst_err"], r["err"])
        w["checks"] += 1
    with open(path, "w") as f:
        json.dump({"per_test": worst, "all": RECORDED}, f, indent=1)
