import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch

        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    """Writes the parity figures the GPU tests collected (near-tie counts, largest
    relative errors per test) to the JSON file DFLASH_PARITY_RECORD names."""
    path = os.environ.get("DFLASH_PARITY_RECORD")
    if not path:
        return
    mod = sys.modules.get("tests.gpu_common")
    rec = getattr(mod, "RECORD", None) if mod else None
    if not rec:
        return
    import json

    with open(path, "w") as f:
        json.dump({"exitstatus": int(exitstatus), "tests": rec}, f, indent=1, sort_keys=True)
        f.write("\n")
