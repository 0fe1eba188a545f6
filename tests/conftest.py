import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The worst forward-output errors of the GPU parity tests in this run: the raw
    max |O - O_ref| next to the gated value the tests bound by 1e-2."""
    mod = sys.modules.get("gpu_util")
    rec = getattr(mod, "O_RECORD", None) if mod else None
    if rec and rec.get("n"):
        terminalreporter.write_line(
            f"O parity over {rec['n']} compared elements: raw max |O - O_ref| = {rec['raw']:.3e}, "
            f"gated (plain below |O_ref| = 2, beyond half a bf16 ulp above) = {rec['gate']:.3e}")
