import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a device; skip them cleanly when there is none
    # so that `-m "not gpu"` and an unfiltered run on a CPU machine both pass.
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
    """Achieved parity margins of every comparison run in this session."""
    try:
        from gdla_testutil import MARGINS
    except Exception:  # pragma: no cover
        return
    if not MARGINS:
        return
    tr = terminalreporter
    tr.write_sep("-", f"parity margins ({len(MARGINS)} comparisons)")
    tr.write_line("dtype  max|e|      rms(e)/rms  max(|e|-2^-6|ref|)/rms  bound  case")
    for what, dt, err, rel_rms, rel_elem, bound in MARGINS:
        if dt == "fp32":
            tr.write_line(f"fp32   {err:.3e}   -           -                       {bound:.0e}  {what}")
        else:
            tr.write_line(f"bf16   {err:.3e}   {rel_rms:.3e}   {rel_elem:+.3e}              {bound:.3g}   {what}")
