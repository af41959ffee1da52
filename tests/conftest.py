import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    """Per output-irrep-block parity of the GPU tests that recorded it: the worst block of each
    tensor, as max|err| / max|ref| of the tensor and of the block itself."""
    try:
        from gpu_util import BLOCK_RECORDS
    except Exception:  # noqa: BLE001
        return
    if not BLOCK_RECORDS:
        return
    tr = terminalreporter
    tr.section("parity per irreps block (max|err| / max|ref|: of the tensor, of the block)")
    by = {}
    for name, lab, a, b in BLOCK_RECORDS:
        by.setdefault(name, []).append((lab, a, b))
    for name, rows in by.items():
        cells = ", ".join(f"{lab} {a:.1e}/{b:.1e}" for lab, a, b in rows)
        tr.write_line(f"{name}: {cells}")
