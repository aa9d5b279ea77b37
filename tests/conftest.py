import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


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


def pytest_terminal_summary(terminalreporter):
    """Pooled excused-mismatch counts of the GPU parity tests run here."""
    mod = sys.modules.get("tests.parity")
    if mod is None or not getattr(mod, "SUMMARY", None):
        return
    terminalreporter.section("parity: excused mismatches (oracle margin < 1e-5) per test")
    tot_d = tot_e = 0
    for name, t in mod.SUMMARY.items():
        tot_d += t["decisions"]
        tot_e += t["excused"]
        kinds = ", ".join(f"{k} {v[1]}/{v[0]}" for k, v in sorted(t["by_kind"].items()))
        terminalreporter.write_line(f"{name}: {t['excused']}/{t['decisions']} "
                                    f"({100.0 * t['excused'] / max(1, t['decisions']):.4f}%); {kinds}")
    terminalreporter.write_line(f"all: {tot_e}/{tot_d} ({100.0 * tot_e / max(1, tot_d):.4f}%)")
