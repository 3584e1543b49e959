"""Shared test configuration.

Tests marked ``gpu`` need a CUDA device and the built ``libna2d.so``; the
driver runs them with ``-m gpu`` on a B200 and everything else with
``-m "not gpu"`` on a CPU-only box.
"""
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parent.parent
for p in (str(ROOT), str(Path(__file__).resolve().parent)):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libna2d.so")
