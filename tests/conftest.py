"""Shared pytest setup: repo root on sys.path and the ``gpu`` marker.

Tests marked ``gpu`` need a CUDA device (a B200) and the built ``libafd_ffn.so``; all other
tests run on the CPU and cover the oracle, its pins, the host-side logic and that the
C-ABI library loads and exports every declared symbol.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device and the built CUDA library")
