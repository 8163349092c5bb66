"""Shared pytest configuration.

Tests marked ``gpu`` need a CUDA device (parity of the CUDA path against the
oracle); everything else runs on CPU only.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
