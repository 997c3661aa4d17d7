"""Shared pytest configuration: the ``gpu`` marker is registered in pytest.ini.

GPU tests fail loudly (never skip) when CUDA or the compiled library is
missing, so a GPU run can never pass on a fallback path.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
