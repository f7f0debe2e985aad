"""Test configuration: the ``gpu`` marker and import paths.

Tests marked ``gpu`` need a CUDA device and the built CUDA library; every
other test runs on the CPU.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running oracle checks")


def golden_facts():
    """Parse tests/golden/pcast_facts.txt into a dict of floats."""
    path = os.path.join(ROOT, "tests", "golden", "pcast_facts.txt")
    facts = {}
    with open(path) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (x.strip() for x in line.split("=", 1))
            facts[key] = float(val)
    return facts
