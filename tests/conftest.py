"""Shared test set-up: the ``gpu`` marker, the repo on ``sys.path`` and the
golden-fixture reader."""
import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200)")


def golden_lines(name):
    """Non-comment lines of a golden fixture."""
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


@pytest.fixture(scope="session")
def golden():
    return golden_lines


PICKER_HEADER = os.path.join(ROOT, "ring_all_reduce_virtual_b200", "csrc", "rr_picker_table.h")


def picker_table():
    """The picker's generated table: (header text, [(nranks, log2 bytes,
    alignment class, algo, margin)], the sweep record it was generated from)."""
    text = open(PICKER_HEADER, encoding="utf-8").read()
    rows = [(int(a), int(b), int(c), d.lower(), float(e))
            for a, b, c, d, e in re.findall(r"\{(\d+), (\d+), (\d), RR_ALGO_(\w+), ([\d.]+)f\}", text)]
    src = re.search(r"from\n// (\S+);", text).group(1)
    return text, rows, src
