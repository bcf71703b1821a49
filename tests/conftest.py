import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")

# Tolerances for the floating-point GEMM results (bf16 inputs, fp32 accumulate):
# relative Frobenius error and max-abs error relative to max |Y_ref|.
REL_FRO_TOL = 5e-3
MAX_ABS_REL_TOL = 1e-2
# SVID vectors: cosine similarity with the oracle's singular vectors.
SVID_COS_TOL = 0.9999


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture
def golden():
    return load_golden
