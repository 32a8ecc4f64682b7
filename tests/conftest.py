import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)

IQ1S_ANCHOR = 0.61  # the pages' flat IQ1_S anchor
IQ2XS_ANCHOR = 0.9  # fixed once by a seeded sweep on non-evaluation data (design notes)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: runs CUDA kernels on a GPU through the C-ABI library")


@pytest.fixture(scope="session")
def grids():
    from ggml_iq_codebook_b200 import synth
    return {"iq1_s": synth.iq1s_grid(), "iq2_xs": synth.iq2xs_grid(), "iq1_m": synth.iq1s_grid(),
            "iq2_s": synth.iq2s_grid()}


@pytest.fixture(scope="session")
def anchors():
    return {"iq1_s": IQ1S_ANCHOR, "iq2_xs": IQ2XS_ANCHOR, "iq1_m": 1.0, "iq2_s": IQ2XS_ANCHOR}
