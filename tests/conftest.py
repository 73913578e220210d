import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (runs on the B200 box)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_sessionstart(session):
    # Build the in-tree CUDA library and the oracle if their sources changed.
    from binarized_convolution_b200 import build as _build

    _build.build()
    import oracle

    oracle.build()


@pytest.fixture(autouse=True)
def _default_cta_mode():
    """Tests may force the tensor-core spread of the layers they create; put it back."""
    yield
    from binarized_convolution_b200 import _native

    if _native._lib is not None:
        _native.bconv_set_cta_mode(_native.CTA_AUTO)
        _native.bconv_set_tc_codes(_native.CODES_AUTO)
        _native.bconv_set_staging(_native.STAGING_AUTO)
