import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built libmx.so")
    config.addinivalue_line("markers", "slow: long-running full-size case")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) when no CUDA device is visible.
    try:
        import torch

        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(params=[0, 1], ids=["pair", "single"])
def gemm_variant(request):
    """Runs a GEMM test with the CTA-pair kernel (0, the default) and the single-CTA kernel (1)."""
    from mxfp8_block_scaled_07_b200 import mx

    mx.set_gemm_variant(request.param)
    yield request.param
    mx.set_gemm_variant(0)


@pytest.fixture(params=[0, 1, 2], ids=["regs", "tma", "split"])
def quant_variant(request):
    """Runs a quantizer test with the register-staged kernels (0, the default), the TMA-staged
    kernel (1) and the register-staged kernels with split loads for every rowwise call (2)."""
    from mxfp8_block_scaled_07_b200 import mx

    mx.set_quantize_variant(request.param)
    yield request.param
    mx.set_quantize_variant(0)


@pytest.fixture(params=[0, 1], ids=["pair", "single"])
def grouped_variant(request):
    """Runs a grouped-GEMM test with the CTA-pair kernel (0, the default) and the single-CTA
    kernel (1)."""
    from mxfp8_block_scaled_07_b200 import mx

    mx.set_gemm_variant(request.param)
    yield request.param
    mx.set_gemm_variant(0)
