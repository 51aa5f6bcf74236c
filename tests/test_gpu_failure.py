"""Failure detection on the device without a GPU fault: a kernel whose bounded wait cannot
complete (an mbarrier nothing arrives on) gives up, records NVFP4_ERR_TIMEOUT in the library's
status word and returns; nvfp4_sync_status reports it once, and the context keeps working."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_14_b200 as nv
import oracle as O
from gpu_helpers import assert_quant_equal, gpu_quantize
from nvfp4_block_scaled_14_b200 import _lib as L
from nvfp4_block_scaled_14_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    nv.load()


def test_wait_timeout_is_reported_and_cleared():
    lib = L.load()
    assert nv.sync_status() == 0
    assert lib.nvfp4_selftest_wait_timeout(None) == L.NVFP4_OK
    assert lib.nvfp4_sync_status(None) == L.NVFP4_ERR_TIMEOUT
    assert lib.nvfp4_sync_status(None) == L.NVFP4_OK  # reported once, then cleared


def test_context_usable_after_timeout():
    lib = L.load()
    assert lib.nvfp4_selftest_wait_timeout(None) == L.NVFP4_OK
    assert lib.nvfp4_sync_status(None) == L.NVFP4_ERR_TIMEOUT
    x = W.to_bf16_bits(W.normal((64, 256), 1.0, 34, 0))
    assert_quant_equal(gpu_quantize(x), O.quantize(x))
    assert nv.sync_status() == 0


def test_timeout_reported_on_the_callers_stream():
    lib = L.load()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        assert lib.nvfp4_selftest_wait_timeout(s.cuda_stream) == L.NVFP4_OK
    assert lib.nvfp4_sync_status(s.cuda_stream) == L.NVFP4_ERR_TIMEOUT
    assert np.int32(lib.nvfp4_sync_status(s.cuda_stream)) == 0
