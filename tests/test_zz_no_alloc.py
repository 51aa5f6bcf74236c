"""nvfp4_linear_noalloc: the linear layer for callers that cannot allocate device memory (an
engine or plugin host that owns all device memory, latency-critical loops that forbid an
allocation, callers with no buffer to lend). Its split-K partial sums go to a fixed 4 MiB
array inside the library instead of a caller workspace.

Checked through the C ABI against nvfp4_linear (which takes a caller workspace) on the same
quantized operands, on two calls in a row, within the GEMM tolerance of the other tests.
This file is collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_14_b200 as nv
from gpu_helpers import gemm_tolerance, to_numpy_f64
from nvfp4_block_scaled_14_b200 import _lib as L
from nvfp4_block_scaled_14_b200 import workloads as W

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    nv.load()


def _operands(M, N, K, seed):
    a = torch.from_numpy(W.to_bf16_bits(W.normal((M, K), 1.0, 60, seed)).view(np.int16)) \
        .cuda().view(torch.bfloat16)
    w = torch.from_numpy(W.to_bf16_bits(W.normal((N, K), 0.02, 61, seed)).view(np.int16)) \
        .cuda().view(torch.bfloat16)
    return nv.quantize(a), nv.quantize(w)


def _call_noalloc(qa, qw, M, N, K, y):
    lib = L.load()
    stream = torch.cuda.current_stream().cuda_stream
    return lib.nvfp4_linear_noalloc(
        qa.codes.data_ptr(), qa.scales_swz.data_ptr(), qa.global_scale.data_ptr(),
        qw.codes.data_ptr(), qw.scales_swz.data_ptr(), qw.global_scale.data_ptr(),
        M, N, K, L.NVFP4_BF16, y.data_ptr(), stream or None)


@pytest.mark.parametrize("M,N,K", [(256, 256, 2048), (8, 1024, 4096), (1, 384, 2048),
                                   (64, 512, 1024), (8, 12288, 4096)])
def test_noalloc_matches_linear_on_two_calls(M, N, K):
    lib = L.load()
    need = lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, M, N, K)
    assert need <= SCRATCH_BYTES
    qa, qw = _operands(M, N, K, M + N)
    ref = to_numpy_f64(nv.linear(qa, qw))  # the existing entry point, caller workspace
    tol = gemm_tolerance(ref, True)
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(qa, qw, M, N, K, y) == L.NVFP4_OK
        torch.cuda.synchronize()
        got = to_numpy_f64(y)
        assert np.all(np.abs(got - ref) <= tol), f"call {call}: max err {np.abs(got - ref).max()}"
    assert nv.sync_status() == 0


def test_noalloc_uses_the_scratch_for_split_k():
    # the first shape above splits K across CTAs, so its partial sums really go to the array
    lib = L.load()
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, 256, 256, 2048) > 0


def test_noalloc_rejects_shapes_beyond_the_scratch():
    lib = L.load()
    M, N, K = 300, 520, 1056  # split-K partials of this plan need more than 4 MiB
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, M, N, K) > SCRATCH_BYTES
    qa, qw = _operands(M, N, K, 7)
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(qa, qw, M, N, K, y) == L.NVFP4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not y.float().abs().sum().item()  # rejected before any launch
