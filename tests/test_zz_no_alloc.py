"""nvfp4_linear_noalloc: the linear layer for callers that cannot allocate device memory (an
engine or plugin host that owns all device memory, latency-critical loops that forbid an
allocation, callers with no buffer to lend). Its split-K partial sums go to a fixed 4 MiB
array inside the library instead of a caller workspace.

Checked through the C ABI on two calls in a row: against nvfp4_linear (which takes a caller
workspace) on the same quantized operands -- bit for bit, since both run the same plan and the
same deterministic kernels -- and against the oracle's exact product within the GEMM tolerance
of the other tests. The second call uses other operands of the same shape, so a partial sum
left in the array by the first call cannot pass for its own. This file is collected last so
that a run stopping at the first failure has already run every other test; it also passes on
its own in a fresh process."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_14_b200 as nv
import oracle as O
from gpu_helpers import assert_gemm_close, to_numpy_f64
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
    """Quantized operands on the device and their oracle quantization."""
    xa = W.to_bf16_bits(W.normal((M, K), 1.0, 60, seed))
    xw = W.to_bf16_bits(W.normal((N, K), 0.02, 61, seed))
    a = torch.from_numpy(xa.view(np.int16)).cuda().view(torch.bfloat16)
    w = torch.from_numpy(xw.view(np.int16)).cuda().view(torch.bfloat16)
    return nv.quantize(a), nv.quantize(w), O.quantize(xa), O.quantize(xw)


def _call_noalloc(qa, qw, M, N, K, y):
    lib = L.load()
    stream = torch.cuda.current_stream().cuda_stream
    return lib.nvfp4_linear_noalloc(
        qa.codes.data_ptr(), qa.scales_swz.data_ptr(), qa.global_scale.data_ptr(),
        qw.codes.data_ptr(), qw.scales_swz.data_ptr(), qw.global_scale.data_ptr(),
        M, N, K, L.NVFP4_BF16, y.data_ptr(), stream or None)


# (256, 256, 2048) and (129, 256, 1024) split K across CTAs (their partial sums go through
# the array); the small-M shapes reduce their K split on chip and never touch it
@pytest.mark.parametrize("M,N,K", [(256, 256, 2048), (129, 256, 1024), (64, 512, 1024),
                                   (8, 1024, 4096), (1, 384, 2048), (8, 12288, 4096)])
def test_noalloc_matches_linear_and_oracle_on_two_calls(M, N, K):
    lib = L.load()
    need = lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, M, N, K)
    assert need <= SCRATCH_BYTES
    for call, seed in enumerate((M + N, M + N + 1)):
        qa, qw, ra, rw = _operands(M, N, K, seed)
        ref = to_numpy_f64(nv.linear(qa, qw))  # the existing entry point, caller workspace
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(qa, qw, M, N, K, y) == L.NVFP4_OK
        torch.cuda.synchronize()
        got = to_numpy_f64(y)
        assert np.array_equal(got, ref), f"call {call}: differs from nvfp4_linear"
        assert_gemm_close(got, O.gemm(ra, rw), True, what=f"call {call}")
    assert nv.sync_status() == 0


def test_noalloc_split_k_shapes_use_the_scratch():
    # the split-K shapes above need partial sums, so the array is what holds them
    lib = L.load()
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, 256, 256, 2048) > 0
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, 129, 256, 1024) > 0


def test_noalloc_at_the_size_limit():
    # 256 x 256 x 4096 splits K into 16 parts: 16 x 256 x 256 fp32 partials, exactly 4 MiB,
    # accepted (and correct); one more k-tile makes 17 parts, 4.25 MiB, rejected
    lib = L.load()
    M, N, K = 256, 256, 4096
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, M, N, K) == SCRATCH_BYTES
    qa, qw, ra, rw = _operands(M, N, K, 9)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(qa, qw, M, N, K, y) == L.NVFP4_OK
    torch.cuda.synchronize()
    got = to_numpy_f64(y)
    assert np.array_equal(got, to_numpy_f64(nv.linear(qa, qw)))
    assert_gemm_close(got, O.gemm(ra, rw), True, what="4 MiB of partials")
    K2 = K + 256
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, M, N, K2) > SCRATCH_BYTES
    qa, qw, _, _ = _operands(M, N, K2, 10)
    torch.cuda.synchronize()
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(qa, qw, M, N, K2, y) == L.NVFP4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all()


def test_noalloc_rejects_shapes_beyond_the_scratch():
    lib = L.load()
    M, N, K = 300, 520, 1056  # split-K partials of this plan need more than 4 MiB
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR, M, N, K) > SCRATCH_BYTES
    qa, qw, _, _ = _operands(M, N, K, 7)
    torch.cuda.synchronize()
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    before = y.view(torch.int16).clone()
    assert _call_noalloc(qa, qw, M, N, K, y) == L.NVFP4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), before)  # the NaN sentinel: nothing was launched
