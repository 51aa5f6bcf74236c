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


# ---- the single-pass quantizers' bounded grid-wide exchange ----------------------------------

def _ws():
    lib = L.load()
    n = lib.nvfp4_workspace_bytes(L.NVFP4_OP_QUANTIZE, 1, 0, 32)
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    # arbitrary contents: the exchange needs no clearing
    return torch.randint(0, 256, (n,), dtype=torch.uint8, device="cuda", generator=g)


def _exchange(vals, ws, skip=-1, late=-1, late_ns=0, limit=1 << 21, out=None):
    lib = L.load()
    v = vals if isinstance(vals, torch.Tensor) else torch.tensor(vals, dtype=torch.float32,
                                                                 device="cuda")
    if out is None:
        out = torch.full((2,), -1.0, dtype=torch.float32, device="cuda")
    st = lib.nvfp4_selftest_grid_exchange(v.numel(), v.data_ptr(), skip, late, late_ns, limit,
                                          out.data_ptr(), ws.data_ptr(), ws.numel(),
                                          torch.cuda.current_stream().cuda_stream or None)
    return st, out


def test_grid_exchange_all_arrive():
    ws = _ws()
    n = torch.cuda.get_device_properties(0).multi_processor_count
    for vals in (np.arange(1, n + 1, dtype=np.float32), np.full(n, 3.5, np.float32)):
        st, out = _exchange(vals.tolist(), ws)
        assert st == L.NVFP4_OK
        assert nv.sync_status() == 0
        assert out.cpu().tolist() == [float(vals.max()), float(vals.max()) / 2]


def test_grid_exchange_missing_cta_times_out():
    # CTA 5 never arrives; its slot still holds the previous launch's token, which must not
    # count: the others give up after 64 poll rounds, report a timeout and return
    ws = _ws()
    n = 148
    st, out = _exchange([1.0] * n, ws)
    assert st == L.NVFP4_OK and nv.sync_status() == 0
    st, out = _exchange([2.0] * n, ws, skip=5, limit=64)
    assert st == L.NVFP4_OK
    assert nv.sync_status() == L.NVFP4_ERR_TIMEOUT
    assert out.cpu().tolist() == [-1.0, -1.0]
    assert nv.sync_status() == 0
    x = W.to_bf16_bits(W.normal((64, 256), 1.0, 34, 1))  # the context keeps working
    assert_quant_equal(gpu_quantize(x), O.quantize(x))


def test_grid_exchange_waits_for_a_late_cta():
    # the largest value sits in a CTA that arrives 0.2 ms late; consecutive launches in the
    # same workspace, with different values, each get their own maxima
    ws = _ws()
    n = 148
    for big in (1000.0, 500.0, 750.0):
        vals = [1.0] * n
        vals[n - 1] = big
        st, out = _exchange(vals, ws, late=n - 1, late_ns=200_000)
        assert st == L.NVFP4_OK
        assert nv.sync_status() == 0
        assert out.cpu().tolist() == [big, big / 2]


def test_grid_exchange_in_graph_replays():
    # a captured exchange replayed with new values each time: every replay is a new launch
    # with its own token, so the slots of the previous replay never satisfy the next one
    ws = _ws()
    n = 148
    vals = torch.ones(n, dtype=torch.float32, device="cuda")
    out = torch.full((2,), -1.0, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        _exchange(vals, ws, late=n - 1, late_ns=200_000, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _exchange(vals, ws, late=n - 1, late_ns=200_000, out=out)
    for big in (900.0, 300.0, 600.0):
        vals.fill_(1.0)
        vals[n - 1] = big
        g.replay()
        torch.cuda.synchronize()
        assert out.cpu().tolist() == [big, big / 2]
    assert nv.sync_status() == 0
    del g


def test_quantizers_on_two_streams_at_once():
    # single-pass quantizers (X1-sized, fused) and streamed ones (X2-sized) launched on two
    # streams without ordering between them: each stream has its own grid barrier and its own
    # workspace, so every result equals the one-at-a-time result
    xs = [W.to_bf16_bits(W.normal((4096, 3072), 1.0, 90, 1)),
          W.to_bf16_bits(W.normal((4096, 3072), 3.0, 90, 2)),
          W.to_bf16_bits(W.normal((4096, 12288), 1.0, 90, 3)),
          W.to_bf16_bits(W.normal((4096, 12288), 0.5, 90, 4))]
    dx = [torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16) for x in xs]
    ref = [nv.quantize(x) for x in dx]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [nv.quantize(x) for x in dx]
    for _ in range(3):
        torch.cuda.synchronize()
        for o in outs:
            o.codes.zero_()
            o.scales_swz.zero_()
        torch.cuda.synchronize()
        for i, x in enumerate(dx):
            with torch.cuda.stream(streams[i % 2]):
                nv.quantize(x, out=outs[i])
        torch.cuda.synchronize()
        assert nv.sync_status() == 0
        for o, r in zip(outs, ref):
            assert torch.equal(o.codes, r.codes)
            assert torch.equal(o.scales_swz, r.scales_swz)
            assert torch.equal(o.global_scale, r.global_scale)
