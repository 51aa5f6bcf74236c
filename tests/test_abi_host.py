"""Host-side checks of the C ABI (no GPU needed): the library builds and loads, exports every
function include/nvfp4.h declares, sizes the buffers correctly, and rejects bad arguments on
the host before touching the device."""
import ctypes

import pytest

from nvfp4_block_scaled_14_b200 import _lib as L


@pytest.fixture(scope="module")
def lib():
    return L.load()


def test_exports_every_declared_symbol(lib):
    names = L.declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L._SIGNATURES)


def test_status_strings(lib):
    for st in range(8):
        assert lib.nvfp4_status_str(st)
    assert lib.nvfp4_status_str(99) == b"unknown status"


def test_buffer_sizes(lib):
    assert lib.nvfp4_codes_bytes(4096, 3072) == 4096 * 1536
    assert lib.nvfp4_scales_bytes(4096, 3072, 0) == 4096 * 192
    assert lib.nvfp4_scales_bytes(4096, 3072, 1) == 4096 * 192
    # padding to 128-row x 4-block atoms
    assert lib.nvfp4_scales_bytes(1, 32, 1) == 512
    assert lib.nvfp4_scales_bytes(129, 96, 1) == 2 * 128 * 8
    # 4.5 bits per weight (codes + linear scales)
    assert (lib.nvfp4_codes_bytes(64, 256) + lib.nvfp4_scales_bytes(64, 256, 0)) * 8 == \
        64 * 256 * 4.5
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_QUANTIZE, 10, 0, 64) >= 4
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_CALIB_BF16, 0, 0, 0) > 0
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_CALIB_F32, 0, 0, 0) > \
        lib.nvfp4_workspace_bytes(L.NVFP4_OP_CALIB_BF16, 0, 0, 0)
    assert lib.nvfp4_workspace_bytes(99, 1, 1, 1) == 0


FAKE = 0x10000  # never dereferenced: every call below fails its host-side check first


def test_quantize_argument_checks(lib):
    q = lib.nvfp4_quantize
    ws = lib.nvfp4_workspace_bytes(L.NVFP4_OP_QUANTIZE, 8, 0, 64)
    # cols not a multiple of 32, negative rows
    assert q(FAKE, 1, 8, 48, None, FAKE, FAKE, None, FAKE, FAKE, ws, None) == L.NVFP4_ERR_SHAPE
    assert q(FAKE, 1, -1, 64, None, FAKE, FAKE, None, FAKE, FAKE, ws, None) == L.NVFP4_ERR_SHAPE
    assert q(FAKE, 1, 8, 1 << 31, None, FAKE, FAKE, None, FAKE, FAKE, ws, None) == \
        L.NVFP4_ERR_SHAPE
    # bad dtype, missing outputs
    assert q(FAKE, 7, 8, 64, None, FAKE, FAKE, None, FAKE, FAKE, ws, None) == \
        L.NVFP4_ERR_INVALID_ARG
    assert q(FAKE, 1, 8, 64, None, FAKE, None, None, FAKE, FAKE, ws, None) == \
        L.NVFP4_ERR_INVALID_ARG
    assert q(FAKE, 1, 8, 64, None, FAKE, FAKE, None, None, FAKE, ws, None) == \
        L.NVFP4_ERR_INVALID_ARG
    assert q(None, 1, 8, 64, None, FAKE, FAKE, None, FAKE, FAKE, ws, None) == \
        L.NVFP4_ERR_INVALID_ARG
    # misaligned input / codes
    assert q(FAKE + 8, 1, 8, 64, None, FAKE, FAKE, None, FAKE, FAKE, ws, None) == \
        L.NVFP4_ERR_ALIGNMENT
    assert q(FAKE, 1, 8, 64, None, FAKE + 4, FAKE, None, FAKE, FAKE, ws, None) == \
        L.NVFP4_ERR_ALIGNMENT
    # dynamic amax needs the workspace
    assert q(FAKE, 1, 8, 64, None, FAKE, FAKE, None, FAKE, None, 0, None) == \
        L.NVFP4_ERR_WORKSPACE
    assert q(FAKE, 1, 8, 64, None, FAKE, FAKE, None, FAKE, FAKE, ws - 4, None) == \
        L.NVFP4_ERR_WORKSPACE


def test_fp8_and_dequant_checks(lib):
    f = lib.nvfp4_quantize_fp8_src
    assert f(FAKE, FAKE + 2, 8, 64, None, FAKE, FAKE, None, FAKE, FAKE, 1 << 20, None) == \
        L.NVFP4_ERR_ALIGNMENT
    assert f(FAKE, None, 8, 40, None, FAKE, FAKE, None, FAKE, FAKE, 1 << 20, None) == \
        L.NVFP4_ERR_SHAPE
    d = lib.nvfp4_dequantize
    assert d(FAKE, FAKE, FAKE, 8, 48, 0, FAKE, None) == L.NVFP4_ERR_SHAPE
    assert d(FAKE, FAKE, FAKE, 8, 64, 5, FAKE, None) == L.NVFP4_ERR_INVALID_ARG
    assert d(None, FAKE, FAKE, 8, 64, 0, FAKE, None) == L.NVFP4_ERR_INVALID_ARG
    assert d(FAKE, FAKE, FAKE, 8, 64, 0, FAKE + 8, None) == L.NVFP4_ERR_ALIGNMENT
    # empty input is a no-op
    assert d(None, None, None, 0, 64, 0, None, None) == L.NVFP4_OK


def test_linear_and_calib_checks(lib):
    li = lib.nvfp4_linear
    args = [FAKE] * 6
    assert li(*args, 64, 64, 48, 1, FAKE, None, 0, None) == L.NVFP4_ERR_SHAPE
    assert li(*args, -1, 64, 64, 1, FAKE, None, 0, None) == L.NVFP4_ERR_SHAPE
    assert li(*args, 64, 64, 64, 3, FAKE, None, 0, None) == L.NVFP4_ERR_INVALID_ARG
    assert li(*args, 0, 64, 64, 1, None, None, 0, None) == L.NVFP4_OK  # empty output
    assert li(*args, 64, 64, 64, 1, None, None, 0, None) == L.NVFP4_ERR_INVALID_ARG
    c = lib.nvfp4_calib_percentile_amax
    one = (ctypes.c_void_p * 1)(FAKE)
    assert c(one, 1, 1024, 1, 1001, 1000, FAKE, FAKE, FAKE, 1 << 20, None) == \
        L.NVFP4_ERR_INVALID_ARG
    assert c(one, 1, 1024, 1, 0, 1000, FAKE, FAKE, FAKE, 1 << 20, None) == \
        L.NVFP4_ERR_INVALID_ARG
    assert c(one, 0, 1024, 1, 999, 1000, FAKE, FAKE, FAKE, 1 << 20, None) == \
        L.NVFP4_ERR_INVALID_ARG
    assert c(one, 1, 0, 1, 999, 1000, FAKE, FAKE, FAKE, 1 << 20, None) == L.NVFP4_ERR_SHAPE
    mis = (ctypes.c_void_p * 1)(FAKE + 2)
    assert c(mis, 1, 1024, 1, 999, 1000, FAKE, FAKE, FAKE, 1 << 20, None) == \
        L.NVFP4_ERR_ALIGNMENT
    assert c(one, 1, 1024, 1, 999, 1000, FAKE, FAKE, FAKE, 16, None) == L.NVFP4_ERR_WORKSPACE


def test_product_path_never_imports_oracle():
    import os
    import re
    pkg = os.path.dirname(L.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, re.M), f
                assert "nvfp4_oracle" not in text, f


def test_linear_lowrank_checks(lib):
    lr = lib.nvfp4_linear_lowrank
    ops = [FAKE] * 9  # a codes / scales / gs, w codes / scales / gs, x, down, up
    ws = 256 * 128 * 2
    assert lr(*ops, 256, 256, 48, 128, FAKE, FAKE, ws, None) == L.NVFP4_ERR_SHAPE  # K % 32
    assert lr(*ops, 256, 256, 0, 128, FAKE, FAKE, ws, None) == L.NVFP4_ERR_SHAPE   # K == 0
    assert lr(*ops, 256, 260, 64, 128, FAKE, FAKE, ws, None) == L.NVFP4_ERR_SHAPE  # N % 8
    assert lr(*ops, 256, 256, 64, 24, FAKE, FAKE, ws, None) == L.NVFP4_ERR_SHAPE   # rank % 16
    assert lr(*ops, 256, 256, 64, 272, FAKE, FAKE, ws, None) == L.NVFP4_ERR_SHAPE  # rank > 256
    assert lr(*ops, 0, 256, 64, 128, None, None, 0, None) == L.NVFP4_OK            # empty
    assert lr(*([FAKE] * 6), None, FAKE, FAKE, 256, 256, 64, 128, FAKE, FAKE, ws, None) == \
        L.NVFP4_ERR_INVALID_ARG
    assert lr(*ops, 256, 256, 64, 128, FAKE + 8, FAKE, ws, None) == L.NVFP4_ERR_ALIGNMENT
    assert lr(*ops, 256, 256, 64, 128, FAKE, FAKE, ws - 2, None) == L.NVFP4_ERR_WORKSPACE
    assert lr(*ops, 256, 256, 64, 128, FAKE, None, 0, None) == L.NVFP4_ERR_WORKSPACE
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR_LOWRANK, 4096, 128, 0) == 4096 * 128 * 2
    assert lib.nvfp4_workspace_bytes(L.NVFP4_OP_LINEAR_LOWRANK, 4096, 512, 0) == 0


def test_free_workspaces_empties_the_cache():
    # host logic only: the binding's per-(device, stream) workspace cache and its reset
    import nvfp4_block_scaled_14_b200 as nv
    nv._ws_cache[(0, 12345)] = object()
    assert "free_workspaces" in nv.__all__
    nv.free_workspaces()
    assert nv._ws_cache == {}


def test_scalar_pointers_must_be_4_byte_aligned(lib):
    # a static amax or an fp8 scale is one fp32 the kernels load as such
    q = lib.nvfp4_quantize
    assert q(FAKE, 1, 8, 64, FAKE + 2, FAKE, FAKE, None, FAKE, None, 0, None) == \
        L.NVFP4_ERR_ALIGNMENT
    f = lib.nvfp4_quantize_fp8_src
    assert f(FAKE, FAKE, 8, 64, FAKE + 1, FAKE, FAKE, None, FAKE, None, 0, None) == \
        L.NVFP4_ERR_ALIGNMENT
    jobs = (L.QuantJob * 2)()
    for j in jobs:
        j.x, j.rows, j.cols, j.codes, j.scales_swz, j.global_scale = FAKE, 8, 64, FAKE, FAKE, FAKE
        j.static_amax = FAKE
    jobs[0].src, jobs[1].src = L.NVFP4_SRC_BF16, L.NVFP4_SRC_E4M3
    jobs[1].fp8_scale = FAKE + 2
    assert lib.nvfp4_quantize_batch(jobs, 2, None, 0, None) == L.NVFP4_ERR_ALIGNMENT
    jobs[1].fp8_scale = FAKE
    jobs[0].static_amax = FAKE + 2
    assert lib.nvfp4_quantize_batch(jobs, 2, None, 0, None) == L.NVFP4_ERR_ALIGNMENT
