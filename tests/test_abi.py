"""CPU-side checks of the C ABI: the library builds/loads, exports every symbol
include/bitlinear.h declares, and host-side validation rejects bad arguments
before any CUDA work (no GPU needed)."""
import ctypes
import os
import re

import pytest

from bit_ternary_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build_library()
    return _lib.lib()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "bitlinear.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"BL_API\s+[\w\s\*]*?\b(bitlinear_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_symbols()
    for must in ("bitlinear_pack_weights", "bitlinear_quant_act", "bitlinear_forward"):
        assert must in names
    assert set(names) == set(_lib.SIGNATURES)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_abi_version_and_status_strings(L):
    assert L.bitlinear_abi_version() == 1
    for st in range(0, 10):
        s = L.bitlinear_status_string(st)
        assert s and isinstance(s, bytes)
    assert L.bitlinear_status_string(99) == b"unknown status"


def test_workspace_queries(L):
    assert L.bitlinear_pack_workspace_size(10, 32) >= 256 + 2048
    ws = L.bitlinear_workspace_size(4096, 13824, 2560)
    assert ws >= 4096 * 2560 + 8 * 4096
    assert ws % 256 == 0
    assert L.bitlinear_host_workspace_size(4096, 13824, 2560) >= ws + 4 * 4096 * (2560 + 13824)
    assert L.bitlinear_workspace_size(0, 5, 16) == 256


FAKE = 0x10000  # never dereferenced: validation fails first


@pytest.mark.parametrize("K", [0, -16, 8, 24, 131072 + 16])
def test_bad_k_rejected_before_cuda(L, K):
    assert L.bitlinear_forward(FAKE, 1, 1, K, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert L.bitlinear_quant_act(FAKE, 1, K, FAKE, FAKE, None, None) == 2
    assert L.bitlinear_pack_weights(FAKE, 1, K, FAKE, FAKE, FAKE, 4096, None) == 2


def test_empty_is_noop(L):
    assert L.bitlinear_forward(None, 0, 5, 16, None, None, None, None, 0, None) == 0
    assert L.bitlinear_forward(None, 3, 0, 16, None, None, None, None, 0, None) == 0
    assert L.bitlinear_quant_act(None, 0, 16, None, None, None, None) == 0


def test_null_and_alignment_rejected(L):
    assert L.bitlinear_forward(None, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.bitlinear_forward(FAKE + 4, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 3
    assert L.bitlinear_forward(FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE + 16, 1 << 20, None) == 3
    assert L.bitlinear_forward(FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 10, None) == 4
    assert L.bitlinear_pack_weights(FAKE, 0, 16, FAKE, FAKE, FAKE, 4096, None) == 2
    assert L.bitlinear_pack_weights(FAKE, 4, 16, FAKE, FAKE, FAKE, 16, None) == 4
    assert L.bitlinear_forward_acc(FAKE, 1, 1, 16, FAKE, None, FAKE, 1 << 20, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()


def test_product_path_does_not_import_oracle():
    pkg = os.path.join(ROOT, "bit_ternary_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, fn)) as f:
                    src = f.read()
                assert "import oracle" not in src and "from oracle" not in src, fn


def test_batch_validation_before_cuda(L):
    calls = (_lib.LinearCall * 2)()
    calls[0] = _lib.LinearCall(FAKE, 1, 8, 64, FAKE, FAKE, FAKE)
    calls[1] = _lib.LinearCall(FAKE, 1, 8, 24, FAKE, FAKE, FAKE)  # K % 16 != 0
    assert L.bitlinear_forward_batch(calls, 2, 0, FAKE, 1 << 20, None) == 2
    calls[1] = _lib.LinearCall(None, 1, 8, 64, FAKE, FAKE, FAKE)
    assert L.bitlinear_forward_batch(calls, 2, 0, FAKE, 1 << 20, None) == 1
    calls[1] = _lib.LinearCall(FAKE, 1, 8, 64, FAKE, FAKE, FAKE)
    assert L.bitlinear_forward_batch(calls, 2, 0x80, FAKE, 1 << 20, None) == 2  # unknown flag
    assert L.bitlinear_forward_batch(calls, 2, 0x4, FAKE, 1 << 20, None) == 2  # first undefined bit
    assert _lib.BL_FLAG_STREAM_WEIGHTS_EARLY == 1 and _lib.BL_FLAG_ONE_LAUNCH_PER_CALL == 2
    assert L.bitlinear_forward_batch(calls, 0, 0, None, 0, None) == 0
    assert L.bitlinear_batch_workspace_size(calls, 2) == 256 + 256 + 256 + 256  # header, s_x, sums, q


def test_forward_q_and_async_host_validation_before_cuda(L):
    # bitlinear_forward_q(q, s_x, M, N, K, packed, D, y, ws, ws_bytes, stream)
    assert L.bitlinear_forward_q(FAKE, FAKE, 1, 1, 24, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert L.bitlinear_forward_q(None, FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.bitlinear_forward_q(FAKE, None, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.bitlinear_forward_q(FAKE + 8, FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 3
    assert L.bitlinear_forward_q(FAKE, FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 16, None) == 4
    assert L.bitlinear_forward_q(None, None, 0, 4, 16, None, None, None, None, 0, None) == 0
    # bitlinear_forward_host_async(x_host, M, N, K, packed, D, y_host, ws, ws_bytes, stream)
    assert L.bitlinear_forward_host_async(None, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.bitlinear_forward_host_async(FAKE, 1, 1, 40, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert L.bitlinear_forward_host_async(FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE + 16, 1 << 20, None) == 3
    assert L.bitlinear_forward_host_async(FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, 8, None) == 4


def test_rmsnorm_validation_before_cuda(L):
    # bitlinear_rmsnorm_quant_act(x, g, eps, M, K, q, s_x, rowsum, stream)
    assert L.bitlinear_rmsnorm_quant_act(FAKE, FAKE, 1e-6, 1, 16384 + 16, FAKE, FAKE, None, None) == 2
    assert L.bitlinear_rmsnorm_quant_act(FAKE, None, 1e-6, 1, 64, FAKE, FAKE, None, None) == 1
    assert L.bitlinear_rmsnorm_quant_act(FAKE, FAKE, -1.0, 1, 64, FAKE, FAKE, None, None) == 2
    assert L.bitlinear_rmsnorm_quant_act(FAKE, FAKE + 4, 1e-6, 1, 64, FAKE, FAKE, None, None) == 3
    assert L.bitlinear_rmsnorm_quant_act(None, None, 1e-6, 0, 64, None, None, None, None) == 0
    # bitlinear_forward_rmsnorm(x, g, eps, M, N, K, packed, D, y, ws, ws_bytes, stream)
    assert L.bitlinear_forward_rmsnorm(FAKE, FAKE, 1e-6, 1, 1, 20000 - 20000 % 16, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                       None) == 2
    assert L.bitlinear_forward_rmsnorm(FAKE, None, 1e-6, 1, 1, 64, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.bitlinear_forward_rmsnorm(FAKE, FAKE, 1e-6, 1, 1, 64, FAKE, FAKE, FAKE, FAKE, 16, None) == 4


def test_batch_host_validation_before_cuda(L):
    calls = (_lib.LinearCall * 3)()
    calls[0] = _lib.LinearCall(FAKE, 1, 8, 64, FAKE, FAKE, FAKE)
    calls[1] = _lib.LinearCall(FAKE, 3, 5, 32, FAKE, FAKE, FAKE)
    calls[2] = _lib.LinearCall(None, 0, 8, 64, None, None, None)  # empty: stages nothing
    need = L.bitlinear_batch_host_workspace_size(calls, 3)
    # batch workspace, then x blocks (256 + 384 bytes) and y blocks (32 + 60 -> 64 bytes), 256-aligned each
    assert need == L.bitlinear_batch_workspace_size(calls, 3) + 768 + 256
    # bitlinear_forward_batch_host(calls, count, flags, ws, ws_bytes, stream)
    assert L.bitlinear_forward_batch_host(calls, 3, 0, FAKE, need - 1, None) == 4
    assert L.bitlinear_forward_batch_host(calls, 3, 0, FAKE + 16, need, None) == 3
    assert L.bitlinear_forward_batch_host(calls, 3, 0x80, FAKE, need, None) == 2
    assert L.bitlinear_forward_batch_host(calls, -1, 0, FAKE, need, None) == 2
    assert L.bitlinear_forward_batch_host(calls, 0, 0, None, 0, None) == 0
    calls[1] = _lib.LinearCall(FAKE, 3, 5, 40, FAKE, FAKE, FAKE)  # K % 16 != 0
    assert L.bitlinear_forward_batch_host(calls, 3, 0, FAKE, 1 << 20, None) == 2
    calls[1] = _lib.LinearCall(FAKE, 3, 5, 32, FAKE, FAKE, None)  # no y
    assert L.bitlinear_forward_batch_host(calls, 3, 0, FAKE, 1 << 20, None) == 1
    calls[1] = _lib.LinearCall(FAKE, 3, 5, 32, FAKE + 4, FAKE, FAKE)  # packed not 16-byte aligned
    assert L.bitlinear_forward_batch_host(calls, 3, 0, FAKE, 1 << 20, None) == 3
    assert L.bitlinear_batch_host_workspace_size(None, 3) == 0


def test_i2s_sizes_and_validation_before_cuda(L):
    assert L.bitlinear_i2s_bytes(3, 48) == 68
    assert L.bitlinear_i2s_bytes(2560, 2560) == 2560 * 2560 // 4 + 4
    assert L.bitlinear_i2s_bytes(1, 16) == 36
    assert L.bitlinear_i2s_bytes(-1, 16) == 0
    assert L.bitlinear_i2s_workspace_size() == 256
    # bitlinear_i2s_export(packed, D, N, K, layout, i2s, ws, ws_bytes, stream)
    assert L.bitlinear_i2s_export(FAKE, FAKE, 3, 24, 0, FAKE, FAKE, 256, None) == 2
    assert L.bitlinear_i2s_export(FAKE, FAKE, 0, 48, 0, FAKE, FAKE, 256, None) == 2
    assert L.bitlinear_i2s_export(FAKE, FAKE, 3, 48, 2, FAKE, FAKE, 256, None) == 2
    assert L.bitlinear_i2s_export(None, FAKE, 3, 48, 0, FAKE, FAKE, 256, None) == 1
    assert L.bitlinear_i2s_export(FAKE, FAKE, 3, 48, 1, FAKE + 4, FAKE, 256, None) == 3
    assert L.bitlinear_i2s_export(FAKE, FAKE + 2, 3, 48, 1, FAKE, FAKE, 256, None) == 3
    assert L.bitlinear_i2s_export(FAKE, FAKE, 3, 48, 0, FAKE, FAKE, 128, None) == 4
    # bitlinear_i2s_import(i2s, N, K, layout, packed, D, ws, ws_bytes, stream)
    assert L.bitlinear_i2s_import(FAKE, 3, 40, 0, FAKE, FAKE, FAKE, 256, None) == 2
    assert L.bitlinear_i2s_import(FAKE, 3, 48, -1, FAKE, FAKE, FAKE, 256, None) == 2
    assert L.bitlinear_i2s_import(FAKE, 3, 48, 0, FAKE, None, FAKE, 256, None) == 1
    assert L.bitlinear_i2s_import(FAKE, 3, 48, 0, FAKE + 8, FAKE, FAKE, 256, None) == 3
    assert L.bitlinear_i2s_import(FAKE, 3, 48, 0, FAKE, FAKE, FAKE + 16, 256, None) == 3
    assert L.bitlinear_i2s_import(FAKE, 3, 48, 0, FAKE, FAKE, FAKE, 8, None) == 4
    assert L.bitlinear_status_string(9) == b"I2_S: field holding 3, bad scale, or rows of D that differ"


def test_i2s_async_and_status_validation_before_cuda(L):
    assert L.bitlinear_i2s_export_async(FAKE, FAKE, 3, 24, 0, FAKE, FAKE, 256, None) == 2
    assert L.bitlinear_i2s_export_async(FAKE, FAKE, 3, 48, 0, FAKE + 4, FAKE, 256, None) == 3
    assert L.bitlinear_i2s_import_async(FAKE, 3, 48, 7, FAKE, FAKE, FAKE, 256, None) == 2
    assert L.bitlinear_i2s_import_async(FAKE, 3, 48, 0, FAKE, FAKE, FAKE, 0, None) == 4
    assert L.bitlinear_i2s_status(None, 256, None) == 1
    assert L.bitlinear_i2s_status(FAKE + 16, 256, None) == 3
    assert L.bitlinear_i2s_status(FAKE, 16, None) == 4


def test_python_constants_match_header_defines():
    with open(os.path.join(ROOT, "include", "bitlinear.h")) as f:
        text = f.read()
    defines = {k: int(v) for k, v in re.findall(r"#define\s+(BL_\w+)\s+(\d+)u?\b", text)}
    for name in ("BL_FLAG_STREAM_WEIGHTS_EARLY", "BL_FLAG_ONE_LAUNCH_PER_CALL", "BL_I2S_CONSECUTIVE",
                 "BL_I2S_QUARTERS"):
        assert getattr(_lib, name) == defines[name], name
    statuses = dict((k, int(v)) for k, v in re.findall(r"(BL_(?:OK|ERR_\w+))\s*=\s*(\d+)", text))
    for code, name in _lib.STATUS_NAMES.items():
        assert statuses[name] == code, name


# ------------------------------------------------- per-256-block scale variant
@pytest.mark.parametrize("K,nb", [(16, 1), (256, 1), (272, 2), (2560, 10), (6912, 27), (4304, 17), (131072, 512)])
def test_block_scales_count(L, K, nb):
    assert L.bitlinear_block_scales(K) == nb


@pytest.mark.parametrize("K", [0, -16, 24, 131072 + 16])
def test_block_scales_invalid_k(L, K):
    assert L.bitlinear_block_scales(K) == 0
    assert L.bitlinear_blocks_workspace_size(4, 4, K) == 0


def test_blocks_workspace_adds_row_sums_per_block(L):
    for M, K in ((1, 2560), (200, 272), (4096, 6912)):
        base = L.bitlinear_workspace_size(M, 8, K)
        blk = L.bitlinear_blocks_workspace_size(M, 8, K)
        nb = L.bitlinear_block_scales(K)
        assert blk >= base + 4 * M * nb and blk % 256 == 0


@pytest.mark.parametrize("K", [0, 8, 24, 131072 + 16])
def test_block_entry_points_reject_bad_k(L, K):
    assert L.bitlinear_forward_blocks(FAKE, 1, 1, K, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert L.bitlinear_pack_weights_blocks(FAKE, 1, K, FAKE, FAKE, FAKE, 1 << 16, None) == 2


def test_block_entry_points_validate_before_cuda(L):
    big = 1 << 24
    assert L.bitlinear_forward_blocks(None, 0, 5, 16, None, None, None, None, 0, None) == 0  # empty: no-op
    assert L.bitlinear_forward_blocks(None, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, big, None) == 1
    assert L.bitlinear_forward_blocks(FAKE, 1, 1, 16, FAKE, None, FAKE, FAKE, big, None) == 1
    assert L.bitlinear_forward_blocks(FAKE + 4, 1, 1, 16, FAKE, FAKE, FAKE, FAKE, big, None) == 3
    assert L.bitlinear_forward_blocks(FAKE, 1, 1, 16, FAKE, FAKE, FAKE, FAKE + 16, big, None) == 3
    # the plain forward workspace is short for the block route (it also holds per-block row sums)
    short = L.bitlinear_workspace_size(200, 8, 272)
    assert L.bitlinear_forward_blocks(FAKE, 200, 8, 272, FAKE, FAKE, FAKE, FAKE, short, None) == 4
    assert L.bitlinear_pack_weights_blocks(FAKE, 0, 16, FAKE, FAKE, FAKE, big, None) == 2
    assert L.bitlinear_pack_weights_blocks(None, 4, 16, FAKE, FAKE, FAKE, big, None) == 1
    assert L.bitlinear_pack_weights_blocks(FAKE, 4, 16, FAKE, FAKE, FAKE, 16, None) == 4


def test_async_pack_and_status_validate_before_cuda(L):
    ws = L.bitlinear_pack_workspace_size(1, 16)
    assert L.bitlinear_pack_weights_async(FAKE, 1, 24, FAKE, FAKE, FAKE, ws, None) == 2
    assert L.bitlinear_pack_weights_async(FAKE, 4, 16, FAKE, FAKE, FAKE, 16, None) == 4
    assert L.bitlinear_pack_weights_async(FAKE + 4, 4, 16, FAKE, FAKE, FAKE, ws, None) == 3
    assert L.bitlinear_pack_status(None, ws, None) == 1
    assert L.bitlinear_pack_status(FAKE + 16, ws, None) == 3
    assert L.bitlinear_pack_status(FAKE, 16, None) == 4
