"""The C-ABI library without a GPU: it loads, exports every entry point that
include/fp8gemm.h declares, and rejects bad arguments synchronously (before
any CUDA call), so these run on a CPU-only machine."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8gemm.h")


@pytest.fixture(scope="module")
def lib():
    from moe_grouped_gemm_04_b200 import build as b
    b.build()
    import moe_grouped_gemm_04_b200 as m
    return m.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("per_token_cast_to_fp8", "per_block_cast_to_fp8", "fp8_gemm_nt",
              "fp8_grouped_gemm_contiguous", "fp8_grouped_gemm_masked",
              "fg_get_device_status", "fg_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_binding_names_match_header():
    import moe_grouped_gemm_04_b200 as m
    assert set(m.EXPORTED) == set(declared_functions())


def test_sfa_stride_and_status_strings(lib):
    assert [lib.fg_sfa_stride(m) for m in (1, 4, 5, 64, 65, 14208)] == [4, 4, 8, 64, 68, 14208]
    assert lib.fg_status_string(1) == b"FG_ERR_INVALID_ARG"
    assert lib.fg_status_string(0) == b"FG_OK"


FAKE = 0x10000   # never dereferenced: validation fails before any CUDA call
MISALIGNED = 0x10008


def test_validation_rejects_without_touching_the_device(lib):
    P = ctypes.c_void_p
    ok = P(FAKE)
    # K not a multiple of 128
    assert lib.fp8_gemm_nt(ok, ok, ok, ok, ok, 64, 256, 100, None) == 1
    # N not a multiple of 16
    assert lib.fp8_gemm_nt(ok, ok, ok, ok, ok, 64, 250, 256, None) == 1
    # null and misaligned pointers
    assert lib.fp8_gemm_nt(None, ok, ok, ok, ok, 64, 256, 256, None) == 1
    assert lib.fp8_gemm_nt(ok, ok, P(MISALIGNED), ok, ok, 64, 256, 256, None) == 1
    assert b"aligned" in lib.fg_last_error()
    # contiguous: M_total must be a multiple of 128
    assert lib.fp8_grouped_gemm_contiguous(ok, ok, ok, ok, ok, ok, 100, 256, 256, 2, None) == 1
    assert lib.fp8_grouped_gemm_contiguous(ok, ok, ok, ok, ok, ok, 128, 256, 256, 0, None) == 1
    # masked: G and M_max positive
    assert lib.fp8_grouped_gemm_masked(ok, ok, ok, ok, ok, ok, 0, 64, 256, 256, 64, None) == 1
    assert lib.fp8_grouped_gemm_masked(ok, ok, ok, ok, ok, ok, 2, 0, 256, 256, 64, None) == 1
    assert lib.fp8_grouped_gemm_masked(ok, ok, ok, ok, ok, None, 2, 64, 256, 256, 64, None) == 1
    # quantizers
    assert lib.per_token_cast_to_fp8(ok, ok, ok, 1, 64, 100, None) == 1
    assert lib.per_token_cast_to_fp8(ok, ok, ok, 0, 64, 128, None) == 1
    assert lib.per_block_cast_to_fp8(ok, ok, ok, 1, 0, 128, None) == 1
    assert lib.per_block_cast_to_fp8(ok, P(MISALIGNED), ok, 1, 64, 128, None) == 1
    assert lib.fg_selftest_wait_timeout(0, None) == 1
    # weight dequantization
    assert lib.per_block_dequant_to_bf16(ok, ok, ok, 1, 64, 100, None) == 1
    assert lib.per_block_dequant_to_bf16(ok, ok, ok, 0, 64, 128, None) == 1
    assert lib.per_block_dequant_to_bf16(ok, ok, ok, 1, 0, 128, None) == 1
    assert lib.per_block_dequant_to_bf16(ok, ok, P(MISALIGNED), 1, 64, 128, None) == 1
    # tensor-core rate kernel: launch length and output pointer
    assert lib.fg_fp8_mma_peak(0, ok, None) == 1
    assert lib.fg_fp8_mma_peak(32769, ok, None) == 1
    assert lib.fg_fp8_mma_peak(16, None, None) == 1
    # empty problems are a no-op success
    assert lib.fp8_gemm_nt(ok, ok, ok, ok, ok, 0, 256, 256, None) == 0
    assert lib.per_token_cast_to_fp8(ok, ok, ok, 1, 0, 128, None) == 0
    assert lib.fp8_grouped_gemm_contiguous(ok, ok, ok, ok, ok, ok, 0, 256, 256, 2, None) == 0


def test_ue8m0_gemm_validation_without_the_device(lib):
    P = ctypes.c_void_p
    ok = P(FAKE)
    assert lib.fp8_gemm_nt_ue8m0(ok, ok, ok, ok, ok, 64, 256, 100, None) == 1
    assert lib.fp8_gemm_nt_ue8m0(ok, ok, ok, ok, ok, 256, 250, 256, None) == 1
    assert lib.fp8_gemm_nt_ue8m0(ok, ok, ok, ok, None, 256, 256, 256, None) == 1
    assert lib.fp8_grouped_gemm_contiguous_ue8m0(ok, ok, ok, ok, ok, ok, 100, 256, 256, 2, None) == 1
    assert lib.fp8_grouped_gemm_contiguous_ue8m0(ok, ok, ok, ok, ok, None, 128, 256, 256, 2, None) == 1
    assert lib.fp8_grouped_gemm_masked_ue8m0(ok, ok, ok, ok, ok, ok, 0, 64, 256, 256, 64, None) == 1
    assert lib.fp8_grouped_gemm_masked_ue8m0(ok, ok, P(MISALIGNED), ok, ok, ok, 2, 64, 256, 256, 64,
                                             None) == 1
    assert lib.fp8_gemm_nt_ue8m0(ok, ok, ok, ok, ok, 0, 256, 256, None) == 0
    assert lib.fp8_grouped_gemm_contiguous_ue8m0(ok, ok, ok, ok, ok, ok, 0, 256, 256, 2, None) == 0
    # the tile knob takes 0, 128, 224 and 256 single-CTA and 224 as a pair
    for w, pair in ((0, 0), (128, 0), (224, 0), (256, 0), (224, 1), (192, 1), (0, 1)):
        assert lib.fg_set_ue8m0_tile(w, pair) == 0
    for w, pair in ((-1, 0), (64, 0), (192, 0), (512, 0), (128, 1), (256, 1)):
        assert lib.fg_set_ue8m0_tile(w, pair) == 1
    assert lib.fg_set_ue8m0_tile(0, 0) == 0


def test_ffn_validation_without_the_device(lib):
    P = ctypes.c_void_p
    ok = P(FAKE)
    args = [ok] * 11
    ws = [ok, 1 << 20]  # workspace and its size
    # I and H must be positive multiples of 128; M_total a multiple of 128
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*args, 256, 256, 100, 2, *ws, None) == 1
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*args, 256, 200, 128, 2, *ws, None) == 1
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*args, 100, 256, 128, 2, *ws, None) == 1
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*args, 256, 256, 128, 0, *ws, None) == 1
    bad = list(args)
    bad[6] = P(MISALIGNED)  # Hq
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*bad, 256, 256, 128, 2, *ws, None) == 1
    margs = list(args)
    margs[10] = None  # masked_m
    assert lib.fp8_moe_ffn_masked_ue8m0(*margs, 2, 64, 256, 128, 32, *ws, None) == 1
    assert lib.fp8_moe_ffn_masked_ue8m0(*args, 2, 0, 256, 128, 32, *ws, None) == 1
    # the workspace: present, aligned and at least fg_moe_ffn_workspace_bytes
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*args, 256, 256, 128, 2, None, 1 << 20, None) == 1
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*args, 256, 256, 128, 2, P(MISALIGNED), 1 << 20, None) == 1
    need = lib.fg_moe_ffn_workspace_bytes(0, 256, 2)
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*args, 256, 256, 128, 2, ok, need - 1, None) == 1
    assert lib.fp8_moe_ffn_masked_ue8m0(*args, 2, 64, 256, 128, 32, ok,
                                        lib.fg_moe_ffn_workspace_bytes(1, 64, 2) - 1, None) == 1
    # an empty contiguous problem is a no-op success; GU may be NULL
    nogu = list(args)
    nogu[8] = None
    assert lib.fp8_moe_ffn_contiguous_ue8m0(*nogu, 0, 256, 128, 2, *ws, None) == 0


def test_ffn_mode_knob(lib):
    for m in (0, 1, 2):
        assert lib.fg_set_ffn_mode(m) == 0
    for m in (-1, 3):
        assert lib.fg_set_ffn_mode(m) == 1
    assert lib.fg_set_ffn_mode(0) == 0


def test_ffn_workspace_bytes(lib):
    """One int counter per 128-token tile (masked: per expert and tile of its
    slab), rounded up to 256 bytes; 0 for invalid arguments."""
    assert lib.fg_moe_ffn_workspace_bytes(0, 13952, 8) == 512          # 109 tiles: 436 bytes
    assert lib.fg_moe_ffn_workspace_bytes(0, 128 * 100, 8) == 512      # 100 tiles
    assert lib.fg_moe_ffn_workspace_bytes(1, 256, 32) == 256           # 32 x 2 tiles
    assert lib.fg_moe_ffn_workspace_bytes(1, 200, 100) == 1024         # 100 x 2 tiles
    assert lib.fg_moe_ffn_workspace_bytes(2, 256, 8) == 0
    assert lib.fg_moe_ffn_workspace_bytes(0, 256, 0) == 0


def test_k_grouped_validation_without_the_device(lib):
    P = ctypes.c_void_p
    ok = P(FAKE)
    args = [ok] * 6
    assert lib.fp8_k_grouped_gemm_nt_ue8m0(*args, 0, 128, 256, 256, None) == 1   # G
    assert lib.fp8_k_grouped_gemm_nt_ue8m0(*args, 2, 0, 256, 256, None) == 1     # M
    assert lib.fp8_k_grouped_gemm_nt_ue8m0(*args, 2, 128, 250, 256, None) == 1   # N % 16
    assert lib.fp8_k_grouped_gemm_nt_ue8m0(*args, 2, 128, 256, 200, None) == 1   # T % 128
    bad = list(args)
    bad[5] = None  # ks
    assert lib.fp8_k_grouped_gemm_nt_ue8m0(*bad, 2, 128, 256, 256, None) == 1
    bad = list(args)
    bad[4] = P(MISALIGNED)  # D
    assert lib.fp8_k_grouped_gemm_nt_ue8m0(*bad, 2, 128, 256, 256, None) == 1
