"""The C-ABI library builds, loads and exports every symbol the header declares (no GPU needed).

Only host-side entry points are exercised here: the size helpers, the status
strings, and argument checks that reject a call before any CUDA call is made.
"""
import ctypes
import re

import pytest

from w3a16_gemv_b200 import _binding, build

NULL = None
FAKE_A = 0x10000  # 16-byte aligned addresses that are never dereferenced:
FAKE_B = 0x20000  # every call below is rejected by the host checks first
FAKE_C = 0x30000
FAKE_D = 0x40000


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _binding.lib()


def declared_functions():
    text = open(build.HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w3\w*)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("w3_pack", "w3_unpack", "w3_dequant_f32", "w3a16_gemm", "w3_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert sorted(n for n, _, _ in _binding.SIGNATURES) == declared_functions()


def test_host_helpers(lib):
    assert lib.w3_abi_version() == 1
    assert lib.w3_packed_words_per_row(8192) == 768  # the card's gate_proj example
    assert lib.w3_groups_per_row(8192) == 64
    assert lib.w3_packed_words_per_row(100) == -1 and lib.w3_groups_per_row(64) == -1
    for s in range(8):
        assert lib.w3_status_string(s)
    assert lib.w3_status_string(99) == b"unknown status"


def test_host_argument_checks(lib):
    g = lib.w3a16_gemm
    assert g(NULL, FAKE_B, FAKE_C, FAKE_D, 1, 16, 128, NULL) == 1  # W3_ERR_NULL
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 0, 16, 128, NULL) == 2  # M < 1
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 1, 0, 128, NULL) == 2  # N < 1
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 1, 16, 192, NULL) == 2  # K % 128
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 1, 16, 0, NULL) == 2
    assert g(FAKE_A + 2, FAKE_B, FAKE_C, FAKE_D, 1, 16, 128, NULL) == 3  # misaligned x
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_B, 1, 16, 128, NULL) == 7  # y overlaps packed
    assert lib.w3_pack(FAKE_A, FAKE_A, 4, 128, NULL) == 7
    assert lib.w3_unpack(FAKE_A, NULL, 4, 128, NULL) == 1
    assert lib.w3_dequant_f32(FAKE_A, FAKE_B, FAKE_C, 4, 130, NULL) == 2
    r = lib.w3_repack_ct4
    assert r(NULL, FAKE_B, 4, 128, NULL, NULL) == 1  # W3_ERR_NULL
    assert r(FAKE_A, FAKE_B, 4, 96, NULL, NULL) == 2  # K % 128
    assert r(FAKE_A + 4, FAKE_B, 4, 128, NULL, NULL) == 3  # misaligned container
    assert r(FAKE_A, FAKE_B, 4, 128, FAKE_C + 4, NULL) == 3  # misaligned counter
    assert r(FAKE_A, FAKE_A + 16, 4, 128, NULL, NULL) == 7  # output overlaps the container


def test_native_order_host_checks(lib):
    assert lib.w3_native_words(40, 256) == 64 * 24  # two 32-row blocks of 24 words per row
    assert lib.w3_native_words(32, 8192) == 32 * 768
    assert lib.w3_native_words(1, 100) == -1
    assert lib.w3_pack_native(NULL, FAKE_B, 4, 128, NULL) == 1
    assert lib.w3_native_from_packed(FAKE_A, FAKE_B, 4, 96, NULL) == 2
    assert lib.w3_packed_from_native(FAKE_A + 4, FAKE_B, 4, 128, NULL) == 3
    assert lib.w3_native_from_packed(FAKE_A, FAKE_A + 16, 40, 256, NULL) == 7  # overlap
    g = lib.w3a16_gemm_native
    assert g(NULL, FAKE_B, FAKE_C, FAKE_D, 1, 64, 128, NULL) == 1
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 0, 64, 128, NULL) == 2
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 17, 64, 128, NULL) == 5  # batches above 16: row-major path
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 1, 16, 128, NULL) == 5   # fewer than 32 rows
    assert g(FAKE_A, FAKE_B, FAKE_C, FAKE_B, 1, 64, 128, NULL) == 7   # y overlaps the weights


def test_no_silent_fallback_without_a_device(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    # valid arguments reach the device set-up, which must fail loudly
    st = lib.w3a16_gemm(FAKE_A, FAKE_B, FAKE_C, FAKE_D, 1, 16, 128, NULL)
    assert st in (4, 5)  # W3_ERR_CUDA or W3_ERR_UNSUPPORTED, never W3_OK
