"""W3A16 group-128 fused dequantize-and-multiply for NVIDIA B200 (sm_100a).

The product is ``libw3a16.so`` (C ABI, ``include/w3a16.h``); this package is its
thin Python binding.  Importing the package loads nothing; the library is
loaded on the first call and a missing library raises.

    from w3a16_gemv_b200 import w3_pack, w3a16_gemm
    packed = w3_pack(codes)                # uint8 [N,K] -> int32 [N, 3K/32]
    y = w3a16_gemm(x, packed, scales)      # bf16 [M,K] x W^T -> bf16 [M,N]
"""
from ._binding import (  # noqa: F401
    W3Error,
    lib,
    status_string,
    w3_check_device_error,
    w3_dequant_f32,
    w3_groups_per_row,
    w3_native_from_packed,
    w3_native_words,
    w3_pack,
    w3_pack_native,
    w3_packed_from_native,
    w3_packed_words_per_row,
    w3_repack_ct4,
    w3_unpack,
    w3a16_gemm,
    w3a16_gemm_native,
    w3a16_gemm_noalloc,
    w3a16_gemm_launches,
    w3a16_gemm_route,
)

__all__ = [
    "W3Error",
    "lib",
    "status_string",
    "w3_check_device_error",
    "w3_dequant_f32",
    "w3_groups_per_row",
    "w3_native_from_packed",
    "w3_native_words",
    "w3_pack",
    "w3_pack_native",
    "w3_packed_from_native",
    "w3_packed_words_per_row",
    "w3_repack_ct4",
    "w3_unpack",
    "w3a16_gemm",
    "w3a16_gemm_native",
    "w3a16_gemm_noalloc",
    "w3a16_gemm_launches",
    "w3a16_gemm_route",
]
