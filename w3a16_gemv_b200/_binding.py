"""ctypes binding of libw3a16.so: argument marshalling only.

Each function here has the name of the C entry point it calls (see
``include/w3a16.h``), takes torch CUDA tensors, checks dtypes and shapes,
allocates outputs with torch when none are given, and passes raw pointers and
torch's current CUDA stream to the library.  No arithmetic of the format or of
the product happens in Python, and there is no fallback: if the library is
missing or the device is not a B200, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw3a16.so")

W3_OK = 0
STATUS_NAMES = {
    0: "W3_OK",
    1: "W3_ERR_NULL",
    2: "W3_ERR_SHAPE",
    3: "W3_ERR_ALIGN",
    4: "W3_ERR_CUDA",
    5: "W3_ERR_UNSUPPORTED",
    6: "W3_ERR_TIMEOUT",
    7: "W3_ERR_ALIAS",
}

# (name, restype, argtypes) of every entry point declared in include/w3a16.h
_P, _I64 = ctypes.c_void_p, ctypes.c_int64
SIGNATURES = [
    ("w3_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("w3_abi_version", ctypes.c_int32, []),
    ("w3_packed_words_per_row", _I64, [_I64]),
    ("w3_groups_per_row", _I64, [_I64]),
    ("w3_pack", ctypes.c_int, [_P, _P, _I64, _I64, _P]),
    ("w3_unpack", ctypes.c_int, [_P, _P, _I64, _I64, _P]),
    ("w3_dequant_f32", ctypes.c_int, [_P, _P, _P, _I64, _I64, _P]),
    ("w3_repack_ct4", ctypes.c_int, [_P, _P, _I64, _I64, _P, _P]),
    ("w3a16_gemm", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    ("w3a16_gemm_noalloc", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    ("w3_native_words", _I64, [_I64, _I64]),
    ("w3_pack_native", ctypes.c_int, [_P, _P, _I64, _I64, _P]),
    ("w3_native_from_packed", ctypes.c_int, [_P, _P, _I64, _I64, _P]),
    ("w3_packed_from_native", ctypes.c_int, [_P, _P, _I64, _I64, _P]),
    ("w3a16_gemm_native", ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    ("w3a16_gemm_route", ctypes.c_char_p, [_I64, _I64, _I64, ctypes.c_int32]),
    ("w3a16_gemm_launches", ctypes.c_int32, [_I64, _I64, _I64, ctypes.c_int32]),
    ("w3_check_device_error", ctypes.c_int, [_P]),
]

_lock = threading.Lock()
_lib: ctypes.CDLL | None = None


class W3Error(RuntimeError):
    """A non-zero w3_status returned by the library."""

    def __init__(self, status: int, what: str):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{what}: {name} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """The loaded library with its signatures declared.  Raises if it was not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m w3a16_gemv_b200.build` "
                    "(there is no fallback implementation)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, res, args in SIGNATURES:
                f = getattr(handle, name)
                f.restype = res
                f.argtypes = args
            _lib = handle
        return _lib


def status_string(status: int) -> str:
    return lib().w3_status_string(int(status)).decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, what: str) -> None:
    if status != W3_OK:
        raise W3Error(status, what)


def _need(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def w3_packed_words_per_row(K: int) -> int:
    return int(lib().w3_packed_words_per_row(K))


def w3_groups_per_row(K: int) -> int:
    return int(lib().w3_groups_per_row(K))


def w3_pack(codes: torch.Tensor, packed: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """codes uint8 [N,K] (0..7) -> packed int32 [N, 3K/32]."""
    _need(codes, torch.uint8, "codes")
    N, K = codes.shape
    if packed is None:
        packed = torch.empty((N, max(w3_packed_words_per_row(K), 1)), dtype=torch.int32, device=codes.device)
    _need(packed, torch.int32, "packed")
    _check(lib().w3_pack(codes.data_ptr(), packed.data_ptr(), N, K, _stream(stream)), "w3_pack")
    return packed


def w3_unpack(packed: torch.Tensor, K: int, codes: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """packed int32 [N, 3K/32] -> codes uint8 [N,K]."""
    _need(packed, torch.int32, "packed")
    N = packed.shape[0]
    if packed.shape[1] != w3_packed_words_per_row(K):
        raise ValueError("packed width does not match K")
    if codes is None:
        codes = torch.empty((N, K), dtype=torch.uint8, device=packed.device)
    _need(codes, torch.uint8, "codes")
    _check(lib().w3_unpack(packed.data_ptr(), codes.data_ptr(), N, K, _stream(stream)), "w3_unpack")
    return codes


def w3_repack_ct4(ct4: torch.Tensor, K: int, packed: torch.Tensor | None = None, count_out_of_range: bool = False,
                  stream=None):
    """4-bit container int32 [N, K/8] -> exact-width packed int32 [N, 3K/32].

    With count_out_of_range, returns (packed, count) where count is a device int64 tensor holding the
    number of levels outside -4..3 that were clamped."""
    _need(ct4, torch.int32, "ct4")
    N = ct4.shape[0]
    if ct4.dim() != 2 or ct4.shape[1] * 8 != K:
        raise ValueError("ct4 must be [N, K/8]")
    if packed is None:
        packed = torch.empty((N, w3_packed_words_per_row(K)), dtype=torch.int32, device=ct4.device)
    _need(packed, torch.int32, "packed")
    count = torch.zeros(1, dtype=torch.int64, device=ct4.device) if count_out_of_range else None
    _check(lib().w3_repack_ct4(ct4.data_ptr(), packed.data_ptr(), N, K, count.data_ptr() if count is not None else None,
                               _stream(stream)), "w3_repack_ct4")
    return (packed, count) if count_out_of_range else packed


def w3_dequant_f32(packed: torch.Tensor, scales: torch.Tensor, K: int, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """W[n,k] = (c-4) * scales[n,k//128] as float32 [N,K]."""
    _need(packed, torch.int32, "packed")
    _need(scales, torch.bfloat16, "scales")
    N = packed.shape[0]
    if packed.shape[1] != w3_packed_words_per_row(K) or tuple(scales.shape) != (N, w3_groups_per_row(K)):
        raise ValueError("packed/scales shapes do not match N, K")
    if out is None:
        out = torch.empty((N, K), dtype=torch.float32, device=packed.device)
    _need(out, torch.float32, "out")
    _check(lib().w3_dequant_f32(packed.data_ptr(), scales.data_ptr(), out.data_ptr(), N, K, _stream(stream)),
           "w3_dequant_f32")
    return out


def w3a16_gemm(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """y = x W^T, x bf16 [M,K], packed int32 [N,3K/32], scales bf16 [N,K/128] -> y bf16 [M,N]."""
    return _gemm("w3a16_gemm", x, packed, scales, out, stream)


def w3a16_gemm_noalloc(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                       out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """w3a16_gemm with the library's fixed scratch instead of an allocation (overlapping calls race)."""
    return _gemm("w3a16_gemm_noalloc", x, packed, scales, out, stream)


def _gemm(entry: str, x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, out: torch.Tensor | None,
          stream) -> torch.Tensor:
    _need(x, torch.bfloat16, "x")
    _need(packed, torch.int32, "packed")
    _need(scales, torch.bfloat16, "scales")
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] != w3_packed_words_per_row(K) or tuple(scales.shape) != (N, w3_groups_per_row(K)):
        raise ValueError("packed/scales shapes do not match x's K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, "out")
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be [M, N]")
    _check(getattr(lib(), entry)(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), out.data_ptr(), M, N, K,
                                 _stream(stream)), entry)
    return out


def w3_native_words(N: int, K: int) -> int:
    return int(lib().w3_native_words(N, K))


def _native_out(N: int, K: int, device, out: torch.Tensor | None) -> torch.Tensor:
    n = w3_native_words(N, K)
    if n < 0:
        raise ValueError(f"no native order for N={N}, K={K}")
    if out is None:
        out = torch.empty((n,), dtype=torch.int32, device=device)
    _need(out, torch.int32, "native")
    if out.numel() != n:
        raise ValueError(f"native must hold {n} words")
    return out


def w3_pack_native(codes: torch.Tensor, native: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """codes uint8 [N,K] (0..7) -> the native block order, int32 [w3_native_words(N, K)]."""
    _need(codes, torch.uint8, "codes")
    N, K = codes.shape
    native = _native_out(N, K, codes.device, native)
    _check(lib().w3_pack_native(codes.data_ptr(), native.data_ptr(), N, K, _stream(stream)), "w3_pack_native")
    return native


def w3_native_from_packed(packed: torch.Tensor, K: int, native: torch.Tensor | None = None, stream=None):
    """packed int32 [N, 3K/32] -> the native block order (a permutation of the words)."""
    _need(packed, torch.int32, "packed")
    N = packed.shape[0]
    if packed.shape[1] != w3_packed_words_per_row(K):
        raise ValueError("packed width does not match K")
    native = _native_out(N, K, packed.device, native)
    _check(lib().w3_native_from_packed(packed.data_ptr(), native.data_ptr(), N, K, _stream(stream)),
           "w3_native_from_packed")
    return native


def w3_packed_from_native(native: torch.Tensor, N: int, K: int, packed: torch.Tensor | None = None, stream=None):
    """The native block order -> packed int32 [N, 3K/32]."""
    _need(native, torch.int32, "native")
    if native.numel() != w3_native_words(N, K):
        raise ValueError("native size does not match N, K")
    if packed is None:
        packed = torch.empty((N, w3_packed_words_per_row(K)), dtype=torch.int32, device=native.device)
    _need(packed, torch.int32, "packed")
    _check(lib().w3_packed_from_native(native.data_ptr(), packed.data_ptr(), N, K, _stream(stream)),
           "w3_packed_from_native")
    return packed


def w3a16_gemm_native(x: torch.Tensor, native: torch.Tensor, scales: torch.Tensor, N: int,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x W^T with W in the native block order (decode batches, M <= 16)."""
    _need(x, torch.bfloat16, "x")
    _need(native, torch.int32, "native")
    _need(scales, torch.bfloat16, "scales")
    M, K = x.shape
    if native.numel() != w3_native_words(N, K) or tuple(scales.shape) != (N, w3_groups_per_row(K)):
        raise ValueError("native/scales sizes do not match N, K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, "out")
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be [M, N]")
    _check(lib().w3a16_gemm_native(x.data_ptr(), native.data_ptr(), scales.data_ptr(), out.data_ptr(), M, N, K,
                                   _stream(stream)), "w3a16_gemm_native")
    return out


def w3a16_gemm_route(M: int, N: int, K: int, num_sms: int | None = None) -> str:
    """The kernel route w3a16_gemm takes for M x N x K (see include/w3a16.h).  num_sms defaults to
    the current CUDA device's SM count; pass it explicitly to ask without a GPU."""
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    r = lib().w3a16_gemm_route(M, N, K, num_sms)
    if r is None:
        raise ValueError(f"w3a16_gemm_route: no route for M={M} N={N} K={K} num_sms={num_sms}")
    return r.decode()


def w3a16_gemm_launches(M: int, N: int, K: int, num_sms: int | None = None) -> int:
    """How many kernels one w3a16_gemm call launches for M x N x K (see include/w3a16.h).
    num_sms defaults to the current CUDA device's SM count."""
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    n = lib().w3a16_gemm_launches(M, N, K, num_sms)
    if n < 0:
        raise ValueError(f"w3a16_gemm_launches: no route for M={M} N={N} K={K} num_sms={num_sms}")
    return n


def w3_check_device_error(stream=None) -> None:
    """Synchronise the stream and raise W3Error if a kernel recorded a timeout."""
    _check(lib().w3_check_device_error(_stream(stream)), "w3_check_device_error")
