"""CPU oracle for the W3A16 group-128 format (test infrastructure only).

This package is the reference the CUDA library is checked against.  It is used
only by ``tests/``, by ``__graft_entry__.smoke()`` and by the CPU-baseline leg of
``bench.py``; the product path (``w3a16_gemv_b200``) never imports it.  It shares
no code with the CUDA kernels.  The arithmetic lives in ``w3_oracle.c`` (plain
C, bit-level pack/unpack, exact fp32 dequantization, fp64 triple loop); this
module only compiles it with the host C compiler and marshals numpy arrays.

Format followed: the GSQ model card "Llama-3.1-70B-Instruct-3Bit-GSQ", section
"Storage layout (why the HF UI shows I32 + BF16)" -- uint3 codes packed with
exact width ([N, K] -> [N, 3K/32] int32), bf16 scales [N, K/128], symmetric with
no zero point; section "Quantization details" -- group size 128 and the GSQ
5-level codebook {-2..2} x scale.  The bit order (LSB-first bitstream per row)
and the signed level q = c - 4 are readings stated in ``w3_oracle.c``.

Every function is pinned by ``tests/test_oracle_pins.py`` against facts the
card fixes and against closed forms and brute force; none of its pins re-types
its own formula.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

GROUP = 128

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w3_oracle.c")
_LIB = os.path.join(_HERE, "libw3oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``w3_oracle.c`` into ``libw3oracle.so`` with the host C compiler."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-fopenmp", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load the compiled oracle (building it first if needed) and declare its signatures."""
    global _lib
    with _lock:
        if path is None and _lib is not None:
            return _lib
        lib = ctypes.CDLL(path or build())
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_words_per_row.argtypes = [i64]
        lib.oracle_words_per_row.restype = i64
        lib.oracle_groups_per_row.argtypes = [i64]
        lib.oracle_groups_per_row.restype = i64
        for name, nargs in (("oracle_pack", 2), ("oracle_unpack", 2)):
            f = getattr(lib, name)
            f.argtypes = [p] * nargs + [i64, i64]
            f.restype = ctypes.c_int
        lib.oracle_dequant_f32.argtypes = [p, p, p, i64, i64]
        lib.oracle_dequant_f32.restype = ctypes.c_int
        lib.oracle_gemm_f64.argtypes = [p, p, p, p, i64, i64, i64]
        lib.oracle_gemm_f64.restype = ctypes.c_int
        lib.oracle_gemm_f64_threads.argtypes = [p, p, p, p, i64, i64, i64, ctypes.c_int]
        lib.oracle_gemm_f64_threads.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_gemm_f64_entries.argtypes = [p, p, p, i64, i64, i64, p, p, i64, p]
        lib.oracle_gemm_f64_entries.restype = ctypes.c_int
        lib.oracle_weight_row_norms.argtypes = [p, p, i64, i64, p]
        lib.oracle_weight_row_norms.restype = ctypes.c_int
        lib.oracle_native_words.argtypes = [i64, i64]
        lib.oracle_native_words.restype = i64
        for name in ("oracle_native_from_packed", "oracle_packed_from_native"):
            f = getattr(lib, name)
            f.argtypes = [p, p, i64, i64]
            f.restype = ctypes.c_int
        lib.oracle_ct4_words_per_row.argtypes = [i64]
        lib.oracle_ct4_words_per_row.restype = i64
        lib.oracle_pack_ct4.argtypes = [p, p, i64, i64]
        lib.oracle_pack_ct4.restype = ctypes.c_int
        lib.oracle_repack_ct4.argtypes = [p, p, i64, i64, p]
        lib.oracle_repack_ct4.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"{what}: invalid argument")


class Oracle:
    """Numpy front end over one loaded copy of the oracle library."""

    def __init__(self, lib: ctypes.CDLL | None = None):
        self.lib = lib if lib is not None else load_library()

    def words_per_row(self, K: int) -> int:
        return int(self.lib.oracle_words_per_row(K))

    def groups_per_row(self, K: int) -> int:
        return int(self.lib.oracle_groups_per_row(K))

    def pack(self, codes: np.ndarray) -> np.ndarray:
        """codes uint8 [N,K] (0..7) -> packed uint32 [N, 3K/32]."""
        codes = _c(codes, np.uint8)
        N, K = codes.shape
        out = np.empty((N, max(self.words_per_row(K), 0)), dtype=np.uint32)
        _check(self.lib.oracle_pack(_ptr(codes), _ptr(out), N, K), "oracle_pack")
        return out

    def unpack(self, packed: np.ndarray, K: int) -> np.ndarray:
        """packed uint32 [N, 3K/32] -> codes uint8 [N,K]."""
        packed = _c(packed.view(np.uint32), np.uint32)
        N = packed.shape[0]
        if packed.shape[1] != self.words_per_row(K):
            raise ValueError("packed width does not match K")
        out = np.empty((N, K), dtype=np.uint8)
        _check(self.lib.oracle_unpack(_ptr(packed), _ptr(out), N, K), "oracle_unpack")
        return out

    def native_words(self, N: int, K: int) -> int:
        """Words of the kernel-native block layout of an N x K weight (rows padded to 32)."""
        return int(self.lib.oracle_native_words(N, K))

    def native_from_packed(self, packed: np.ndarray, K: int) -> np.ndarray:
        """packed uint32 [N, 3K/32] (row order) -> the native block order, uint32 [native_words]."""
        packed = _c(packed.view(np.uint32), np.uint32)
        N = packed.shape[0]
        if packed.shape[1] != self.words_per_row(K):
            raise ValueError("packed width does not match K")
        out = np.empty(max(self.native_words(N, K), 0), dtype=np.uint32)
        _check(self.lib.oracle_native_from_packed(_ptr(packed), _ptr(out), N, K), "oracle_native_from_packed")
        return out

    def packed_from_native(self, native: np.ndarray, N: int, K: int) -> np.ndarray:
        """The inverse: native block order -> packed uint32 [N, 3K/32]."""
        native = _c(native.view(np.uint32), np.uint32)
        if native.size != self.native_words(N, K):
            raise ValueError("native size does not match N, K")
        out = np.empty((N, max(self.words_per_row(K), 0)), dtype=np.uint32)
        _check(self.lib.oracle_packed_from_native(_ptr(native), _ptr(out), N, K), "oracle_packed_from_native")
        return out

    def ct4_words_per_row(self, K: int) -> int:
        return int(self.lib.oracle_ct4_words_per_row(K))

    def pack_ct4(self, codes: np.ndarray) -> np.ndarray:
        """codes uint8 [N,K] (0..7) -> 4-bit container uint32 [N, K/8] (level + 8 per nibble, LSB first)."""
        codes = _c(codes, np.uint8)
        N, K = codes.shape
        out = np.empty((N, max(self.ct4_words_per_row(K), 0)), dtype=np.uint32)
        _check(self.lib.oracle_pack_ct4(_ptr(codes), _ptr(out), N, K), "oracle_pack_ct4")
        return out

    def repack_ct4(self, ct4: np.ndarray, K: int) -> tuple[np.ndarray, int]:
        """4-bit container uint32 [N, K/8] -> (exact-width packed uint32 [N, 3K/32], levels clamped)."""
        ct4 = _c(ct4.view(np.uint32), np.uint32)
        N = ct4.shape[0]
        if ct4.shape[1] != self.ct4_words_per_row(K):
            raise ValueError("container width does not match K")
        out = np.empty((N, max(self.words_per_row(K), 0)), dtype=np.uint32)
        count = np.zeros(1, dtype=np.int64)
        _check(self.lib.oracle_repack_ct4(_ptr(ct4), _ptr(out), N, K, _ptr(count)), "oracle_repack_ct4")
        return out, int(count[0])

    def dequant_f32(self, packed: np.ndarray, scales_bf16: np.ndarray, K: int) -> np.ndarray:
        """W[n,k] = (c-4) * s[n,k//128] as fp32 [N,K] (exact)."""
        packed = _c(packed.view(np.uint32), np.uint32)
        scales_bf16 = _c(scales_bf16.view(np.uint16), np.uint16)
        N = packed.shape[0]
        self._shapes(packed, scales_bf16, N, K)
        out = np.empty((N, K), dtype=np.float32)
        _check(self.lib.oracle_dequant_f32(_ptr(packed), _ptr(scales_bf16), _ptr(out), N, K),
               "oracle_dequant_f32")
        return out

    def max_threads(self) -> int:
        """Threads a multi-threaded call uses by default (all cores)."""
        return int(self.lib.oracle_max_threads())

    def gemm_f64(self, x_bf16: np.ndarray, packed: np.ndarray, scales_bf16: np.ndarray,
                 threads: int | None = None) -> np.ndarray:
        """y = x W^T in fp64, [M,N].  threads: None = one thread; 0 = all cores; n = n threads
        (rows n spread over threads; every element is the same k-ordered fp64 sum)."""
        x_bf16 = _c(x_bf16.view(np.uint16), np.uint16)
        packed = _c(packed.view(np.uint32), np.uint32)
        scales_bf16 = _c(scales_bf16.view(np.uint16), np.uint16)
        M, K = x_bf16.shape
        N = packed.shape[0]
        self._shapes(packed, scales_bf16, N, K)
        out = np.empty((M, N), dtype=np.float64)
        if threads is None:
            _check(self.lib.oracle_gemm_f64(_ptr(x_bf16), _ptr(packed), _ptr(scales_bf16), _ptr(out), M, N, K),
                   "oracle_gemm_f64")
        else:
            _check(self.lib.oracle_gemm_f64_threads(_ptr(x_bf16), _ptr(packed), _ptr(scales_bf16), _ptr(out),
                                                    M, N, K, int(threads)), "oracle_gemm_f64_threads")
        return out

    def gemm_f64_entries(self, x_bf16, packed, scales_bf16, ms, ns) -> np.ndarray:
        """y[ms[i], ns[i]] for each i, fp64."""
        x_bf16 = _c(x_bf16.view(np.uint16), np.uint16)
        packed = _c(packed.view(np.uint32), np.uint32)
        scales_bf16 = _c(scales_bf16.view(np.uint16), np.uint16)
        ms = _c(np.asarray(ms, dtype=np.int64), np.int64)
        ns = _c(np.asarray(ns, dtype=np.int64), np.int64)
        M, K = x_bf16.shape
        N = packed.shape[0]
        self._shapes(packed, scales_bf16, N, K)
        out = np.empty(ms.shape[0], dtype=np.float64)
        _check(self.lib.oracle_gemm_f64_entries(_ptr(x_bf16), _ptr(packed), _ptr(scales_bf16), M, N, K,
                                                _ptr(ms), _ptr(ns), ms.shape[0], _ptr(out)),
               "oracle_gemm_f64_entries")
        return out

    def weight_row_norms(self, packed: np.ndarray, scales_bf16: np.ndarray, K: int) -> np.ndarray:
        """||W[n,:]||_2 in fp64, [N]."""
        packed = _c(packed.view(np.uint32), np.uint32)
        scales_bf16 = _c(scales_bf16.view(np.uint16), np.uint16)
        N = packed.shape[0]
        self._shapes(packed, scales_bf16, N, K)
        out = np.empty(N, dtype=np.float64)
        _check(self.lib.oracle_weight_row_norms(_ptr(packed), _ptr(scales_bf16), N, K, _ptr(out)),
               "oracle_weight_row_norms")
        return out

    def _shapes(self, packed, scales, N, K):
        if packed.shape != (N, self.words_per_row(K)):
            raise ValueError(f"packed shape {packed.shape} does not match N={N}, K={K}")
        if scales.shape != (N, self.groups_per_row(K)):
            raise ValueError(f"scales shape {scales.shape} does not match N={N}, K={K}")


_default: Oracle | None = None


def get() -> Oracle:
    """The process-wide oracle instance."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    u = np.ascontiguousarray(a).view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
