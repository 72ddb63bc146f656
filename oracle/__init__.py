"""CPU oracle for the TurboQuant paged KV cache -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (``libtq.so`` and
``quantized_paged_kv_tq_b200``) never imports it and shares no code with it.

The arithmetic lives in ``tq_oracle.c`` (plain single-threaded C, built with
``-ffp-contract=off``: fp32 quantiser, fp64 attention); this module only
marshals numpy arrays through ctypes.  Method source: "xInfer: Pure-Rust LLM
Inference Without a Python Runtime", sections "What actually sits between the
request and the tokens" (Walsh-Hadamard rotation + per-head absmax
quantisation) and "TurboQuant is a memory trade" (dequantise on every
attention step).

Parity pins: every function below is pinned by ``tests/test_oracle_pins.py``
against closed forms, library routines (scipy's Hadamard matrix, numpy's
bit packing, torch's scaled_dot_product_attention in fp64) and hand-derived
fixtures in ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "libtq_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra"]

FORMAT_BITS = {2: 2, 3: 3, 4: 4, 8: 8, 16: 0, 17: 8}
FP8 = 17          # the fp8 (E4M3) format id


def build(force: bool = False) -> str:
    """Compile tq_oracle.c into libtq_oracle.so (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or (
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC)):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        _lib.oracle_block_bytes.restype = ctypes.c_int64
        _lib.oracle_block_bytes.argtypes = [I, I, I]
        for name in ("oracle_fwht_f32", "oracle_fwht_f64"):
            getattr(_lib, name).argtypes = [P, I]
            getattr(_lib, name).restype = None
        _lib.oracle_rotate_f32.argtypes = [P, I, P]
        _lib.oracle_rotate_f32.restype = None
        _lib.oracle_quantize_rotated.argtypes = [P, I, I, P, P]
        _lib.oracle_quantize_rotated.restype = None
        _lib.oracle_pack_codes.argtypes = [P, I, I, P]
        _lib.oracle_pack_codes.restype = None
        _lib.oracle_unpack_codes.argtypes = [P, I, I, P]
        _lib.oracle_unpack_codes.restype = None
        _lib.oracle_quantize_vector.argtypes = [P, I, I, P, P]
        _lib.oracle_quantize_vector.restype = None
        _lib.oracle_quantize_append.argtypes = [P, P, P, I, I, I, I, I, I, P, P]
        _lib.oracle_quantize_append.restype = I
        _lib.oracle_append_bf16.argtypes = [P, P, P, I, I, I, I, I, P, P]
        _lib.oracle_append_bf16.restype = I
        _lib.oracle_paged_decode.argtypes = [P, I, I, I, I, I, P, P, P, I, P,
                                             I, I, I, P]
        _lib.oracle_paged_decode.restype = I
        _lib.oracle_attention_f64.argtypes = [P, P, P, I, I, I, P]
        _lib.oracle_attention_f64.restype = None
        _lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_value.restype = ctypes.c_double
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        _lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        _lib.oracle_fp8_quantize_vector.argtypes = [P, I, P, P]
        _lib.oracle_fp8_quantize_vector.restype = None
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def block_bytes(fmt: int, d: int, page_size: int) -> int:
    return int(lib().oracle_block_bytes(fmt, d, page_size))


def fwht_f32(x) -> np.ndarray:
    """Unnormalised Sylvester WHT in fp32 (copy)."""
    y = _c(x, np.float32).copy()
    lib().oracle_fwht_f32(_ptr(y), y.shape[-1])
    return y


def fwht_f64(x) -> np.ndarray:
    y = _c(x, np.float64).copy()
    lib().oracle_fwht_f64(_ptr(y), y.shape[-1])
    return y


def rotate_f32(x_bf16) -> np.ndarray:
    """y = H x / sqrt(d) in fp32 for one bf16 vector given as uint16 bits."""
    x = _c(x_bf16, np.uint16)
    y = np.empty(x.shape[-1], np.float32)
    lib().oracle_rotate_f32(_ptr(x), x.shape[-1], _ptr(y))
    return y


def quantize_rotated(y, bits: int):
    """(codes int32[d], scale fp32) of an already-rotated fp32 vector."""
    y = _c(y, np.float32)
    codes = np.empty(y.shape[-1], np.int32)
    s = np.zeros(1, np.float32)
    lib().oracle_quantize_rotated(_ptr(y), y.shape[-1], bits, _ptr(codes), _ptr(s))
    return codes, s[0]


def pack_codes(codes, bits: int) -> np.ndarray:
    codes = _c(codes, np.int32)
    d = codes.shape[-1]
    out = np.empty(d * bits // 8, np.uint8)
    lib().oracle_pack_codes(_ptr(codes), d, bits, _ptr(out))
    return out


def unpack_codes(packed, d: int, bits: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    codes = np.empty(d, np.int32)
    lib().oracle_unpack_codes(_ptr(packed), d, bits, _ptr(codes))
    return codes


def quantize_vector(x_bf16, bits: int):
    """(packed bytes, scale) of one bf16 head vector: rotate, quantise, pack."""
    x = _c(x_bf16, np.uint16)
    d = x.shape[-1]
    out = np.empty(d * bits // 8, np.uint8)
    s = np.zeros(1, np.float32)
    lib().oracle_quantize_vector(_ptr(x), d, bits, _ptr(out), _ptr(s))
    return out, s[0]


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(code))


def e4m3_encode(y: float) -> int:
    return int(lib().oracle_e4m3_encode(y))


def fp8_quantize_vector(x_bf16):
    """(E4M3 code bytes, fp32 scale) of one bf16 head vector (no rotation)."""
    x = _c(x_bf16, np.uint16)
    out = np.empty(x.shape[-1], np.uint8)
    s = np.zeros(1, np.float32)
    lib().oracle_fp8_quantize_vector(_ptr(x), x.shape[-1], _ptr(out), _ptr(s))
    return out, s[0]


def quantize_append(k_bf16, v_bf16, slot_mapping, bits: int, page_size: int,
                    k_pages: np.ndarray, v_pages: np.ndarray) -> None:
    """Append into uint8 page pools shaped [num_pages][num_kv_heads][block];
    `bits` is the format: 2, 3, 4, 8 (turbo) or FP8 (17)."""
    k = _c(k_bf16, np.uint16)
    v = _c(v_bf16, np.uint16)
    slots = _c(slot_mapping, np.int64)
    T, H, d = k.shape
    num_pages = k_pages.shape[0]
    rc = lib().oracle_quantize_append(_ptr(k), _ptr(v), _ptr(slots), T, H, d,
                                      bits, page_size, num_pages,
                                      _ptr(k_pages), _ptr(v_pages))
    if rc:
        raise ValueError(f"oracle_quantize_append failed: {rc}")


def append_bf16(k_bf16, v_bf16, slot_mapping, page_size: int,
                k_pages: np.ndarray, v_pages: np.ndarray) -> None:
    """Append into uint16 pools shaped [num_pages][num_kv_heads][P][d]."""
    k = _c(k_bf16, np.uint16)
    v = _c(v_bf16, np.uint16)
    slots = _c(slot_mapping, np.int64)
    T, H, d = k.shape
    rc = lib().oracle_append_bf16(_ptr(k), _ptr(v), _ptr(slots), T, H, d,
                                  page_size, k_pages.shape[0], _ptr(k_pages),
                                  _ptr(v_pages))
    if rc:
        raise ValueError(f"oracle_append_bf16 failed: {rc}")


def attention_f64(q, K, V, rotated: bool) -> np.ndarray:
    """One query row over n keys (fp64); rotated=True attends in the
    Hadamard basis: K, V already rotated, q rotated and the output rotated
    back inside."""
    q = _c(q, np.float64)
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    n, d = K.shape
    out = np.empty(d, np.float64)
    lib().oracle_attention_f64(_ptr(q), _ptr(K), _ptr(V), n, d, int(rotated),
                               _ptr(out))
    return out


def paged_decode(q_bf16, fmt: int, page_size: int, k_pages: np.ndarray,
                 v_pages: np.ndarray, page_table, seq_lens,
                 num_kv_heads: int) -> np.ndarray:
    """fp64 attention output [batch][q_len][num_q_heads][d]."""
    q = _c(q_bf16, np.uint16)
    B, q_len, Hq, d = q.shape
    pt = _c(page_table, np.int32)
    sl = _c(seq_lens, np.int32)
    assert pt.shape[0] == B and sl.shape[0] == B
    out = np.zeros((B, q_len, Hq, d), np.float64)
    rc = lib().oracle_paged_decode(_ptr(q), fmt, d, num_kv_heads, page_size,
                                   k_pages.shape[0], _ptr(k_pages),
                                   _ptr(v_pages), _ptr(pt), pt.shape[1],
                                   _ptr(sl), B, q_len, Hq, _ptr(out))
    if rc:
        raise ValueError(f"oracle_paged_decode failed: {rc}")
    return out
