"""ctypes binding of libtq.so (declared in include/tq.h).

Argument marshalling only: every step of the append and decode path runs in
the library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  Importing this module loads ``libtq.so`` from the package directory
and raises ImportError when it has not been built (there is no CPU
fallback).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m quantized_paged_kv_tq_b200.build` "
        "(nvcc, sm_100a); there is no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

TQ_OK = 0
TQ_ERR_INVALID_ARG = 1
TQ_ERR_UNSUPPORTED = 2
TQ_ERR_CUDA = 3
TQ_ERR_TIMEOUT = 4
TQ_ERR_DEVICE_CHECK = 5
TQ_ERR_WORKSPACE = 6
TQ_ERR_NO_PAGES = 7

TQ_TURBO2, TQ_TURBO3, TQ_TURBO4, TQ_TURBO8, TQ_BF16 = 2, 3, 4, 8, 16
FORMATS = (TQ_TURBO2, TQ_TURBO3, TQ_TURBO4, TQ_TURBO8, TQ_BF16)

# every entry point include/tq.h declares
SYMBOLS = ("tq_abi_version", "tq_status_string", "tq_page_block_bytes",
           "tq_quantize_append", "tq_append_bf16", "tq_decode_workspace_size",
           "tq_decode_workspace_init", "tq_paged_decode", "tq_paged_decode_bf16",
           "tq_paged_decode_noalloc", "tq_read_device_error", "tq_hbm_copy", "tq_hbm_read",
           "tq_prefix_cache_create", "tq_prefix_cache_destroy", "tq_prefix_cache_begin",
           "tq_prefix_cache_extend", "tq_prefix_cache_finish", "tq_prefix_cache_stats",
           "tq_prefix_cache_page_refs", "tq_step_graph_create", "tq_step_graph_launch",
           "tq_step_graph_destroy")


class tq_cache(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("pages", ctypes.c_void_p),
                ("dev_error", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t
_CP = ctypes.POINTER(tq_cache)
_lib.tq_abi_version.restype = _I
_lib.tq_abi_version.argtypes = []
_lib.tq_status_string.restype = ctypes.c_char_p
_lib.tq_status_string.argtypes = [_I]
_lib.tq_page_block_bytes.restype = _S
_lib.tq_page_block_bytes.argtypes = [_I, _I, _I]
_lib.tq_quantize_append.restype = _I
_lib.tq_quantize_append.argtypes = [_P, _P, _P, _I, _I, _CP, _P]
_lib.tq_append_bf16.restype = _I
_lib.tq_append_bf16.argtypes = [_P, _P, _P, _I, _CP, _P]
_lib.tq_decode_workspace_size.restype = _S
_lib.tq_decode_workspace_size.argtypes = [_I, _I, _I, _I, _CP]
_lib.tq_decode_workspace_init.restype = _I
_lib.tq_decode_workspace_init.argtypes = [_P, _S, _P]
for _name in ("tq_paged_decode", "tq_paged_decode_bf16"):
    getattr(_lib, _name).restype = _I
    getattr(_lib, _name).argtypes = [_P, _CP, _P, _I, _P, _I, _I, _I, _I, _P, _P, _S, _P]
_lib.tq_paged_decode_noalloc.restype = _I
_lib.tq_paged_decode_noalloc.argtypes = [_P, _CP, _P, _I, _P, _I, _I, _I, _I, _P, _P]
_lib.tq_read_device_error.restype = _I
_lib.tq_read_device_error.argtypes = [_CP, ctypes.POINTER(ctypes.c_uint32), _I, _P]
_lib.tq_hbm_copy.restype = _I
_lib.tq_hbm_copy.argtypes = [_P, _P, _S, _P]
_lib.tq_hbm_read.restype = _I
_lib.tq_hbm_read.argtypes = [_P, _S, _P, _P]


class tq_step(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("slot_mapping", ctypes.c_void_p), ("num_tokens", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("max_pages_per_seq", ctypes.c_int32), ("seq_lens", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("q_len", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
                ("out", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


_lib.tq_step_graph_create.restype = _I
_lib.tq_step_graph_create.argtypes = [_CP, ctypes.POINTER(tq_step), _P, ctypes.POINTER(_P)]
_lib.tq_step_graph_launch.restype = _I
_lib.tq_step_graph_launch.argtypes = [_P, _P]
_lib.tq_step_graph_destroy.restype = None
_lib.tq_step_graph_destroy.argtypes = [_P]


class tq_prefix_stats(ctypes.Structure):
    _fields_ = [("free_pages", ctypes.c_int64), ("cached_blocks", ctypes.c_int64),
                ("live_sequences", ctypes.c_int64), ("hit_tokens", ctypes.c_int64),
                ("prompt_tokens", ctypes.c_int64), ("evictions", ctypes.c_int64)]


_IP = ctypes.POINTER(ctypes.c_int32)
_lib.tq_prefix_cache_create.restype = _P
_lib.tq_prefix_cache_create.argtypes = [_I, _I, ctypes.c_int64]
_lib.tq_prefix_cache_destroy.restype = None
_lib.tq_prefix_cache_destroy.argtypes = [_P]
_lib.tq_prefix_cache_begin.restype = _I
_lib.tq_prefix_cache_begin.argtypes = [_P, _IP, _I, _IP, _I, _IP, _IP]
_lib.tq_prefix_cache_extend.restype = _I
_lib.tq_prefix_cache_extend.argtypes = [_P, _I, _I, _IP, _I]
_lib.tq_prefix_cache_finish.restype = _I
_lib.tq_prefix_cache_finish.argtypes = [_P, _I, _IP, _I]
_lib.tq_prefix_cache_stats.restype = _I
_lib.tq_prefix_cache_stats.argtypes = [_P, ctypes.POINTER(tq_prefix_stats)]
_lib.tq_prefix_cache_page_refs.restype = _I
_lib.tq_prefix_cache_page_refs.argtypes = [_P, _I]


class TqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    return _lib


def abi_version() -> int:
    return _lib.tq_abi_version()


def status_string(status: int) -> str:
    return _lib.tq_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != TQ_OK:
        raise TqError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def tq_page_block_bytes(fmt: int, head_dim: int = 128, page_size: int = 16) -> int:
    return int(_lib.tq_page_block_bytes(fmt, head_dim, page_size))


class Cache:
    """Paged K/V pool of one layer plus its C descriptor.

    ``pages`` is a zeroed torch uint8 tensor [num_pages][num_kv_heads][2][block]
    (the K block, then the V block); ``k_pages`` and ``v_pages`` are its
    [num_pages][num_kv_heads][block] views.  ``dev_error`` is a one-word int32 tensor
    the kernels report to.
    """

    def __init__(self, fmt: int, num_pages: int, num_kv_heads: int, page_size: int = 16,
                 head_dim: int = 128, device="cuda"):
        bb = tq_page_block_bytes(fmt, head_dim, page_size)
        if bb == 0:
            raise ValueError("unsupported cache shape")
        self.format, self.num_pages, self.num_kv_heads = fmt, num_pages, num_kv_heads
        self.page_size, self.head_dim, self.block_bytes = page_size, head_dim, bb
        # one pool [page][kv head][K block, V block]; k_pages / v_pages are views
        self.pages = torch.zeros((num_pages, num_kv_heads, 2, bb), dtype=torch.uint8,
                                 device=device)
        self.k_pages = self.pages[:, :, 0]
        self.v_pages = self.pages[:, :, 1]
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=device)
        self.desc = tq_cache(fmt, head_dim, num_kv_heads, page_size, num_pages,
                             self.pages.data_ptr(), self.dev_error.data_ptr())
        self._ws = None

    def workspace(self, batch: int, q_len: int, num_q_heads: int, max_seq_len: int,
                  stream=None):
        n = tq_decode_workspace_size(batch, q_len, num_q_heads, max_seq_len, self)
        if n == 0:
            return None
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.k_pages.device)
            tq_decode_workspace_init(self._ws, stream)
        return self._ws

    def read_error(self, clear: bool = True, stream=None) -> int:
        return tq_read_device_error(self, clear, stream)


def _desc(cache) -> tq_cache:
    return cache.desc if isinstance(cache, Cache) else cache


def tq_quantize_append(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, bits: int,
                       cache, stream=None) -> None:
    """Rotate, quantise, pack and store new K/V rows ([T][Hkv][128] bf16)."""
    T = k.shape[0] if k.dim() else 0
    _check(_lib.tq_quantize_append(_dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"),
                                   _dev(slot_mapping, torch.int64, "slot_mapping"), T, bits,
                                   ctypes.byref(_desc(cache)), _stream(stream)),
           "tq_quantize_append")


def tq_append_bf16(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, cache,
                   stream=None) -> None:
    T = k.shape[0] if k.dim() else 0
    _check(_lib.tq_append_bf16(_dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"),
                               _dev(slot_mapping, torch.int64, "slot_mapping"), T,
                               ctypes.byref(_desc(cache)), _stream(stream)),
           "tq_append_bf16")


def tq_decode_workspace_size(batch: int, q_len: int, num_q_heads: int, max_seq_len: int,
                             cache) -> int:
    return int(_lib.tq_decode_workspace_size(batch, q_len, num_q_heads, max_seq_len,
                                             ctypes.byref(_desc(cache))))


def tq_decode_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(_lib.tq_decode_workspace_init(workspace.data_ptr(), workspace.numel(),
                                         _stream(stream)), "tq_decode_workspace_init")


def _decode(fn, name, q, cache, page_table, seq_lens, q_len, out, max_seq_len, workspace,
            stream):
    B = q.shape[0]
    Hq = q.shape[2]
    if q.shape[1] != q_len:
        raise ValueError("q must be [batch][q_len][num_q_heads][head_dim]")
    if max_seq_len is None:
        raise ValueError("max_seq_len (a host bound on seq_lens) is required")
    if workspace is None and isinstance(cache, Cache):
        workspace = cache.workspace(B, q_len, Hq, max_seq_len, stream)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_n = workspace.numel() if workspace is not None else 0
    _check(fn(_dev(q, torch.bfloat16, "q"), ctypes.byref(_desc(cache)),
              _dev(page_table, torch.int32, "page_table"), page_table.shape[1],
              _dev(seq_lens, torch.int32, "seq_lens"), B, q_len, Hq, max_seq_len,
              _dev(out, torch.float32, "out"), ws_ptr, ws_n, _stream(stream)), name)


def tq_paged_decode(q, cache, page_table, seq_lens, q_len, out, max_seq_len=None,
                    workspace=None, stream=None) -> None:
    """Decode attention over a turbo cache; out[b][t][h][:] fp32."""
    _decode(_lib.tq_paged_decode, "tq_paged_decode", q, cache, page_table, seq_lens, q_len,
            out, max_seq_len, workspace, stream)


def tq_paged_decode_bf16(q, cache, page_table, seq_lens, q_len, out, max_seq_len=None,
                         workspace=None, stream=None) -> None:
    """The same decode over a bf16 cache (uncompressed reference point)."""
    _decode(_lib.tq_paged_decode_bf16, "tq_paged_decode_bf16", q, cache, page_table, seq_lens,
            q_len, out, max_seq_len, workspace, stream)


def tq_paged_decode_noalloc(q, cache, page_table, seq_lens, q_len, out, max_seq_len,
                            stream=None) -> None:
    """tq_paged_decode without a workspace argument, for callers that may not
    allocate device memory while running: the scratch is a fixed 64 MiB array
    inside libtq.so (shared by all calls, so overlapping calls on one GPU
    must be serialised by the caller)."""
    if q.shape[1] != q_len:
        raise ValueError("q must be [batch][q_len][num_q_heads][head_dim]")
    _check(_lib.tq_paged_decode_noalloc(
        _dev(q, torch.bfloat16, "q"), ctypes.byref(_desc(cache)),
        _dev(page_table, torch.int32, "page_table"), page_table.shape[1],
        _dev(seq_lens, torch.int32, "seq_lens"), q.shape[0], q_len, q.shape[2], max_seq_len,
        _dev(out, torch.float32, "out"), _stream(stream)), "tq_paged_decode_noalloc")


def tq_read_device_error(cache, clear: bool = True, stream=None) -> int:
    code = ctypes.c_uint32(0)
    _check(_lib.tq_read_device_error(ctypes.byref(_desc(cache)), ctypes.byref(code),
                                     int(clear), _stream(stream)), "tq_read_device_error")
    return code.value


def tq_hbm_copy(src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    _check(_lib.tq_hbm_copy(src.data_ptr(), dst.data_ptr(), src.numel() * src.element_size(),
                            _stream(stream)), "tq_hbm_copy")


def tq_hbm_read(src: torch.Tensor, sink: torch.Tensor, stream=None) -> None:
    _check(_lib.tq_hbm_read(src.data_ptr(), src.numel() * src.element_size(), sink.data_ptr(),
                            _stream(stream)), "tq_hbm_read")


class PrefixCache:
    """Host-side prefix-block manager of a pool of `num_pages` pages
    (tq_prefix_cache_* in include/tq.h).  Token ids are int32; page tables
    come back as numpy int32 arrays for the caller to copy to the device."""

    def __init__(self, num_pages: int, page_size: int = 16, max_cached_tokens: int = 0):
        self.page_size = page_size
        self.h = _lib.tq_prefix_cache_create(num_pages, page_size, max_cached_tokens)
        if not self.h:
            raise ValueError("tq_prefix_cache_create failed")

    def __del__(self):
        h = getattr(self, "h", None)
        if h:
            _lib.tq_prefix_cache_destroy(h)
            self.h = None

    @staticmethod
    def _ids(tokens):
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        return t, t.ctypes.data_as(_IP)

    def begin(self, tokens, max_pages: int):
        """(seq handle, cached token count, page table int32 [n pages])."""
        import numpy as np
        t, tp = self._ids(tokens)
        pt = np.full(max_pages, -1, np.int32)
        cached = ctypes.c_int32(0)
        seq = ctypes.c_int32(-1)
        _check(_lib.tq_prefix_cache_begin(self.h, tp, len(t), pt.ctypes.data_as(_IP), max_pages,
                                          ctypes.byref(cached), ctypes.byref(seq)),
               "tq_prefix_cache_begin")
        n = -(-len(t) // self.page_size)
        return seq.value, cached.value, pt[:n].copy()

    def extend(self, seq: int, new_len: int, max_pages: int):
        import numpy as np
        pt = np.full(max_pages, -1, np.int32)
        _check(_lib.tq_prefix_cache_extend(self.h, seq, new_len, pt.ctypes.data_as(_IP),
                                           max_pages), "tq_prefix_cache_extend")
        return pt[:-(-new_len // self.page_size)].copy()

    def finish(self, seq: int, tokens) -> None:
        t, tp = self._ids(tokens)
        _check(_lib.tq_prefix_cache_finish(self.h, seq, tp, len(t)), "tq_prefix_cache_finish")

    def stats(self) -> dict:
        st = tq_prefix_stats()
        _check(_lib.tq_prefix_cache_stats(self.h, ctypes.byref(st)), "tq_prefix_cache_stats")
        return {name: getattr(st, name) for name, _ in tq_prefix_stats._fields_}

    def page_refs(self, page: int) -> int:
        return _lib.tq_prefix_cache_page_refs(self.h, page)


class StepGraph:
    """One append + decode step captured as a CUDA graph on `stream` (a
    torch.cuda.Stream, not the default stream) with the given tensors fixed;
    refresh the tensors' contents between launch() calls."""

    def __init__(self, cache, stream, q, page_table, seq_lens, q_len, out, max_seq_len,
                 k=None, v=None, slot_mapping=None, workspace=None):
        B = q.shape[0]
        if workspace is None and isinstance(cache, Cache):
            workspace = cache.workspace(B, q_len, q.shape[2], max_seq_len)
        T = k.shape[0] if k is not None else 0
        self.step = tq_step(
            k.data_ptr() if T else None, v.data_ptr() if T else None,
            slot_mapping.data_ptr() if T else None, T,
            _dev(q, torch.bfloat16, "q"), _dev(page_table, torch.int32, "page_table"),
            page_table.shape[1], _dev(seq_lens, torch.int32, "seq_lens"), B, q_len, q.shape[2],
            max_seq_len, _dev(out, torch.float32, "out"),
            workspace.data_ptr() if workspace is not None else None,
            workspace.numel() if workspace is not None else 0)
        self._keep = (cache, q, page_table, seq_lens, out, k, v, slot_mapping, workspace)
        h = ctypes.c_void_p()
        _check(_lib.tq_step_graph_create(ctypes.byref(_desc(cache)), ctypes.byref(self.step),
                                         _stream(stream), ctypes.byref(h)),
               "tq_step_graph_create")
        self.h = h.value

    def launch(self, stream=None) -> None:
        _check(_lib.tq_step_graph_launch(self.h, _stream(stream)), "tq_step_graph_launch")

    def __del__(self):
        h = getattr(self, "h", None)
        if h:
            _lib.tq_step_graph_destroy(h)
            self.h = None
