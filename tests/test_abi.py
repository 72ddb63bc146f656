"""The C ABI on the host (no GPU): symbols, sizes, status codes.

Every call here fails host validation or is a documented no-op, so nothing
reaches the CUDA runtime."""
import ctypes
import os
import re

import pytest

from conftest import ROOT
from quantized_paged_kv_tq_b200 import build as tqbuild

tqbuild.build()
from quantized_paged_kv_tq_b200 import tq  # noqa: E402


def header_functions():
    with open(os.path.join(ROOT, "include", "tq.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_header_and_binding_agree():
    assert header_functions() == sorted(tq.SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(tq.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name


def test_abi_version_and_strings():
    assert tq.abi_version() == 3
    for s in range(8):
        assert tq.status_string(s).startswith("TQ_")
    assert tq.status_string(99) == "TQ_ERR_UNKNOWN"


def test_block_bytes():
    # page of 16 tokens: d*b/8 code bytes + a 4-byte scale per token
    assert tq.tq_page_block_bytes(tq.TQ_TURBO4, 128, 16) == 16 * 68
    assert tq.tq_page_block_bytes(tq.TQ_TURBO3, 128, 16) == 16 * 52
    assert tq.tq_page_block_bytes(tq.TQ_TURBO8, 128, 16) == 16 * 132
    assert tq.tq_page_block_bytes(tq.TQ_TURBO2, 128, 64) == 64 * 36
    assert tq.tq_page_block_bytes(tq.TQ_BF16, 128, 16) == 16 * 256
    assert tq.tq_page_block_bytes(tq.TQ_TURBO4, 64, 16) == 0
    assert tq.tq_page_block_bytes(tq.TQ_TURBO4, 128, 24) == 0
    assert tq.tq_page_block_bytes(5, 128, 16) == 0
    for fmt in tq.FORMATS:
        for P in (16, 32, 64):
            assert tq.tq_page_block_bytes(fmt, 128, P) % 16 == 0


FAKE = 0x10000  # never dereferenced: every call below stops in host checks


def desc(fmt=4, d=128, H=8, P=16, pages=10, kv=FAKE, err=None):
    return tq.tq_cache(fmt, d, H, P, pages, kv, err)


def qa(c, k=FAKE, v=FAKE, s=FAKE, n=4, bits=None):
    return tq.lib().tq_quantize_append(k, v, s, n, c.format if bits is None else bits,
                                       ctypes.byref(c), None)


def test_quantize_append_validation():
    I, U = tq.TQ_ERR_INVALID_ARG, tq.TQ_ERR_UNSUPPORTED
    assert tq.lib().tq_quantize_append(FAKE, FAKE, FAKE, 4, 4, None, None) == I
    assert qa(desc(fmt=16)) == I                      # bf16 cache
    assert qa(desc(fmt=5)) == I                       # unknown format
    assert qa(desc(), bits=3) == I                    # bits != cache format
    assert qa(desc(d=64)) == U
    assert qa(desc(P=24)) == U
    assert qa(desc(H=0)) == I
    assert qa(desc(pages=0)) == I
    assert qa(desc(kv=None)) == I
    assert qa(desc(kv=FAKE + 8)) == I                 # 16-byte alignment
    assert qa(desc(), k=None) == I
    assert qa(desc(), v=FAKE + 2) == I
    assert qa(desc(), s=FAKE + 4) == I
    assert qa(desc(), n=-1) == I
    assert qa(desc(), n=0) == tq.TQ_OK                # no-op, nothing launched
    assert tq.lib().tq_append_bf16(FAKE, FAKE, FAKE, 4, ctypes.byref(desc(fmt=4)), None) == I
    assert tq.lib().tq_append_bf16(FAKE, FAKE, FAKE, 0, ctypes.byref(desc(fmt=16)), None) == 0


def dec(c, q=FAKE, pt=FAKE, maxp=512, sl=FAKE, B=8, q_len=1, Hq=32, max_len=4096, out=FAKE,
        ws=FAKE, ws_n=1 << 30, bf16=False):
    fn = tq.lib().tq_paged_decode_bf16 if bf16 else tq.lib().tq_paged_decode
    return fn(q, ctypes.byref(c), pt, maxp, sl, B, q_len, Hq, max_len, out, ws, ws_n, None)


def test_decode_validation():
    I, U, W = tq.TQ_ERR_INVALID_ARG, tq.TQ_ERR_UNSUPPORTED, tq.TQ_ERR_WORKSPACE
    c = desc()
    assert dec(desc(fmt=16)) == I                     # turbo call on a bf16 cache
    assert dec(c, bf16=True) == I                     # bf16 call on a turbo cache
    assert dec(c, Hq=30) == I                         # not a multiple of kv heads
    assert dec(c, q_len=0) == I
    assert dec(c, max_len=0) == I
    assert dec(c, maxp=255) == I                      # too few page-table columns
    assert dec(c, q_len=1025, Hq=32) == U             # 4100 rows per kv head > 4096
    assert dec(c, q_len=1024, Hq=32, max_len=1024, ws=None, ws_n=0) != U   # 4096 rows
    assert dec(c, B=70000) == U
    assert dec(c, q=FAKE + 4) == I
    assert dec(c, out=FAKE + 8) == I
    assert dec(c, pt=None) == I
    assert dec(c, ws=None, ws_n=0) == W
    assert dec(c, ws_n=1024) == W
    assert dec(c, B=0) == tq.TQ_OK                    # empty batch: no-op
    assert dec(c, max_len=4, q_len=8) == I            # max_seq_len < q_len


def _expected_workspace(batch, Hkv, G, seq, P, fmt):
    """Workspace layout the decode kernels use: merge counters, then (m, l)
    and the 128-float partial output of every (unit, split, row), where a
    unit is one (sequence, kv head, row group).  Rows per CTA: 8 for the bf16
    cache; 4, 8 or 16 for the turbo formats.  Splits are 2048 tokens (1024
    with 64-token pages)."""
    split = 1024 if P == 64 else 2048
    nsplit = -(-seq // split)
    if nsplit <= 1:
        return 0
    if fmt == 16:
        rows = 8
    else:
        rows = 4 if G <= 4 else (8 if G <= 8 else 16)
    units = batch * Hkv * -(-G // rows)
    r256 = lambda x: -(-x // 256) * 256
    return r256(units * 4) + r256(units * nsplit * rows * 8) + units * nsplit * rows * 128 * 4


def test_workspace_size():
    ws = tq.lib().tq_decode_workspace_size
    c = desc()
    # one split (<= 2048 tokens with 16-token pages): no workspace
    assert ws(8, 1, 32, 2048, ctypes.byref(c)) == 0
    assert ws(8, 1, 32, 2049, ctypes.byref(c)) == _expected_workspace(8, 8, 4, 2049, 16, 4)
    # 4 splits x 64 (seq, kv head) units x 4 rows x (128 + 2) floats + counters
    assert ws(8, 1, 32, 8192, ctypes.byref(c)) == 4 * 64 * 4 * 130 * 4 + 256
    assert ws(8, 1, 30, 4096, ctypes.byref(c)) == 0   # invalid
    for fmt in (2, 3, 4, 8, 16):
        for q_len, Hq in ((1, 32), (1, 64), (4, 32), (8, 64), (3, 40)):
            cf = desc(fmt=fmt)
            assert ws(8, q_len, Hq, 8192, ctypes.byref(cf)) == \
                _expected_workspace(8, 8, q_len * Hq // 8, 8192, 16, fmt), (fmt, q_len, Hq)
    c64 = desc(P=64)
    assert ws(4, 1, 40, 131072, ctypes.byref(c64)) == _expected_workspace(4, 8, 5, 131072, 64, 4)
    assert ws(4, 1, 40, 131072, ctypes.byref(c64)) >= 4 * 8 * 128 * 8 * 130 * 4


def test_hbm_probe_validation():
    assert tq.lib().tq_hbm_copy(FAKE, FAKE, 0, None) == 0
    assert tq.lib().tq_hbm_copy(FAKE, FAKE, 24, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib().tq_hbm_read(FAKE + 4, 32, FAKE, None) == tq.TQ_ERR_INVALID_ARG


def test_read_device_error_without_word():
    code = ctypes.c_uint32(7)
    assert tq.lib().tq_read_device_error(ctypes.byref(desc(err=None)), ctypes.byref(code), 1,
                                         None) == 0
    assert code.value == 0


def test_descriptor_layout_matches_the_c_header(tmp_path):
    """The ctypes descriptor has the size and field offsets a C compiler
    gives tq_cache, and the enum values the header defines."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "tq.h"\n'
        "int main(void) {\n"
        '  printf("%zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(tq_cache),\n'
        "         offsetof(tq_cache, format), offsetof(tq_cache, head_dim),\n"
        "         offsetof(tq_cache, num_kv_heads), offsetof(tq_cache, page_size),\n"
        "         offsetof(tq_cache, num_pages), offsetof(tq_cache, pages),\n"
        "         offsetof(tq_cache, dev_error));\n"
        '  printf("%d %d %d %d %d %d\\n", TQ_TURBO2, TQ_TURBO3, TQ_TURBO4, TQ_TURBO8, TQ_BF16,\n'
        "         TQ_ABI_VERSION);\n"
        '  printf("%d %d %d %d %d %d %d %d\\n", TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED,\n'
        "         TQ_ERR_CUDA, TQ_ERR_TIMEOUT, TQ_ERR_DEVICE_CHECK, TQ_ERR_WORKSPACE,\n"
        "         TQ_ERR_NO_PAGES);\n"
        '  printf("%zu %zu %zu %zu %zu %zu %zu\\n", sizeof(tq_prefix_stats),\n'
        "         offsetof(tq_prefix_stats, free_pages), offsetof(tq_prefix_stats, cached_blocks),\n"
        "         offsetof(tq_prefix_stats, live_sequences), offsetof(tq_prefix_stats, hit_tokens),\n"
        "         offsetof(tq_prefix_stats, prompt_tokens), offsetof(tq_prefix_stats, evictions));\n"
        "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                           str(exe)])
    lines = subprocess.check_output([str(exe)], text=True).split("\n")
    sizes = [int(x) for x in lines[0].split()]
    C = tq.tq_cache
    assert sizes[0] == ctypes.sizeof(C)
    assert sizes[1:] == [getattr(C, f).offset for f in
                         ("format", "head_dim", "num_kv_heads", "page_size", "num_pages",
                          "pages", "dev_error")]
    assert [int(x) for x in lines[1].split()] == [tq.TQ_TURBO2, tq.TQ_TURBO3, tq.TQ_TURBO4,
                                                  tq.TQ_TURBO8, tq.TQ_BF16, tq.abi_version()]
    assert [int(x) for x in lines[2].split()] == [
        tq.TQ_OK, tq.TQ_ERR_INVALID_ARG, tq.TQ_ERR_UNSUPPORTED, tq.TQ_ERR_CUDA,
        tq.TQ_ERR_TIMEOUT, tq.TQ_ERR_DEVICE_CHECK, tq.TQ_ERR_WORKSPACE, tq.TQ_ERR_NO_PAGES]
    S = tq.tq_prefix_stats
    assert [int(x) for x in lines[3].split()] == [ctypes.sizeof(S)] + [
        getattr(S, f).offset for f, _ in S._fields_]


def test_step_graph_validation_on_the_host():
    """The graph step checks its arguments like the two calls it captures
    and refuses the legacy stream; nothing reaches the CUDA runtime."""
    c = desc()
    st = tq.tq_step()
    h = ctypes.c_void_p()
    create = tq.lib().tq_step_graph_create
    assert create(ctypes.byref(c), ctypes.byref(st), None, ctypes.byref(h)) == tq.TQ_ERR_INVALID_ARG
    st.batch, st.q_len, st.num_q_heads, st.max_seq_len = 1, 1, 8, 16
    st.max_pages_per_seq = 1
    # fake stream handle: validation fails (no q / out pointers) before any capture
    assert create(ctypes.byref(c), ctypes.byref(st), FAKE, ctypes.byref(h)) == tq.TQ_ERR_INVALID_ARG
    assert h.value is None
    assert tq.lib().tq_step_graph_launch(None, None) == tq.TQ_ERR_INVALID_ARG
    tq.lib().tq_step_graph_destroy(None)
