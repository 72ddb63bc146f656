"""tq_paged_decode_noalloc: the decode for callers that may not allocate.

Some callers cannot allocate device memory while they run -- a plugin
called from an inference runtime's fixed memory plan, or a service that
reserves all of its device memory at start-up.  For them the library keeps
the split-KV scratch in a fixed array of its own.  This test calls that
entry point through the C ABI and checks its output against the regular
tq_paged_decode (caller-provided workspace) on two calls in a row, the
second one reusing the scratch the first one left behind.  Both entry
points launch the same kernel with the same fixed splits and the same merge
order, so the outputs must agree bit for bit; the no-alloc output is also
checked against the CPU oracle's fp64 result at the parity tolerances.

The file name sorts last so that, in a run that stops at the first failure,
every other test has already run; it also builds and sets up everything it
needs, so it passes when run on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ATOL = 2e-3      # the tolerances the parity tests use
RTOL_L2 = 1e-3


def _close(got: np.ndarray, ref: np.ndarray):
    got = got.astype(np.float64)
    assert np.all(np.isfinite(got))
    assert np.abs(got - ref).max() <= ATOL
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= RTOL_L2


def _oracle_decode(w, fmt):
    """fp64 oracle output from a cache the oracle builds itself from the
    same generator values (never from GPU output)."""
    import oracle
    bb = oracle.block_bytes(fmt, w.head_dim, w.page_size)
    kp = np.zeros((w.num_pages, w.num_kv_heads, bb), np.uint8)
    vp = np.zeros_like(kp)
    for slots, k, v in w.iter_fill():
        oracle.quantize_append(k, v, slots, fmt, w.page_size, kp, vp)
    return oracle.paged_decode(w.queries(), fmt, w.page_size, kp, vp, w.page_table,
                               w.seq_lens, w.num_kv_heads)


def test_noalloc_matches_workspace_decode_twice():
    from quantized_paged_kv_tq_b200 import build as tqbuild
    tqbuild.build()
    from quantized_paged_kv_tq_b200 import tq
    from quantized_paged_kv_tq_b200 import workloads as W

    def d_bf16(u16):
        return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(
            torch.bfloat16).cuda()

    for fmt, q_len in ((4, 1), (3, 4)):
        # several splits per sequence, so the scratch (partials + counters) is used
        w = W.custom(seq_lens=(1300, 700, 2049), num_q_heads=8, num_kv_heads=2, q_len=q_len,
                     fmt=fmt, seed=31 + fmt)
        cache = tq.Cache(fmt, w.num_pages, w.num_kv_heads, w.page_size)
        for slots, k, v in w.iter_fill():
            tq.tq_quantize_append(d_bf16(k), d_bf16(v), torch.from_numpy(slots).cuda(), fmt,
                                  cache)
        q = d_bf16(w.queries())
        pt = torch.from_numpy(w.page_table).cuda()
        sl = torch.from_numpy(w.seq_lens).cuda()
        shape = (w.batch, q_len, w.num_q_heads, w.head_dim)
        ref = torch.full(shape, float("nan"), device="cuda")
        tq.tq_paged_decode(q, cache, pt, sl, q_len, ref, max_seq_len=w.max_seq_len)
        stream = torch.cuda.current_stream().cuda_stream
        torch.cuda.synchronize()
        for _ in range(2):
            out = torch.full(shape, float("nan"), device="cuda")
            st = tq.lib().tq_paged_decode_noalloc(
                q.data_ptr(), ctypes.byref(cache.desc), pt.data_ptr(), pt.shape[1],
                sl.data_ptr(), w.batch, q_len, w.num_q_heads, w.max_seq_len, out.data_ptr(),
                stream)
            assert st == tq.TQ_OK, tq.status_string(st)
            torch.cuda.synchronize()
            assert torch.equal(out, ref)           # same kernel, splits and merge order
        assert cache.read_error() == 0
        _close(out.cpu().numpy(), _oracle_decode(w, fmt))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from quantized_paged_kv_tq_b200 import build as tqbuild
    tqbuild.build()
    from quantized_paged_kv_tq_b200 import tq
    cache = tq.Cache(4, 4, 8, 16)
    q = torch.zeros((4096, 1, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((4096, 1, 32, 128), device="cuda")
    pt = torch.zeros((4096, 8192), dtype=torch.int32, device="cuda")
    sl = torch.zeros(4096, dtype=torch.int32, device="cuda")
    # 4096 sequences x 8 kv heads x 256 splits of partials: far above 64 MiB
    st = tq.lib().tq_paged_decode_noalloc(q.data_ptr(), ctypes.byref(cache.desc), pt.data_ptr(),
                                          pt.shape[1], sl.data_ptr(), 4096, 1, 32, 131072,
                                          out.data_ptr(), None)
    assert st == tq.TQ_ERR_WORKSPACE
