"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Codes and scales must be bit-exact; attention outputs within max-abs 2e-3
and relative-L2 1e-3 of the oracle's fp64 result on the same dequantised
cache.  Small workloads are compared element by element everywhere; the
full-size workloads on sampled slots and sampled sequences (the oracle
rebuilds those sequences' caches itself from the generator's values)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (check_close, dev, dev_bf16, gpu_decode, gpu_fill, gpu_rows, k_pool_logical,
                         oracle_decode, oracle_pools, oracle_rows)
from quantized_paged_kv_tq_b200 import workloads as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from quantized_paged_kv_tq_b200 import build as _b
    _b.build()
    from quantized_paged_kv_tq_b200 import tq

TURBO = (2, 3, 4, 8)
FP8 = 17


def small(fmt, **kw):
    base = dict(num_q_heads=8, num_kv_heads=2, page_size=16, q_len=1,
                seq_lens=(2600, 37, 2049), fmt=fmt, seed=11 + fmt)
    base.update(kw)
    return W.custom(**base)


# ------------------------------------------------------------ quantiser
@pytest.mark.parametrize("fmt", TURBO + (FP8,))
@pytest.mark.parametrize("P", [16, 32, 64])
def test_quantize_append_bit_exact_small(fmt, P):
    """Every byte of both pools equals the oracle's (ragged last pages,
    permuted pages, outlier channels)."""
    w = small(fmt, page_size=P, seq_lens=(300, 37, 129))
    cache = gpu_fill(w, fmt)
    kp, vp = oracle_pools(fmt, w.num_pages, w)
    for slots, k, v in w.iter_fill():
        oracle.quantize_append(k, v, slots, fmt, P, kp, vp)
    assert np.array_equal(k_pool_logical(cache.k_pages.cpu().numpy(), fmt, P), kp)
    assert np.array_equal(cache.v_pages.cpu().numpy(), vp)
    assert cache.read_error() == 0


@pytest.mark.parametrize("fmt", TURBO)
def test_quantize_special_vectors(fmt):
    """All-zero rows (s = 0), +-powers of two, e_0, constant rows, huge and
    tiny magnitudes, and slot -1 (skipped)."""
    rng = np.random.default_rng(fmt)
    rows = [np.zeros(128, np.float32), np.full(128, 3.0, np.float32), np.eye(128)[0],
            -np.eye(128)[5] * 1024, rng.standard_normal(128) * 1e30,
            rng.standard_normal(128) * 1e-30, rng.standard_normal(128) * 2.0 ** 100,
            np.where(np.arange(128) % 2 == 0, 0.5, -0.5)]
    n = len(rows)
    x = np.stack(rows).astype(np.float32)
    k = W.f32_to_bf16_bits(np.repeat(x[:, None], 2, 1))
    v = W.f32_to_bf16_bits(np.repeat(-x[:, None], 2, 1))
    slots = np.arange(n, dtype=np.int64) * 3
    slots[2] = -1
    from quantized_paged_kv_tq_b200 import tq as T
    cache = T.Cache(fmt, 2, 2, 16)
    T.tq_quantize_append(dev_bf16(k), dev_bf16(v), dev(slots), fmt, cache)
    torch.cuda.synchronize()
    kp, vp = oracle_pools(fmt, 2, W.custom(num_kv_heads=2, page_size=16))
    oracle.quantize_append(k, v, slots, fmt, 16, kp, vp)
    assert np.array_equal(k_pool_logical(cache.k_pages.cpu().numpy(), fmt, 16), kp)
    assert np.array_equal(cache.v_pages.cpu().numpy(), vp)


@pytest.mark.parametrize("name,fmt", [("tiny", 4), ("batch8", 4), ("cbatch64", 3),
                                      ("cbatch64", 8), ("target64x8k", 4),
                                      ("long128k", 4), ("long128k", 2),
                                      ("specverify", 4)])
def test_quantize_full_size_sampled(name, fmt):
    w = W.make(name)
    cache = gpu_fill(w, fmt)
    slots = w.fill_slots()
    pick = np.sort(np.random.default_rng(5).choice(len(slots), min(1500, len(slots)),
                                                   replace=False))
    s = slots[pick]
    got = gpu_rows(cache, s, w.page_size, fmt)
    ref = oracle_rows(w, s, fmt)
    for a, b in zip(got, ref):
        assert a.shape == b.shape and np.array_equal(np.asarray(a), np.asarray(b))
    assert cache.read_error() == 0


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("fmt", TURBO + (16, FP8))
@pytest.mark.parametrize("q_len,Hq,Hkv", [(1, 8, 2), (1, 10, 2), (4, 8, 2), (3, 6, 1),
                                          (1, 16, 1), (8, 64, 8), (2, 4, 2), (2, 8, 2)])
def test_decode_small(fmt, q_len, Hq, Hkv):
    """Ragged lengths (2600 = 2 splits + tail, 37 < one tile, 2049 = one
    token past a split), 1-8 query rows per kv head up to 16 and 64; q_len 2
    with 4 and 8 rows per kv head takes the causal path of the 4- and 8-row
    kernels, q_len 3-8 with more rows that of the 16-row one."""
    w = small(fmt, q_len=q_len, num_q_heads=Hq, num_kv_heads=Hkv,
              seq_lens=(2600, 37 + q_len, 2049))
    cache = gpu_fill(w, fmt)
    got = gpu_decode(w, fmt, cache)
    ref = oracle_decode(w, fmt, np.arange(w.batch))
    check_close(got, ref, f"fmt {fmt} q_len {q_len} {Hq}/{Hkv}")
    assert cache.read_error() == 0


@pytest.mark.parametrize("fmt", (4, 2, FP8))
def test_decode_page64(fmt):
    w = small(fmt, page_size=64, seq_lens=(2500, 64, 1025), num_q_heads=10)
    cache = gpu_fill(w, fmt)
    check_close(gpu_decode(w, fmt, cache), oracle_decode(w, fmt, np.arange(w.batch)))


@pytest.mark.parametrize("fmt", TURBO + (16, FP8))
@pytest.mark.parametrize("q_len", [1, 4])
def test_decode_page32(fmt, q_len):
    """32-token pages: 4 pages per 128-token tile, 4 and 16 rows per kv head."""
    w = small(fmt, page_size=32, q_len=q_len, seq_lens=(2600, 40 + q_len, 2049))
    cache = gpu_fill(w, fmt)
    check_close(gpu_decode(w, fmt, cache), oracle_decode(w, fmt, np.arange(w.batch)),
                f"fmt {fmt} page 32 q_len {q_len}")
    assert cache.read_error() == 0


CONFIG_RUNS = [("tiny", 4, None), ("batch8", 4, (0, 5)), ("cbatch64", 3, "minmax"),
               ("cbatch64", 8, "minmax"), ("cbatch64", 16, "minmax"), ("cbatch64", FP8, "minmax"),
               ("target64x8k", 4, (0, 63)), ("long128k", 4, (2,)), ("long128k", 2, (1,)),
               ("specverify", 4, (0, 7, 20))]


@pytest.mark.parametrize("name,fmt,seqs", CONFIG_RUNS)
def test_decode_configs(name, fmt, seqs):
    """Every configuration at full size; the oracle checks sampled sequences
    (all of them for the tiny one) and every output must be finite."""
    w = W.make(name)
    cache = gpu_fill(w, fmt)
    got = gpu_decode(w, fmt, cache)
    assert np.all(np.isfinite(got))
    if seqs is None:
        seqs = np.arange(w.batch)
    elif seqs == "minmax":
        seqs = (int(np.argmin(w.seq_lens)), int(np.argmax(w.seq_lens)), 17)
    seqs = np.asarray(seqs)
    ref = oracle_decode(w, fmt, seqs)
    check_close(got[seqs], ref, f"{name} fmt {fmt}")
    assert cache.read_error() == 0


# ------------------------------------------------------------ properties
@pytest.mark.parametrize("fmt", (4, 16))
def test_batch_invariance(fmt):
    """A sequence's output is bit-identical alone and inside a batch."""
    w = small(fmt, seq_lens=(2600, 37, 2049, 4100))
    cache = gpu_fill(w, fmt)
    full = gpu_decode(w, fmt, cache)
    q = w.queries()
    for b in range(w.batch):
        one = gpu_decode(w, fmt, cache, q=q[b:b + 1], page_table=w.page_table[b:b + 1],
                         seq_lens=w.seq_lens[b:b + 1])
        assert np.array_equal(one[0], full[b])


def test_page_permutation_invariance():
    """Moving pages to other physical slots changes nothing, bit for bit."""
    w = small(4, seq_lens=(700, 300))
    cache = gpu_fill(w, 4)
    out = gpu_decode(w, 4, cache)
    perm = np.random.default_rng(3).permutation(w.num_pages)
    from quantized_paged_kv_tq_b200 import tq as T
    c2 = T.Cache(4, w.num_pages, w.num_kv_heads, w.page_size)
    inv = torch.as_tensor(perm, device="cuda")
    c2.k_pages[inv] = cache.k_pages
    c2.v_pages[inv] = cache.v_pages
    pt = np.where(w.page_table >= 0, perm[np.maximum(w.page_table, 0)], -1)
    assert np.array_equal(gpu_decode(w, 4, c2, page_table=pt), out)


def test_shared_prefix_equals_private_copies():
    """Sequences reading one physical copy of a prefix give the same bits as
    sequences holding private copies of the same prefix values."""
    shared = W.custom(seq_lens=(2600, 3000, 2300), q_len=4, num_q_heads=8,
                      num_kv_heads=2, shared_prefix_seqs=3, shared_prefix_tokens=1024,
                      permute_pages=False, fmt=4, seed=9)
    cache = gpu_fill(shared, 4)
    out = gpu_decode(shared, 4, cache)
    # private layout: copy the prefix pages for sequences 1 and 2
    from quantized_paged_kv_tq_b200 import tq as T
    P = shared.page_size
    npre = 1024 // P
    extra = 2 * npre
    c2 = T.Cache(4, shared.num_pages + extra, 2, P)
    c2.k_pages[:shared.num_pages] = cache.k_pages
    c2.v_pages[:shared.num_pages] = cache.v_pages
    pt = shared.page_table.copy()
    for i, b in enumerate((1, 2)):
        new = shared.num_pages + i * npre + np.arange(npre)
        c2.k_pages[torch.as_tensor(new, device="cuda")] = cache.k_pages[:npre]
        c2.v_pages[torch.as_tensor(new, device="cuda")] = cache.v_pages[:npre]
        pt[b, :npre] = new
    assert np.array_equal(gpu_decode(shared, 4, c2, page_table=pt), out)
    check_close(out, oracle_decode(shared, 4, np.arange(3)))


def test_append_order_independence():
    w = small(3, seq_lens=(500, 77))
    a = gpu_fill(w, 3)
    b = gpu_fill(w, 3, shuffle_seed=1)
    c = gpu_fill(w, 3, chunk=7)
    for x in (b, c):
        assert torch.equal(a.k_pages, x.k_pages) and torch.equal(a.v_pages, x.v_pages)


@pytest.mark.parametrize("q_len,lens", [(4, (2050, 2052)), (2, (2049, 2050)), (2, (1025, 1026))])
def test_causal_last_split_fully_masked_rows(q_len, lens):
    """q_len 4 at seq_len 2050 (16 rows per kv head): the second split holds
    keys 2048-2049 only, which rows t = 0, 1 must not see (their partial is
    empty); q_len 2 at 2049 (8 rows): row t = 0 sees nothing of key 2048;
    q_len 2 at 1025 with 64-token pages (1024-token splits): the same at
    key 1024."""
    if lens[0] == 1025:
        w = small(4, q_len=q_len, seq_lens=lens, page_size=64)
        cache = gpu_fill(w, 4)
        check_close(gpu_decode(w, 4, cache), oracle_decode(w, 4, np.arange(2)))
        return
    w = small(4, q_len=q_len, seq_lens=lens)
    cache = gpu_fill(w, 4)
    check_close(gpu_decode(w, 4, cache), oracle_decode(w, 4, np.arange(2)))


@pytest.mark.parametrize("fmt,q_len,lens", [
    (4, 64, (700, 2300)),        # 256 rows per kv head; the chunk crosses a split boundary
    (3, 200, (2300, 200)),       # 800 rows; the second sequence is the chunk alone
    (16, 96, (2200, 500)),       # bf16 cache: 8-row groups
    (2, 256, (4096, 2400)),      # 1024 rows; a chunk at the end of two splits
    (FP8, 48, (2100, 60)),
    (8, 32, (1500, 40)),         # exactly 128 rows: one query-major CTA per kv head
    (4, 33, (900, 2049)),        # 132 rows: a second row block of 4 rows
    (3, 40, (129, 3000)),        # 160 rows, a context of 89 tokens before the chunk
])
def test_chunked_prefill_over_quantised_pages(fmt, q_len, lens):
    """A chunk of q_len prefill tokens, appended first, attends causally over
    the cache: row t sees keys j <= seq_len - q_len + t.  Every row of every
    chunk against the oracle (128 or more rows per kv head take the
    query-major kernel for turbo formats)."""
    w = small(fmt, q_len=q_len, seq_lens=lens)
    cache = gpu_fill(w, fmt)
    check_close(gpu_decode(w, fmt, cache), oracle_decode(w, fmt, np.arange(len(lens))),
                f"fmt {fmt} chunk {q_len}")
    assert cache.read_error() == 0


@pytest.mark.parametrize("fmt", (4, 2, 8))
def test_mixed_lengths_in_one_batch(fmt):
    """Lengths of 1 token, exactly one split, one token past it, many
    splits and a partial tile, in one batch, all against the oracle."""
    w = small(fmt, seq_lens=(1, 2048, 2049, 20000, 129, 5000, 1))
    cache = gpu_fill(w, fmt)
    check_close(gpu_decode(w, fmt, cache), oracle_decode(w, fmt, np.arange(w.batch)),
                f"fmt {fmt} mixed lengths")
    assert cache.read_error() == 0


def test_invalid_length_mid_batch_skips_only_that_sequence():
    """A sequence whose length is above max_seq_len is reported and skipped;
    the sequences before and after it in the batch are still exact."""
    from quantized_paged_kv_tq_b200 import tq as T
    w = small(4, seq_lens=(1500, 3000, 700))
    cache = gpu_fill(w, 4)
    out = torch.full((3, 1, 8, 128), float("nan"), device="cuda")
    T.tq_paged_decode(dev_bf16(w.queries()), cache, dev(w.page_table), dev(w.seq_lens), 1, out,
                      max_seq_len=2000)
    code = cache.read_error()
    assert code & 0xff == T.TQ_ERR_DEVICE_CHECK and code >> 8 == 3
    got = out.cpu().numpy()
    ref = oracle_decode(w, 4, np.array([0, 2]))
    check_close(got[[0, 2]], ref, "neighbours of a skipped sequence")


def test_repeated_calls_reuse_workspace():
    """The merge counters return to zero: many calls on one workspace agree."""
    w = small(4)
    cache = gpu_fill(w, 4)
    first = gpu_decode(w, 4, cache)
    for _ in range(5):
        assert np.array_equal(gpu_decode(w, 4, cache), first)


# ------------------------------------------------------- device findings
def test_device_checks_report_and_skip():
    from quantized_paged_kv_tq_b200 import tq as T
    w = small(4, seq_lens=(100, 40))
    cache = gpu_fill(w, 4)
    assert cache.read_error() == 0
    # slot past the pool: skipped, reported
    k = dev_bf16(np.zeros((1, 2, 128), np.uint16))
    T.tq_quantize_append(k, k, dev(np.array([w.num_pages * 16 + 3], np.int64)), 4, cache)
    code = cache.read_error()
    assert code & 0xff == T.TQ_ERR_DEVICE_CHECK and code >> 8 == 1
    # page-table entry out of range: reported
    pt = w.page_table.copy()
    pt[1, 0] = w.num_pages + 5
    gpu_decode(w, 4, cache, page_table=pt)
    code = cache.read_error()
    assert code & 0xff == T.TQ_ERR_DEVICE_CHECK and code >> 8 == 2
    # seq_len above max_seq_len: reported, sequence skipped
    out = torch.zeros((2, 1, 8, 128), device="cuda")
    sl = dev(np.array([100, 40], np.int32))
    T.tq_paged_decode(dev_bf16(w.queries()), cache, dev(w.page_table), sl, 1, out,
                      max_seq_len=50)
    code = cache.read_error()
    assert code & 0xff == T.TQ_ERR_DEVICE_CHECK and code >> 8 == 3
    assert cache.read_error() == 0


def test_empty_batch_and_zero_tokens():
    from quantized_paged_kv_tq_b200 import tq as T
    cache = T.Cache(4, 4, 2, 16)
    e = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    T.tq_quantize_append(e, e, torch.empty(0, dtype=torch.int64, device="cuda"), 4, cache)
    out = torch.empty((0, 1, 8, 128), device="cuda")
    T.tq_paged_decode(torch.empty((0, 1, 8, 128), dtype=torch.bfloat16, device="cuda"), cache,
                      torch.zeros((0, 4), dtype=torch.int32, device="cuda"),
                      torch.zeros(0, dtype=torch.int32, device="cuda"), 1, out, max_seq_len=64)
    torch.cuda.synchronize()
    assert not cache.k_pages.any()


def test_hbm_probes():
    from quantized_paged_kv_tq_b200 import tq as T
    src = torch.randint(0, 255, (1 << 24,), dtype=torch.uint8, device="cuda")
    dst = torch.zeros_like(src)
    T.tq_hbm_copy(src, dst)
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    T.tq_hbm_read(src, sink)
    torch.cuda.synchronize()
    assert torch.equal(src, dst)


# ------------------------------------------------ prefix-block manager
def _kv_of_tokens(tokens, num_kv_heads, seed):
    """K/V of a token as a function of (token id, position) only, so a
    cached block is valid for every prompt that starts with the same ids."""
    n = len(tokens)
    k = np.empty((n, num_kv_heads, 128), np.uint16)
    v = np.empty_like(k)
    for j, t in enumerate(tokens):
        x = np.random.default_rng([seed, int(t), j]).standard_normal(
            (2, num_kv_heads, 128)).astype(np.float32)
        k[j], v[j] = W.f32_to_bf16_bits(x[0]), W.f32_to_bf16_bits(x[1])
    return k, v


def test_decode_through_prefix_cache_page_tables():
    """Page tables from the prefix-block manager: B reuses 9 blocks of A and
    prefills the rest, C is cached at a block boundary and prefills its last
    block again; decoding B and C together matches the oracle on private
    copies of their K/V."""
    from quantized_paged_kv_tq_b200 import tq as T
    P, H, Hq, fmt, seed = 16, 2, 8, 4, 41
    pool_pages, max_pages = 64, 16
    pc = T.PrefixCache(pool_pages, P)
    cache = T.Cache(fmt, pool_pages, H, P)
    rng = np.random.default_rng(40)
    a = rng.integers(0, 30000, 200).astype(np.int32)
    b = np.concatenate([a[:150], rng.integers(0, 30000, 70).astype(np.int32)])
    c = a[:160].copy()

    def admit(tokens):
        seq, cached, pt = pc.begin(tokens, max_pages)
        k, v = _kv_of_tokens(tokens, H, seed)
        pos = np.arange(cached, len(tokens))
        slots = pt[pos // P].astype(np.int64) * P + pos % P
        T.tq_quantize_append(dev_bf16(k[cached:]), dev_bf16(v[cached:]), dev(slots), fmt, cache)
        return seq, cached, pt

    sa, ca, pta = admit(a)
    assert ca == 0
    pc.finish(sa, a)
    sb, cb, ptb = admit(b)
    sc, cc, ptc = admit(c)
    assert cb == 144 and cc == 144
    assert np.array_equal(ptb[:9], pta[:9]) and np.array_equal(ptc[:9], pta[:9])
    assert ptc[9] != pta[9]
    table = np.full((2, max_pages), -1, np.int32)
    table[0, :len(ptb)] = ptb
    table[1, :len(ptc)] = ptc
    lens = np.array([len(b), len(c)], np.int32)
    q = W.f32_to_bf16_bits(rng.standard_normal((2, 1, Hq, 128)).astype(np.float32))
    out = torch.full((2, 1, Hq, 128), float("nan"), device="cuda")
    T.tq_paged_decode(dev_bf16(q), cache, dev(table), dev(lens), 1, out, max_seq_len=int(lens.max()))
    torch.cuda.synchronize()
    assert cache.read_error() == 0
    got = out.cpu().numpy()
    for i, toks in enumerate((b, c)):
        k, v = _kv_of_tokens(toks, H, seed)
        npg = -(-len(toks) // P)
        bb = oracle.block_bytes(fmt, 128, P)
        kp = np.zeros((npg, H, bb), np.uint8)
        vp = np.zeros_like(kp)
        oracle.quantize_append(k, v, np.arange(len(toks)), fmt, P, kp, vp)
        ref = oracle.paged_decode(np.ascontiguousarray(q[i:i + 1]), fmt, P, kp, vp,
                                  np.arange(npg, dtype=np.int32)[None],
                                  np.array([len(toks)], np.int32), H)
        check_close(got[i:i + 1], ref, f"prefix-cache sequence {i}")
    pc.finish(sb, b)
    pc.finish(sc, c)


# ------------------------------------------------------ graph-captured step
@pytest.mark.parametrize("fmt", (4, 3, 16))
def test_step_graph_replays_the_eager_step(fmt):
    """An append + decode step captured once as a CUDA graph and replayed
    with new token values each time gives the same cache bytes and the same
    outputs, bit for bit, as the two calls made eagerly."""
    from quantized_paged_kv_tq_b200 import tq as T
    w = small(fmt, seq_lens=(2600, 38, 2049))
    stream = torch.cuda.Stream()
    c_eager = T.Cache(fmt, w.num_pages, w.num_kv_heads, w.page_size)
    c_graph = T.Cache(fmt, w.num_pages, w.num_kv_heads, w.page_size)
    append = (lambda k, v, s, c: T.tq_append_bf16(k, v, s, c, stream=stream)) if fmt == 16 else \
        (lambda k, v, s, c: T.tq_quantize_append(k, v, s, fmt, c, stream=stream))
    decode = T.tq_paged_decode_bf16 if fmt == 16 else T.tq_paged_decode
    with torch.cuda.stream(stream):
        for slots, k, v in w.iter_fill(upto=w.seq_lens - 1):
            for c in (c_eager, c_graph):
                append(dev_bf16(k), dev_bf16(v), dev(slots.astype(np.int64)), c)
        new_slots = dev(np.array([w.slots_of(b, [int(w.seq_lens[b]) - 1])[0]
                                  for b in range(w.batch)], np.int64))
        q, pt, sl = dev_bf16(w.queries()), dev(w.page_table), dev(w.seq_lens)
        shape = (w.batch, 1, w.num_q_heads, 128)
        k_buf = torch.empty((w.batch, w.num_kv_heads, 128), dtype=torch.bfloat16, device="cuda")
        v_buf = torch.empty_like(k_buf)
        out_g = torch.full(shape, float("nan"), device="cuda")
        graph = T.StepGraph(c_graph, stream, q, pt, sl, 1, out_g, w.max_seq_len,
                            k=k_buf, v=v_buf, slot_mapping=new_slots)
        for i in range(3):
            k_new, v_new = (dev_bf16(x) for x in w.new_tokens(i, w.batch))
            k_buf.copy_(k_new)
            v_buf.copy_(v_new)
            graph.launch(stream)
            append(k_new, v_new, new_slots, c_eager)
            out_e = torch.full(shape, float("nan"), device="cuda")
            decode(q, c_eager, pt, sl, 1, out_e, max_seq_len=w.max_seq_len, stream=stream)
            stream.synchronize()
            assert torch.equal(c_graph.pages, c_eager.pages)
            assert torch.equal(out_g, out_e)
    assert c_graph.read_error() == 0 and c_eager.read_error() == 0


def test_fp8_special_vectors():
    """fp8 codes of all-zero rows (s = 0), signed zeros, exact powers of
    two, values at E4M3 ties, tiny and huge magnitudes: every byte of both
    pools equals the oracle's."""
    rng = np.random.default_rng(70)
    rows = [np.zeros(128, np.float32), np.eye(128)[3] * -2.0,
            np.where(np.arange(128) % 3 == 0, -0.0, 1.0625),
            rng.standard_normal(128) * 1e-30, rng.standard_normal(128) * 3e37,
            np.linspace(-448, 448, 128), rng.standard_normal(128)]
    x = np.stack(rows).astype(np.float32)
    n = len(rows)
    k = W.f32_to_bf16_bits(np.repeat(x[:, None], 2, 1))
    v = W.f32_to_bf16_bits(np.repeat(x[::-1, None], 2, 1))
    P = 16
    slots = np.arange(n, dtype=np.int64)
    from quantized_paged_kv_tq_b200 import tq as T
    cache = T.Cache(FP8, 1, 2, P)
    T.tq_quantize_append(dev_bf16(k), dev_bf16(v), dev(slots), FP8, cache)
    torch.cuda.synchronize()
    kp, vp = oracle_pools(FP8, 1, W.custom(page_size=P, num_kv_heads=2, fmt=FP8))
    oracle.quantize_append(k, v, slots, FP8, P, kp, vp)
    assert np.array_equal(k_pool_logical(cache.k_pages.cpu().numpy(), FP8, P), kp)
    assert np.array_equal(cache.v_pages.cpu().numpy(), vp)
    assert cache.read_error() == 0
