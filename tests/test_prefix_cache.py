"""The prefix-block manager (tq_prefix_cache_*), host only.

Each rule of "xinfer-ai" package docs, "Prefix Cache (KV Reuse)" is checked
on its own: finished sequences give their full blocks to the cache; a new
prompt reuses the longest cached block-aligned prefix; a common prefix that
ends inside a block has that block recomputed; a prompt cached entirely at
block boundaries recomputes its last block; the cache is capped in tokens,
rounded down to whole blocks; it shares the pool with live sequences.
"""
import numpy as np
import pytest

from quantized_paged_kv_tq_b200 import build as tqbuild

tqbuild.build()
from quantized_paged_kv_tq_b200 import tq  # noqa: E402

P = 16


def prompt(n, seed):
    return np.random.default_rng(seed).integers(0, 50000, size=n).astype(np.int32)


def test_first_prompt_misses_and_finish_caches_full_blocks():
    pc = tq.PrefixCache(64, P, max_cached_tokens=64 * P)
    a = prompt(100, 1)
    seq, cached, pt = pc.begin(a, 16)
    assert cached == 0 and len(pt) == 7 and len(set(pt)) == 7
    assert pc.stats()["free_pages"] == 64 - 7 and pc.stats()["live_sequences"] == 1
    pc.finish(seq, a)
    st = pc.stats()
    # 6 full blocks cached, the partial 7th page freed
    assert st["cached_blocks"] == 6 and st["free_pages"] == 64 - 6 and st["live_sequences"] == 0
    assert all(pc.page_refs(int(p)) == 1 for p in pt[:6]) and pc.page_refs(int(pt[6])) == 0


def test_longest_block_aligned_prefix_is_reused():
    pc = tq.PrefixCache(64, P)
    a = prompt(100, 2)
    sa, _, pta = pc.begin(a, 16)
    pc.finish(sa, a)
    b = np.concatenate([a[:80], prompt(30, 3)])          # 5 full common blocks
    sb, cached, ptb = pc.begin(b, 16)
    assert cached == 80
    assert np.array_equal(ptb[:5], pta[:5])
    assert not set(ptb[5:]) & set(pta[:6])               # not among the cached pages
    assert pc.stats()["hit_tokens"] == 80
    # shared pages: the cache and sequence b hold them
    assert all(pc.page_refs(int(p)) == 2 for p in ptb[:5])


def test_common_prefix_ending_mid_block_recomputes_that_block():
    pc = tq.PrefixCache(64, P)
    a = prompt(100, 4)
    sa, _, pta = pc.begin(a, 16)
    pc.finish(sa, a)
    b = a.copy()[:100]
    b[85] += 1                                           # differs inside block 5
    _, cached, ptb = pc.begin(b, 16)
    assert cached == 80                                  # blocks 0-4 only
    assert np.array_equal(ptb[:5], pta[:5]) and ptb[5] != pta[5]


def test_prompt_cached_at_block_boundaries_recomputes_last_block():
    pc = tq.PrefixCache(64, P)
    a = prompt(100, 5)
    sa, _, pta = pc.begin(a, 16)
    pc.finish(sa, a)
    c = a[:96].copy()                                    # exactly the 6 cached blocks
    _, cached, ptc = pc.begin(c, 16)
    assert cached == 80                                  # the last block is prefilled again
    assert np.array_equal(ptc[:5], pta[:5]) and ptc[5] != pta[5]
    # a one-block prompt that is cached: nothing reused, one block prefilled
    pc2 = tq.PrefixCache(8, P)
    one = prompt(16, 6)
    s1, _, _ = pc2.begin(one, 4)
    pc2.finish(s1, one)
    _, cached1, _ = pc2.begin(one, 4)
    assert cached1 == 0


def test_blocks_are_keyed_by_position_not_only_content():
    """The same 16 token ids as block 1 of one prompt and block 0 of another
    are different blocks (the cache is a prefix trie)."""
    pc = tq.PrefixCache(64, P)
    blk = prompt(16, 7)
    a = np.concatenate([prompt(16, 8), blk])
    sa, _, _ = pc.begin(a, 8)
    pc.finish(sa, a)
    _, cached, _ = pc.begin(np.concatenate([blk, prompt(20, 9)]), 8)
    assert cached == 0


def test_identical_blocks_finished_twice_are_cached_once():
    pc = tq.PrefixCache(64, P)
    a = prompt(64, 10)
    s1, _, pt1 = pc.begin(a, 8)
    s2, _, pt2 = pc.begin(a, 8)                          # both miss: nothing cached yet
    assert not set(pt1) & set(pt2)
    pc.finish(s1, a)
    pc.finish(s2, a)
    st = pc.stats()
    assert st["cached_blocks"] == 4 and st["free_pages"] == 64 - 4
    _, cached, pt3 = pc.begin(a, 8)
    assert cached == 48 and np.array_equal(pt3[:3], pt1[:3])


def test_generated_tokens_join_the_cache_through_extend():
    pc = tq.PrefixCache(64, P)
    a = prompt(20, 11)
    sa, _, pt = pc.begin(a, 8)
    pt = pc.extend(sa, 40, 8)                            # decode grew it to 40 tokens
    assert len(pt) == 3
    full = np.concatenate([a, prompt(20, 12)])
    pc.finish(sa, full)
    assert pc.stats()["cached_blocks"] == 2
    _, cached, _ = pc.begin(np.concatenate([full[:32], prompt(5, 13)]), 8)
    assert cached == 32


def test_cap_keeps_the_prefix_end_of_a_chain():
    """With room for 4 blocks, an 8-block sequence leaves its first 4 cached:
    only blocks without cached children can go, least recently used first."""
    pc = tq.PrefixCache(64, P, max_cached_tokens=4 * P + 7)   # rounded down to 4 blocks
    a = prompt(8 * P, 14)
    sa, _, pta = pc.begin(a, 16)
    pc.finish(sa, a)
    st = pc.stats()
    assert st["cached_blocks"] == 4 and st["evictions"] == 4
    _, cached, ptb = pc.begin(a[:6 * P], 16)
    assert cached == 4 * P and np.array_equal(ptb[:4], pta[:4])


def test_eviction_when_the_pool_runs_out_spares_live_sequences():
    pc = tq.PrefixCache(12, P, max_cached_tokens=12 * P)
    a, b = prompt(4 * P, 15), prompt(4 * P, 16)
    sa, _, pta = pc.begin(a, 8)
    pc.finish(sa, a)                                     # a: 4 cached blocks (oldest)
    sb, _, ptb = pc.begin(b, 8)
    pc.finish(sb, b)                                     # b: 4 cached blocks
    # a live sequence reusing a's first 2 blocks holds them
    sl, cached, ptl = pc.begin(np.concatenate([a[:2 * P], prompt(P, 17)]), 8)
    assert cached == 2 * P
    # 12 pages: 8 cached + 1 fresh for sl -> 3 free; a 6-page prompt must evict 3
    sn, cached_n, ptn = pc.begin(prompt(6 * P, 18), 8)
    assert cached_n == 0 and pc.stats()["evictions"] == 3
    # a's blocks 0-1 are held by sl and survive; a's leaves went first (LRU)
    _, hit, _ = pc.begin(a[:3 * P], 8)
    assert hit == 2 * P
    assert all(pc.page_refs(int(p)) >= 2 for p in ptl[:2])


def test_no_pages_leaves_the_state_unchanged():
    pc = tq.PrefixCache(4, P)
    s, _, _ = pc.begin(prompt(3 * P, 19), 8)
    before = pc.stats()
    with pytest.raises(tq.TqError) as e:
        pc.begin(prompt(2 * P, 20), 8)
    assert e.value.status == tq.TQ_ERR_NO_PAGES
    assert pc.stats() == before
    with pytest.raises(tq.TqError) as e:
        pc.extend(s, 5 * P, 8)
    assert e.value.status == tq.TQ_ERR_NO_PAGES and pc.stats() == before


def test_invalid_arguments():
    pc = tq.PrefixCache(8, P)
    with pytest.raises(tq.TqError):
        pc.begin(np.zeros(0, np.int32), 4)               # empty prompt
    with pytest.raises(tq.TqError):
        pc.begin(prompt(5 * P, 21), 4)                   # table too short
    with pytest.raises(tq.TqError):
        pc.finish(3, prompt(4, 22))                      # unknown handle
    s, _, _ = pc.begin(prompt(P, 23), 4)
    pc.finish(s, prompt(P, 23))
    with pytest.raises(tq.TqError):
        pc.finish(s, prompt(P, 23))                      # finished already
    with pytest.raises(tq.TqError):
        pc.extend(s, 2 * P, 4)
    assert tq.lib().tq_prefix_cache_create(0, 16, 0) is None
    assert pc.page_refs(-1) == -1 and pc.page_refs(8) == -1
