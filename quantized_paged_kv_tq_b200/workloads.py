"""Seeded synthetic workloads for the TurboQuant paged KV cache.

This module only draws inputs: sequence lengths, page tables, slot lists and
bf16 K/V/q values.  It holds none of the method's arithmetic and imports
neither the CUDA binding nor the oracle, so both sides can be fed the same
bytes.

Every value is a deterministic function of (workload seed, physical slot
chunk) or (workload seed, stream id), drawn with numpy's PCG64
(``default_rng``): any subset of slots can be regenerated on its own, which
lets a test check sampled tokens of a 131072-token context without holding
all of it twice.

The shapes and value mixes stand in for the KV traffic of the serving
workloads on the pages (xInfer's turbo4/turbo3 KV cache, "TurboQuant is a
memory trade"; infero's paged continuous batching, "Continuous batching";
xInfer's MTP verify with --num-speculative-tokens 3, "Getting a server up";
block-granular prefix sharing, xinfer-ai docs "Prefix Cache (KV Reuse)").
No model, prompt or dataset is used: values are N(0,1) with a few channels
scaled x20 (the outliers a Hadamard rotation is meant to spread) or
Student-t(3) for heavy-tailed keys.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128
SLOT_CHUNK = 4096          # slots per independently seeded K/V chunk

# stream ids mixed into the seed sequence
_S_CHANNELS = 11
_S_LENS = 12
_S_PERM = 13
_S_Q = 14
_S_K = 21
_S_V = 22
_S_NEW = 31


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Workload:
    """One synthetic decode workload (shapes, lengths, page tables)."""
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    page_size: int
    q_len: int
    formats: tuple
    seed: int
    k_dist: str = "normal"          # "normal" | "student_t3"
    k_outliers: int = 0
    v_outliers: int = 0
    permute_pages: bool = False
    shared_prefix_seqs: int = 0     # sequences 0..n-1 share their prefix pages
    shared_prefix_tokens: int = 0
    head_dim: int = HEAD_DIM
    seq_lens: np.ndarray = field(default=None, repr=False)
    page_table: np.ndarray = field(default=None, repr=False)
    num_pages: int = 0
    k_channels: np.ndarray = field(default=None, repr=False)
    v_channels: np.ndarray = field(default=None, repr=False)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.batch else 0

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.page_table.shape[1])

    # ------------------------------------------------------------------ slots
    def slots_of(self, b: int, positions: np.ndarray) -> np.ndarray:
        pos = np.asarray(positions, np.int64)
        pages = self.page_table[b, pos // self.page_size].astype(np.int64)
        return pages * self.page_size + pos % self.page_size

    def fill_slots(self, upto: np.ndarray | None = None) -> np.ndarray:
        """Distinct physical slots holding positions [0, upto[b]) of every
        sequence (default: the whole seq_len).  Shared prefix pages are
        listed once, by their first owner."""
        lens = self.seq_lens if upto is None else np.asarray(upto)
        out = []
        for b in range(self.batch):
            start = 0
            if 0 < b < self.shared_prefix_seqs:
                start = self.shared_prefix_tokens
            n = int(lens[b])
            if n > start:
                out.append(self.slots_of(b, np.arange(start, n)))
        return np.concatenate(out) if out else np.zeros(0, np.int64)

    # ----------------------------------------------------------------- values
    def _chunk_kv(self, chunk: int, which: int) -> np.ndarray:
        """bf16 bits [SLOT_CHUNK][num_kv_heads][d] of one slot chunk."""
        rng = np.random.default_rng([self.seed, which, chunk])
        shape = (SLOT_CHUNK, self.num_kv_heads, self.head_dim)
        if which == _S_K and self.k_dist == "student_t3":
            x = rng.standard_t(3, size=shape).astype(np.float32)
        else:
            x = rng.standard_normal(shape, dtype=np.float32)
        ch = self.k_channels if which == _S_K else self.v_channels
        if ch is not None and len(ch):
            x[:, :, ch] *= np.float32(20.0)
        return f32_to_bf16_bits(x)

    def kv_for_slots(self, slots: np.ndarray):
        """(k, v) bf16 bits [len(slots)][num_kv_heads][d] for physical slots."""
        slots = np.asarray(slots, np.int64)
        k = np.empty((len(slots), self.num_kv_heads, self.head_dim), np.uint16)
        v = np.empty_like(k)
        if len(slots) == 0:
            return k, v
        chunks = slots // SLOT_CHUNK
        for c in np.unique(chunks):
            sel = np.nonzero(chunks == c)[0]
            off = slots[sel] - c * SLOT_CHUNK
            k[sel] = self._chunk_kv(int(c), _S_K)[off]
            v[sel] = self._chunk_kv(int(c), _S_V)[off]
        return k, v

    def iter_fill(self, max_tokens: int = 1 << 16, upto=None):
        """Yield (slots, k, v) batches covering fill_slots(), chunk-aligned
        so each seeded chunk is drawn once."""
        slots = self.fill_slots(upto)
        order = np.argsort(slots, kind="stable")
        slots = slots[order]
        i = 0
        while i < len(slots):
            j = min(len(slots), i + max_tokens)
            yield (slots[i:j],) + self.kv_for_slots(slots[i:j])
            i = j

    def queries(self) -> np.ndarray:
        """bf16 bits [batch][q_len][num_q_heads][d], N(0,1)."""
        rng = np.random.default_rng([self.seed, _S_Q])
        x = rng.standard_normal((self.batch, self.q_len, self.num_q_heads,
                                 self.head_dim), dtype=np.float32)
        return f32_to_bf16_bits(x)

    def new_tokens(self, step: int, n: int):
        """(k, v) bf16 bits [n][num_kv_heads][d] for an appended step."""
        rng = np.random.default_rng([self.seed, _S_NEW, step])
        shape = (n, self.num_kv_heads, self.head_dim)
        out = []
        for which, ch in ((_S_K, self.k_channels), (_S_V, self.v_channels)):
            if which == _S_K and self.k_dist == "student_t3":
                x = rng.standard_t(3, size=shape).astype(np.float32)
            else:
                x = rng.standard_normal(shape, dtype=np.float32)
            if ch is not None and len(ch):
                x[:, :, ch] *= np.float32(20.0)
            out.append(f32_to_bf16_bits(x))
        return out[0], out[1]

    # ------------------------------------------------------------- accounting
    def tokens_read(self) -> int:
        """Logical (token, kv head) rows one decode step reads."""
        return int(self.seq_lens.astype(np.int64).sum()) * self.num_kv_heads

    def unique_tokens_read(self) -> int:
        return len(self.fill_slots()) * self.num_kv_heads


def row_bytes(fmt: int, d: int = HEAD_DIM) -> int:
    """Cache bytes of one (token, kv head) row of K or of V: codes + scale."""
    if fmt == 16:
        return 2 * d
    if fmt == 17:                       # fp8: one byte per code
        return d + 4
    return d * fmt // 8 + 4


def _finish(w: Workload, rng_lens=None) -> Workload:
    P = w.page_size
    rng = np.random.default_rng([w.seed, _S_CHANNELS])
    w.k_channels = (np.sort(rng.choice(w.head_dim, w.k_outliers, replace=False))
                    if w.k_outliers else np.zeros(0, np.int64))
    w.v_channels = (np.sort(rng.choice(w.head_dim, w.v_outliers, replace=False))
                    if w.v_outliers else np.zeros(0, np.int64))
    lens = w.seq_lens
    pages_per = (lens + P - 1) // P
    maxp = int(pages_per.max()) if w.batch else 1
    pt = np.full((w.batch, max(maxp, 1)), -1, np.int32)
    nxt = 0
    shared = w.shared_prefix_tokens // P if w.shared_prefix_seqs else 0
    if shared:
        prefix_pages = np.arange(shared, dtype=np.int32)
        nxt = shared
    for b in range(w.batch):
        n = int(pages_per[b])
        if b < w.shared_prefix_seqs and shared:
            pt[b, :shared] = prefix_pages
            k = n - shared
            pt[b, shared:n] = np.arange(nxt, nxt + k, dtype=np.int32)
            nxt += k
        else:
            pt[b, :n] = np.arange(nxt, nxt + n, dtype=np.int32)
            nxt += n
    w.num_pages = nxt
    if w.permute_pages:
        perm = np.random.default_rng([w.seed, _S_PERM]).permutation(nxt).astype(np.int32)
        pt = np.where(pt >= 0, perm[np.maximum(pt, 0)], -1).astype(np.int32)
    w.page_table = pt
    return w


def make(name: str) -> Workload:
    """The named synthetic workloads.

    tiny        batch 1, 4 q / 1 kv head, context 256, page 16, turbo4,
                2 key outlier channels x20, seed 0, q_len 1.
    batch8      batch 8, 32 q / 8 kv heads, context 4096, page 16, turbo4,
                physical pages randomly permuted, 4 outlier channels x20 in
                K and in V, seed 1.
    cbatch64    batch 64, 32 / 8, lengths uniform in [128, 8192], page 16,
                turbo3 and turbo8 plus a bf16 cache, 4 outlier channels,
                seed 2; each step appends one token per sequence.
    target64x8k the cbatch64 shapes with every length 8192, turbo4.
    long128k    batch 4, 40 / 8 heads, context 131072, page 64, turbo4 and
                turbo2, keys Student-t(3), seed 3.
    specverify  batch 32, 32 / 8, q_len 4 (causal among the draft tokens),
                sequences 0-15 share a 2048-token prefix through the same
                physical pages, private suffixes of 256-4096 tokens, page 16,
                turbo4, 4 outlier channels, seed 4.
    prefill256  batch 4, 32 / 8, context 4096 whose last 256 tokens are a
                prefill chunk (q_len 256: 1024 query rows per kv head,
                causal), page 16, turbo4, 2 key and 1 value outlier channels,
                seed 9.
    """
    if name == "tiny":
        w = Workload(name, 1, 4, 1, 16, 1, (4,), 0, k_outliers=2)
        w.seq_lens = np.array([256], np.int32)
    elif name == "batch8":
        w = Workload(name, 8, 32, 8, 16, 1, (4,), 1, k_outliers=4, v_outliers=4,
                     permute_pages=True)
        w.seq_lens = np.full(8, 4096, np.int32)
    elif name == "cbatch64":
        w = Workload(name, 64, 32, 8, 16, 1, (3, 8, 16), 2, k_outliers=4,
                     v_outliers=4)
        w.seq_lens = np.random.default_rng([2, _S_LENS]).integers(
            128, 8192, size=64, endpoint=True).astype(np.int32)
    elif name == "target64x8k":
        w = Workload(name, 64, 32, 8, 16, 1, (4,), 2, k_outliers=4, v_outliers=4)
        w.seq_lens = np.full(64, 8192, np.int32)
    elif name == "long128k":
        w = Workload(name, 4, 40, 8, 64, 1, (4, 2), 3, k_dist="student_t3")
        w.seq_lens = np.full(4, 131072, np.int32)
    elif name == "specverify":
        w = Workload(name, 32, 32, 8, 16, 4, (4,), 4, k_outliers=4, v_outliers=4,
                     shared_prefix_seqs=16, shared_prefix_tokens=2048)
        w.seq_lens = (2048 + np.random.default_rng([4, _S_LENS]).integers(
            256, 4096, size=32, endpoint=True)).astype(np.int32)
    elif name == "prefill256":
        w = Workload(name, 4, 32, 8, 16, 256, (4,), 9, k_outliers=2, v_outliers=1,
                     permute_pages=True)
        w.seq_lens = np.full(4, 4096, np.int32)
    else:
        raise KeyError(name)
    return _finish(w)


def custom(name="custom", batch=2, num_q_heads=8, num_kv_heads=2, page_size=16,
           q_len=1, seq_lens=(40, 17), fmt=4, seed=123, k_outliers=2,
           v_outliers=1, permute_pages=True, shared_prefix_seqs=0,
           shared_prefix_tokens=0, k_dist="normal") -> Workload:
    """A small workload of arbitrary shape for edge-case tests (the batch is
    len(seq_lens))."""
    batch = len(seq_lens)
    w = Workload(name, batch, num_q_heads, num_kv_heads, page_size, q_len,
                 (fmt,), seed, k_dist=k_dist, k_outliers=k_outliers,
                 v_outliers=v_outliers, permute_pages=permute_pages,
                 shared_prefix_seqs=shared_prefix_seqs,
                 shared_prefix_tokens=shared_prefix_tokens)
    w.seq_lens = np.asarray(seq_lens, np.int32)
    return _finish(w)


ALL = ("tiny", "batch8", "cbatch64", "target64x8k", "long128k", "specverify", "prefill256")
