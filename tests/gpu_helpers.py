"""Shared plumbing for the GPU parity tests.

The GPU side fills its cache through tq_quantize_append / tq_append_bf16 from
the seeded generator's values and decodes through tq_paged_decode*.  The
oracle side builds its OWN cache from the same generator values (never from
GPU output) for the sequences it checks, remapping their physical pages to a
compact pool, and decodes it in fp64.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_paged_kv_tq_b200 import tq
from quantized_paged_kv_tq_b200 import workloads as W

ATOL = 2e-3      # max-abs error bound on attention outputs
RTOL_L2 = 1e-3   # relative L2 error bound on attention outputs


def dev_bf16(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_fill(w: W.Workload, fmt: int, chunk: int = 1 << 16, cache=None,
             shuffle_seed: int | None = None) -> tq.Cache:
    """Allocate and fill a GPU cache with every context token of w
    (optionally appending each chunk's tokens in a shuffled order)."""
    if cache is None:
        cache = tq.Cache(fmt, w.num_pages, w.num_kv_heads, w.page_size)
    for slots, k, v in w.iter_fill(chunk):
        if shuffle_seed is not None:
            p = np.random.default_rng(shuffle_seed).permutation(len(slots))
            slots, k, v = slots[p], k[p], v[p]
        ks, vs, ss = dev_bf16(k), dev_bf16(v), dev(slots.astype(np.int64))
        if fmt == 16:
            tq.tq_append_bf16(ks, vs, ss, cache)
        else:
            tq.tq_quantize_append(ks, vs, ss, fmt, cache)
    torch.cuda.synchronize()
    return cache


def gpu_decode(w: W.Workload, fmt: int, cache: tq.Cache, q: np.ndarray | None = None,
               page_table=None, seq_lens=None) -> np.ndarray:
    q = w.queries() if q is None else q
    pt = w.page_table if page_table is None else page_table
    sl = w.seq_lens if seq_lens is None else seq_lens
    out = torch.full((q.shape[0], w.q_len, w.num_q_heads, w.head_dim), float("nan"),
                     dtype=torch.float32, device="cuda")
    fn = tq.tq_paged_decode_bf16 if fmt == 16 else tq.tq_paged_decode
    fn(dev_bf16(q), cache, dev(pt.astype(np.int32)), dev(sl.astype(np.int32)), w.q_len, out,
       max_seq_len=int(np.max(sl)))
    torch.cuda.synchronize()
    return out.cpu().numpy()


def oracle_pools(fmt: int, npages: int, w: W.Workload):
    bb = oracle.block_bytes(fmt, w.head_dim, w.page_size)
    if fmt == 16:
        shape = (npages, w.num_kv_heads, w.page_size, w.head_dim)
        return np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    return (np.zeros((npages, w.num_kv_heads, bb), np.uint8),
            np.zeros((npages, w.num_kv_heads, bb), np.uint8))


def oracle_decode(w: W.Workload, fmt: int, seqs, q: np.ndarray | None = None) -> np.ndarray:
    """fp64 oracle output for sequences `seqs`, from an oracle-built cache."""
    seqs = np.asarray(seqs)
    q = w.queries() if q is None else q
    P = w.page_size
    pt = w.page_table[seqs]
    lens = w.seq_lens[seqs]
    used = sorted({int(p) for i, b in enumerate(seqs)
                   for p in pt[i, :(int(lens[i]) + P - 1) // P]})
    remap = {p: i for i, p in enumerate(used)}
    cpt = np.full(pt.shape, -1, np.int32)
    for i in range(len(seqs)):
        n = (int(lens[i]) + P - 1) // P
        cpt[i, :n] = [remap[int(p)] for p in pt[i, :n]]
    kp, vp = oracle_pools(fmt, len(used), w)
    phys = np.array(used, np.int64)
    for j in range(0, len(phys), 4096):
        blk = phys[j:j + 4096]
        slots = (blk[:, None] * P + np.arange(P)[None, :]).ravel()
        k, v = w.kv_for_slots(slots)
        cslots = ((np.arange(j, j + len(blk))[:, None]) * P + np.arange(P)[None, :]).ravel()
        if fmt == 16:
            oracle.append_bf16(k, v, cslots, P, kp, vp)
        else:
            oracle.quantize_append(k, v, cslots, fmt, P, kp, vp)
    return oracle.paged_decode(np.ascontiguousarray(q[seqs]), fmt, P, kp, vp, cpt, lens,
                               w.num_kv_heads)


def check_close(got: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    got = got.astype(np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max())
    rel_l2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= ATOL, f"{what}: max-abs {max_abs:.3e} > {ATOL}"
    assert rel_l2 <= RTOL_L2, f"{what}: rel-L2 {rel_l2:.3e} > {RTOL_L2}"
    return {"max_abs": max_abs, "rel_l2": rel_l2}


FP8 = 17


def code_bits(fmt: int) -> int:
    """Bits per code of a cache format (fp8 codes are bytes)."""
    return 8 if fmt == FP8 else fmt


def k_unswizzle(rows: np.ndarray, off: int, fmt: int) -> np.ndarray:
    """Undo the documented 16-byte chunk permutation of a K token row at
    offset `off` in its page (include/tq.h: logical chunk c is stored at
    chunk c ^ w(off))."""
    w = {2: (off >> 2) & 1, 4: (off >> 1) & 3, 8: off & 7}.get(code_bits(fmt), 0)
    if w == 0:
        return rows
    n = rows.shape[-1] // 16
    chunks = rows.reshape(rows.shape[:-1] + (n, 16))
    return chunks[..., [c ^ w for c in range(n)], :].reshape(rows.shape)


def k_pool_logical(kp: np.ndarray, fmt: int, P: int) -> np.ndarray:
    """A K pool [pages][heads][block] with every token row's chunk
    permutation undone (token rows in plain packed order, scales as they
    are)."""
    out = kp.copy()
    cb = 128 * code_bits(fmt) // 8
    for r in range(P):
        out[..., r * cb:(r + 1) * cb] = k_unswizzle(kp[..., r * cb:(r + 1) * cb], r, fmt)
    return out


def gpu_rows(cache: tq.Cache, slots: np.ndarray, P: int, fmt: int):
    """K packed rows, V offset-binary values (read from the dim-major V
    block) and the fp32 scales of K and V at `slots` (host copy)."""
    pages = torch.as_tensor(slots // P, device="cuda")
    offs = slots % P
    kb = cache.k_pages[pages].cpu().numpy()
    vb = cache.v_pages[pages].cpu().numpy()
    cb = 128 * fmt // 8
    idx = np.arange(len(slots))
    kc = np.stack([k_unswizzle(kb[i, :, offs[i] * cb:(offs[i] + 1) * cb], int(offs[i]), fmt)
                   for i in idx])
    vbits = np.unpackbits(vb[:, :, :P * cb], axis=-1, bitorder="little")
    vbits = vbits.reshape(len(slots), vb.shape[1], 128, P, fmt)[idx, :, :, offs]
    vu = (vbits * (1 << np.arange(fmt))).sum(-1)
    so = P * cb
    ks = np.stack([kb[i, :, so + 4 * offs[i]:so + 4 * offs[i] + 4] for i in idx]).view(np.float32)
    vs = np.stack([vb[i, :, so + 4 * offs[i]:so + 4 * offs[i] + 4] for i in idx]).view(np.float32)
    return kc, vu, ks[..., 0], vs[..., 0]


def oracle_rows(w: W.Workload, slots: np.ndarray, fmt: int):
    k, v = w.kv_for_slots(slots)
    n, H = len(slots), w.num_kv_heads
    cb = 128 * fmt // 8
    L = (1 << (fmt - 1)) - 1
    kc = np.zeros((n, H, cb), np.uint8)
    vu = np.zeros((n, H, 128), np.int64)
    ks = np.zeros((n, H), np.float32)
    vs = np.zeros_like(ks)
    for i in range(n):
        for h in range(H):
            kc[i, h], ks[i, h] = oracle.quantize_vector(k[i, h], fmt)
            codes, vs[i, h] = oracle.quantize_rotated(oracle.rotate_f32(v[i, h]), fmt)
            vu[i, h] = codes + L
    return kc, vu, ks, vs
