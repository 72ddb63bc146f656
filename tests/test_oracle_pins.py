"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here re-types the oracle's own formulas: every check compares it to
a closed form, a hand-derived fixture (tests/golden), a library routine
(scipy's Sylvester Hadamard matrix, numpy's little-endian bit packing,
torch's scaled_dot_product_attention in fp64) or an invariant of the
method (orthonormality, rotation invariance of exact attention, the
quantiser's error bound, power-of-two and sign equivariance, causality).
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from conftest import read_golden
from quantized_paged_kv_tq_b200 import workloads as W

BITS = (2, 3, 4, 8)


def Lof(b):
    return (1 << (b - 1)) - 1


def rand_bf16(rng, shape, scale=1.0):
    return W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * scale)


# --------------------------------------------------------------------- WHT
@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128])
def test_fwht_is_sylvester_hadamard(d):
    """Columns of the oracle's transform are the Sylvester Hadamard matrix:
    scipy.linalg.hadamard and the closed form (-1)^popcount(i & j)."""
    H32 = np.stack([oracle.fwht_f32(np.eye(d, dtype=np.float32)[j]) for j in range(d)], 1)
    H64 = np.stack([oracle.fwht_f64(np.eye(d)[j]) for j in range(d)], 1)
    ref = scipy.linalg.hadamard(d)
    i, j = np.meshgrid(np.arange(d), np.arange(d), indexing="ij")
    closed = np.where(np.vectorize(lambda a: bin(a).count("1") % 2)(i & j), -1, 1)
    assert np.array_equal(H32, ref) and np.array_equal(H64, ref)
    assert np.array_equal(ref, closed)
    # H H = d I exactly
    assert np.array_equal(H64 @ H64, d * np.eye(d))


def test_fwht_golden_h4():
    rows = np.array(read_golden("hadamard_d4.txt"), dtype=np.int64)
    H = np.stack([oracle.fwht_f64(np.eye(4)[j]) for j in range(4)], 1)
    assert np.array_equal(H, rows)


def test_rotate_d2_closed_form():
    """d = 2: y = [[1, 1], [1, -1]] x / sqrt(2)."""
    for a, b in [(1.0, 0.5), (-3.0, 2.0), (0.25, 0.25)]:
        x = W.f32_to_bf16_bits(np.array([a, b], np.float32))
        y = oracle.rotate_f32(x)
        assert np.allclose(y, [(a + b) / math.sqrt(2), (a - b) / math.sqrt(2)],
                           rtol=2e-7, atol=0)


def test_rotation_matches_fp64_hadamard_and_preserves_norm():
    rng = np.random.default_rng(5)
    H = scipy.linalg.hadamard(128).astype(np.float64)
    for _ in range(50):
        x = rand_bf16(rng, 128, scale=rng.uniform(0.01, 30))
        xf = W.bf16_bits_to_f32(x).astype(np.float64)
        y = oracle.rotate_f32(x).astype(np.float64)
        ref = H @ xf / math.sqrt(128)
        assert np.max(np.abs(y - ref)) <= 8 * 2.0 ** -24 * np.max(np.abs(ref)) * 8
        assert abs(np.linalg.norm(y) / np.linalg.norm(xf) - 1.0) < 1e-6


# --------------------------------------------------------------- quantiser
def test_golden_e0_codes():
    """x = e_0: every rotated entry is fp32(1/sqrt(128)), so every code is +L."""
    x = np.zeros(128, np.uint16)
    x[0] = 0x3F80  # bf16 1.0
    for bits_s, scale_hex, pattern in read_golden("quant_e0.txt"):
        bits = int(bits_s)
        packed, s = oracle.quantize_vector(x, bits)
        assert np.float32(s).view(np.uint32) == int(scale_hex, 16)
        pat = bytes.fromhex(pattern)
        assert packed.tobytes() == pat * (len(packed) // len(pat))


@pytest.mark.parametrize("bits", BITS)
def test_constant_vector_exact(bits):
    """x = a * 1: the rotation concentrates everything in y_0 = a sqrt(d)
    (exactly, in fp32), so code_0 = sign(a) L and every other code is 0."""
    for a in (1.0, -2.5, 0.375):
        x = W.f32_to_bf16_bits(np.full(128, a, np.float32))
        y = oracle.rotate_f32(x)
        assert y[0] == np.float32(np.float32(128 * a) * np.float32(1 / math.sqrt(128)))
        assert np.all(y[1:] == 0)
        codes, s = oracle.quantize_rotated(y, bits)
        assert codes[0] == (Lof(bits) if a > 0 else -Lof(bits))
        assert np.all(codes[1:] == 0)
        assert s == abs(y[0])


@pytest.mark.parametrize("bits", BITS)
def test_dequant_error_bound(bits):
    """|code s / L - y| <= s / (2L) for every element (plus fp32 slack)."""
    rng = np.random.default_rng(bits)
    L = Lof(bits)
    for _ in range(200):
        x = rand_bf16(rng, 128, scale=rng.uniform(0.1, 10))
        x_f = W.bf16_bits_to_f32(x)
        x_f[rng.choice(128, 3, replace=False)] *= 20
        x = W.f32_to_bf16_bits(x_f)
        y = oracle.rotate_f32(x).astype(np.float64)
        codes, s = oracle.quantize_rotated(y.astype(np.float32), bits)
        assert s == np.max(np.abs(y))
        assert np.all(np.abs(codes) <= L)
        err = np.abs(codes * float(s) / L - y)
        assert np.all(err <= float(s) / (2 * L) * (1 + 2.0 ** -20))
        # the absmax element is represented exactly by +-L
        i = int(np.argmax(np.abs(y)))
        assert abs(codes[i]) == L


@pytest.mark.parametrize("bits", BITS)
def test_pow2_scale_equivariance(bits):
    """x * 2^k gives identical codes and scale * 2^k (bit-exact)."""
    rng = np.random.default_rng(10 + bits)
    for _ in range(50):
        x = rand_bf16(rng, 128)
        p0, s0 = oracle.quantize_vector(x, bits)
        for k in (-3, 1, 5):
            xk = W.f32_to_bf16_bits(W.bf16_bits_to_f32(x) * np.float32(2.0 ** k))
            pk, sk = oracle.quantize_vector(xk, bits)
            assert np.array_equal(p0, pk)
            assert sk == np.float32(s0 * np.float32(2.0 ** k))


@pytest.mark.parametrize("bits", BITS)
def test_sign_symmetry(bits):
    rng = np.random.default_rng(20 + bits)
    for _ in range(50):
        x = rand_bf16(rng, 128)
        neg = x ^ np.uint16(0x8000)
        y, yn = oracle.rotate_f32(x), oracle.rotate_f32(neg)
        c, s = oracle.quantize_rotated(y, bits)
        cn, sn = oracle.quantize_rotated(yn, bits)
        assert s == sn and np.array_equal(c, -cn)


@pytest.mark.parametrize("bits", BITS)
def test_zero_vector(bits):
    packed, s = oracle.quantize_vector(np.zeros(128, np.uint16), bits)
    assert s == 0.0
    assert np.array_equal(oracle.unpack_codes(packed, 128, bits), np.zeros(128))


def test_round_half_away_from_zero_at_ties():
    """Constructed ties: with s a multiple of L chosen so that y*L/s is exact,
    n + 1/2 rounds away from zero."""
    y = np.zeros(128, np.float32)
    y[:6] = [7.0, 2.5, -2.5, 0.5, -0.5, 1.5]
    c, s = oracle.quantize_rotated(y, 4)                      # L = 7, s = 7
    assert s == 7 and list(c[:6]) == [7, 3, -3, 1, -1, 2]
    y = np.zeros(128, np.float32)
    y[:4] = [1.0, 0.5, -0.5, 0.25]
    c, s = oracle.quantize_rotated(y, 2)                      # L = 1
    assert list(c[:4]) == [1, 1, -1, 0]
    y = np.zeros(128, np.float32)
    y[:4] = [3.0, 0.5, -1.5, 2.5]
    c, s = oracle.quantize_rotated(y, 3)                      # L = 3
    assert list(c[:4]) == [3, 1, -2, 3]
    y = np.zeros(128, np.float32)
    y[:3] = [127.0, 2.5, -126.5]
    c, s = oracle.quantize_rotated(y, 8)                      # L = 127
    assert list(c[:3]) == [127, 3, -127]


def _fl32(q):
    """Nearest fp32 (ties to even) of an exact rational q (normal range)."""
    from fractions import Fraction
    if q == 0:
        return Fraction(0)
    sgn = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    m = a / ulp
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sgn * n * ulp


def _round_half_away(q):
    from fractions import Fraction
    sgn = -1 if q < 0 else 1
    a = abs(q)
    n = a.numerator // a.denominator
    return sgn * (n + (1 if a - n >= Fraction(1, 2) else 0))


def test_division_order_golden():
    """fl32(y L) / s with an IEEE division, not y fl32(L / s) nor
    fl32(y / s) L: on each fixture row the three orders give different
    codes; the expected one is derived again here with exact rationals."""
    from fractions import Fraction
    rows = read_golden("quant_division_order.txt")
    assert len(rows) >= 9
    for bits_s, y_hex, s_hex, code_s, other_s in rows:
        bits, L = int(bits_s), Lof(int(bits_s))
        y = np.uint32(int(y_hex, 16)).view(np.float32)
        s = np.uint32(int(s_hex, 16)).view(np.float32)
        Y, S = Fraction(float(y)), Fraction(float(s))
        want = _round_half_away(_fl32(_fl32(Y * L) / S))
        recip = _round_half_away(_fl32(Y * _fl32(Fraction(L) / S)))
        late = _round_half_away(_fl32(_fl32(Y / S) * L))
        assert want == int(code_s) and recip == late == int(other_s) != want
        vec = np.zeros(128, np.float32)
        vec[0], vec[1], vec[2] = s, y, -y
        codes, scale = oracle.quantize_rotated(vec, bits)
        assert scale == s and codes[0] == L
        assert codes[1] == want and codes[2] == -want


@pytest.mark.parametrize("bits,y,s,code", [(4, 1.25, 3.5, 3), (3, 1.25, 1.5, 3),
                                           (8, 0.25, 5.0, 6), (2, 0.75, 1.5, 1)])
def test_exact_ties_with_scale_not_L(bits, y, s, code):
    """Ties y L / s = n + 1/2 that are exact at every fp32 step with s != L
    (and s not a power of two for turbo4/3/8): 1.25*7/3.5 = 2.5 -> 3,
    1.25*3/1.5 = 2.5 -> 3, 0.25*127/5 = 6.35 -> 6 (no tie, a plain case),
    0.75*1/1.5 = 0.5 -> 1; negatives mirror them."""
    vec = np.zeros(128, np.float32)
    vec[0], vec[1], vec[2] = s, y, -y
    codes, scale = oracle.quantize_rotated(vec, bits)
    assert scale == np.float32(s) and list(codes[1:3]) == [code, -code]


def test_fwht_stage_order_golden():
    """Strides 1, 2, 4 in that order, each butterfly rounded to fp32: the
    hand-derived d = 8 fixture differs bit for bit from the reverse order
    (and from the exact transform)."""
    want = np.array([int(h, 16) for _, h in read_golden("fwht_stage_order_d8.txt")],
                    np.uint32).view(np.float32)
    x = np.array([1.0, 2.0 ** -24, -1.0, 2.0 ** -24, 0, 0, 0, 0], np.float32)
    got = oracle.fwht_f32(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    # the rotation: the same butterflies, then one multiply by fp32(1/sqrt(8))
    c = np.float32(1 / math.sqrt(8))
    y = oracle.rotate_f32(W.f32_to_bf16_bits(x))
    assert np.array_equal(y.view(np.uint32), (want * c).view(np.uint32))
    # embedded in a 128-vector: strides 8..64 only meet zeros, so entries
    # 0..7 carry the same values and entries 8i..8i+7 copy them
    x128 = np.zeros(128, np.float32)
    x128[:8] = x
    y128 = oracle.rotate_f32(W.f32_to_bf16_bits(x128))
    c128 = np.float32(1 / math.sqrt(128))
    assert np.array_equal(y128.view(np.uint32), np.tile(want * c128, 16).view(np.uint32))


@pytest.mark.parametrize("bits", BITS)
def test_packing_matches_numpy_little_endian_bits(bits):
    rng = np.random.default_rng(30 + bits)
    L = Lof(bits)
    for _ in range(50):
        codes = rng.integers(-L, L, size=128, endpoint=True).astype(np.int32)
        u = (codes + L).astype(np.uint32)
        bitmat = ((u[:, None] >> np.arange(bits)) & 1).astype(np.uint8)
        ref = np.packbits(bitmat.ravel(), bitorder="little")
        got = oracle.pack_codes(codes, bits)
        assert np.array_equal(got, ref)
        assert np.array_equal(oracle.unpack_codes(got, 128, bits), codes)


def test_packing_golden():
    for bits_s, codes_s, hexbytes in read_golden("pack_examples.txt"):
        bits = int(bits_s)
        codes = np.array([int(c) for c in codes_s.split(",")], np.int32)
        assert oracle.pack_codes(codes, bits).tobytes() == bytes.fromhex(hexbytes)


def test_compression_ratio_turbo4():
    """The page's compression table gives 3.7x for turbo4 over BF16 ("TurboQuant
    is a memory trade"; xinfer-ai performance tips: "turbo4 gives 3.7x
    compression"): 256 B of bf16 vs 64 B of 4-bit codes + a 4 B fp32 scale."""
    bf16 = oracle.block_bytes(16, 128, 16)
    t4 = oracle.block_bytes(4, 128, 16)
    assert bf16 == 16 * 256 and t4 == 16 * 68
    assert abs(bf16 / t4 - 3.7) < 0.1


# --------------------------------------------------------------- attention
def _sdpa(q, K, V, causal_last):
    """torch fp64 SDPA of rows q [R][d] over K/V [n][d]; row r sees keys
    0..causal_last[r]."""
    n = K.shape[0]
    mask = torch.tensor(np.arange(n)[None, :] <= np.asarray(causal_last)[:, None])
    return torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(K)[None], torch.tensor(V)[None],
        attn_mask=mask[None]).numpy()[0]


def _pools(w, fmt):
    bb = oracle.block_bytes(fmt, w.head_dim, w.page_size)
    if fmt == 16:
        shape = (w.num_pages, w.num_kv_heads, w.page_size, w.head_dim)
        return np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    shape = (w.num_pages, w.num_kv_heads, bb)
    return np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)


def _fill(w, fmt):
    kp, vp = _pools(w, fmt)
    for slots, k, v in w.iter_fill():
        if fmt == 16:
            oracle.append_bf16(k, v, slots, w.page_size, kp, vp)
        else:
            oracle.quantize_append(k, v, slots, fmt, w.page_size, kp, vp)
    return kp, vp


def _unpack_u(pool, fmt, page, kvh, off, P, dim_major, d=128):
    """Offset-binary values u of one token via numpy's little-endian
    unpackbits: K blocks hold token rows, V blocks dimension rows."""
    cb = d * fmt // 8
    blk = pool[page, kvh]
    if dim_major:
        bits = np.unpackbits(blk[:P * cb], bitorder="little").reshape(d, P, fmt)[:, off]
    else:
        bits = np.unpackbits(blk[off * cb:(off + 1) * cb], bitorder="little").reshape(d, fmt)
    return (bits * (1 << np.arange(fmt))).sum(1)


def _dequant_numpy(pool, fmt, page, kvh, off, P, dim_major=False, d=128):
    """Rotated dequantised row (code * s / L)."""
    cb = d * fmt // 8
    blk = pool[page, kvh]
    u = _unpack_u(pool, fmt, page, kvh, off, P, dim_major, d)
    s = blk[P * cb + 4 * off:P * cb + 4 * off + 4].view(np.float32)[0]
    L = Lof(fmt)
    return (u - L) * float(s) / L


@pytest.mark.parametrize("fmt", [16, 4, 3, 8, 2])
@pytest.mark.parametrize("q_len", [1, 3])
def test_paged_decode_matches_sdpa(fmt, q_len):
    """The paged decode equals textbook softmax attention (torch SDPA, fp64)
    on the de-rotated dequantised K/V gathered through the page table, with
    the causal limit j <= seq_len - q_len + t and GQA group h // group."""
    w = W.custom(batch=3, num_q_heads=6, num_kv_heads=2, page_size=16,
                 q_len=q_len, seq_lens=(37, 16, 5 + q_len), fmt=fmt, seed=fmt)
    kp, vp = _fill(w, fmt)
    q = w.queries()
    out = oracle.paged_decode(q, fmt, w.page_size, kp, vp, w.page_table,
                              w.seq_lens, w.num_kv_heads)
    H = scipy.linalg.hadamard(128) / math.sqrt(128)
    P = w.page_size
    for b in range(w.batch):
        n = int(w.seq_lens[b])
        for h in range(w.num_q_heads):
            kvh = h // w.group
            K = np.zeros((n, 128))
            V = np.zeros((n, 128))
            for j in range(n):
                page, off = int(w.page_table[b, j // P]), j % P
                if fmt == 16:
                    K[j] = W.bf16_bits_to_f32(kp[page, kvh, off])
                    V[j] = W.bf16_bits_to_f32(vp[page, kvh, off])
                else:
                    K[j] = H @ _dequant_numpy(kp, fmt, page, kvh, off, P)
                    V[j] = H @ _dequant_numpy(vp, fmt, page, kvh, off, P, dim_major=True)
            qr = W.bf16_bits_to_f32(q[b, :, h]).astype(np.float64)
            ref = _sdpa(qr, K, V, [n - q_len + t for t in range(q_len)])
            assert np.max(np.abs(out[b, :, h] - ref)) < 1e-11


def test_rotation_invariance_of_exact_attention():
    """Attending in the Hadamard basis (q, K, V rotated, output rotated back)
    equals plain attention when nothing is quantised."""
    rng = np.random.default_rng(40)
    for n in (1, 7, 300):
        q = rng.standard_normal(128)
        K = rng.standard_normal((n, 128)) * 2
        V = rng.standard_normal((n, 128))
        Kr = np.stack([oracle.fwht_f64(k) / math.sqrt(128) for k in K])
        Vr = np.stack([oracle.fwht_f64(v) / math.sqrt(128) for v in V])
        a = oracle.attention_f64(q, K, V, rotated=False)
        b = oracle.attention_f64(q, Kr, Vr, rotated=True)
        assert np.max(np.abs(a - b)) < 1e-5
        assert np.max(np.abs(a - b)) < 1e-12


def test_single_key_and_identical_keys():
    rng = np.random.default_rng(41)
    q = rng.standard_normal(128)
    v = rng.standard_normal(128)
    k = rng.standard_normal(128)
    # one key: output is that value, whatever the score
    assert np.allclose(oracle.attention_f64(q, k[None], v[None], False), v, atol=1e-15)
    vr = oracle.fwht_f64(v) / math.sqrt(128)
    assert np.allclose(oracle.attention_f64(q, k[None], vr[None], True), v, atol=1e-13)
    # identical keys: output is the mean of the values
    V = rng.standard_normal((9, 128))
    K = np.repeat(k[None], 9, 0)
    assert np.allclose(oracle.attention_f64(q, K, V, False), V.mean(0), atol=1e-14)


def test_brute_force_softmax_tiny():
    """Explicit exp/sum on a 4-dimensional, 3-key case."""
    q = np.array([0.5, -1.0, 2.0, 0.0])
    K = np.array([[1.0, 0, 0, 0], [0, 1.0, 0, 0], [0, 0, 1.0, 1.0]])
    V = np.array([[1.0, 2, 3, 4], [-1.0, 0, 1, 0], [0.0, 0, 0, 8]])
    s = [0.5 / 2, -1.0 / 2, 2.0 / 2]
    e = [math.exp(x) for x in s]
    ref = sum(ei * V[i] for i, ei in enumerate(e)) / sum(e)
    assert np.allclose(oracle.attention_f64(q, K, V, False), ref, atol=1e-15)


@pytest.mark.parametrize("fmt", [4, 16])
def test_causal_rows_equal_shorter_single_token_decode(fmt):
    """Row t of a q_len = 4 verify equals a q_len = 1 decode of the same
    query at seq_len - 3 + t."""
    w = W.custom(batch=2, num_q_heads=4, num_kv_heads=1, q_len=4,
                 seq_lens=(50, 21), fmt=fmt, seed=7)
    kp, vp = _fill(w, fmt)
    q = w.queries()
    out = oracle.paged_decode(q, fmt, w.page_size, kp, vp, w.page_table,
                              w.seq_lens, w.num_kv_heads)
    for t in range(4):
        lens = w.seq_lens - 3 + t
        single = oracle.paged_decode(np.ascontiguousarray(q[:, t:t + 1]), fmt,
                                     w.page_size, kp, vp, w.page_table, lens,
                                     w.num_kv_heads)
        assert np.array_equal(single[:, 0], out[:, t])


@pytest.mark.parametrize("bits,P", [(4, 16), (3, 16), (2, 32), (8, 64), (3, 64)])
def test_quantize_append_layout_and_skip(bits, P):
    """K rows land at block (page, head), token row `offset`; V codes land
    dim-major (dimension i's row holds every token's field i); scales follow
    the codes; slot -1 writes nothing; other tokens' fields are untouched."""
    rng = np.random.default_rng(50 + bits)
    k = rand_bf16(rng, (4, 2, 128))
    v = rand_bf16(rng, (4, 2, 128))
    cb = 128 * bits // 8
    kp = np.zeros((4, 2, oracle.block_bytes(bits, 128, P)), np.uint8)
    vp = np.zeros_like(kp)
    slots = np.array([5, -1, P * 3 + P - 1, 6])
    oracle.quantize_append(k, v, slots, bits, P, kp, vp)
    L = Lof(bits)
    for t, (page, off) in ((0, (0, 5)), (2, (3, P - 1)), (3, (0, 6))):
        for h in range(2):
            pk, sk = oracle.quantize_vector(k[t, h], bits)
            yv = oracle.rotate_f32(v[t, h])
            cv, sv = oracle.quantize_rotated(yv, bits)
            assert np.array_equal(kp[page, h, off * cb:(off + 1) * cb], pk)
            assert np.array_equal(_unpack_u(vp, bits, page, h, off, P, True), cv + L)
            so = P * cb + 4 * off
            assert kp[page, h, so:so + 4].view(np.float32)[0] == sk
            assert vp[page, h, so:so + 4].view(np.float32)[0] == sv
    written = {(0, 5), (3, P - 1), (0, 6)}
    for page in range(4):
        for off in range(P):
            if (page, off) not in written:
                assert not kp[page, :, off * cb:(off + 1) * cb].any()
                for h in range(2):
                    assert not _unpack_u(vp, bits, page, h, off, P, True).any()


# ----------------------------------------------------------------- fp8
FP8 = oracle.FP8


def test_e4m3_values_match_torch_float8():
    """Every E4M3 code's value equals torch's float8_e4m3fn (a library
    routine), NaN codes included."""
    codes = torch.arange(256, dtype=torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    assert np.array_equal(np.isnan(lib_vals), np.isnan(ours))
    ok = ~np.isnan(ours)
    assert np.array_equal(lib_vals[ok], ours[ok])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_rounding_golden():
    for v_hex, c_hex in read_golden("e4m3_rounding.txt"):
        v = np.uint32(int(v_hex, 16)).view(np.float32)
        assert oracle.e4m3_encode(float(v)) == int(c_hex, 16), v_hex


def test_e4m3_encode_matches_torch_cast():
    """Round to nearest, ties to even, saturating below the NaN midpoint:
    the same codes as torch's fp32 -> float8_e4m3fn cast on values spread
    over every binade and the subnormals."""
    rng = np.random.default_rng(60)
    x = rng.standard_normal(20000) * 10.0 ** rng.uniform(-4.5, 2.6, 20000)
    x = np.clip(x, -460.0, 460.0).astype(np.float32)
    lib_codes = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    assert np.array_equal(lib_codes, ours)


def test_fp8_quantizer_closed_forms():
    """x = a e_j: s = |a| and y_j = fl(fl(a 448) / |a|) = +-448 exactly, so
    code j is 0x7E or 0xFE and every other code is +0; x = 0 gives s = 0 and
    codes 0."""
    for a, j in ((1.0, 0), (-3.5, 7), (0.0078125, 127)):
        x = np.zeros(128, np.float32)
        x[j] = a
        codes, s = oracle.fp8_quantize_vector(W.f32_to_bf16_bits(x))
        assert s == abs(a)
        assert codes[j] == (0x7E if a > 0 else 0xFE)
        assert np.all(np.delete(codes, j) == 0)
    codes, s = oracle.fp8_quantize_vector(np.zeros(128, np.uint16))
    assert s == 0 and not codes.any()


def test_fp8_pow2_equivariance_and_error_bound():
    """x 2^k keeps every code (bit-exact) and scales s by 2^k; the
    dequantised value is within half an E4M3 step of x: |xhat - x| <=
    s/448 * max(|y| 2^-4, 2^-10) (plus fp32 slack)."""
    rng = np.random.default_rng(61)
    for _ in range(100):
        xb = rand_bf16(rng, 128, scale=rng.uniform(0.01, 50))
        c0, s0 = oracle.fp8_quantize_vector(xb)
        for k in (-4, 3):
            xk = W.f32_to_bf16_bits(W.bf16_bits_to_f32(xb) * np.float32(2.0 ** k))
            ck, sk = oracle.fp8_quantize_vector(xk)
            assert np.array_equal(c0, ck) and sk == np.float32(s0 * np.float32(2.0 ** k))
        x = W.bf16_bits_to_f32(xb).astype(np.float64)
        xhat = np.array([oracle.e4m3_value(c) for c in c0]) * float(s0) / 448.0
        y = np.abs(x) * 448.0 / float(s0)
        bound = float(s0) / 448.0 * np.maximum(y * 2.0 ** -4, 2.0 ** -10) * (1 + 2.0 ** -20)
        assert np.all(np.abs(xhat - x) <= bound + 1e-30)
        assert np.max(np.abs(xhat)) == float(s0)          # the absmax element is exact


def test_fp8_append_layout():
    """fp8 blocks have turbo8's layout: K token rows of 128 code bytes, V
    dimension rows of page_size code bytes, fp32 scales after the codes."""
    rng = np.random.default_rng(62)
    P = 16
    k = rand_bf16(rng, (3, 2, 128))
    v = rand_bf16(rng, (3, 2, 128))
    bb = oracle.block_bytes(FP8, 128, P)
    assert bb == P * 132
    kp = np.zeros((2, 2, bb), np.uint8)
    vp = np.zeros_like(kp)
    slots = np.array([3, -1, P + 15])
    oracle.quantize_append(k, v, slots, FP8, P, kp, vp)
    for t, (page, off) in ((0, (0, 3)), (2, (1, 15))):
        for h in range(2):
            ck, sk = oracle.fp8_quantize_vector(k[t, h])
            cv, sv = oracle.fp8_quantize_vector(v[t, h])
            assert np.array_equal(kp[page, h, off * 128:(off + 1) * 128], ck)
            assert np.array_equal(vp[page, h, :P * 128].reshape(128, P)[:, off], cv)
            assert kp[page, h, P * 128 + 4 * off:P * 128 + 4 * off + 4].view(np.float32)[0] == sk
            assert vp[page, h, P * 128 + 4 * off:P * 128 + 4 * off + 4].view(np.float32)[0] == sv


@pytest.mark.parametrize("q_len", [1, 3])
def test_fp8_paged_decode_matches_sdpa(q_len):
    """fp8 decode is plain softmax attention (no rotation) on the
    dequantised K and V: torch SDPA in fp64 on the same values."""
    w = W.custom(batch=2, num_q_heads=4, num_kv_heads=2, page_size=16, q_len=q_len,
                 seq_lens=(45, 17 + q_len), fmt=FP8, seed=63)
    kp, vp = _pools(w, FP8)
    for slots, k, v in w.iter_fill():
        oracle.quantize_append(k, v, slots, FP8, w.page_size, kp, vp)
    q = w.queries()
    out = oracle.paged_decode(q, FP8, w.page_size, kp, vp, w.page_table, w.seq_lens,
                              w.num_kv_heads)
    P = w.page_size
    for b in range(w.batch):
        n = int(w.seq_lens[b])
        for h in range(w.num_q_heads):
            kvh = h // w.group
            K = np.zeros((n, 128))
            V = np.zeros((n, 128))
            for j in range(n):
                page, off = int(w.page_table[b, j // P]), j % P
                blk_k, blk_v = kp[page, kvh], vp[page, kvh]
                sk = blk_k[P * 128 + 4 * off:P * 128 + 4 * off + 4].view(np.float32)[0]
                sv = blk_v[P * 128 + 4 * off:P * 128 + 4 * off + 4].view(np.float32)[0]
                K[j] = torch.from_numpy(blk_k[off * 128:(off + 1) * 128].copy()).view(
                    torch.float8_e4m3fn).double().numpy() * float(sk) / 448.0
                V[j] = torch.from_numpy(blk_v[:P * 128].reshape(128, P)[:, off].copy()).view(
                    torch.float8_e4m3fn).double().numpy() * float(sv) / 448.0
            qr = W.bf16_bits_to_f32(q[b, :, h]).astype(np.float64)
            ref = _sdpa(qr, K, V, [n - q_len + t for t in range(q_len)])
            assert np.max(np.abs(out[b, :, h] - ref)) < 1e-11


def test_fp8_division_order_golden():
    """fl(fl(x 448) / s): on each row the exact quotient is an E4M3
    midpoint reached exactly, so the code is the even neighbour; the
    reciprocal multiply (rows 1-3) or the late multiply (rows 4-6) would
    give the odd one."""
    from fractions import Fraction
    for x_hex, s_hex, code_s, other_s in read_golden("fp8_division_order.txt"):
        x = np.uint32(int(x_hex, 16)).view(np.float32)
        s = np.uint32(int(s_hex, 16)).view(np.float32)
        X, S = Fraction(float(x)), Fraction(float(s))
        y = _fl32(_fl32(X * 448) / S)
        assert y == X * 448 / S                        # both steps exact: the midpoint itself
        lo_hi = sorted(oracle.e4m3_value(c) for c in (int(code_s, 16), int(other_s, 16)))
        assert y == (Fraction(lo_hi[0]) + Fraction(lo_hi[1])) / 2
        assert int(code_s, 16) % 2 == 0 and int(other_s, 16) % 2 == 1
        vec = np.zeros(128, np.float32)
        vec[0], vec[1] = s, x
        codes, scale = oracle.fp8_quantize_vector(W.f32_to_bf16_bits(vec))
        assert scale == s and codes[0] == 0x7E and codes[1] == int(code_s, 16)
        recip = oracle.e4m3_encode(float(_fl32(X * _fl32(Fraction(448) / S))))
        late = oracle.e4m3_encode(float(_fl32(_fl32(X / S) * 448)))
        assert int(other_s, 16) in (recip, late)
