"""The quantiser's fast path, checked in fp32 on the CPU.

The definition of a code ("xInfer: Pure-Rust LLM Inference Without a Python
Runtime", section "What actually sits between the request and the tokens":
per-head absmax quantisation after the rotation) is
code = clamp(round_half_away(fl(y L) / s), -L, L), with an IEEE fp32
division.  The CUDA quantiser replaces the division by a multiplication with
fl(1/s) and rounds with rint, and takes the division only when
q = fl(fl(y L) * fl(1/s)) lies within a margin of a half-integer.  Its
argument is that q and the IEEE quotient differ by less than 3.001 L 2^-24,
so the margin is the smallest power of two >= 4 L, times 2^-24.  This test
restates those steps with numpy's IEEE fp32 arithmetic and checks on values
placed next to half-integers that wherever the fast path decides, it
decides the code of the definition.  It exercises no CUDA code.
"""
import numpy as np
import pytest

F32 = np.float32


def margin(L):
    m = 2.0 ** -24
    p = 1
    while p < 4 * L:
        p *= 2
        m *= 2.0
    return m


def roundf(x):
    return np.sign(x) * np.floor(np.abs(x) + F32(0.5))


def adversarial(L, n, rng):
    """(y, s) with y L / s spread over [-L, L], half of them within 2^-26 ..
    2^-8 of a half-integer; s over 2^-100 .. 2^100."""
    s = ((rng.random(n, dtype=np.float32) * F32(2) + F32(0.5)) *
         F32(2.0) ** rng.integers(-100, 100, n).astype(np.float32)).astype(F32)
    half = rng.integers(-L, L, n).astype(F32) + F32(0.5)
    jitter = ((rng.random(n, dtype=np.float32) - F32(0.5)) *
              F32(2.0) ** rng.integers(-26, -8, n).astype(np.float32))
    y = ((half + jitter) * s / F32(L)).astype(F32)
    y[: n // 2] = ((rng.random(n // 2, dtype=np.float32) * F32(2) - F32(1)) * s[: n // 2]).astype(F32)
    return np.clip(y, -s, s).astype(F32), s


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_fast_path_agrees_with_the_ieee_quotient(bits):
    L = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(100 + bits)
    y, s = adversarial(L, 1 << 18, rng)
    t = (y * F32(L)).astype(F32)
    q = (t * (F32(1) / s).astype(F32)).astype(F32)
    magic = F32(12582912.0)                       # 1.5 2^23: fp32 spacing 1 above 2^23
    n = ((q + magic).astype(F32) - magic).astype(F32)
    assert np.array_equal(n, np.rint(q))          # the add rounds to nearest even
    d = (q - n).astype(F32)
    fast = np.abs(d) <= F32(0.5 - margin(L))
    ref = np.clip(roundf((t / s).astype(F32)), -L, L)
    assert np.array_equal(n[fast], ref[fast])
    assert np.all(np.abs(n[fast]) <= L)
    # the adversarial half of the sample reaches the fallback, the rest
    # almost never does (about 2 margin per value)
    assert (~fast).sum() > 0
    assert (~fast[: len(fast) // 2]).mean() < 64 * margin(L)


def test_margin_is_needed():
    """A margin 16 times smaller than the stated one lets the fast path
    decide some codes against the definition (turbo8, L = 127), so the test
    above has the power to catch a margin that is too small."""
    L = 127
    rng = np.random.default_rng(7)
    wrong = 0
    for _ in range(8):
        y, s = adversarial(L, 1 << 18, rng)
        t = (y * F32(L)).astype(F32)
        q = (t * (F32(1) / s).astype(F32)).astype(F32)
        n = np.rint(q).astype(F32)
        fast = np.abs((q - n).astype(F32)) <= F32(0.5 - margin(L) / 16)
        ref = np.clip(roundf((t / s).astype(F32)), -L, L)
        wrong += int((n[fast] != ref[fast]).sum())
    assert wrong > 0
