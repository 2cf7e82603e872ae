"""The integer widening of E2M1 codes the NVFP4 decode tiles use, restated in Python and pinned to the
oracle's E2M1 decoding (the format's value table).

The tiles widen a 32-bit word of eight codes into four f16x2 values, pair i holding codes i and i + 4
times 2^-14. Two integer forms do this. The pair-at-a-time form places a code's sign at f16 bit 15 and its
exponent and mantissa at bits 9-11. The whole-word form moves each code's sign from bit 3 to bit 6 of its
byte with one multiply-add (n + 7 (n & 8)) and then places the bytes with byte permutes. Here both forms
are checked against each other and against the E2M1 values for every code in every position."""
import numpy as np

import oracle.pkv_oracle as O

MASK = 0xFFFFFFFF


def pair_form(w: int, i: int) -> int:
    x = (w << (12 - 4 * i)) & MASK
    return ((x >> 3) & 0x0E000E00) | (x & 0x80008000)


def byte_perm(a: int, b: int, sel: int) -> int:
    src = [(a >> (8 * k)) & 0xFF for k in range(4)] + [(b >> (8 * k)) & 0xFF for k in range(4)]
    return sum(src[(sel >> (4 * k)) & 7] << (8 * k) for k in range(4))


def word_form(w: int) -> list:
    e, o = w & 0x0F0F0F0F, (w >> 4) & 0x0F0F0F0F
    es = (((e + 7 * (e & 0x08080808)) & MASK) << 1) & MASK
    os_ = (((o + 7 * (o & 0x08080808)) & MASK) << 1) & MASK
    return [byte_perm(es, 0, 0x2404), byte_perm(os_, 0, 0x2404), byte_perm(es, 0, 0x3414), byte_perm(os_, 0, 0x3414)]


def f16x2_values(v: int) -> tuple:
    h = np.array([v & 0xFFFF, v >> 16], dtype=np.uint16).view(np.float16).astype(np.float64)
    return float(h[0]), float(h[1])


def test_word_form_equals_pair_form_and_the_e2m1_values():
    rng = np.random.default_rng(7)
    words = [int(x) for x in rng.integers(0, 2**32, size=2000, dtype=np.uint64)]
    # Every code in every nibble position, its neighbours set to every other code.
    for pos in range(8):
        for c in range(16):
            for other in range(16):
                words.append((c << (4 * pos)) | sum(other << (4 * q) for q in range(8) if q != pos))
    for w in words:
        nib = [(w >> (4 * k)) & 0xF for k in range(8)]
        values = O.e2m1_decode(np.array(nib, dtype=np.uint8)).astype(np.float64)
        got = word_form(w)
        for i in range(4):
            assert got[i] == pair_form(w, i), (hex(w), i)
            lo, hi = f16x2_values(got[i])
            assert lo == values[i] * 2.0**-14 and hi == values[i + 4] * 2.0**-14, (hex(w), i)


def test_a_planted_sign_slip_is_caught():
    """The check above fails for a form that moves the sign one bit short."""
    w = 0x89ABCDEF
    e = w & 0x0F0F0F0F
    wrong = byte_perm((((e + 3 * (e & 0x08080808)) & MASK) << 1) & MASK, 0, 0x2404)
    nib = [(w >> (4 * k)) & 0xF for k in range(8)]
    values = O.e2m1_decode(np.array(nib, dtype=np.uint8)).astype(np.float64)
    assert f16x2_values(wrong) != (values[0] * 2.0**-14, values[4] * 2.0**-14)
