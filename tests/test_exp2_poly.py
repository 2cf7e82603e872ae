"""The FMA-pipe exp2 of the tcgen05 kernel (exp2_fma2 in csrc/common.cuh), evaluated
step for step in float32 on the host: its relative error stays below 1e-4 over
every exponent the softmax can produce (x <= 8 after the lazy max update; x far
below 0 only for negligible terms)."""
import pathlib
import re

import numpy as np

CSRC = pathlib.Path(__file__).resolve().parents[1] / "paged_kv_attention_block_b200" / "csrc"


def _constants():
    text = (CSRC / "common.cuh").read_text()
    c = [float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f", text).group(1)) for i in range(4)]
    shift = float(re.search(r"kRoundShift = ([0-9.]+)f", text).group(1))
    return [np.float32(x) for x in c], np.float32(shift)


def _f32_fma(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma(x):
    c, shift = _constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + shift).astype(np.float32)
    j = (t - shift).astype(np.float32)
    f = _f32_fma(j, np.float32(-1.0), x)
    p = _f32_fma(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = _f32_fma(p, f, np.full_like(f, c[1]))
    p = _f32_fma(p, f, np.full_like(f, c[0]))
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-120.0, 8.0, 400001), np.arange(-120, 9, dtype=np.float64)]).astype(np.float32)
    got = exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-4


def test_round_trip_of_the_exponent_field():
    # Integers and half-integers: the range reduction lands exactly on them.
    x = np.arange(-124, 9, 0.5, dtype=np.float32)
    got = exp2_fma(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1.0) < 1e-4)
    assert np.all(np.isfinite(got)) and np.all(got > 0)


def test_masked_scores_vanish():
    got = exp2_fma(np.array([-np.inf, -1e30, -300.0], np.float32))
    assert np.all(got < 2.0 ** -120) and np.all(got >= 0)
