"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function raises ``AssertionError`` when the oracle disagrees
with what the pages or the mathematics fix.  ``test_oracle_pins.py`` runs them
on the real oracle; ``test_oracle_mutations.py`` plants plausible mistakes in
the oracle and checks that at least one pin fails for each.

Independent references used here:
* torch's ``float8_e4m3fn`` and ``bfloat16`` CPU conversions (library codecs);
* the E2M1 value table (the eight magnitudes the 4-bit format defines) and a
  rounding written here as scaled round-half-even per binade, for NVFP4;
* ``torch.nn.functional.scaled_dot_product_attention`` in float64 on a
  contiguous ``[heads, seq, dim]`` layout built straight from the generator's
  values (so the paged write/read path is bypassed);
* a pure-Python brute force on tiny inputs;
* closed forms (single token, constant keys, zero query, two tokens, one
  dominant logit) and the worked block mapping of the TensorRT-LLM deep dive
  (gentlecold.top, §9: logical blocks 0/1/2 -> physical blocks 17/3/91).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle.pkv_oracle as O
from paged_kv_attention_block_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# Helpers (test side)
# ---------------------------------------------------------------------------

def oracle_pool_for(w: W.Workload, upto: str = "all"):
    """Oracle pool holding every token of ``w`` (``upto="all"``) or only history."""
    pool = O.new_pool(w.num_blocks, w.num_layers, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype,
                      w.k_scale, w.v_scale)
    k, v, cu, sp = w.packed_kv(upto)
    O.kv_append(pool, w.layer, k, v, w.kv_in_dtype, cu, sp, w.block_tables)
    return pool


def q64(w: W.Workload) -> np.ndarray:
    return O.decode_bits(w.q, w.q_dtype) if w.q_dtype != "f32" else w.q.astype(np.float64)


def run_oracle(w: W.Workload, pool=None):
    pool = pool if pool is not None else oracle_pool_for(w)
    return O.paged_attention(pool, w.layer, q64(w), w.cu_q_lens, w.seq_lens, w.block_tables, w.num_q_heads,
                             w.softmax_scale, w.causal, window=w.window)


def _values64(w: W.Workload, s: int):
    """Contiguous K/V [seq_len][Hkv][D] of sequence s as the cache holds them (library codecs)."""
    k, v = w.kv_values(s)
    if w.kv_dtype == "e4m3":
        out = []
        for which, x in ((0, k), (1, v)):
            sc = (w.k_scale if which == 0 else w.v_scale)[w.layer].astype(np.float32)
            y = torch.from_numpy(np.ascontiguousarray(x, np.float32) / sc[None, :, None])
            out.append(y.to(torch.float8_e4m3fn).to(torch.float64).numpy() * sc.astype(np.float64)[None, :, None])
        return out[0], out[1]
    if w.kv_dtype == "nvfp4":
        # Codes from the (separately pinned) quantiser, values through the E2M1 table and torch's
        # E4M3 conversion: the paged write and read paths are bypassed.
        out = []
        for which, x in ((0, k), (1, v)):
            g = (w.k_scale if which == 0 else w.v_scale)[w.layer].astype(np.float32)
            codes, sc = O.nvfp4_quantize(np.ascontiguousarray(x, np.float32), g[None, :])
            mag = np.array(E2M1_MAGNITUDES)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
            blk = torch.from_numpy(sc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
            out.append(mag * np.repeat(blk, 16, axis=-1) * g.astype(np.float64)[None, :, None])
        return out[0], out[1]
    if w.kv_dtype == "f32":
        return k.astype(np.float64), v.astype(np.float64)
    tdt = torch.bfloat16 if w.kv_dtype == "bf16" else torch.float16
    conv = lambda x: torch.from_numpy(x.view(np.int16)).view(tdt).to(torch.float64).numpy()  # noqa: E731
    return conv(k), conv(v)


def dense_sdpa(w: W.Workload):
    """softmax(scale q K^T) V per sequence with torch SDPA, contiguous layout, float64."""
    qq = q64(w)
    out = np.full(qq.shape, np.nan)
    g = w.num_q_heads // w.num_kv_heads
    cu = w.cu_q_lens
    for s in range(w.num_seqs):
        ql, L = int(w.q_lens[s]), int(w.seq_lens[s])
        if ql == 0:
            continue
        k, v = _values64(w, s)
        K = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2))).repeat_interleave(g, dim=0)
        V = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2))).repeat_interleave(g, dim=0)
        Q = torch.from_numpy(np.ascontiguousarray(qq[cu[s]:cu[s + 1]].transpose(1, 0, 2)))
        pos = L - ql + torch.arange(ql)
        mask = torch.arange(L)[None, :] <= pos[:, None] if w.causal else torch.ones(ql, L, dtype=torch.bool)
        if w.window:
            mask &= torch.arange(L)[None, :] > pos[:, None] - w.window
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=w.softmax_scale)
        out[cu[s]:cu[s + 1]] = o.numpy().transpose(1, 0, 2)
    return out


def small_workloads():
    """Small copies of each workload shape (several tiles, ragged tails)."""
    return [
        W.tiny_fp32(seq_lens=(17, 5, 33)),
        W.llama3_8b_decode_bf16(batch=3, lo=60, hi=200),
        W.mixed_bf16(n_decode=3, n_prefill=2, chunk=40, dec_lo=30, dec_hi=300, cached_lo_blocks=1,
                     cached_hi_blocks=3, block_size=16),
        W.longctx_fp8(batch=2, seq_len=150),
        W.prefix_reuse_bf16(n_req=3, prefix=256, suf_lo=3, suf_hi=40),
    ]


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def pin_e4m3_decode_table():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin]) and np.array_equal(np.signbit(got[fin]), np.signbit(ref[fin]))
    # Values the OCP E4M3 definition fixes.
    assert got[0x7E] == 448.0 and got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9 and got[0x07] == 7 * 2.0 ** -9
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and got[0x80] == 0.0 and np.signbit(got[0x80])


def pin_e4m3_encode():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    fin = ~np.isnan(vals)
    # encode(decode(c)) == c for every finite code (including -0).
    assert np.array_equal(O.e4m3_encode(vals[fin].astype(np.float32)), codes[fin])
    # Ties go to the even code at every midpoint between neighbouring magnitudes.
    pos = np.arange(0, 0x7E)
    lo, hi = O.e4m3_decode(pos), O.e4m3_decode(pos + 1)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (lo + hi) / 2)
    want = np.where(pos % 2 == 0, pos, pos + 1)
    assert np.array_equal(O.e4m3_encode(mid), want.astype(np.uint8))
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(0))
    assert np.array_equal(O.e4m3_encode(up), (pos + 1).astype(np.uint8))
    assert np.array_equal(O.e4m3_encode(dn), pos.astype(np.uint8))
    # Random values inside the range where torch's (non-saturating) RNE agrees.
    r = np.random.default_rng(7)
    x = np.concatenate([r.standard_normal(200000) * 40, r.standard_normal(20000) * 1e-2,
                        r.uniform(-463.9, 463.9, 20000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), ref)
    # Saturation to the largest finite value, NaN kept.
    big = np.array([448, 463.99, 464, 1e6, np.inf, -500, -np.inf, np.nan], np.float32)
    assert O.e4m3_encode(big).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F]


# The eight E2M1 magnitudes (codes 0..7); code | 8 is the negative.
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _e2m1_round_here(y):
    """Nearest E2M1 value with ties to even, written independently of the oracle: spacing 0.5
    below 2, 1 in [2, 4), 2 from 4; np.rint breaks ties to the even multiple; clamp at 6."""
    y = np.asarray(y, np.float64)
    a = np.abs(y)
    r = np.where(a < 2, np.rint(a * 2) / 2, np.where(a < 4, np.rint(a), 2 * np.rint(a / 2)))
    r = np.minimum(r, 6.0)
    return np.where(np.signbit(y), -r, r)


def pin_e2m1_table():
    got = O.e2m1_decode(np.arange(16))
    assert np.array_equal(got[:8], np.array(E2M1_MAGNITUDES))
    assert np.array_equal(got[8:], -np.array(E2M1_MAGNITUDES)) and np.signbit(got[8])


def pin_e2m1_encode():
    codes = np.arange(16)
    vals = np.array(E2M1_MAGNITUDES + tuple(-m for m in E2M1_MAGNITUDES), np.float32)
    vals[8] = -0.0
    assert np.array_equal(O.e2m1_encode(vals), codes.astype(np.uint8))
    # Midpoints: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4 (even codes).
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    assert O.e2m1_encode(mids).tolist() == [0, 2, 2, 4, 4, 6, 6]
    assert O.e2m1_encode(-mids).tolist() == [8, 10, 10, 12, 12, 14, 14]
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    assert O.e2m1_encode(up).tolist() == [1, 2, 3, 4, 5, 6, 7]
    assert O.e2m1_encode(dn).tolist() == [0, 1, 2, 3, 4, 5, 6]
    assert O.e2m1_encode(np.array([6.0, 6.5, 100.0, -1e30], np.float32)).tolist() == [7, 7, 7, 15]
    r = np.random.default_rng(5)
    y = np.concatenate([r.uniform(-7, 7, 100000), r.standard_normal(20000) * 0.3]).astype(np.float32)
    got = O.e2m1_decode(O.e2m1_encode(y))
    assert np.array_equal(got, _e2m1_round_here(y))


def pin_nvfp4_worked_group():
    """Groups worked by hand from the format: with g = 1 and max |x| = 6 the block scale is 1.0
    (E4M3 code 0x38) and each value on the E2M1 grid keeps its own code; 0.25 is a tie that goes
    to the even code 0.  Doubling g halves the block scale (0x30); an all-zero group stores
    zero codes and a zero scale.  The byte image puts dimension 2i in the low nibble."""
    x = np.array([-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6, 0.25], np.float32)
    want = [0xF, 0xE, 0xD, 0xC, 0xB, 0xA, 0x9, 0x0, 0x1, 0x2, 0x3, 0x4, 0x5, 0x6, 0x7, 0x0]
    codes, sc = O.nvfp4_quantize(x[None, :], np.float32(1.0))
    assert codes[0].tolist() == want and sc[0].tolist() == [0x38]
    codes, sc = O.nvfp4_quantize(x[None, :], np.float32(2.0))
    assert codes[0].tolist() == want and sc[0].tolist() == [0x30]
    codes, sc = O.nvfp4_quantize(np.zeros((1, 32), np.float32), np.float32(0.01))
    assert not codes.any() and not sc.any()
    # amax 3 with g = 1: scale 0.5 (0x30), so 3 -> 6 (code 7) and 0.2 / 0.5 = 0.4 -> 0.5 (code 1).
    y = np.zeros(16, np.float32)
    y[0], y[1], y[2] = 3.0, -0.2, 0.7
    codes, sc = O.nvfp4_quantize(y[None, :], np.float32(1.0))
    assert sc[0].tolist() == [0x30] and codes[0, :3].tolist() == [0x7, 0x9, 0x3]
    # Byte image of a 1-block, 1-head, 2-slot pool of head_dim 32 (64 bytes per run of K or V).
    pool = O.new_pool(1, 1, 1, 2, 32, "nvfp4", np.ones((1, 1), np.float32), np.ones((1, 1), np.float32))
    row = np.array([1, 2, 3, 4, 6, 0.5, 1.5, 0] * 4, np.float32).reshape(1, 1, 32)
    O.kv_append(pool, 0, row, row, "f32", np.array([0, 1]), np.array([1]), np.array([[0]]))
    img = O.nvfp4_pool_bytes(pool)
    assert img.shape == (1, 1, 2, 1, 2 * 16 + 2 * 2)
    # Slot 1 of K: codes 2, 4, 5, 6 | 7, 1, 3, 0 (scale 1.0: max 6) -> bytes 0x42, 0x65, 0x17, 0x03.
    assert img[0, 0, 0, 0, 16:20].tolist() == [0x42, 0x65, 0x17, 0x03]
    assert img[0, 0, 0, 0, 32 + 2:32 + 4].tolist() == [0x38, 0x38]
    assert img[0, 0, 0, 0, 0:16].tolist() == [0x7F] * 16  # slot 0 untouched


def pin_nvfp4_scale_invariance():
    """Scaling the values and the global scale by the same power of two changes no stored code
    (all quantities stay exact and inside the E4M3 normal range)."""
    r = np.random.default_rng(9)
    x = (r.standard_normal((50, 4, 128)) * 0.7).astype(np.float32)
    g = (np.abs(x).max(axis=(0, 2)) / (6 * 448)).astype(np.float32)[None, :]
    c0, s0 = O.nvfp4_quantize(x, g)
    for k in (-3, 2, 5):
        c1, s1 = O.nvfp4_quantize(x * np.float32(2.0 ** k), g * np.float32(2.0 ** k))
        assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


def pin_nvfp4_error_bound():
    """Dequantised values stay within half an E2M1 step (at most 1, at the top binade) of
    x / (s g), and the block scale is E4M3's rounding of max |x| / (6 g): relative error at
    most 2^-4 in the normal range."""
    r = np.random.default_rng(10)
    x = (r.standard_normal((200, 2, 128)) * r.uniform(0.01, 3, (200, 2, 1))).astype(np.float32)
    g = (np.abs(x).max(axis=(0, 2)) / (6 * 448)).astype(np.float32)[None, :]
    codes, sc = O.nvfp4_quantize(x, g)
    s = torch.from_numpy(sc).view(torch.float8_e4m3fn).to(torch.float64).numpy()  # [n][H][8]
    gg = g.astype(np.float64)[..., None]
    amax = np.abs(x.astype(np.float64)).reshape(200, 2, 8, 16).max(axis=-1)
    target = amax / (6 * gg)
    normal = target >= 2.0 ** -6
    assert (np.abs(s - target)[normal] <= target[normal] * 2.0 ** -4 * (1 + 1e-12)).all()
    mag = np.array(E2M1_MAGNITUDES)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    y = x.astype(np.float64) / (np.repeat(s, 16, axis=-1) * gg)
    step = np.where(np.abs(y) < 2, 0.25, np.where(np.abs(y) < 4, 0.5, 1.0))
    assert (np.abs(mag - np.clip(y, -6, 6)) <= step * (1 + 1e-6)).all()


def pin_bf16_decode():
    bits = np.arange(0, 65536, 7, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = O.decode_bits(bits, "bf16")
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


# ---------------------------------------------------------------------------
# Paged addressing
# ---------------------------------------------------------------------------

def pin_block_mapping_example():
    with open(os.path.join(GOLDEN, "block_mapping_example.json")) as f:
        g = json.load(f)
    table = np.array(g["block_table"], np.int32)
    for case in g["cases"]:
        B = case["block_size"]
        for p, (phys, slot) in zip(case["positions"], case["expect"]):
            got = O.block_address(table, p, B)
            assert (int(got[0]), int(got[1])) == (phys, slot), (p, got, phys, slot)
    # Append through that table writes exactly those slots and nothing else.
    B = g["cases"][0]["block_size"]
    n = 3 * B
    pool = O.new_pool(100, 1, 1, B, 4, "f32")
    vals = np.arange(n * 4, dtype=np.float32).reshape(n, 1, 4)
    O.kv_append(pool, 0, vals, -vals, "f32", np.array([0, n]), np.array([0]), table[None, :])
    for t in range(n):
        phys = g["block_table"][t // B]
        assert np.array_equal(pool.bits[phys, 0, 0, 0, t % B], vals[t, 0])
        assert np.array_equal(pool.bits[phys, 0, 1, 0, t % B], -vals[t, 0])
    touched = np.zeros(100, bool)
    touched[g["block_table"]] = True
    assert np.isnan(pool.bits[~touched]).all()


def pin_partial_reuse_example():
    """The deep dive's partial-reuse example: block [A, B, C, D], a new request [A, B, X, Y] matching two
    tokens; the matched tokens are copied into a new block, the request appends X and Y after them, and the
    existing block is left as it was (tests/golden/partial_reuse_example.json)."""
    with open(os.path.join(GOLDEN, "partial_reuse_example.json")) as f:
        g = json.load(f)
    B, n = g["block_size"], g["matched_tokens"]
    labels = sorted(set(g["existing_block"]) | set(g["new_request"]))
    row = {lab: np.full((1, 8), 10.0 * (i + 1), np.float32) + np.arange(8, dtype=np.float32) for i, lab in enumerate(labels)}
    kv = lambda toks, sign: np.stack([sign * row[t] for t in toks])  # noqa: E731  [T][Hkv=1][D=8]
    pool = O.new_pool(6, 1, 1, B, 8, "f32")
    old, new = 1, 4  # physical blocks
    O.kv_append(pool, 0, kv(g["existing_block"], 1), kv(g["existing_block"], -1), "f32", np.array([0, B]),
                np.array([0]), np.array([[old]]))
    O.copy_block_prefix(pool, [old], [new], [n])
    tail = g["new_request"][n:]
    O.kv_append(pool, 0, kv(tail, 1), kv(tail, -1), "f32", np.array([0, len(tail)]), np.array([n]),
                np.array([[new]]))
    for blk, want in ((old, g["expect_existing"]), (new, g["expect_new"])):
        for which, sign in ((0, 1), (1, -1)):
            got = O.gather_rows(pool, 0, np.array([blk]), 0, which, B)
            assert np.array_equal(got, kv(want, sign)[:, 0, :].astype(np.float64)), (blk, which)
    others = [b for b in range(6) if b not in (old, new)]
    assert np.isnan(pool.bits[others]).all()


def pin_append_roundtrip():
    for w in small_workloads():
        pool = oracle_pool_for(w)
        used = np.zeros(w.num_blocks, bool)
        for s in range(w.num_seqs):
            k64, v64 = _values64(w, s)
            L = int(w.seq_lens[s])
            for h in range(w.num_kv_heads):
                got_k = O.gather_rows(pool, w.layer, w.block_tables[s], h, 0, L)
                got_v = O.gather_rows(pool, w.layer, w.block_tables[s], h, 1, L)
                assert np.array_equal(got_k, k64[:, h, :]) and np.array_equal(got_v, v64[:, h, :]), (w.name, s, h)
            used[w.block_tables[s][: (L + w.block_size - 1) // w.block_size]] = True
        sent = O.sentinel_bits(w.kv_dtype)
        untouched = pool.bits[~used]
        if w.kv_dtype == "f32":
            assert np.isnan(untouched).all()
        else:
            assert (untouched == sent).all()


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def pin_dense_equivalence():
    for w in small_workloads():
        out, _ = run_oracle(w)
        ref = dense_sdpa(w)
        err = np.abs(out - ref).max()
        assert err <= 1e-12, (w.name, err)


def pin_nvfp4_dense():
    """An NVFP4 cache: the paged oracle against SDPA over values dequantised here (E2M1 table,
    torch's E4M3 conversion), prefill chunk and decode rows, several blocks and a ragged tail."""
    w = W.build("nv", seed=21, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=8,
                num_kv_heads=2, head_dim=128, block_size=16, seq_lens=[70, 33, 5], q_lens=[20, 1, 1])
    out, _ = run_oracle(w)
    assert np.abs(out - dense_sdpa(w)).max() <= 1e-12


def pin_noncausal_dense():
    w = W.mixed_bf16(n_decode=2, n_prefill=2, chunk=24, dec_lo=20, dec_hi=70, cached_lo_blocks=1,
                     cached_hi_blocks=2, block_size=16)
    w.causal = False
    out, _ = run_oracle(w)
    assert np.abs(out - dense_sdpa(w)).max() <= 1e-12


def pin_brute_force():
    """Pure-Python loops on a tiny mixed batch (one prefill chunk, one decode)."""
    w = W.build("brute", seed=5, kv_dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=3, block_size=2,
                seq_lens=[5, 4], q_lens=[3, 1], num_blocks=9)
    out, lse = run_oracle(w)
    qq = q64(w)
    cu = w.cu_q_lens
    for s in range(2):
        k, v = w.kv_values(s)
        L, ql = int(w.seq_lens[s]), int(w.q_lens[s])
        for j in range(ql):
            p = L - ql + j
            for h in range(4):
                kvh = h // 2
                z = [w.softmax_scale * sum(float(qq[cu[s] + j, h, d]) * float(k[t, kvh, d]) for d in range(3))
                     for t in range(p + 1)]
                m = max(z)
                e = [math.exp(x - m) for x in z]
                den = sum(e)
                for d in range(3):
                    ref = sum(e[t] * float(v[t, kvh, d]) for t in range(p + 1)) / den
                    assert abs(out[cu[s] + j, h, d] - ref) <= 1e-13, (s, j, h, d)
                assert abs(lse[cu[s] + j, h] - (m + math.log(den))) <= 1e-13


def pin_lse_logsumexp():
    from scipy.special import logsumexp

    w = W.llama3_8b_decode_bf16(batch=2, lo=30, hi=90)
    pool = oracle_pool_for(w)
    _, lse = run_oracle(w, pool)
    qq = q64(w)
    for s in range(2):
        for h in (0, 5, 31):
            k, _ = _values64(w, s)
            z = w.softmax_scale * (k[:, h // 4, :] @ qq[s, h])
            assert abs(lse[s, h] - logsumexp(z)) <= 1e-12


def pin_permutation_invariance():
    base = W.llama3_8b_decode_bf16(batch=3, lo=40, hi=300)
    w2 = W.llama3_8b_decode_bf16(batch=3, lo=40, hi=300)
    # Same values, another physical placement: reshuffle the block ids.
    perm = np.random.default_rng(99).permutation(base.num_blocks).astype(np.int32)
    w2.block_tables = np.where(base.block_tables >= 0, perm[np.maximum(base.block_tables, 0)], -1)
    o1, l1 = run_oracle(base)
    o2, l2 = run_oracle(w2)
    assert not np.array_equal(base.block_tables, w2.block_tables)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_softmax_rows():
    w = W.mixed_bf16(n_decode=2, n_prefill=1, chunk=20, dec_lo=20, dec_hi=90, cached_lo_blocks=1,
                     cached_hi_blocks=2, block_size=16)
    pool = oracle_pool_for(w)
    qq = q64(w)
    for s in range(w.num_seqs):
        for j in range(int(w.q_lens[s])):
            for h in (0, 9, 31):
                p = O.attention_row_probs(pool, 0, qq, w.cu_q_lens, w.seq_lens, w.block_tables, w.num_q_heads,
                                          w.softmax_scale, True, s, j, h)
                assert abs(p.sum() - 1.0) <= 1e-12 and (p >= 0).all()
                lim = int(w.seq_lens[s]) - int(w.q_lens[s]) + j + 1
                assert (p[lim:] == 0).all() and (p[:lim] > 0).all()


def _one_seq(kvals, vvals, qvals, B=4, causal=True, q_len=1):
    """Oracle on hand-made values: one sequence, Hq=2, Hkv=1, f32."""
    L, D = kvals.shape
    nb = (L + B - 1) // B
    pool = O.new_pool(nb + 3, 1, 1, B, D, "f32")
    table = (np.arange(nb)[::-1] + 2).astype(np.int32)[None, :]  # reversed, offset placement
    O.kv_append(pool, 0, kvals[:, None, :].astype(np.float32), vvals[:, None, :].astype(np.float32), "f32",
                np.array([0, L]), np.array([0]), table)
    return O.paged_attention(pool, 0, qvals.astype(np.float64), np.array([0, q_len]), np.array([L]), table, 2,
                             0.125, causal)


def pin_closed_forms():
    r = np.random.default_rng(3)
    D = 8
    # seq_len = 1 -> v0 exactly
    k = r.standard_normal((1, D)).astype(np.float32)
    v = r.standard_normal((1, D)).astype(np.float32)
    o, lse = _one_seq(k, v, r.standard_normal((1, 2, D)))
    assert np.array_equal(o[0, 0], v[0].astype(np.float64)) and np.array_equal(o[0, 1], v[0].astype(np.float64))
    # q = 0 -> exact mean of V; lse = ln L
    L = 13
    k = r.standard_normal((L, D)).astype(np.float32)
    v = r.standard_normal((L, D)).astype(np.float32)
    o, lse = _one_seq(k, v, np.zeros((1, 2, D)))
    assert np.abs(o[0, 0] - v.astype(np.float64).mean(0)).max() <= 1e-15
    assert abs(lse[0, 0] - math.log(L)) <= 1e-15
    # all keys equal -> mean of V
    k = np.tile(r.standard_normal((1, D)).astype(np.float32), (L, 1))
    o, _ = _one_seq(k, v, r.standard_normal((1, 2, D)))
    assert np.abs(o[0, 1] - v.astype(np.float64).mean(0)).max() <= 1e-15
    # two tokens -> (v0 e^z0 + v1 e^z1) / (e^z0 + e^z1)
    k = r.standard_normal((2, D)).astype(np.float32)
    v = r.standard_normal((2, D)).astype(np.float32)
    q = r.standard_normal((1, 2, D))
    o, _ = _one_seq(k, v, q)
    z = 0.125 * (k.astype(np.float64) @ q[0, 0])
    v64 = v.astype(np.float64)
    ref = (v64[0] * math.exp(z[0]) + v64[1] * math.exp(z[1])) / (math.exp(z[0]) + math.exp(z[1]))
    assert np.abs(o[0, 0] - ref).max() <= 1e-14
    # one dominant logit -> v_t
    L = 9
    k = r.standard_normal((L, D)).astype(np.float32)
    v = r.standard_normal((L, D)).astype(np.float32)
    q = np.zeros((1, 2, D))
    q[0, :] = 50.0 * 8 * k[4]
    o, _ = _one_seq(k, v, q)
    assert np.abs(o[0, 0] - v[4]).max() <= 1e-12
    # first row of a chunk with nothing cached sees only its own key -> v0
    L = 6
    k = r.standard_normal((L, D)).astype(np.float32)
    v = r.standard_normal((L, D)).astype(np.float32)
    o, _ = _one_seq(k, v, r.standard_normal((L, 2, D)), q_len=L)
    assert np.array_equal(o[0, 0], v[0].astype(np.float64))
    # the last row of that chunk sees every key: it equals the non-causal answer,
    # while the non-causal first row differs from v0
    q = r.standard_normal((L, 2, D))
    oc, _ = _one_seq(k, v, q, q_len=L)
    on, _ = _one_seq(k, v, q, q_len=L, causal=False)
    assert np.array_equal(oc[L - 1], on[L - 1]) and not np.allclose(on[0, 0], v[0])


def pin_split_reduce():
    """Partials over arbitrary (some empty) key ranges merge back to the unsplit result."""
    w = W.llama3_8b_decode_bf16(batch=2, lo=100, hi=300)
    pool = oracle_pool_for(w)
    out, lse = run_oracle(w, pool)
    qq = q64(w)
    r = np.random.default_rng(11)
    for s in range(2):
        L = int(w.seq_lens[s])
        cuts = np.sort(np.concatenate([[0, L, L, 0], r.integers(0, L, 5)]))
        for h in (0, 7, 30):
            k, v = _values64(w, s)
            K, V = k[:, h // 4], v[:, h // 4]
            po, pl = [], []
            for a, b in zip(cuts[:-1], cuts[1:]):
                if b <= a:
                    po.append(np.full((1, w.head_dim), 7.0))  # content of an empty part is ignored
                    pl.append(np.array([-np.inf]))
                    continue
                z = w.softmax_scale * (K[a:b] @ qq[s, h])
                m = z.max()
                e = np.exp(z - m)
                po.append(((e @ V[a:b]) / e.sum())[None, :])
                pl.append(np.array([m + math.log(e.sum())]))
            o, l = O.split_kv_reduce(np.stack(po), np.stack(pl))
            assert np.abs(o[0] - out[s, h]).max() <= 1e-13 and abs(l[0] - lse[s, h]) <= 1e-13
    o, l = O.split_kv_reduce(np.zeros((2, 1, 4)), np.full((2, 1), -np.inf))
    assert (o == 0).all() and l[0] == -np.inf


def pin_prefix_sharing():
    """Shared prefix blocks give the same result as private copies of them."""
    w = W.prefix_reuse_bf16(n_req=4, prefix=256, suf_lo=5, suf_hi=60)
    shared, _ = run_oracle(w)
    B = w.block_size
    P = w.shared_prefix_tokens // B
    assert (w.block_tables[:, :P] == w.block_tables[0, :P]).all()
    w2 = W.prefix_reuse_bf16(n_req=4, prefix=256, suf_lo=5, suf_hi=60)
    extra = w2.num_blocks
    w2.num_blocks = extra + P * w2.num_seqs
    for s in range(w2.num_seqs):
        w2.block_tables[s, :P] = extra + s * P + np.arange(P)
    private, _ = run_oracle(w2)
    assert np.array_equal(shared, private)


# ---------------------------------------------------------------------------
# Limited attention window (deep dive §11)
# ---------------------------------------------------------------------------

def pin_window_dense():
    """Banded causal mask on the contiguous layout (torch SDPA) for several windows."""
    for W_ in (1, 3, 17, 70):
        for w in (W.mixed_bf16(n_decode=3, n_prefill=2, chunk=40, dec_lo=30, dec_hi=300, cached_lo_blocks=1,
                               cached_hi_blocks=3, block_size=16),
                  W.longctx_fp8(batch=2, seq_len=150)):
            w.window = W_
            out, _ = run_oracle(w)
            assert np.abs(out - dense_sdpa(w)).max() <= 1e-12, (w.name, W_)


def pin_window_limits():
    """A window of one position leaves only the row's own token (o = v_p exactly); a window at
    least as long as the sequence changes nothing, bit for bit."""
    w = W.mixed_bf16(n_decode=3, n_prefill=2, chunk=24, dec_lo=20, dec_hi=90, cached_lo_blocks=1,
                     cached_hi_blocks=2, block_size=16)
    pool = oracle_pool_for(w)
    full, full_lse = run_oracle(w, pool)
    w.window = int(w.seq_lens.max())
    same, same_lse = run_oracle(w, pool)
    assert np.array_equal(full, same) and np.array_equal(full_lse, same_lse)
    w.window = 1
    one, _ = run_oracle(w, pool)
    g = w.num_q_heads // w.num_kv_heads
    for s in range(w.num_seqs):
        k, v = _values64(w, s)
        L, ql = int(w.seq_lens[s]), int(w.q_lens[s])
        for j in range(ql):
            tok = int(w.cu_q_lens[s]) + j
            for h in range(w.num_q_heads):
                assert np.array_equal(one[tok, h], v[L - ql + j, h // g]), (s, j, h)


def pin_window_brute_force():
    """Pure-Python loops with a window of 3 on a tiny mixed batch."""
    w = W.build("brute_w", seed=6, kv_dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=3, block_size=2,
                seq_lens=[7, 5], q_lens=[4, 1], num_blocks=12, window=3)
    out, lse = run_oracle(w)
    qq = q64(w)
    cu = w.cu_q_lens
    for s in range(2):
        k, v = w.kv_values(s)
        L, ql = int(w.seq_lens[s]), int(w.q_lens[s])
        for j in range(ql):
            p = L - ql + j
            keys = range(max(0, p - 2), p + 1)
            for h in range(4):
                kvh = h // 2
                z = {t: w.softmax_scale * sum(float(qq[cu[s] + j, h, d]) * float(k[t, kvh, d]) for d in range(3))
                     for t in keys}
                m = max(z.values())
                e = {t: math.exp(x - m) for t, x in z.items()}
                den = sum(e.values())
                for d in range(3):
                    ref = sum(e[t] * float(v[t, kvh, d]) for t in keys) / den
                    assert abs(out[cu[s] + j, h, d] - ref) <= 1e-13, (s, j, h, d)
                assert abs(lse[cu[s] + j, h] - (m + math.log(den))) <= 1e-13


# ---------------------------------------------------------------------------
# Partial reuse: block prefix copy (deep dive §11)
# ---------------------------------------------------------------------------

def pin_block_copy():
    """Copy a sequence's blocks, whole and in part, into free blocks: a table pointing at the
    copies gathers the same rows bit for bit up to the copied length; the rest of a partially
    copied block keeps its sentinels; attention of a request that reuses the copied prefix equals
    attention over the original tokens."""
    w = W.build("copy", seed=19, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=16, block_size=8,
                seq_lens=[61, 20, 35], q_lens=[1, 1, 1], pool_factor=3.0)
    pool = oracle_pool_for(w)
    B = w.block_size
    used = set(int(b) for b in w.block_tables.ravel() if b >= 0)
    free = [b for b in range(w.num_blocks) if b not in used]
    s, L = 0, int(w.seq_lens[0])
    nblk = (L + B - 1) // B
    n_last = L - (nblk - 1) * B
    src = w.block_tables[s, :nblk].copy()
    dst = np.array(free[:nblk], np.int32)
    ns = np.array([B] * (nblk - 1) + [max(1, n_last // 2)], np.int32)
    before = pool.bits.copy()
    O.copy_block_prefix(pool, src, dst, ns)
    table = w.block_tables[s].copy()
    table[:nblk] = dst
    n_copied = (nblk - 1) * B + int(ns[-1])
    for kvh in range(w.num_kv_heads):
        for which in (0, 1):
            a = O.gather_rows(pool, w.layer, w.block_tables[s], kvh, which, n_copied)
            b = O.gather_rows(pool, w.layer, table, kvh, which, n_copied)
            assert np.array_equal(a, b)
    # Untouched: slots past the copied prefix of the last block, and every other block.
    last = int(dst[-1])
    assert np.array_equal(pool.bits[last, :, :, :, int(ns[-1]):], before[last, :, :, :, int(ns[-1]):])
    others = np.ones(w.num_blocks, bool)
    others[dst] = False
    assert np.array_equal(pool.bits[others], before[others])
    # A request reusing the copied prefix (its own table) attends like the original over those tokens.
    q = q64(w)[:1]
    o1, l1 = O.paged_attention(pool, w.layer, q, np.array([0, 1]), np.array([n_copied]),
                               w.block_tables[s:s + 1], w.num_q_heads, w.softmax_scale, True)
    o2, l2 = O.paged_attention(pool, w.layer, q, np.array([0, 1]), np.array([n_copied]), table[None, :],
                               w.num_q_heads, w.softmax_scale, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


ALL_PINS = [
    pin_e4m3_decode_table, pin_e4m3_encode, pin_bf16_decode, pin_block_mapping_example, pin_partial_reuse_example,
    pin_append_roundtrip,
    pin_dense_equivalence, pin_noncausal_dense, pin_brute_force, pin_lse_logsumexp, pin_permutation_invariance,
    pin_softmax_rows, pin_closed_forms, pin_split_reduce, pin_prefix_sharing, pin_window_dense, pin_window_limits,
    pin_window_brute_force, pin_block_copy, pin_e2m1_table, pin_e2m1_encode, pin_nvfp4_worked_group,
    pin_nvfp4_scale_invariance, pin_nvfp4_error_bound, pin_nvfp4_dense,
]
