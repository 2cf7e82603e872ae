"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

A pin suite that still passes with a mistake planted would not be pinning
that part of the oracle.  Every mutation below must make at least one pin in
``oracle_pins.ALL_PINS`` fail.
"""
import numpy as np
import pytest

import oracle.pkv_oracle as O
import oracle_pins as P

_orig_block_address = O.block_address
_orig_softmax_rows = O._softmax_rows
_orig_gather = O.gather_rows
_orig_decode = O.decode_bits
_orig_split = O.split_kv_reduce
_orig_start = O.key_start
_orig_copy = O.copy_block_prefix
_orig_e2m1_encode = O.e2m1_encode
_orig_e2m1_decode = O.e2m1_decode
_orig_pool_bytes = O.nvfp4_pool_bytes
_orig_quantize = O.nvfp4_quantize


def _gqa_modulo(h, hq, hkv):
    return h % hkv


def _slot_reversed(row, pos, B):
    phys, slot = _orig_block_address(row, pos, B)
    return phys, B - 1 - slot


def _block_shifted(row, pos, B):
    pos = np.asarray(pos)
    return row[np.minimum(pos // B + (pos % B == B - 1), len(row) - 1)], pos % B


def _causal_excludes_self(L, ql, j, causal):
    j = np.asarray(j)
    return np.full(j.shape, L) if not causal else L - ql + j


def _causal_ignored(L, ql, j, causal):
    return np.full(np.asarray(j).shape, L)


def _truncating_round(x):
    return np.floor(x)


def _half_up_round(x):
    return np.floor(x + 0.5)


def _scale_twice(z):
    return _orig_softmax_rows(2.0 * z)


def _lse_without_max(z):
    w, m, l = _orig_softmax_rows(z)
    return w, 0.0 * m, l


def _kv_swapped(pool, layer, row, kvh, which, n):
    return _orig_gather(pool, layer, row, kvh, 1 - which, n)


def _e4m3_bias8(codes):
    c = np.asarray(codes, dtype=np.int64)
    v = _orig_decode(codes, "e4m3")
    return np.where((c & 0x78) != 0, v / 2.0, v)


def _decode_e4m3_bias8(bits, dtype):
    return _e4m3_bias8(bits) if dtype == "e4m3" else _orig_decode(bits, dtype)


def _bf16_wrong_shift(bits, dtype):
    if dtype == "bf16":
        u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(15)
        return u.view(np.float32).astype(np.float64)
    return _orig_decode(bits, dtype)


def _window_one_too_wide(L, ql, j, window):
    return np.maximum(0, _orig_start(L, ql, j, window) - (1 if window > 0 else 0))


def _copy_whole_block(pool, src, dst, n):
    return _orig_copy(pool, src, dst, [pool.block_size] * len(list(n)))


def _copy_off_by_one(pool, src, dst, n):
    return _orig_copy(pool, src, dst, [max(0, int(x) - 1) for x in n])


def _e2m1_ties_up(y32):
    """Ties of the E2M1 rounding go to the larger magnitude instead of the even code."""
    y = np.asarray(y32, np.float32)
    a = np.abs(y)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    bump = np.isin(a, mids)
    return _orig_e2m1_encode(np.where(bump, np.nextafter(a, np.float32(np.inf)) * np.sign(y), y).astype(np.float32))


def _e2m1_exponent_bias_0(codes):
    c = np.asarray(codes, dtype=np.int64)
    v = _orig_e2m1_decode(codes)
    return np.where(((c >> 1) & 3) != 0, 2.0 * v, v)


def _nibbles_swapped(pool):
    img = _orig_pool_bytes(pool).copy()
    n = pool.bits.shape[4] * pool.bits.shape[5] // 2
    img[..., :n] = ((img[..., :n] >> 4) | (img[..., :n] << 4)) & 0xFF
    return img


def _quantize_scale_over_4(x32, g):
    """Block scale max / (4 g) instead of max / (6 g); element codes against that scale."""
    x = np.asarray(x32, np.float32)
    D = x.shape[-1]
    grp = x.reshape(x.shape[:-1] + (D // 16, 16))
    gg = np.asarray(g, np.float32)[..., None]
    sc = O.e4m3_encode((np.abs(grp).max(axis=-1) / (np.float32(4.0) * gg)).astype(np.float32))
    s = O.e4m3_decode(sc).astype(np.float32)
    denom = np.where(s == 0, 1, s * gg).astype(np.float32)
    codes = O.e2m1_encode((grp / denom[..., None]).astype(np.float32))
    return np.where((s == 0)[..., None], 0, codes).reshape(x.shape).astype(np.uint8), sc


def _quantize_without_global(x32, g):
    """Element codes from x / s, dropping the global scale."""
    codes, sc = _orig_quantize(x32, g)
    x = np.asarray(x32, np.float32)
    D = x.shape[-1]
    s = O.e4m3_decode(sc).astype(np.float32)
    y = x.reshape(x.shape[:-1] + (D // 16, 16)) / np.where(s == 0, 1, s)[..., None]
    return O.e2m1_encode(y.astype(np.float32)).reshape(x.shape), sc


def _gather_without_block_scale(pool, layer, row, kvh, which, n):
    if pool.dtype != "nvfp4":
        return _orig_gather(pool, layer, row, kvh, which, n)
    t = np.arange(n)
    phys, slot = O.block_address(row, t, pool.block_size)
    return O.e2m1_decode(pool.bits[phys, layer, which, kvh, slot, :]) * np.float64(pool.scale(which, layer)[kvh])


def _split_sign(po, pl):
    return _orig_split(po, -np.asarray(pl))


MUTATIONS = {
    "gqa_modulo_mapping": [("kv_head_of", _gqa_modulo)],
    "slot_reversed": [("block_address", _slot_reversed)],
    "block_index_off_by_one": [("block_address", _block_shifted)],
    "causal_excludes_own_token": [("key_limit", _causal_excludes_self)],
    "causal_mask_ignored": [("key_limit", _causal_ignored)],
    "e4m3_truncates": [("rne", _truncating_round)],
    "e4m3_ties_away": [("rne", _half_up_round)],
    "softmax_scale_doubled": [("_softmax_rows", _scale_twice)],
    "lse_drops_max": [("_softmax_rows", _lse_without_max)],
    "k_v_swapped": [("gather_rows", _kv_swapped)],
    "e4m3_bias_8": [("e4m3_decode", _e4m3_bias8), ("decode_bits", _decode_e4m3_bias8)],
    "bf16_decode_shift": [("decode_bits", _bf16_wrong_shift)],
    "split_merge_sign": [("split_kv_reduce", _split_sign)],
    "window_one_too_wide": [("key_start", _window_one_too_wide)],
    "copy_whole_block": [("copy_block_prefix", _copy_whole_block)],
    "copy_one_token_short": [("copy_block_prefix", _copy_off_by_one)],
    "e2m1_ties_up": [("e2m1_encode", _e2m1_ties_up)],
    "e2m1_exponent_bias_0": [("e2m1_decode", _e2m1_exponent_bias_0)],
    "nvfp4_nibbles_swapped": [("nvfp4_pool_bytes", _nibbles_swapped)],
    "nvfp4_block_scale_over_4": [("nvfp4_quantize", _quantize_scale_over_4)],
    "nvfp4_codes_without_global_scale": [("nvfp4_quantize", _quantize_without_global)],
    "nvfp4_gather_drops_block_scale": [("gather_rows", _gather_without_block_scale)],
    "nvfp4_group_32": [("NVFP4_GROUP", 32)],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    for attr, fn in MUTATIONS[name]:
        monkeypatch.setattr(O, attr, fn)
    caught = []
    for pin in P.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except Exception as e:  # noqa: BLE001 - any failure of a pin counts
            caught.append((pin.__name__, type(e).__name__))
            break
    assert caught, f"no pin catches the planted mistake {name}"
