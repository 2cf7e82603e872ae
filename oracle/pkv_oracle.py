"""CPU oracle for paged KV-cache attention, in float64.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this module.  The CUDA
path never calls it and shares no code with it.

What it computes, step by step, with the passage each step follows:

* Paged storage (TensorRT-LLM deep dive, gentlecold.top, §9 "KV cache系统":
  the block pool, the per-request block table mapping logical block 0/1/2 to
  physical blocks 17/3/91, and the contiguous ``[batch, 2, heads, max_seq_len,
  head_dim]`` layout paging replaces).  Token ``p`` of a request lives in
  physical block ``table[p // B]`` at slot ``p % B``; one pool block holds, per
  layer, K then V, per KV head, ``B`` token rows of ``head_dim`` values.
* ``kv_append`` (TensorRT-LLM concept explainer, compassingai.com, "技术原理":
  page-table lookup nodes for KV reads and writes; deep dive §2: decode writes
  the new token's KV; §8: each prefill chunk appends its KV before the next
  chunk): copy each new token's K and V rows into its slot.  With an fp8-e4m3
  cache (deep dive §13, ``KvCacheConfig(dtype="fp8")``) the stored byte is the
  E4M3 encoding, round-to-nearest-even with saturation to +-448, of
  ``x / scale`` computed in float32, with one scale per (layer, KV head) for K
  and one for V.  With an NVFP4 cache (deep dive §13, ``NVFP4 KV cache`` and
  ``KvCacheConfig(dtype="nvfp4")``; the pages name the format but print none
  of it, so the reading is the published NVFP4 definition: 4-bit E2M1 values in
  groups of 16 sharing an E4M3 scale, under a float32 scale per tensor, here
  per (layer, KV head, K|V)), each 16-value group ``x`` of a row with global
  scale ``g`` stores the block scale code ``c = E4M3(max|x| / (6 g))`` and the
  element codes ``E2M1(x_i / (value(c) g))`` (nearest even, saturating at 6;
  all zero when the block scale is 0), every quotient and product in float32.
* ``paged_attention`` (deep dive §2: decode reads the whole KV history of the
  request to do attention; §6: context and generation requests in one packed
  batch; §8: a chunk attends to the cached KV plus itself): for sequence ``s``,
  query row ``j`` at absolute position ``p = seq_len - q_len + j`` and query
  head ``h`` with KV head ``h // (Hq / Hkv)``, scores ``z_t = scale * q . k_t``
  for keys ``t <= p`` (all ``t < seq_len`` when not causal), then the plain
  softmax ``w = exp(z - max z) / sum`` and ``o = sum_t w_t v_t``; also
  ``lse = max z + ln sum exp(z - max z)``.  No tiling, no online softmax.
  ``copy_block_prefix`` (deep dive §11, partial reuse with
  ``copy_on_partial_reuse``): the first ``n`` slots of a block, every layer, K
  and V and KV head, copied into the same slots of another block.
  With a limited attention window ``W`` (deep dive §11, "有限attention window":
  tokens outside the window no longer take part in attention), row ``j`` sees
  only the ``W`` most recent positions up to its own: keys ``p - W < t <= p``.
* ``split_kv_reduce``: partial states over disjoint key sets ``(o_i, lse_i)``
  (``o_i`` normalised, natural-log ``lse_i``; an empty set has ``lse = -inf``)
  merge as ``M = max lse_i``, ``w_i = exp(lse_i - M)``, ``o = sum w_i o_i / sum
  w_i``, ``lse = M + ln sum w_i``.  This is the exact identity behind splitting
  a softmax over key ranges; the pages do not print it (they never describe
  split-KV), so it is pinned against the unsplit computation.

Every floating-point step is float64 except the ones the fp8 and NVFP4
encodings decide: their quotients and products are taken in float32 because the
stored bytes depend on them.

Helper functions (``kv_head_of``, ``block_address``, ``key_limit``,
``rne``) are module-level so that tests can plant a mistake in one of them and
check that a pin catches it.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "E4M3_MAX", "e4m3_decode", "e4m3_encode", "e2m1_decode", "e2m1_encode", "nvfp4_quantize", "nvfp4_pool_bytes",
    "NVFP4_GROUP", "decode_bits", "kv_head_of", "block_address",
    "key_limit", "key_start", "copy_block_prefix", "OraclePool", "new_pool", "kv_append", "gather_rows", "paged_attention",
    "attention_row_probs", "split_kv_reduce", "sentinel_bits",
]

E4M3_MAX = 448.0
NVFP4_GROUP = 16  # values sharing one E4M3 block scale


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def rne(x: np.ndarray) -> np.ndarray:
    """Round half to even (IEEE roundTiesToEven) on exactly representable float64 inputs."""
    return np.rint(x)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """OCP 8-bit floating point, E4M3 variant: 1 sign, 4 exponent (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal ``m * 2^-9``; otherwise ``(1 + m/8) * 2^(e-7)``.
    There is no infinity; ``S.1111.111`` is NaN, so the largest finite value is
    ``1.75 * 2^8 = 448``.
    """
    c = np.asarray(codes, dtype=np.int64)
    sign = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (c & 7 == 7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


def e4m3_encode(x32: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 code, round to nearest even, saturating finite overflow to +-448.

    NaN maps to 0x7F.  The sign of zero is kept.
    """
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    out = np.zeros(a.shape, dtype=np.int64)
    finite = np.isfinite(a)
    sat = (~finite) | (a >= E4M3_MAX)
    # Subnormal binade and zero: multiples of 2^-9 below 2^-6 (a code of 8 is 2^-6 itself).
    sub = finite & (a < 2.0 ** -6)
    out = np.where(sub, rne(np.where(sub, a, 0.0) * 2.0 ** 9).astype(np.int64), out)
    # Normal binades: a = f * 2^E with f in [0.5, 1); exponent e = E - 1, mantissa (2f - 1) * 8.
    nrm = finite & ~sub & ~sat
    f, E = np.frexp(np.where(nrm, a, 1.0))
    e = E.astype(np.int64) - 1
    m = rne((2.0 * f - 1.0) * 8.0).astype(np.int64)
    carry = m == 8
    e = np.where(carry, e + 1, e)
    m = np.where(carry, 0, m)
    code_n = ((e + 7) << 3) | m
    out = np.where(nrm, np.minimum(code_n, 0x7E), out)
    out = np.where(sat, 0x7E, out)
    out = np.where(neg, out | 0x80, out)
    out = np.where(np.isnan(x), 0x7F, out)
    return out.astype(np.uint8)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no infinity or NaN.

    Exponent field 0 is subnormal ``m * 0.5``; otherwise ``(1 + m/2) * 2^(e-1)``, so the
    magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.
    """
    c = np.asarray(codes, dtype=np.int64)
    sign = (c >> 3) & 1
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e.astype(np.float64) - 1.0))
    return np.where(sign == 1, -mag, mag)


def e2m1_encode(y32: np.ndarray) -> np.ndarray:
    """float32 (finite) -> E2M1 code: the nearest of the eight magnitudes, a tie going to the
    code with mantissa bit 0 (round half to even), beyond 6 saturating to 6; the sign bit is
    the sign of the input (so -0.1 gives the code of -0)."""
    y = np.asarray(y32, dtype=np.float32).astype(np.float64)
    mags = e2m1_decode(np.arange(8))
    a = np.minimum(np.abs(y), mags[-1])  # saturation first: huge inputs are 6, not a far tie
    dist = np.abs(a[..., None] - mags)  # [..., 8]
    best = dist.min(axis=-1, keepdims=True)
    tied = dist == best
    # Among the nearest codes take the even one (mantissa bit 0); at most two are nearest.
    even = tied & ((np.arange(8) & 1) == 0)
    pick = np.where(even.any(axis=-1), even.argmax(axis=-1), tied.argmax(axis=-1))
    return (pick | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def nvfp4_quantize(x32: np.ndarray, g) -> tuple[np.ndarray, np.ndarray]:
    """Rows ``x32`` [..., D] (float32) with global scale ``g`` (float32, broadcast over [...]) ->
    (E2M1 codes uint8 [..., D], E4M3 block scale codes uint8 [..., D / 16]).

    Per 16-value group: ``a = max |x|``, ``c = E4M3(a / (6 g))``, ``s = value(c)``; codes
    ``E2M1(x / (s g))``, all zero when ``s`` is 0.  Products and quotients in float32."""
    x = np.asarray(x32, dtype=np.float32)
    D = x.shape[-1]
    grp = x.reshape(x.shape[:-1] + (D // NVFP4_GROUP, NVFP4_GROUP))
    gg = np.asarray(g, dtype=np.float32)[..., None]  # broadcast over the group axis
    amax = np.abs(grp).max(axis=-1)
    six_g = (np.float32(6.0) * gg).astype(np.float32)
    scale_codes = e4m3_encode((amax / six_g).astype(np.float32))
    s = e4m3_decode(scale_codes).astype(np.float32)
    denom = (s * gg).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (grp / denom[..., None]).astype(np.float32)
    codes = np.where((s == 0)[..., None], np.uint8(0), e2m1_encode(np.where((s == 0)[..., None], 0, y)))
    return codes.reshape(x.shape).astype(np.uint8), scale_codes


def decode_bits(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Stored bits -> float64, exactly."""
    if dtype == "f32":
        return np.asarray(bits, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        with np.errstate(invalid="ignore"):
            return u.view(np.float32).astype(np.float64)
    if dtype == "f16":
        return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    if dtype == "e4m3":
        return e4m3_decode(bits)
    raise ValueError(dtype)


def _to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    return decode_bits(bits, dtype).astype(np.float32)  # exact for every input dtype


def sentinel_bits(dtype: str):
    """NaN pattern that fills pool slots no sequence owns."""
    return {"f32": np.float32(np.nan), "bf16": np.uint16(0x7FC0), "f16": np.uint16(0x7E00),
            "e4m3": np.uint8(0x7F), "nvfp4": np.uint8(0x7F)}[dtype]


# ---------------------------------------------------------------------------
# Paged addressing
# ---------------------------------------------------------------------------

def kv_head_of(h, num_q_heads: int, num_kv_heads: int):
    """GQA: consecutive groups of Hq/Hkv query heads share one KV head."""
    return h // (num_q_heads // num_kv_heads)


def block_address(table_row: np.ndarray, pos, block_size: int):
    """Logical token position -> (physical block id, slot in block)."""
    pos = np.asarray(pos)
    return table_row[pos // block_size], pos % block_size


def key_limit(seq_len: int, q_len: int, j, causal: bool):
    """Number of keys query row ``j`` of a ``q_len``-token step may attend to."""
    j = np.asarray(j)
    if not causal:
        return np.full(j.shape, seq_len)
    return seq_len - q_len + j + 1


def key_start(seq_len: int, q_len: int, j, window: int):
    """First key query row ``j`` may attend to: 0, or ``p - W + 1`` under a window ``W``."""
    j = np.asarray(j)
    if window <= 0:
        return np.zeros(j.shape, dtype=np.int64)
    return np.maximum(0, seq_len - q_len + j + 1 - window)


class OraclePool:
    """Host copy of a pool: ``bits[num_blocks][num_layers][2][Hkv][B][D]`` in storage bits.

    NVFP4 pools hold one E2M1 code per element in ``bits`` and the E4M3 block scale codes in
    ``block_scales[num_blocks][num_layers][2][Hkv][B][D / 16]``; ``nvfp4_pool_bytes`` packs
    both into the pool's byte image."""

    def __init__(self, bits: np.ndarray, dtype: str, k_scale=None, v_scale=None, block_scales=None):
        self.bits = bits
        self.dtype = dtype
        self.block_scales = block_scales
        self.k_scale = None if k_scale is None else np.asarray(k_scale, np.float32)
        self.v_scale = None if v_scale is None else np.asarray(v_scale, np.float32)

    @property
    def block_size(self) -> int:
        return self.bits.shape[4]

    @property
    def num_kv_heads(self) -> int:
        return self.bits.shape[3]

    @property
    def head_dim(self) -> int:
        return self.bits.shape[5]

    def scale(self, which: int, layer: int) -> np.ndarray:
        s = self.k_scale if which == 0 else self.v_scale
        return s[layer]


def new_pool(num_blocks, num_layers, num_kv_heads, block_size, head_dim, dtype, k_scale=None, v_scale=None):
    shape = (num_blocks, num_layers, 2, num_kv_heads, block_size, head_dim)
    if dtype == "nvfp4":
        # The 0x7F fill byte: codes 0xF (dimension 2i) and 0x7 (2i+1), block scales E4M3 NaN.
        bits = np.empty(shape, np.uint8)
        bits[..., 0::2] = 0xF
        bits[..., 1::2] = 0x7
        scales = np.full(shape[:-1] + (head_dim // NVFP4_GROUP,), 0x7F, np.uint8)
        return OraclePool(bits, dtype, k_scale, v_scale, scales)
    storage = {"f32": np.float32, "bf16": np.uint16, "f16": np.uint16, "e4m3": np.uint8}[dtype]
    bits = np.full(shape, sentinel_bits(dtype), storage)
    return OraclePool(bits, dtype, k_scale, v_scale)


def nvfp4_pool_bytes(pool: OraclePool) -> np.ndarray:
    """The pool's byte image: per (block, layer, K|V, head), B rows of D/2 bytes (dimension 2i in
    the low nibble of byte i, 2i+1 in the high one) then B rows of D/16 block scale bytes."""
    c = pool.bits
    packed = (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)
    lead = c.shape[:4]
    return np.concatenate([packed.reshape(lead + (-1,)), pool.block_scales.reshape(lead + (-1,))], axis=-1)


def _store(pool: OraclePool, which: int, layer: int, x_bits: np.ndarray, in_dtype: str):
    """Values [n][Hkv][D] in ``in_dtype`` -> stored bits for the pool dtype (NVFP4: codes and
    block scale codes)."""
    if pool.dtype == "nvfp4":
        x32 = _to_f32(x_bits, in_dtype)
        return nvfp4_quantize(x32, pool.scale(which, layer).astype(np.float32)[None, :])
    if pool.dtype == "e4m3":
        x32 = _to_f32(x_bits, in_dtype)
        scale = pool.scale(which, layer).astype(np.float32)[None, :, None]
        return e4m3_encode(x32 / scale)
    if pool.dtype != in_dtype:
        raise ValueError(f"kv_append into a {pool.dtype} pool takes {pool.dtype} values, got {in_dtype}")
    return np.asarray(x_bits)


def kv_append(pool: OraclePool, layer: int, k_new, v_new, in_dtype: str, cu_new, start_pos, block_tables):
    """Write each new token's K and V rows into its (block, slot).

    ``k_new``/``v_new`` are packed ``[T][Hkv][D]``; sequence ``s`` owns rows
    ``cu_new[s]:cu_new[s+1]`` at positions ``start_pos[s] + i``.
    """
    B = pool.block_size
    for s in range(len(start_pos)):
        lo, hi = int(cu_new[s]), int(cu_new[s + 1])
        if hi <= lo:
            continue
        pos = int(start_pos[s]) + np.arange(hi - lo)
        phys, slot = block_address(block_tables[s], pos, B)
        if np.any(phys < 0) or np.any(phys >= pool.bits.shape[0]):
            raise IndexError(f"sequence {s}: block id out of range")
        for which, src in ((0, k_new), (1, v_new)):
            stored = _store(pool, which, layer, src[lo:hi], in_dtype)
            if pool.dtype == "nvfp4":
                pool.bits[phys, layer, which, :, slot, :] = stored[0]
                pool.block_scales[phys, layer, which, :, slot, :] = stored[1]
            else:
                pool.bits[phys, layer, which, :, slot, :] = stored


def copy_block_prefix(pool: OraclePool, src_blocks, dst_blocks, n_tokens):
    """Partial reuse (deep dive §11, copy_on_partial_reuse): slots ``0 .. n-1`` of block ``src``
    go to the same slots of block ``dst``, for every layer, K and V and KV head; in order, as a
    plain copy of the stored values."""
    for src, dst, n in zip(np.asarray(src_blocks), np.asarray(dst_blocks), np.asarray(n_tokens)):
        pool.bits[int(dst), :, :, :, :int(n), :] = pool.bits[int(src), :, :, :, :int(n), :]
        if pool.block_scales is not None:
            pool.block_scales[int(dst), :, :, :, :int(n), :] = pool.block_scales[int(src), :, :, :, :int(n), :]


def gather_rows(pool: OraclePool, layer: int, table_row, kvh: int, which: int, n: int) -> np.ndarray:
    """Dequantised K (which=0) or V (which=1) of tokens ``0..n-1`` for one KV head, float64 [n][D]."""
    t = np.arange(n)
    phys, slot = block_address(table_row, t, pool.block_size)
    if pool.dtype == "nvfp4":
        codes = pool.bits[phys, layer, which, kvh, slot, :]
        block = e4m3_decode(pool.block_scales[phys, layer, which, kvh, slot, :])  # [n][D/16]
        vals = e2m1_decode(codes) * np.repeat(block, NVFP4_GROUP, axis=-1)
        return vals * np.float64(pool.scale(which, layer)[kvh])
    vals = decode_bits(pool.bits[phys, layer, which, kvh, slot, :], pool.dtype)
    if pool.dtype == "e4m3":
        vals = vals * np.float64(pool.scale(which, layer)[kvh])
    return vals


def _softmax_rows(z: np.ndarray):
    m = z.max(axis=1)
    w = np.exp(z - m[:, None])
    l = w.sum(axis=1)
    return w, m, l


def paged_attention(pool: OraclePool, layer: int, q: np.ndarray, cu_q_lens, seq_lens, block_tables,
                    num_q_heads: int, softmax_scale: float, causal: bool = True, seqs=None, window: int = 0):
    """softmax(scale * q K^T) V over each sequence's paged K/V.

    ``q`` is float64 ``[T_q][Hq][D]`` (already decoded).  Returns ``(out, lse)``
    with ``out`` float64 ``[T_q][Hq][D]`` and ``lse`` float64 ``[T_q][Hq]``; rows
    of sequences outside ``seqs`` stay NaN.  ``window`` > 0 (causal only) limits
    every row to its ``window`` most recent positions.
    """
    if window > 0 and not causal:
        raise ValueError("a window needs causal positions")
    T, Hq, D = q.shape
    Hkv = pool.num_kv_heads
    out = np.full((T, Hq, D), np.nan)
    lse = np.full((T, Hq), np.nan)
    seqs = range(len(seq_lens)) if seqs is None else seqs
    for s in seqs:
        q0, q1 = int(cu_q_lens[s]), int(cu_q_lens[s + 1])
        ql, L = q1 - q0, int(seq_lens[s])
        if ql == 0:
            continue
        lim = key_limit(L, ql, np.arange(ql), causal)
        lo = key_start(L, ql, np.arange(ql), window)
        kv_cache = {}
        for h in range(Hq):
            kvh = int(kv_head_of(h, num_q_heads, Hkv))
            if kvh not in kv_cache:
                kv_cache[kvh] = (gather_rows(pool, layer, block_tables[s], kvh, 0, L),
                                 gather_rows(pool, layer, block_tables[s], kvh, 1, L))
            K, V = kv_cache[kvh]
            z = softmax_scale * (q[q0:q1, h, :] @ K.T)
            t = np.arange(L)[None, :]
            z = np.where((t < lim[:, None]) & (t >= lo[:, None]), z, -np.inf)
            w, m, l = _softmax_rows(z)
            out[q0:q1, h, :] = (w @ V) / l[:, None]
            lse[q0:q1, h] = m + np.log(l)
    return out, lse


def attention_row_probs(pool: OraclePool, layer: int, q: np.ndarray, cu_q_lens, seq_lens, block_tables,
                        num_q_heads: int, softmax_scale: float, causal: bool, s: int, j: int, h: int,
                        window: int = 0):
    """The probability row of one query (sequence ``s``, row ``j``, head ``h``), float64 [seq_len]."""
    L = int(seq_lens[s])
    ql = int(cu_q_lens[s + 1] - cu_q_lens[s])
    kvh = int(kv_head_of(h, num_q_heads, pool.num_kv_heads))
    K = gather_rows(pool, layer, block_tables[s], kvh, 0, L)
    z = softmax_scale * (K @ q[int(cu_q_lens[s]) + j, h, :])
    t = np.arange(L)
    z = np.where((t < key_limit(L, ql, j, causal)) & (t >= key_start(L, ql, j, window)), z, -np.inf)
    w = np.exp(z - z.max())
    return w / w.sum()


def split_kv_reduce(partial_o: np.ndarray, partial_lse: np.ndarray):
    """Merge ``n`` partial states ``[n][R][D]`` / ``[n][R]`` into ``(o [R][D], lse [R])``.

    Parts with ``lse = -inf`` (no keys) carry zero weight.  A row whose parts
    are all empty comes out as ``o = 0``, ``lse = -inf``.
    """
    po = np.asarray(partial_o, np.float64)
    pl = np.asarray(partial_lse, np.float64)
    M = pl.max(axis=0)
    Msafe = np.where(np.isfinite(M), M, 0.0)
    w = np.where(np.isfinite(pl), np.exp(pl - Msafe[None, :]), 0.0)
    tot = w.sum(axis=0)
    o = np.einsum("nr,nrd->rd", w, np.where(np.isfinite(pl)[:, :, None], po, 0.0))
    o = np.where(tot[:, None] > 0, o / np.where(tot > 0, tot, 1.0)[:, None], 0.0)
    lse = np.where(tot > 0, Msafe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return o, lse
