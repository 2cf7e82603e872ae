"""Seeded synthetic workloads for paged KV-cache attention.

This module only draws inputs: sequence lengths, block tables, query and K/V
values and the fp8 calibration scales.  It performs none of the attention
arithmetic and none of the KV-cache writes; both the CUDA path and the CPU
oracle receive exactly the arrays produced here.

Shapes follow the workloads the TensorRT-LLM deep dive (gentlecold.top,
"NVIDIA TensorRT-LLM详解") describes: a block pool with a per-request block table
(§9 "KV cache系统"), in-flight batches that pack context (prefill) requests
before generation (decode) requests (§6 "In-flight batching"), chunked prefill
whose non-final chunks are block multiples (§8 "Chunked prefill"), prefix
blocks shared through radix-tree reuse (§10 "跨请求KV复用") and an fp8 KV cache
(§13 "量化").

Recipe (all draws from numpy PCG64 streams keyed by (seed, stream id)):

* lengths, block permutation, queries and every sequence's K/V come from
  separate streams, so a sequence's K/V can be regenerated alone; a shared
  prefix has a stream of its own (one per prefix group: with
  ``prefix_groups`` = G, sequence s shares the prefix blocks and values of
  group s mod G, so sharers need not be neighbours in the batch);
* values are N(0, 1) float32 times ``data_scale``; bf16/f16 storage rounds
  them to nearest-even through torch's CPU conversion;
* the physical blocks are a seeded permutation of a pool of
  ``ceil(pool_factor * need)`` blocks (or an explicit ``num_blocks``);
  block-table padding is -1;
* fp8 scales are calibration inputs: ``amax / 448`` per (layer, KV head) and
  separately for K and V, over every token of that head; NVFP4 global scales
  are ``amax / (6 * 448)`` on the same footing (the largest E2M1 value times
  the largest E4M3 block scale), so no block scale saturates.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
import os

import numpy as np

# Storage dtype names shared by the binding and the tests.
DTYPES = ("f32", "bf16", "f16", "e4m3", "nvfp4")


def kv_row_bytes(dtype: str, head_dim: int) -> float:
    """Bytes of one token's K (or V) row of one head in a pool of ``dtype`` (NVFP4: head_dim / 2
    bytes of codes and head_dim / 16 bytes of block scales)."""
    if dtype == "nvfp4":
        return head_dim // 2 + head_dim // 16
    return head_dim * {"f32": 4, "bf16": 2, "f16": 2, "e4m3": 1}[dtype]

_STREAM_LENS, _STREAM_PERM, _STREAM_Q, _STREAM_PREFIX = 1, 2, 3, 4
_STREAM_SEQ_BASE = 1000


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


def to_storage(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to a storage dtype (bits as uint16 for 16-bit types)."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "f32":
        return x32
    import torch

    t = torch.from_numpy(x32)
    if dtype == "bf16":
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if dtype == "f16":
        return t.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(f"no direct storage rounding for {dtype}")


@dataclass
class Workload:
    """One step of an in-flight batch over a paged KV cache.

    ``seq_lens[s]`` is the KV length attention sees for sequence ``s``,
    including the ``q_lens[s]`` tokens processed (and appended) this step.
    The first ``seq_lens[s] - q_lens[s]`` tokens are history already in the
    cache; the last ``q_lens[s]`` are appended by this step.
    """

    name: str
    seed: int
    kv_dtype: str
    q_dtype: str
    kv_in_dtype: str  # dtype of the K/V values handed to kv_append
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    num_layers: int
    layer: int
    seq_lens: np.ndarray
    q_lens: np.ndarray
    block_tables: np.ndarray
    softmax_scale: float
    causal: bool
    data_scale: float
    shared_prefix_tokens: int
    k_scale: np.ndarray | None = None  # [num_layers][Hkv] float32, fp8 and NVFP4 only
    v_scale: np.ndarray | None = None
    window: int = 0  # limited attention window (positions); 0 = every cached key
    prefix_groups: int = 1  # sequence s shares the prefix of group s % prefix_groups
    _kv_cache: dict = field(default_factory=dict, repr=False)
    _q: np.ndarray | None = field(default=None, repr=False)

    # ---- derived shapes -------------------------------------------------
    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def cu_q_lens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int32)

    @property
    def total_q(self) -> int:
        return int(self.q_lens.sum())

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def start_pos(self) -> np.ndarray:
        """Position of each sequence's first new token."""
        return (self.seq_lens - self.q_lens).astype(np.int32)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    # ---- values ---------------------------------------------------------
    @property
    def q(self) -> np.ndarray:
        """Queries [total_q][Hq][D] in q storage (float32 or uint16 bits)."""
        if self._q is None:
            r = _rng(self.seed, _STREAM_Q)
            x = r.standard_normal((self.total_q, self.num_q_heads, self.head_dim), dtype=np.float32)
            self._q = to_storage(x * np.float32(self.data_scale), self.q_dtype)
        return self._q

    def _draw_tokens(self, stream: tuple, n: int) -> tuple[np.ndarray, np.ndarray]:
        shape = (n, self.num_kv_heads, self.head_dim)
        r = _rng(self.seed, *stream)
        k = r.standard_normal(shape, dtype=np.float32)
        v = r.standard_normal(shape, dtype=np.float32)
        if self.data_scale != 1.0:
            k *= np.float32(self.data_scale)
            v *= np.float32(self.data_scale)
        return k, v

    def kv_values(self, s: int, cache: bool = True) -> tuple[np.ndarray, np.ndarray]:
        """K and V of every token of sequence ``s`` ([seq_len][Hkv][D]) in ``kv_in_dtype``.

        Tokens inside a shared prefix take their values from one prefix
        stream, so every sharing sequence sees identical prefix K/V.
        """
        if cache and s in self._kv_cache:
            return self._kv_cache[s]
        L = int(self.seq_lens[s])
        P = min(self.shared_prefix_tokens, L)
        parts_k, parts_v = [], []
        if P > 0:
            grp = s % self.prefix_groups
            key = "prefix" if grp == 0 else f"prefix{grp}"
            if key not in self._kv_cache:
                stream = (_STREAM_PREFIX,) if grp == 0 else (_STREAM_PREFIX, grp)
                self._kv_cache[key] = self._draw_tokens(stream, self.shared_prefix_tokens)
            pk, pv = self._kv_cache[key]
            parts_k.append(pk[:P])
            parts_v.append(pv[:P])
        if L - P > 0:
            ok, ov = self._draw_tokens((_STREAM_SEQ_BASE + s,), L - P)
            parts_k.append(ok)
            parts_v.append(ov)
        k = np.concatenate(parts_k) if parts_k else np.zeros((0, self.num_kv_heads, self.head_dim), np.float32)
        v = np.concatenate(parts_v) if parts_v else np.zeros_like(k)
        if self.kv_in_dtype != "f32":
            k, v = to_storage(k, self.kv_in_dtype), to_storage(v, self.kv_in_dtype)
        if cache:
            self._kv_cache[s] = (k, v)
        return k, v

    def packed_kv(self, which: str, seqs=None) -> tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
        """Packed K/V rows for kv_append.

        ``which`` is "new" (this step's tokens), "history" (tokens cached
        before this step) or "all".  Returns (k, v, cu, start_pos) restricted to
        ``seqs`` (default: every sequence); cu and start_pos have one entry per
        listed sequence.
        """
        seqs = range(self.num_seqs) if seqs is None else list(seqs)
        ks, vs, cu, sp = [], [], [0], []
        for s in seqs:
            k, v = self.kv_values(s)
            L, ql = int(self.seq_lens[s]), int(self.q_lens[s])
            lo, hi = {"new": (L - ql, L), "history": (0, L - ql), "all": (0, L)}[which]
            ks.append(k[lo:hi])
            vs.append(v[lo:hi])
            cu.append(cu[-1] + hi - lo)
            sp.append(lo)
        k = np.concatenate(ks) if ks else np.zeros((0, self.num_kv_heads, self.head_dim), np.float32)
        v = np.concatenate(vs) if vs else np.zeros_like(k)
        return k, v, np.asarray(cu, np.int32), np.asarray(sp, np.int32)

    def release(self) -> None:
        self._kv_cache.clear()

    # ---- byte accounting (inputs only) --------------------------------
    def distinct_kv_blocks(self) -> list[tuple[int, int]]:
        """(physical block, tokens used) for every distinct block referenced."""
        used: dict[int, int] = {}
        B = self.block_size
        for s in range(self.num_seqs):
            L = int(self.seq_lens[s])
            for j in range((L + B - 1) // B):
                phys = int(self.block_tables[s, j])
                used[phys] = max(used.get(phys, 0), min(B, L - j * B))
        return sorted(used.items())


def _calibrate_fp8(w: Workload, threads: int, top: float = 448.0) -> None:
    """amax / top scales per (layer, KV head), separately for K and V (top: 448 for fp8,
    6 * 448 for NVFP4 global scales)."""
    H = w.num_kv_heads

    def one(s):
        k, v = w.kv_values(s)
        return np.abs(k).max(axis=(0, 2)) if len(k) else np.zeros(H), np.abs(v).max(axis=(0, 2)) if len(v) else np.zeros(H)

    amax_k = np.zeros(H, np.float64)
    amax_v = np.zeros(H, np.float64)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for ak, av in ex.map(one, range(w.num_seqs)):
            amax_k = np.maximum(amax_k, ak)
            amax_v = np.maximum(amax_v, av)
    ks = np.ones((w.num_layers, H), np.float32)
    vs = np.ones((w.num_layers, H), np.float32)
    ks[w.layer] = (np.maximum(amax_k, 1e-12) / top).astype(np.float32)
    vs[w.layer] = (np.maximum(amax_v, 1e-12) / top).astype(np.float32)
    w.k_scale, w.v_scale = ks, vs


def build(
    name: str,
    *,
    seed: int,
    kv_dtype: str,
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    block_size: int,
    seq_lens,
    q_lens,
    q_dtype: str | None = None,
    kv_in_dtype: str | None = None,
    num_blocks: int | None = None,
    pool_factor: float = 1.25,
    data_scale: float = 1.0,
    shared_prefix_tokens: int = 0,
    num_layers: int = 1,
    layer: int = 0,
    causal: bool = True,
    window: int = 0,
    softmax_scale: float | None = None,
    table_slack: int = 0,
    threads: int | None = None,
    prefix_groups: int = 1,
) -> Workload:
    """Assemble a workload; see the module docstring for the recipe."""
    seq_lens = np.asarray(seq_lens, np.int32)
    q_lens = np.asarray(q_lens, np.int32)
    assert seq_lens.shape == q_lens.shape and np.all(q_lens <= seq_lens) and np.all(q_lens >= 0)
    B = block_size
    if q_dtype is None:
        q_dtype = "f32" if kv_dtype == "f32" else ("f16" if kv_dtype == "f16" else "bf16")
    if kv_in_dtype is None:
        kv_in_dtype = "f32" if kv_dtype in ("f32", "e4m3", "nvfp4") else kv_dtype
    S = len(seq_lens)
    nblk = [(int(L) + B - 1) // B for L in seq_lens]
    P_blocks = shared_prefix_tokens // B
    assert shared_prefix_tokens % B == 0, "shared prefix must be whole blocks"
    if P_blocks:
        assert all(int(L) >= shared_prefix_tokens for L in seq_lens)
    own = [n - P_blocks for n in nblk]
    G = max(1, int(prefix_groups))
    need = G * P_blocks + sum(own)
    if num_blocks is None:
        num_blocks = max(1, math.ceil(pool_factor * need))
    assert num_blocks >= need
    perm = _rng(seed, _STREAM_PERM).permutation(num_blocks).astype(np.int32)
    max_blocks = max(nblk + [1]) + table_slack
    bt = np.full((S, max_blocks), -1, np.int32)
    nxt = G * P_blocks
    for s in range(S):
        grp = s % G  # prefix group: its own physical prefix blocks
        bt[s, :P_blocks] = perm[grp * P_blocks:(grp + 1) * P_blocks]
        bt[s, P_blocks:nblk[s]] = perm[nxt:nxt + own[s]]
        nxt += own[s]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(head_dim)
    w = Workload(
        name=name, seed=seed, kv_dtype=kv_dtype, q_dtype=q_dtype, kv_in_dtype=kv_in_dtype,
        num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=B,
        num_blocks=int(num_blocks), num_layers=num_layers, layer=layer, seq_lens=seq_lens,
        q_lens=q_lens, block_tables=bt, softmax_scale=float(softmax_scale), causal=causal, window=int(window),
        data_scale=data_scale, shared_prefix_tokens=shared_prefix_tokens, prefix_groups=G,
    )
    if kv_dtype in ("e4m3", "nvfp4"):
        _calibrate_fp8(w, threads or min(32, os.cpu_count() or 1), 448.0 if kv_dtype == "e4m3" else 6.0 * 448.0)
    return w


def _lens(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    return _rng(seed, _STREAM_LENS).integers(lo, hi, size=n, endpoint=True).astype(np.int32)


# ---------------------------------------------------------------------------
# The five named workloads.  Each builder takes size knobs so tests can run a
# scaled-down copy with the same structure.
# ---------------------------------------------------------------------------

def tiny_fp32(seed: int = 1001, seq_lens=(17, 64, 100, 200)) -> Workload:
    """4 decode sequences, fp32 KV, Hq 8 / Hkv 2, d 64, block 16, 64-block pool."""
    S = len(seq_lens)
    return build("tiny_fp32", seed=seed, kv_dtype="f32", num_q_heads=8, num_kv_heads=2, head_dim=64,
                 block_size=16, seq_lens=seq_lens, q_lens=[1] * S, num_blocks=64)


def llama3_8b_decode_bf16(seed: int = 1002, batch: int = 64, lo: int = 512, hi: int = 4096) -> Workload:
    """Decode batch, bf16 KV, Hq 32 / Hkv 8, d 128, block 64, lens U[lo, hi], N(0,1)*0.5."""
    return build("llama3_8b_decode_bf16", seed=seed, kv_dtype="bf16", num_q_heads=32, num_kv_heads=8,
                 head_dim=128, block_size=64, seq_lens=_lens(seed, batch, lo, hi), q_lens=[1] * batch,
                 data_scale=0.5)


def mixed_bf16(seed: int = 1003, n_decode: int = 120, n_prefill: int = 4, chunk: int = 512,
               dec_lo: int = 256, dec_hi: int = 8192, cached_lo_blocks: int = 8, cached_hi_blocks: int = 48,
               block_size: int = 128, aligned: bool = True) -> Workload:
    """Prefill chunks (packed first) plus decode sequences in one batch, bf16 KV, block 128.

    Cached prefixes of the prefill requests are block multiples when ``aligned``
    (non-final chunks are block multiples), else drawn at token granularity.
    """
    r = _rng(seed, _STREAM_LENS)
    if aligned:
        cached = r.integers(cached_lo_blocks, cached_hi_blocks, size=n_prefill, endpoint=True) * block_size
    else:
        cached = r.integers(cached_lo_blocks * block_size, cached_hi_blocks * block_size, size=n_prefill, endpoint=True)
    dec = r.integers(dec_lo, dec_hi, size=n_decode, endpoint=True)
    seq_lens = np.concatenate([cached + chunk, dec]).astype(np.int32)
    q_lens = np.concatenate([np.full(n_prefill, chunk), np.ones(n_decode)]).astype(np.int32)
    return build("mixed_bf16", seed=seed, kv_dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                 block_size=block_size, seq_lens=seq_lens, q_lens=q_lens)


def mixed_fp8(seed: int = 1003, **kw) -> Workload:
    """The mixed in-flight batch (same lengths and values as mixed_bf16) over an fp8-e4m3 cache:
    K/V appended from float32 with amax/448 scales per (layer, KV head, K|V), q bf16."""
    w = mixed_bf16(seed=seed, **kw)
    return build("mixed_fp8", seed=seed, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32",
                 num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                 block_size=w.block_size, seq_lens=w.seq_lens, q_lens=w.q_lens)


def llama3_8b_decode_nvfp4(seed: int = 1002, batch: int = 64, lo: int = 512, hi: int = 4096) -> Workload:
    """The Llama-3-8B decode batch (same lengths and values as the bf16 one) over an NVFP4 cache:
    Hq 32 / Hkv 8, d 128, block 64, q bf16, K/V appended from float32."""
    return build("llama3_8b_decode_nvfp4", seed=seed, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32",
                 num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=64, seq_lens=_lens(seed, batch, lo, hi),
                 q_lens=[1] * batch, data_scale=0.5)


def longctx_fp8(seed: int = 1004, batch: int = 8, seq_len: int = 131072) -> Workload:
    """Long-context decode, e4m3 KV with per-(layer, KV-head) scales, q bf16, block 128."""
    return build("longctx_fp8", seed=seed, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32",
                 num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=128,
                 seq_lens=[seq_len] * batch, q_lens=[1] * batch)


def prefix_reuse_bf16(seed: int = 1005, n_req: int = 256, prefix: int = 2048, suf_lo: int = 64,
                      suf_hi: int = 512) -> Workload:
    """Decode requests sharing one prefix's physical blocks, Hq 64 / Hkv 8, d 128, block 128."""
    suffix = _lens(seed, n_req, suf_lo, suf_hi)
    return build("prefix_reuse_bf16", seed=seed, kv_dtype="bf16", num_q_heads=64, num_kv_heads=8,
                 head_dim=128, block_size=128, seq_lens=prefix + suffix, q_lens=[1] * n_req,
                 shared_prefix_tokens=prefix)


NAMED = {
    "tiny_fp32": tiny_fp32,
    "llama3_8b_decode_bf16": llama3_8b_decode_bf16,
    "mixed_bf16": mixed_bf16,
    "longctx_fp8": longctx_fp8,
    "llama3_8b_decode_nvfp4": llama3_8b_decode_nvfp4,
    "prefix_reuse_bf16": prefix_reuse_bf16,
    "mixed_fp8": mixed_fp8,
}
