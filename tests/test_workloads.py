"""The seeded generator: determinism and the structure the pages describe (CPU only)."""
import numpy as np

from paged_kv_attention_block_b200 import workloads as W


def test_deterministic():
    a, b = W.llama3_8b_decode_bf16(batch=4, lo=10, hi=90), W.llama3_8b_decode_bf16(batch=4, lo=10, hi=90)
    assert np.array_equal(a.block_tables, b.block_tables) and np.array_equal(a.q, b.q)
    for s in range(4):
        assert all(np.array_equal(x, y) for x, y in zip(a.kv_values(s), b.kv_values(s)))


def test_named_shapes():
    w = W.tiny_fp32()
    assert list(w.seq_lens) == [17, 64, 100, 200] and w.num_blocks == 64 and w.block_size == 16
    assert (w.block_tables >= 0).sum() == 2 + 4 + 7 + 13
    w = W.llama3_8b_decode_bf16()
    assert w.num_seqs == 64 and w.seq_lens.min() >= 512 and w.seq_lens.max() <= 4096
    assert w.num_blocks == int(np.ceil(1.25 * sum((int(L) + 63) // 64 for L in w.seq_lens)))
    w = W.mixed_bf16()
    assert w.num_seqs == 124 and list(w.q_lens[:4]) == [512] * 4 and (w.q_lens[4:] == 1).all()
    # Context (prefill) requests are packed before generation (decode) requests; cached
    # prefixes of the chunks are block multiples (non-final chunks are block multiples).
    cached = w.seq_lens[:4] - 512
    assert (cached % 128 == 0).all() and cached.min() >= 1024 and cached.max() <= 6144
    w = W.prefix_reuse_bf16()
    assert (w.block_tables[:, :16] == w.block_tables[0, :16]).all()
    assert w.num_q_heads == 64 and w.num_kv_heads == 8


def test_block_tables_distinct_and_in_pool():
    for w in (W.llama3_8b_decode_bf16(batch=6, lo=10, hi=400), W.prefix_reuse_bf16(n_req=5, prefix=256)):
        ids = []
        P = w.shared_prefix_tokens // w.block_size
        for s in range(w.num_seqs):
            n = (int(w.seq_lens[s]) + w.block_size - 1) // w.block_size
            row = w.block_tables[s]
            assert (row[:n] >= 0).all() and (row[:n] < w.num_blocks).all() and (row[n:] == -1).all()
            ids.extend(row[P if s else 0:n].tolist())
        assert len(ids) == len(set(ids))


def test_fp8_scales_are_amax_over_448():
    w = W.longctx_fp8(batch=2, seq_len=70)
    for h in range(w.num_kv_heads):
        amax = max(np.abs(w.kv_values(s)[0][:, h]).max() for s in range(2))
        assert w.k_scale[0, h] == np.float32(amax / 448.0)


def test_nvfp4_global_scales_and_shared_values():
    """NVFP4 global scales are amax / (6 * 448) per (layer, KV head), K and V apart; the NVFP4 decode
    batch draws the same lengths, tables and values as the bf16 one."""
    w = W.llama3_8b_decode_nvfp4(batch=3, lo=20, hi=90)
    for h in range(w.num_kv_heads):
        for which, sc in ((0, w.k_scale), (1, w.v_scale)):
            amax = max(np.abs(w.kv_values(s)[which][:, h]).max() for s in range(3))
            assert sc[0, h] == np.float32(amax / (6.0 * 448.0))
    b = W.llama3_8b_decode_bf16(batch=3, lo=20, hi=90)
    assert np.array_equal(w.seq_lens, b.seq_lens) and np.array_equal(w.block_tables, b.block_tables)
    assert w.kv_in_dtype == "f32" and w.q_dtype == "bf16" and w.block_size == 64
