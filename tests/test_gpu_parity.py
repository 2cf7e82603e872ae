"""CUDA path against the oracle, through the C ABI (needs a B200).

kv_append: the whole pool, byte for byte (sentinel NaNs included).
paged_attention: element by element within the stated tolerance, plus the
log-sum-exp, on scaled-down copies of each workload (several tiles, ragged
tails) and on edge cases; full-size workloads are checked on sampled
sequences in test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

import oracle.pkv_oracle as O
import plan_decode as PD
from gpu_common import TOL, assert_close, gpu_out_f64, oracle_out, oracle_pool, oracle_pool_bytes
from paged_kv_attention_block_b200 import workloads as W

pytestmark = pytest.mark.gpu

O_DEV_BAD_BLOCK_ID, O_DEV_BAD_COPY = 0x1, 0x20  # PKV_DEV_* bits of include/pkv.h


@pytest.fixture(scope="module")
def pkv():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_attention_block_b200 import build
    build.build()
    from paged_kv_attention_block_b200 import api, runner
    return api, runner


def run_case(pkv, w, check_pool=True, check_lse=True, **plan_opts):
    api, runner = pkv
    dw = runner.DeviceWorkload(w)
    dw.append_new()
    plan = dw.plan(**plan_opts)
    lse = torch.full((w.total_q, w.num_q_heads), float("nan"), device="cuda")
    out = torch.full_like(dw.q, float("nan"))
    dw.attention(plan, out=out, out_lse=lse)
    torch.cuda.synchronize()
    assert int(dw.status.item()) == 0
    pool = oracle_pool(w)
    if check_pool:
        got = dw.pool_bytes()
        if w.kv_dtype == "f32":
            same = (got.view(np.uint32) == pool.bits.view(np.uint32))
        else:
            same = got == oracle_pool_bytes(pool)
        assert same.all(), f"kv_append: {int((~same).sum())} pool elements differ"
    ref, ref_lse = oracle_out(w, pool)
    err = assert_close(gpu_out_f64(out), ref, w.kv_dtype)
    if check_lse:
        lse_err = np.abs(lse.cpu().numpy() - ref_lse).max()
        assert lse_err <= (1e-5 if w.kv_dtype == "f32" else 2e-3), lse_err
    return plan, err


# ---- the five workload shapes, scaled down -------------------------------

def test_tiny_fp32_exact_config(pkv):
    run_case(pkv, W.tiny_fp32())


def test_tiny_fp32_lengths_before_append_reading(pkv):
    # The other reading of the tiny config: the listed lengths are the cached
    # lengths before the appended token.
    run_case(pkv, W.tiny_fp32(seq_lens=(18, 65, 101, 201)))


@pytest.mark.parametrize("split", [0, -1, 64, 192])
def test_decode_bf16(pkv, split):
    run_case(pkv, W.llama3_8b_decode_bf16(batch=7, lo=1, hi=1500), kv_split=split, num_ctas=40)


@pytest.mark.parametrize("aligned", [True, False])
def test_mixed_bf16(pkv, aligned):
    w = W.mixed_bf16(n_decode=9, n_prefill=3, chunk=200, dec_lo=1, dec_hi=1200, cached_lo_blocks=1,
                     cached_hi_blocks=6, aligned=aligned)
    run_case(pkv, w, num_ctas=60)


@pytest.mark.parametrize("aligned", [True, False])
def test_mixed_fp8(pkv, aligned):
    """Prefill chunks over an fp8 cache (tensor-memory tiles whose fp8 K/V are widened to f16 in
    shared memory) beside fp8 decode rows."""
    w = W.mixed_fp8(n_decode=9, n_prefill=3, chunk=200, dec_lo=1, dec_hi=1200, cached_lo_blocks=1,
                    cached_hi_blocks=6, aligned=aligned)
    plan, _ = run_case(pkv, w, num_ctas=60)
    assert plan.info["num_tc_items"] > 0


def test_mixed_bf16_split_prefill(pkv):
    w = W.mixed_bf16(n_decode=4, n_prefill=2, chunk=150, dec_lo=100, dec_hi=900, cached_lo_blocks=2,
                     cached_hi_blocks=5, block_size=32)
    run_case(pkv, w, kv_split=64)


def test_noncausal_chunks(pkv):
    w = W.mixed_bf16(n_decode=3, n_prefill=2, chunk=70, dec_lo=10, dec_hi=400, cached_lo_blocks=1,
                     cached_hi_blocks=4, block_size=16)
    w.causal = False
    run_case(pkv, w)


@pytest.mark.parametrize("split", [0, 256])
def test_longctx_fp8(pkv, split):
    run_case(pkv, W.longctx_fp8(batch=3, seq_len=3001), kv_split=split, num_ctas=30)


@pytest.mark.parametrize("cascade", [True, False])
def test_prefix_reuse_bf16(pkv, cascade):
    w = W.prefix_reuse_bf16(n_req=21, prefix=512, suf_lo=1, suf_hi=300)
    plan, _ = run_case(pkv, w, cascade=cascade)
    assert (plan.info["num_groups"] > 0) == cascade


@pytest.mark.parametrize("kv", ["bf16", "f16"])
@pytest.mark.parametrize("split", [0, 64])
def test_prefix_reuse_member_paths(pkv, kv, split):
    """Shared-prefix members on every path: one-token and two-token members (8 and 16 rows: decode
    tiles) and three-token members (24 rows: tcgen05 tiles), whole or split suffixes, all merged
    with their group's state by the merge pass; Hq 64 / Hkv 8, block 16."""
    r = np.random.default_rng(23)
    n = 19
    q_lens = r.integers(1, 4, size=n)
    seq_lens = 256 + q_lens + r.integers(0, 200, size=n)
    w = W.build("members", seed=24, kv_dtype=kv, num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=16,
                seq_lens=seq_lens, q_lens=q_lens, shared_prefix_tokens=256)
    plan, _ = run_case(pkv, w, kv_split=split)
    assert plan.info["num_groups"] >= 1


@pytest.mark.parametrize("kv", ["bf16", "f16", "e4m3"])
@pytest.mark.parametrize("split", [0, 64])
def test_prefix_groups_not_neighbours(pkv, kv, split):
    """Three prefixes alternating through the batch (sequence s shares the prefix blocks of group
    s mod 3): each group's tensor-memory tiles read their listed query tokens, and members of a
    tile of 16 or fewer rows read their prefix themselves."""
    r = np.random.default_rng(31)
    n = 41
    q_lens = r.integers(1, 3, size=n)
    seq_lens = 256 + q_lens + r.integers(0, 300, size=n)
    fp8 = dict(q_dtype="bf16", kv_in_dtype="f32") if kv == "e4m3" else {}
    w = W.build("three", seed=32, kv_dtype=kv, num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=16,
                seq_lens=seq_lens, q_lens=q_lens, shared_prefix_tokens=256, prefix_groups=3, **fp8)
    plan, _ = run_case(pkv, w, kv_split=split)
    d = PD.decode(plan.buffer)
    assert plan.info["num_groups"] == 3 and (d["tc_items"]["pos0"] <= -2).any()


@pytest.mark.parametrize("ctas", [1, 2, 3, 5])
def test_few_ctas_many_items(pkv, ctas):
    """Few persistent CTAs working through many items: the stage and item rings wrap many times,
    alternating decode items (warps own whole tiles) and prefill tiles (warps share every tile)."""
    w = W.mixed_bf16(n_decode=40, n_prefill=3, chunk=100, dec_lo=1, dec_hi=900, cached_lo_blocks=1,
                     cached_hi_blocks=4, block_size=64)
    run_case(pkv, w, num_ctas=ctas, kv_split=128)


@pytest.mark.parametrize("ctas", [1, 3])
def test_few_ctas_decode_fp8(pkv, ctas):
    run_case(pkv, W.longctx_fp8(batch=5, seq_len=2000), num_ctas=ctas, kv_split=192)


SIDE_CASES = {
    "mixed_bf16": lambda: W.mixed_bf16(n_decode=20, n_prefill=3, chunk=200, dec_lo=1, dec_hi=1500, cached_lo_blocks=1,
                                       cached_hi_blocks=8, block_size=32, aligned=False),
    "mixed_fp8": lambda: W.mixed_fp8(n_decode=20, n_prefill=3, chunk=200, dec_lo=1, dec_hi=1500, cached_lo_blocks=1,
                                     cached_hi_blocks=8, block_size=32, aligned=False),
    "prefix_bf16": lambda: W.prefix_reuse_bf16(n_req=21, prefix=512, suf_lo=1, suf_hi=300),
}


@pytest.mark.parametrize("heads", [1, 0])
@pytest.mark.parametrize("ctas", [(40, 4), (7, 2), (200, 60)])
@pytest.mark.parametrize("kind", list(SIDE_CASES))
def test_side_by_side(pkv, kind, ctas, heads):
    """The tcgen05 tiles (prefill chunks, shared-prefix group tiles) and the decode tiles running
    at the same time on disjoint SMs, with forced CTA counts (rings wrapping in both kernels), with
    one-head decode items and with the planner's choice (four-head items where it takes them)."""
    w = SIDE_CASES[kind]()
    plan, _ = run_case(pkv, w, num_ctas=ctas[0], tc_num_ctas=ctas[1], heads_per_item=heads)
    flags = PD.decode(plan.buffer)["header"]["flags"]
    assert flags & PD.PLAN_CORUN and (heads == 0 or not flags & PD.PLAN_HEADS4)


@pytest.mark.parametrize("q_dtype", ["bf16", "f16"])
def test_fp8_prefill_wide_query_rows(pkv, q_dtype):
    """fp8 prefill tiles (S on kind::f8f6f4 with each query row scaled by a power of two and split
    into high and low E4M3 parts): rows whose entries span many binades (a few large, most small,
    some exactly zero, whole rows zero) still match the oracle, and so does their LSE."""
    w = W.build("wideq", seed=41, kv_dtype="e4m3", q_dtype=q_dtype, kv_in_dtype="f32", num_q_heads=32,
                num_kv_heads=8, head_dim=128, block_size=16, seq_lens=[700, 300, 90], q_lens=[160, 300, 1])
    r = np.random.default_rng(42)
    x = r.standard_normal((w.total_q, w.num_q_heads, w.head_dim)).astype(np.float32)
    x *= np.float32(2.0) ** r.integers(-12, 4, size=x.shape).astype(np.float32)  # 16 binades per row
    x[r.random(x.shape) < 0.1] = 0.0
    x[::7, 3] = 0.0  # whole rows of zeros
    x[::5, :, 17] *= 200.0  # a large entry sets the row scale
    w._q = W.to_storage(x, q_dtype)
    plan, _ = run_case(pkv, w)
    assert plan.info["num_tc_items"] > 0


@pytest.mark.parametrize("ctas", [1, 2, 5])
def test_few_ctas_prefill_fp8(pkv, ctas):
    """fp8 prefill tiles on the tcgen05 kernel with few CTAs: the raw-code and f16 rings and the
    converter warps wrap many times, across items of ragged last tiles (block 16)."""
    w = W.mixed_fp8(n_decode=9, n_prefill=3, chunk=200, dec_lo=1, dec_hi=700, cached_lo_blocks=1,
                    cached_hi_blocks=30, block_size=16, aligned=False)
    plan, _ = run_case(pkv, w, num_ctas=ctas, kv_split=256)
    assert plan.info["num_tc_items"] > 0


# ---- shapes and dtypes ----------------------------------------------------

@pytest.mark.parametrize("B", [2, 4, 8, 16, 32, 64, 128, 256])
@pytest.mark.parametrize("D", [64, 128])
def test_block_sizes_and_head_dims(pkv, B, D):
    w = W.build(f"b{B}d{D}", seed=B * 7 + D, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=D,
                block_size=B, seq_lens=[1, B - 1 if B > 1 else 1, B, B + 1, 3 * B + 5, 700], q_lens=[1, 1, 1, 1, 4, 33])
    run_case(pkv, w, num_ctas=16)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (16, 2), (32, 2), (64, 1)])
def test_gqa_groups(pkv, hq, hkv):
    w = W.build(f"g{hq}_{hkv}", seed=hq + hkv, kv_dtype="bf16", num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                block_size=64, seq_lens=[300, 65, 1000, 64], q_lens=[1, 1, 20, 64])
    run_case(pkv, w, num_ctas=32)


@pytest.mark.parametrize("kv,qd", [("f16", "f16"), ("e4m3", "f16"), ("e4m3", "bf16"), ("f32", "f32")])
@pytest.mark.parametrize("D", [64, 128])
def test_dtypes(pkv, kv, qd, D):
    w = W.build(f"{kv}{qd}{D}", seed=D + len(kv), kv_dtype=kv, q_dtype=qd, num_q_heads=16, num_kv_heads=4, head_dim=D,
                block_size=16, seq_lens=[5, 130, 777, 40], q_lens=[1, 1, 9, 40])
    run_case(pkv, w, num_ctas=24)


def test_fp8_from_bf16_values(pkv):
    w = W.build("e4m3_bf16in", seed=11, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="bf16", num_q_heads=8,
                num_kv_heads=2, head_dim=128, block_size=32, seq_lens=[100, 1], q_lens=[1, 1], data_scale=3.0)
    run_case(pkv, w)


# ---- edge cases -------------------------------------------------------------

def test_unscheduled_and_single_token_sequences(pkv):
    w = W.build("edge", seed=5, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                seq_lens=[1, 50, 9, 1, 17], q_lens=[1, 0, 9, 0, 1])
    run_case(pkv, w)


def test_empty_batch(pkv):
    api, runner = pkv
    w = W.build("empty", seed=1, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
                seq_lens=[5], q_lens=[0])
    dw = runner.DeviceWorkload(w)
    plan = dw.plan()
    assert plan.info["num_items"] == 0
    dw.attention(plan, out=torch.empty(0, 8, 64, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()


def test_large_logits_stay_finite(pkv):
    w = W.build("big", seed=9, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=64,
                seq_lens=[500, 90], q_lens=[1, 30], data_scale=8.0)
    run_case(pkv, w)


@pytest.mark.parametrize("kv,qd", [("bf16", "bf16"), ("e4m3", "bf16")])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (64, 8)])
def test_multi_token_causal_decode(pkv, kv, qd, hq, hkv):
    # Speculative verification: 2..8 new tokens per sequence, causal among themselves; with g = 4
    # rows stay decode-sized (<= 16) up to 4 tokens and become tensor-memory tiles past that.
    r = np.random.default_rng(5)
    q_lens = r.integers(2, 9, size=24)
    seq_lens = q_lens + r.integers(30, 1500, size=24)
    w = W.build("spec", seed=12, kv_dtype=kv, q_dtype=qd, kv_in_dtype="f32" if kv == "e4m3" else None,
                num_q_heads=hq, num_kv_heads=hkv, head_dim=128, block_size=64, seq_lens=seq_lens, q_lens=q_lens)
    run_case(pkv, w)


@pytest.mark.parametrize("window", [1, 7, 100, 1000])
@pytest.mark.parametrize("kind", ["mixed_bf16", "decode_f16_d64", "fp8", "block4", "f32"])
def test_limited_attention_window(pkv, window, kind):
    # Every kernel path under a window: decode tiles and tcgen05 prefill tiles (bf16 / f16),
    # fp8 decode and row-split prefill, the cp.async kernel (block 4), the fp32 kernel.
    r = np.random.default_rng(window)
    if kind == "mixed_bf16":
        w = W.build("win", seed=13, kv_dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                    seq_lens=[700, 333, 90, 1500, 41], q_lens=[300, 77, 1, 1, 1], window=window)
    elif kind == "decode_f16_d64":
        w = W.build("win", seed=14, kv_dtype="f16", num_q_heads=16, num_kv_heads=4, head_dim=64, block_size=64,
                    seq_lens=r.integers(1, 3000, size=9), q_lens=[1] * 9, window=window)
    elif kind == "fp8":
        w = W.build("win", seed=15, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32,
                    num_kv_heads=8, head_dim=128, block_size=128, seq_lens=[2000, 400, 77], q_lens=[1, 150, 1],
                    window=window)
    elif kind == "block4":
        w = W.build("win", seed=16, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=4,
                    seq_lens=[300, 45, 180], q_lens=[20, 1, 1], window=window)
    else:
        w = W.build("win", seed=17, kv_dtype="f32", num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
                    seq_lens=[300, 45, 180], q_lens=[20, 1, 1], window=window)
    run_case(pkv, w, kv_split=64)
    run_case(pkv, w, check_pool=False)


@pytest.mark.parametrize("kv", ["bf16", "e4m3", "f32", "nvfp4"])
def test_copy_block_prefix_bit_exact(pkv, kv):
    # Partial reuse: copies of whole and partial block prefixes into free blocks, the whole pool
    # compared byte for byte with the oracle's copy; bad ids and counts are reported, not written.
    api, runner = pkv
    if kv in ("e4m3", "nvfp4"):
        w = W.build("copy", seed=18, kv_dtype=kv, q_dtype="bf16", kv_in_dtype="f32", num_q_heads=8,
                    num_kv_heads=2, head_dim=128, block_size=16, seq_lens=[100, 37, 64], q_lens=[1, 1, 1],
                    num_layers=2, layer=1, pool_factor=3.0)
    else:
        w = W.build("copy", seed=18, kv_dtype=kv, num_q_heads=8, num_kv_heads=2, head_dim=64 if kv == "f32" else 128,
                    block_size=16, seq_lens=[100, 37, 64], q_lens=[1, 1, 1], num_layers=2, layer=1, pool_factor=3.0)
    dw = runner.DeviceWorkload(w)
    dw.append_new()
    used = set(int(b) for b in w.block_tables.ravel() if b >= 0)
    free = [b for b in range(w.num_blocks) if b not in used]
    src = w.block_tables[0, :7]
    ns = [16, 1, 8, 0, 15, 16, 4]
    dst = free[:7]
    pool = oracle_pool(w)
    O.copy_block_prefix(pool, src, dst, ns)
    dev = lambda x: torch.tensor(np.asarray(x, np.int32), device="cuda")  # noqa: E731
    api.copy_block_prefix(dw.cache, dev(src), dev(dst), dev(ns), status=dw.status)
    torch.cuda.synchronize()
    assert int(dw.status.item()) == 0
    got = dw.pool_bytes()
    if kv == "f32":
        assert (got.view(np.uint32) == pool.bits.view(np.uint32)).all()
    else:
        assert (got == oracle_pool_bytes(pool)).all()
    before = dw.pool_bytes().copy()
    api.copy_block_prefix(dw.cache, dev([src[0], w.num_blocks]), dev([free[8], free[9]]), dev([17, 4]),
                          status=dw.status)
    torch.cuda.synchronize()
    assert int(dw.status.item()) == (O_DEV_BAD_BLOCK_ID | O_DEV_BAD_COPY)
    after = dw.pool_bytes()
    assert (after.view(np.uint8) == before.view(np.uint8)).all()


@pytest.mark.parametrize("kv", ["bf16", "f16"])
@pytest.mark.parametrize("D", [64, 128])
def test_prefill_running_max_jumps(pkv, kv, D):
    # Logits spread over hundreds of log2 units: a row's running max keeps
    # jumping by more than 2^8 from tile to tile, so the output accumulator is
    # rescaled many times; long causal chunks span many key tiles.
    w = W.build("jumps", seed=11, kv_dtype=kv, num_q_heads=8, num_kv_heads=2, head_dim=D, block_size=16,
                seq_lens=[700, 333], q_lens=[200, 77], data_scale=6.0)
    run_case(pkv, w)


def test_split_reduce_dense(pkv):
    api, _ = pkv
    r = np.random.default_rng(4)
    n, rows, d = 5, 37, 128
    po = r.standard_normal((n, rows, d)).astype(np.float32)
    pl = (r.standard_normal((n, rows)) * 3).astype(np.float32)
    pl[1, :] = -np.inf
    pl[:, 3] = -np.inf  # a row with no keys at all
    o_ref, l_ref = O.split_kv_reduce(po, pl)
    for dt, tol in ((torch.float32, 1e-6), (torch.bfloat16, 8e-3)):
        lse = torch.empty(rows, device="cuda")
        out, _ = api.split_kv_reduce(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda(), out_dtype=dt,
                                     out_lse=lse)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.abs(got - o_ref).max() <= tol * max(1.0, np.abs(o_ref).max())
        gl = lse.cpu().numpy()
        assert np.isneginf(gl[3]) and np.abs(gl[np.isfinite(l_ref)] - l_ref[np.isfinite(l_ref)]).max() <= 1e-5


# ---- errors reported on the device -------------------------------------------

def test_bad_block_id_is_reported_not_faulted(pkv):
    api, runner = pkv
    w = W.build("badbt", seed=2, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                seq_lens=[40, 40], q_lens=[1, 1])
    dw = runner.DeviceWorkload(w)
    before = dw.cache.pool.clone()
    bt = dw.block_tables.clone()
    bt[1, 2] = w.num_blocks + 1000  # corrupt the table on the host side of the call
    api.kv_append(dw.cache, dw.k_new, dw.v_new, dw.cu_q, dw.start_pos, bt, status=dw.status)
    torch.cuda.synchronize()
    assert int(dw.status.item()) & 0x1
    # Sequence 0 was written, the row aimed at the bad block was not; nothing else changed.
    changed = (dw.cache.pool.view(torch.int16) != before.view(torch.int16)).any(dim=(1, 2, 3, 4, 5))
    assert int(changed.sum()) == 1
    dw.status.zero_()
    plan = dw.plan()
    out = torch.zeros_like(dw.q)
    api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, bt, plan, w.softmax_scale, True, out=out,
                        status=dw.status)
    torch.cuda.synchronize()
    assert int(dw.status.item()) & 0x1


STRAY_CASES = {
    "bf16": lambda: W.build("stray", seed=41, kv_dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128,
                            block_size=64, seq_lens=[1, 63, 65, 700, 2049], q_lens=[1, 1, 1, 30, 1]),
    "e4m3": lambda: W.build("stray", seed=42, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32,
                            num_kv_heads=8, head_dim=128, block_size=64, seq_lens=[1, 63, 65, 700, 2049],
                            q_lens=[1, 1, 1, 30, 1]),
    "nvfp4": lambda: W.build("stray", seed=43, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32,
                             num_kv_heads=8, head_dim=128, block_size=64, seq_lens=[1, 63, 65, 700, 2049],
                             q_lens=[1, 1, 1, 5, 1]),
}


@pytest.mark.parametrize("kv", list(STRAY_CASES))
def test_unowned_slots_do_not_reach_the_output(pkv, kv):
    """Stray reads, for every pool type, including fp8 and NVFP4 whose integer dequantisation turns
    the NaN sentinel into a finite value: the pool bytes no sequence owns are filled with two
    different values (0x7F and 0x3C) before the same appends; the outputs of the same plan must be
    bit-identical, so no byte outside a sequence's slots (tails of partly filled blocks, blocks of
    other sequences, unused blocks) reaches any output, and the result matches the oracle."""
    api, runner = pkv
    w = STRAY_CASES[kv]()
    outs = []
    for fill in (0x7F, 0x3C):
        dw = runner.DeviceWorkload(w, fill_byte=fill)
        dw.append_new()
        out = torch.full_like(dw.q, float("nan"))
        dw.attention(dw.plan(kv_split=64), out=out)
        torch.cuda.synchronize()
        assert int(dw.status.item()) == 0
        outs.append(out)
    assert torch.equal(outs[0], outs[1]), "a pool byte outside the sequences reached the output"
    ref, _ = oracle_out(w, oracle_pool(w))
    assert_close(gpu_out_f64(outs[0]), ref, w.kv_dtype)


# ---- four-head decode items --------------------------------------------------

def _h4_decode(name, seed, kv, hq, hkv, D, B, n, hi, q_len=1, q_dtype=None):
    r = np.random.default_rng(seed)
    extra = {} if q_dtype is None else {"q_dtype": q_dtype, "kv_in_dtype": "f32"}
    return W.build(name, seed=seed, kv_dtype=kv, num_q_heads=hq, num_kv_heads=hkv, head_dim=D, block_size=B,
                   seq_lens=r.integers(q_len, hi, size=n), q_lens=[q_len] * n, **extra)


H4_CASES = {
    "bf16_g4": lambda: W.llama3_8b_decode_bf16(batch=7, lo=1, hi=1500),
    "f16_d64_g2": lambda: _h4_decode("h4a", 41, "f16", 32, 16, 64, 16, 9, 2000),
    "bf16_g8_block8": lambda: _h4_decode("h4b", 42, "bf16", 64, 8, 128, 8, 6, 900),
    "bf16_two_tokens": lambda: _h4_decode("h4c", 43, "bf16", 32, 8, 128, 32, 5, 700, q_len=2),
    "fp8_g4": lambda: _h4_decode("h4d", 44, "e4m3", 32, 8, 128, 64, 6, 3000, q_dtype="bf16"),
    "fp8_f16q_block16": lambda: _h4_decode("h4e", 45, "e4m3", 32, 8, 128, 16, 5, 1200, q_dtype="f16"),
    "nvfp4_g4": lambda: _h4_decode("h4f", 46, "nvfp4", 32, 8, 128, 64, 6, 2500, q_dtype="bf16"),
    "nvfp4_g8_block16": lambda: _h4_decode("h4g", 47, "nvfp4", 64, 8, 128, 16, 4, 900, q_dtype="f16"),
    "prefix_g8": lambda: W.prefix_reuse_bf16(n_req=37, prefix=512, suf_lo=1, suf_hi=300),
}


@pytest.mark.parametrize("split", [0, -1, 64])
@pytest.mark.parametrize("kind", list(H4_CASES))
def test_four_head_items(pkv, kind, split):
    """Plans whose decode items cover four KV heads (one consumer warp a head, no merge between
    warps): every pool kind of the TMA-fed decode kernel, g 2 to 8, one and two query tokens,
    blocks smaller than a tile, split and unsplit key ranges, shared-prefix members' suffixes."""
    w = H4_CASES[kind]()
    plan, _ = run_case(pkv, w, heads_per_item=4, kv_split=split, num_ctas=40)
    assert plan.info["heads_per_item"] == 4
    d = PD.decode(plan.buffer)
    assert d["header"]["flags"] & PD.PLAN_HEADS4 and (d["reg_items"]["kv_head"] % 4 == 0).all()


@pytest.mark.parametrize("heads", [1, 4])
def test_nvfp4_shared_prefix_groups(pkv, heads):
    """NVFP4 pools have no tcgen05 kernel: a run of sharers reads its prefix as decode-tile group
    items (at most 8 rows), one or four KV heads an item, merged with each member's own suffix."""
    w = W.build("nvp", seed=49, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32, num_kv_heads=8,
                head_dim=128, block_size=16, seq_lens=300 + np.arange(9) * 13, q_lens=[1] * 9,
                shared_prefix_tokens=256)
    plan, _ = run_case(pkv, w, heads_per_item=heads, num_ctas=40)
    assert plan.info["num_groups"] == 1 and plan.info["heads_per_item"] == heads


@pytest.mark.parametrize("ctas", [1, 3])
@pytest.mark.parametrize("kind", ["bf16_g4", "nvfp4_g4"])
def test_four_head_items_few_ctas(pkv, kind, ctas):
    """Few CTAs run many four-head items in turn: the warps' stage rings and staging rows carry
    from item to item without an end-of-item barrier."""
    run_case(pkv, H4_CASES[kind](), check_pool=False, heads_per_item=4, num_ctas=ctas)


@pytest.mark.parametrize("window", [1, 100])
def test_four_head_items_window(pkv, window):
    w = _h4_decode("h4w", 48, "bf16", 32, 8, 128, 16, 7, 2000)
    w.window = window
    run_case(pkv, w, heads_per_item=4, num_ctas=40)


@pytest.mark.parametrize("kv", ["e4m3", "nvfp4"])
def test_bad_block_id_in_quantised_pools(pkv, kv):
    """fp8 and NVFP4 decode tiles: a block id outside the pool inside a sequence's range is
    reported (PKV_DEV_BAD_BLOCK_ID), its keys read as zeros rather than from any memory, the
    output stays finite, and every other sequence still matches the oracle."""
    api, runner = pkv
    w = STRAY_CASES[kv]()
    dw = runner.DeviceWorkload(w)
    dw.append_new()
    bt = dw.block_tables.clone()
    bad_seq = 3
    bt[bad_seq, 5] = w.num_blocks + 77
    out = torch.full_like(dw.q, float("nan"))
    api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, bt, dw.plan(), w.softmax_scale, w.causal, out=out,
                        status=dw.status)
    torch.cuda.synchronize()
    assert int(dw.status.item()) & 0x1
    got = gpu_out_f64(out)
    assert np.isfinite(got).all()
    ref, _ = oracle_out(w, oracle_pool(w))
    rows = np.concatenate([np.arange(w.cu_q_lens[s], w.cu_q_lens[s + 1]) for s in range(w.num_seqs) if s != bad_seq])
    assert_close(got, ref, w.kv_dtype, rows=rows)


def test_plan_mismatch_is_reported(pkv):
    api, runner = pkv
    w = W.build("mism", seed=3, kv_dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
                seq_lens=[40, 70], q_lens=[1, 1])
    dw = runner.DeviceWorkload(w)
    plan = dw.plan()
    short = dw.seq_lens.clone()
    short[1] = 10  # device lengths no longer match the plan
    api.paged_attention(dw.cache, dw.q, dw.cu_q, short, dw.block_tables, plan, w.softmax_scale, True,
                        status=dw.status)
    torch.cuda.synchronize()
    assert int(dw.status.item()) & 0x4


TIMEOUT_CASES = {
    # decode tiles (TMA-fed kernel), bf16 and fp8 pools
    "decode_bf16": lambda: W.llama3_8b_decode_bf16(batch=5, lo=100, hi=2000),
    "decode_fp8": lambda: W.longctx_fp8(batch=2, seq_len=3000),
    # a prefill chunk (tcgen05 kernel) beside decode rows
    "mixed_bf16": lambda: W.mixed_bf16(n_decode=3, n_prefill=1, chunk=150, dec_lo=50, dec_hi=900, cached_lo_blocks=1,
                                       cached_hi_blocks=3),
    # the same batch with the two kernels side by side
    "mixed_bf16_side_by_side": lambda: W.mixed_bf16(n_decode=3, n_prefill=1, chunk=150, dec_lo=50, dec_hi=900,
                                                    cached_lo_blocks=1, cached_hi_blocks=3),
    # four-head decode items (no end-of-item barrier between the warps)
    "decode_bf16_heads4": lambda: W.llama3_8b_decode_bf16(batch=5, lo=100, hi=2000),
}


@pytest.mark.parametrize("kind", list(TIMEOUT_CASES))
def test_wait_timeout_is_reported(pkv, kind):
    """The bounded waits' timeout path: with PKV_DEBUG_WITHHOLD_LOADS the producers publish the
    work but load nothing, so with a short wait limit (2e5 SM cycles, about 0.1 ms) every
    consumer wait runs out; the kernels record PKV_DEV_TIMEOUT, drain, free tensor memory and
    return.  The context stays usable: a normal launch on the same pool then matches the oracle."""
    api, runner = pkv
    w = TIMEOUT_CASES[kind]()
    dw = runner.DeviceWorkload(w)
    dw.append_new()
    side = {"tc_num_ctas": 4} if kind.endswith("side_by_side") else {}
    if kind.endswith("heads4"):
        side = {"heads_per_item": 4}
    plan = dw.plan(num_ctas=16, wait_limit_kcycles=200, debug_flags=api.PKV_DEBUG_WITHHOLD_LOADS, **side)
    if side:
        flag = PD.PLAN_HEADS4 if kind.endswith("heads4") else PD.PLAN_CORUN
        assert PD.decode(plan.buffer)["header"]["flags"] == flag
    out = torch.zeros_like(dw.q)
    dw.attention(plan, out=out)
    torch.cuda.synchronize()
    assert int(dw.status.item()) & 0x10, "PKV_DEV_TIMEOUT not reported"
    dw.status.zero_()
    out = torch.full_like(dw.q, float("nan"))
    dw.attention(dw.plan(num_ctas=16, **side), out=out)
    torch.cuda.synchronize()
    assert int(dw.status.item()) == 0
    ref, _ = oracle_out(w, oracle_pool(w))
    assert_close(gpu_out_f64(out), ref, w.kv_dtype)


def test_repeat_launch_is_deterministic(pkv):
    api, runner = pkv
    w = W.llama3_8b_decode_bf16(batch=5, lo=100, hi=3000)
    dw = runner.DeviceWorkload(w)
    dw.append_new()
    plan = dw.plan(num_ctas=20)
    a = dw.attention(plan).clone()
    b = dw.attention(plan).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_graph_step_matches_oracle(pkv):
    """GraphStep (page-locked inputs, host plan, one graph replay per step, output copied back):
    every step's host output equals the oracle's within the bf16 tolerance, on both buffer slots."""
    api, runner = pkv
    w = W.llama3_8b_decode_bf16(batch=6, lo=50, hi=2000)
    dw = runner.DeviceWorkload(w)
    names = {"q": dw.q, "k_new": dw.k_new, "v_new": dw.v_new, "cu_q": dw.cu_q, "seq_lens": dw.seq_lens,
             "start_pos": dw.start_pos, "block_tables": dw.block_tables}
    kw = dict(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
              block_size=w.block_size, kv_dtype=w.kv_dtype, causal=w.causal)
    gs = api.GraphStep(dw.cache, names, kw, w.softmax_scale, w.causal)
    for views in gs.host:
        for k, v in names.items():
            views[k].copy_(v.cpu())
    ref, _ = oracle_out(w, oracle_pool(w))
    slots = [gs.run() for _ in range(3)]
    for s in slots[-2:]:
        got = gs.wait(s).float().numpy().astype(np.float64)
        assert_close(got, ref, w.kv_dtype, what=f"slot {s}")
    assert gs.h2d_bytes >= sum(t.numel() * t.element_size() for t in names.values())



# ---- NVFP4 KV cache (E2M1 codes, E4M3 block scales, float32 scale per (layer, head, K|V)) ----

@pytest.mark.parametrize("B", [16, 32, 64, 128])
@pytest.mark.parametrize("hq", [32, 64])
def test_nvfp4_decode(pkv, B, hq):
    """kv_append byte for byte (codes and block scales) and decode attention, Hkv 8, d 128,
    ragged lengths over several 64-key tiles, blocks smaller and larger than a tile."""
    w = W.build("nv_dec", seed=30 + B, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=hq,
                num_kv_heads=8, head_dim=128, block_size=B, seq_lens=[1, 63, 64, 65, 300, 777, 2049],
                q_lens=[1] * 7, data_scale=0.5)
    run_case(pkv, w)


@pytest.mark.parametrize("split", [-1, 64, 0])
def test_nvfp4_llama3_8b_decode_shape(pkv, split):
    run_case(pkv, W.llama3_8b_decode_nvfp4(batch=9, lo=1, hi=3000), kv_split=split)


@pytest.mark.parametrize("in_dtype", ["bf16", "f16"])
def test_nvfp4_from_16bit_values(pkv, in_dtype):
    w = W.build("nv_in", seed=33, kv_dtype="nvfp4", q_dtype="bf16" if in_dtype == "bf16" else "f16",
                kv_in_dtype=in_dtype, num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=64,
                seq_lens=[130, 5, 700], q_lens=[1, 1, 1])
    run_case(pkv, w)


def test_nvfp4_chunks_and_multi_token(pkv):
    """Prefill chunks and multi-token decode rows over an NVFP4 cache (8-row tiles, causal)."""
    w = W.build("nv_mix", seed=34, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32,
                num_kv_heads=8, head_dim=128, block_size=16, seq_lens=[300, 90, 41, 17], q_lens=[45, 4, 2, 1])
    run_case(pkv, w)


@pytest.mark.parametrize("window", [1, 50, 200])
def test_nvfp4_limited_window(pkv, window):
    w = W.build("nv_win", seed=35, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32,
                num_kv_heads=8, head_dim=128, block_size=32, seq_lens=[700, 64, 250], q_lens=[3, 1, 1],
                window=window)
    run_case(pkv, w)

