"""The C ABI without a GPU: exports, argument checks, and the host planner (CPU only)."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from paged_kv_attention_block_b200 import build as B
from paged_kv_attention_block_b200 import workloads as W
import plan_decode as PD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def api():
    B.build()
    from paged_kv_attention_block_b200 import api as A
    return A


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "pkv.h")).read()
    return sorted(set(re.findall(r"PKV_API\s+[\w\s\*]+?\b(pkv_\w+)\s*\(", text)))


def test_exports_match_header(api):
    names = declared_symbols()
    assert len(names) >= 8
    lib = C.CDLL(api.library_path())
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", api.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (pkv_\w+)", out))
    assert set(names) == exported, (set(names) ^ exported)


def test_version_and_strings(api):
    assert api._lib.pkv_abi_version() == 4
    assert api.status_string(0) == "ok" and api.status_string(4) == "buffer too small"


def _cache(**kw):
    from paged_kv_attention_block_b200 import api as A
    d = dict(pool=0x1000, num_blocks=10, num_layers=1, layer=0, num_kv_heads=2, head_dim=64, block_size=16,
             kv_dtype=A.PKV_BF16, k_scale=None, v_scale=None)
    d.update(kw)
    return A._Cache(**d)


@pytest.mark.parametrize("bad,code", [
    (dict(block_size=24), 1), (dict(block_size=1), 1), (dict(head_dim=96), 2), (dict(layer=1), 1),
    (dict(kv_dtype=7), 1),
])
def test_kv_append_rejects(api, bad, code):
    c = _cache(**bad)
    st = api._lib.pkv_kv_append(C.byref(c), 0x1000, 0x1000, c.kv_dtype, 0x1000, 0x1000, 0x1000, 4, 1, 1, None, None)
    assert st == code, api._lib.pkv_last_error()


def test_kv_append_dtype_rules(api):
    c = _cache()
    assert api._lib.pkv_kv_append(C.byref(c), 0x1000, 0x1000, api.PKV_F32, 0x1000, 0x1000, 0x1000, 4, 1, 1, None,
                                  None) == 1
    c8 = _cache(kv_dtype=api.PKV_FP8_E4M3)
    assert api._lib.pkv_kv_append(C.byref(c8), 0x1000, 0x1000, api.PKV_F32, 0x1000, 0x1000, 0x1000, 4, 1, 1, None,
                                  None) == 1  # no scales
    # NVFP4: head_dim 128 only, scales required, float inputs only.
    c4 = _cache(kv_dtype=api.PKV_NVFP4, head_dim=64, k_scale=0x1000, v_scale=0x1000)
    assert api._lib.pkv_kv_append(C.byref(c4), 0x1000, 0x1000, api.PKV_F32, 0x1000, 0x1000, 0x1000, 4, 1, 1, None,
                                  None) == 2
    c4 = _cache(kv_dtype=api.PKV_NVFP4, head_dim=128)
    assert api._lib.pkv_kv_append(C.byref(c4), 0x1000, 0x1000, api.PKV_F32, 0x1000, 0x1000, 0x1000, 4, 1, 1, None,
                                  None) == 1  # no scales
    c4 = _cache(kv_dtype=api.PKV_NVFP4, head_dim=128, k_scale=0x1000, v_scale=0x1000)
    assert api._lib.pkv_kv_append(C.byref(c4), 0x1000, 0x1000, api.PKV_NVFP4, 0x1000, 0x1000, 0x1000, 4, 1, 1, None,
                                  None) == 1  # codes are not an input dtype
    # Nothing to do is fine and touches no device.
    assert api._lib.pkv_kv_append(C.byref(c), 0, 0, api.PKV_BF16, 0, 0, 0, 4, 0, 0, None, None) == 0


def test_split_reduce_rejects(api):
    assert api._lib.pkv_split_kv_reduce(0x1000, 0x1000, 2, 4, 64, 0x1000, 3, None, None) == 1  # fp8 output
    assert api._lib.pkv_split_kv_reduce(0x1000, 0x1000, -1, 4, 64, 0x1000, 0, None, None) == 1
    assert api._lib.pkv_split_kv_reduce(None, None, 2, 0, 64, None, 0, None, None) == 0


def _plan(api, w, **kw):
    kw.setdefault("num_ctas", 296)
    return api.plan_attention(w.cu_q_lens, w.seq_lens, num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                              head_dim=w.head_dim, block_size=w.block_size, kv_dtype=w.kv_dtype, causal=w.causal,
                              block_tables=w.block_tables, pin=False, **kw)


def test_plan_rejects(api):
    w = W.llama3_8b_decode_bf16(batch=3, lo=10, hi=50)
    with pytest.raises(api.PkvError):
        api.plan_attention(w.cu_q_lens, w.seq_lens, num_q_heads=30, num_kv_heads=8, head_dim=128, block_size=64,
                           kv_dtype="bf16", num_ctas=10, pin=False)
    bad = w.seq_lens.copy()
    bad[1] = 0  # q_len 1 > seq_len 0
    with pytest.raises(api.PkvError):
        api.plan_attention(w.cu_q_lens, bad, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=64,
                           kv_dtype="bf16", num_ctas=10, pin=False)
    with pytest.raises(api.PkvError):  # table row too short for the length
        api.plan_attention(w.cu_q_lens, w.seq_lens * 100, num_q_heads=32, num_kv_heads=8, head_dim=128,
                           block_size=64, kv_dtype="bf16", num_ctas=10, max_blocks=1, pin=False)


CASES = [
    ("decode", lambda: W.llama3_8b_decode_bf16(batch=40, lo=1, hi=5000), {}),
    ("decode_nosplit", lambda: W.llama3_8b_decode_bf16(batch=9, lo=1, hi=900), {"kv_split": -1}),
    ("decode_split64", lambda: W.llama3_8b_decode_bf16(batch=9, lo=1, hi=900), {"kv_split": 64}),
    ("mixed", lambda: W.mixed_bf16(n_decode=30, n_prefill=3, chunk=300, block_size=16, cached_lo_blocks=1,
                                    cached_hi_blocks=40, aligned=False), {}),
    ("mixed_split", lambda: W.mixed_bf16(n_decode=5, n_prefill=2, chunk=77), {"kv_split": 128}),
    ("fp8_long", lambda: W.longctx_fp8(batch=2, seq_len=20000), {"num_ctas": 50}),
    ("prefix", lambda: W.prefix_reuse_bf16(n_req=37, prefix=512, suf_lo=1, suf_hi=300), {}),
    ("prefix_split", lambda: W.prefix_reuse_bf16(n_req=11, prefix=256, suf_lo=1, suf_hi=30), {"kv_split": 64}),
    ("prefix_off", lambda: W.prefix_reuse_bf16(n_req=11, prefix=256), {"cascade": False}),
    ("tiny", lambda: W.tiny_fp32(), {}),
    ("two_prefixes", lambda: W.build("two", seed=24, kv_dtype="bf16", num_q_heads=64, num_kv_heads=8, head_dim=128,
                                     block_size=16, seq_lens=300 + np.arange(37) * 7, q_lens=[1] * 37,
                                     shared_prefix_tokens=256, prefix_groups=2), {}),
    ("two_prefixes_fp8", lambda: W.build("two8", seed=25, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32",
                                         num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                                         seq_lens=[300] * 9, q_lens=[1] * 9, shared_prefix_tokens=256,
                                         prefix_groups=2), {}),
]


@pytest.mark.parametrize("name,make,opts", CASES, ids=[c[0] for c in CASES])
def test_plan_covers_every_key_once(api, name, make, opts):
    w = make()
    p = _plan(api, w, **opts)
    d = PD.decode(p.buffer)
    assert d["header"]["n_items"] + d["header"]["n_tc_items"] == p.info["num_items"]
    PD.check_coverage(d, w.cu_q_lens, w.seq_lens, w.num_q_heads, w.num_kv_heads, w.causal, w.block_tables,
                      w.block_size)
    if name == "prefix":
        assert p.info["num_groups"] >= 1
    if name == "prefix_off":
        assert p.info["num_groups"] == 0


def test_plan_routes_prefill_tiles_to_tensor_memory_list(api):
    """16-bit pools and fp8 pools of head_dim 128: tiles of more than 16 rows go to the tcgen05
    list in 128-row tiles; fp8 pools of head_dim 64 keep 64-row tiles in the register-tile list."""
    w = W.mixed_bf16(n_decode=6, n_prefill=2, chunk=300, block_size=16, cached_lo_blocks=1, cached_hi_blocks=20)
    d = PD.decode(_plan(api, w).buffer)
    g = w.num_q_heads // w.num_kv_heads
    tc, reg = d["tc_items"], d["reg_items"]
    assert len(tc) > 0 and (tc["n_q"] * g > 16).all() and (tc["n_q"] * g).max() == 128
    assert (reg["n_q"] * g <= 16).all()
    w8 = W.build("f8", seed=2, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32, num_kv_heads=8,
                 head_dim=128, block_size=16, seq_lens=[400, 50], q_lens=[200, 1])
    d8 = PD.decode(_plan(api, w8).buffer)
    assert d8["header"]["n_tc_items"] > 0 and (d8["tc_items"]["n_q"] * 4).max() == 128
    assert (d8["reg_items"]["n_q"] * 4 <= 16).all()
    w64 = W.build("f8d64", seed=2, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32,
                  num_kv_heads=8, head_dim=64, block_size=16, seq_lens=[400, 50], q_lens=[200, 1])
    d64 = PD.decode(_plan(api, w64).buffer)
    assert d64["header"]["n_tc_items"] == 0 and (d64["items"]["n_q"] * 4).max() == 64


@pytest.mark.parametrize("window", [1, 5, 64, 200, 100000])
@pytest.mark.parametrize("split", [0, 64])
def test_plan_window_ranges(api, window, split):
    """Under a limited window every row still sees all its visible keys once, and key ranges start
    no later than (and at most a 128-key tile before) the tile's first visible key."""
    w = W.mixed_bf16(n_decode=20, n_prefill=3, chunk=300, block_size=16, cached_lo_blocks=1, cached_hi_blocks=40,
                     aligned=False)
    w.window = window
    p = _plan(api, w, window=window, kv_split=split)
    d = PD.decode(p.buffer)
    assert d["header"]["window"] == window
    PD.check_coverage(d, w.cu_q_lens, w.seq_lens, w.num_q_heads, w.num_kv_heads, w.causal, w.block_tables,
                      w.block_size, window=window)
    if window < 1000:  # the planner skips keys no row of a tile can see
        base = _plan(api, w, kv_split=split)
        keys = lambda pl: int((pl["items"]["k_end"] - pl["items"]["k_begin"]).sum())  # noqa: E731
        assert keys(d) < keys(PD.decode(base.buffer))


def test_plan_nvfp4_rules(api):
    """NVFP4 pools: decode-kernel tiles of at most 8 rows, head_dim 128, blocks of 16+ slots,
    at most 8 query heads per KV head."""
    w = W.build("nv", seed=3, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32, num_kv_heads=8,
                head_dim=128, block_size=16, seq_lens=[300, 40, 9], q_lens=[37, 2, 1])
    d = PD.decode(_plan(api, w).buffer)
    g = w.num_q_heads // w.num_kv_heads
    assert d["header"]["n_tc_items"] == 0 and (d["items"]["n_q"] * g <= 8).all()
    PD.check_coverage(d, w.cu_q_lens, w.seq_lens, w.num_q_heads, w.num_kv_heads, w.causal, w.block_tables,
                      w.block_size)
    for kw in (dict(head_dim=64), dict(block_size=8), dict(num_q_heads=128)):
        args = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16, kv_dtype="nvfp4", num_ctas=10,
                    pin=False)
        args.update(kw)
        with pytest.raises(api.PkvError):
            api.plan_attention(np.array([0, 1], np.int32), np.array([5], np.int32), **args)


def test_plan_window_rejects(api):
    w = W.llama3_8b_decode_bf16(batch=3, lo=10, hi=50)
    with pytest.raises(api.PkvError):
        _plan(api, w, window=-1)
    w.causal = False
    with pytest.raises(api.PkvError):
        _plan(api, w, window=8)


def test_plan_noncausal_and_empty_rows(api):
    w = W.build("mix", seed=3, kv_dtype="bf16", num_q_heads=16, num_kv_heads=2, head_dim=64, block_size=32,
                seq_lens=[40, 7, 300, 1, 90], q_lens=[5, 0, 300, 1, 0], causal=False)
    d = PD.decode(_plan(api, w).buffer)
    PD.check_coverage(d, w.cu_q_lens, w.seq_lens, 16, 2, False)


def test_plan_empty_batch(api):
    p = api.plan_attention(np.zeros(1, np.int32), np.zeros(0, np.int32), num_q_heads=8, num_kv_heads=8,
                           head_dim=64, block_size=16, kv_dtype="f32", num_ctas=4, pin=False)
    assert p.info["num_items"] == 0


def test_plan_balances_decode(api):
    """The automatic split keeps every item within ~2x the mean share per CTA."""
    w = W.llama3_8b_decode_bf16()
    p = _plan(api, w)
    d = PD.decode(p.buffer)
    assert d["header"]["n_tc_items"] == 0  # one-token rows: every item stays in the decode list
    items = d["items"]
    keys = (items["k_end"] - items["k_begin"]).astype(np.int64)
    per_cta = keys.sum() / 296
    assert keys.max() <= max(256, 2 * per_cta / 2 + 64)
    assert p.info["num_items"] >= 296


@pytest.mark.parametrize("name,make,opts", CASES, ids=[c[0] for c in CASES])
def test_plan_orders_heaviest_first(api, name, make, opts):
    """Each list runs heaviest item first (cost = keys x max(1, rows / 16)), so the last items
    the CTAs claim are the short ones; equal costs keep creation order, which for items outside
    shared-prefix groups is (first token, first key, KV head) ascending: the planner splits each
    query tile once and gives every KV head of it the same key pieces."""
    w = make()
    p = _plan(api, w, **opts)
    d = PD.decode(p.buffer)
    g = w.num_q_heads // w.num_kv_heads
    for lst in (d["reg_items"], d["tc_items"]):
        if len(lst) == 0:
            continue
        cost = (lst["k_end"] - lst["k_begin"]).astype(np.float64) * np.maximum(1.0, lst["n_q"] * g / 16.0)
        assert (np.diff(cost) <= 0).all()
        if p.info["num_groups"] == 0:
            for i in range(1, len(lst)):
                if cost[i] == cost[i - 1]:
                    a, b = lst[i - 1], lst[i]
                    assert (a["q_begin"], a["k_begin"], a["kv_head"]) < (b["q_begin"], b["k_begin"], b["kv_head"])


def test_plan_is_deterministic_and_reuses_buffers(api):
    """The same request gives the same bytes; a large enough buffer is planned into in place, a
    too small one is replaced by a fresh buffer holding the same plan."""
    w = W.mixed_bf16(n_decode=12, n_prefill=2, chunk=100, block_size=16, cached_lo_blocks=1, cached_hi_blocks=9)
    a = _plan(api, w)
    b = _plan(api, w)
    n = a.info["plan_bytes"]
    assert torch.equal(a.buffer[:n], b.buffer[:n])
    big = torch.zeros(n + 4096, dtype=torch.uint8)
    c = _plan(api, w, buffer=big)
    assert c.buffer is big and torch.equal(big[:n], a.buffer[:n]) and c.info == a.info
    small = torch.zeros(64, dtype=torch.uint8)
    d = _plan(api, w, buffer=small)
    assert d.buffer is not small and torch.equal(d.buffer[:n], a.buffer[:n]) and not small.any()


def test_plan_avoids_a_tail_round(api):
    """Eight equal 131072-key sequences on 296 CTAs: about two items per CTA would be 640 pieces
    of 13120 keys, leaving 48 CTAs a third round; the planner takes 9 pieces per (sequence, KV
    head) instead (576 items, no CTA beyond two rounds).  Batches of unequal lengths keep the
    two-items-per-CTA split."""
    w = W.longctx_fp8()
    d = PD.decode(_plan(api, w).buffer)
    items = d["items"]
    assert len(items) <= 2 * 296 and len(items) == 8 * 8 * 9
    assert set((items["k_end"] - items["k_begin"]).tolist()) == {14592, 131072 - 8 * 14592}
    PD.check_coverage(d, w.cu_q_lens, w.seq_lens, w.num_q_heads, w.num_kv_heads, w.causal, w.block_tables,
                      w.block_size)
    explicit = PD.decode(_plan(api, w, kv_split=14592).buffer)
    assert np.array_equal(explicit["items"], items)
    dec = W.llama3_8b_decode_bf16()
    two_per_cta = -(-int(dec.seq_lens.sum()) * dec.num_kv_heads // (2 * 296))  # keys, one-row-group weight 1
    auto, fixed = _plan(api, dec), _plan(api, dec, kv_split=-(-two_per_cta // 64) * 64)
    assert torch.equal(auto.buffer[:auto.info["plan_bytes"]], fixed.buffer[:fixed.info["plan_bytes"]])


def test_plan_carries_wait_limit_and_debug_flags(api):
    """The plan header carries the per-launch wait limit and the test switch to the kernels;
    negative limits and unknown flags are refused."""
    w = W.llama3_8b_decode_bf16(batch=3, lo=10, hi=500)
    d = PD.decode(_plan(api, w).buffer)
    assert d["header"]["wait_limit_kcycles"] == 0 and d["header"]["debug_flags"] == 0
    d = PD.decode(_plan(api, w, wait_limit_kcycles=200, debug_flags=api.PKV_DEBUG_WITHHOLD_LOADS).buffer)
    assert d["header"]["wait_limit_kcycles"] == 200 and d["header"]["debug_flags"] == api.PKV_DEBUG_WITHHOLD_LOADS
    with pytest.raises(api.PkvError):
        _plan(api, w, wait_limit_kcycles=-1)
    with pytest.raises(api.PkvError):
        _plan(api, w, debug_flags=0x2)


def test_plan_side_by_side(api):
    """tc_num_ctas > 0: a batch with both kinds of tile is planned side by side (header flag, the
    two CTA counts as given, every row covered once); a decode-only batch, tc_num_ctas < 0, or an
    explicit num_ctas alone is not; tc_num_ctas > 0 without num_ctas is refused."""
    w = W.mixed_bf16(n_decode=30, n_prefill=2, chunk=300, block_size=16, cached_lo_blocks=1, cached_hi_blocks=20)
    d = PD.decode(_plan(api, w, num_ctas=200, tc_num_ctas=48).buffer)
    h = d["header"]
    assert h["flags"] & PD.PLAN_CORUN and h["num_ctas"] == 200 and h["tc_num_ctas"] == 48
    PD.check_coverage(d, w.cu_q_lens, w.seq_lens, w.num_q_heads, w.num_kv_heads, w.causal, w.block_tables,
                      w.block_size)
    assert not PD.decode(_plan(api, w, num_ctas=200, tc_num_ctas=-1).buffer)["header"]["flags"] & PD.PLAN_CORUN
    assert not PD.decode(_plan(api, w, num_ctas=200).buffer)["header"]["flags"] & PD.PLAN_CORUN
    wd = W.llama3_8b_decode_bf16(batch=9, lo=10, hi=900)
    assert not PD.decode(_plan(api, wd, num_ctas=200, tc_num_ctas=48).buffer)["header"]["flags"] & PD.PLAN_CORUN
    with pytest.raises(api.PkvError):
        _plan(api, w, num_ctas=0, tc_num_ctas=48)


def test_plan_groups_sharers_that_are_not_neighbours(api):
    """Two prefixes alternating through the batch (sequence s shares the blocks of prefix s mod 2):
    on a 16-bit pool both prefixes form a group, whose tensor-memory tiles list their query tokens
    (a group tile of 16 or fewer rows would have to run on the decode tiles, so the members of such
    a tile read their prefix themselves); an fp8 pool of head_dim 64 (register tiles only) groups
    only runs of consecutive sharers, so it finds none here."""
    w = W.build("two", seed=24, kv_dtype="bf16", num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=16,
                seq_lens=300 + np.arange(37) * 7, q_lens=[1] * 37, shared_prefix_tokens=256, prefix_groups=2)
    p = _plan(api, w)
    d = PD.decode(p.buffer)
    assert p.info["num_groups"] == 2
    listed = d["tc_items"][d["tc_items"]["pos0"] <= -2]
    # 19 and 18 members of one token: a 16-token tile of 128 rows each, the remaining 3 and 2
    # members (24 and 16 rows) -- the 16-row tile is dropped.
    assert len(listed) == 3 * w.num_kv_heads
    for it in listed[::w.num_kv_heads]:
        tok = PD.item_tokens(d, it)
        assert (np.diff(tok) == 2).all() and len(set(tok % 2)) == 1
    w8 = W.build("two8", seed=25, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32,
                 num_kv_heads=8, head_dim=64, block_size=16, seq_lens=[300] * 9, q_lens=[1] * 9,
                 shared_prefix_tokens=256, prefix_groups=2)
    assert _plan(api, w8).info["num_groups"] == 0


H4_OK = [c for c in CASES if c[0] not in ("tiny",)]


@pytest.mark.parametrize("name,make,opts", H4_OK, ids=[c[0] for c in H4_OK])
def test_plan_four_head_items_cover_every_key_once(api, name, make, opts):
    """heads_per_item = 4: every decode-tile item covers KV heads 4j .. 4j + 3 of one query tile and
    key range, at most 8 rows a head, its heads' partial rows consecutive; expanded per head, the
    plan still covers every (token, KV head) key range once.  The tcgen05 list keeps one head an
    item, and the item count is the tensor-memory items plus a quarter of the one-head decode items
    for the same split."""
    w = make()
    if w.kv_dtype == "e4m3" and w.head_dim != 128:
        pytest.skip("fp8 pools of head_dim 64 run on the cp.async kernel")
    g = w.num_q_heads // w.num_kv_heads
    if any(q * g > PD.HEADS4_ROWS and q * g <= PD.DECODE_ROWS for q in np.diff(w.cu_q_lens)):
        with pytest.raises(api.PkvError):
            _plan(api, w, heads_per_item=4, **opts)
        return
    p = _plan(api, w, heads_per_item=4, **opts)
    d = PD.decode(p.buffer)
    h = d["header"]
    assert p.info["heads_per_item"] == 4 and h["flags"] & PD.PLAN_HEADS4
    reg = d["reg_items"]
    assert (reg["kv_head"] % 4 == 0).all() and (reg["n_q"] * g <= PD.HEADS4_ROWS).all()
    assert (d["tc_items"]["n_q"] * g > PD.DECODE_ROWS).all()
    PD.check_coverage(d, w.cu_q_lens, w.seq_lens, w.num_q_heads, w.num_kv_heads, w.causal, w.block_tables,
                      w.block_size)
    one = _plan(api, w, heads_per_item=1, **opts)
    if opts.get("kv_split", 0) != 0:  # the same pieces: a quarter of the decode items
        d1 = PD.decode(one.buffer)
        assert len(reg) * 4 == len(d1["reg_items"]) and len(d["tc_items"]) == len(d1["tc_items"])
    assert one.info["heads_per_item"] == 1 and not PD.decode(one.buffer)["header"]["flags"] & PD.PLAN_HEADS4


def test_plan_four_head_group_items_on_nvfp4(api):
    """On an NVFP4 pool a run of sharers reads its prefix as decode-tile group items; with four heads
    an item, head hh of a group item still writes member m's rows at part0 + hh * rows + offset, where
    the members' merges look for them."""
    w = W.build("nvp", seed=49, kv_dtype="nvfp4", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32, num_kv_heads=8,
                head_dim=128, block_size=16, seq_lens=300 + np.arange(9) * 13, q_lens=[1] * 9,
                shared_prefix_tokens=256)
    for heads in (1, 4):
        p = _plan(api, w, heads_per_item=heads, num_ctas=40)
        assert p.info["num_groups"] == 1 and p.info["heads_per_item"] == heads
        PD.check_coverage(PD.decode(p.buffer), w.cu_q_lens, w.seq_lens, w.num_q_heads, w.num_kv_heads, w.causal,
                          w.block_tables, w.block_size)


def test_plan_four_head_choice_and_rules(api):
    """Automatic: four-head items for short decode ranges (the shared-prefix batch's suffixes) and
    on NVFP4 pools, one head for long ranges on the others (the 8B decode batch, the long-context
    batch).  Refused: other values,
    KV heads not a multiple of 4, pools without the TMA-fed decode kernel, decode tiles of more
    than 8 rows."""
    assert _plan(api, W.prefix_reuse_bf16()).info["heads_per_item"] == 4
    assert _plan(api, W.llama3_8b_decode_bf16()).info["heads_per_item"] == 1
    assert _plan(api, W.longctx_fp8()).info["heads_per_item"] == 1
    assert _plan(api, W.llama3_8b_decode_nvfp4()).info["heads_per_item"] == 4
    w = W.llama3_8b_decode_bf16(batch=9, lo=10, hi=900)
    for bad in (2, 3, 8, -1):
        with pytest.raises(api.PkvError):
            _plan(api, w, heads_per_item=bad)
    cases = [
        W.build("h6", seed=3, kv_dtype="bf16", num_q_heads=12, num_kv_heads=6, head_dim=128, block_size=16,
                seq_lens=[40, 70], q_lens=[1, 1]),                           # 6 KV heads
        W.build("b4", seed=3, kv_dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=4,
                seq_lens=[40, 70], q_lens=[1, 1]),                           # cp.async kernel
        W.build("f8", seed=3, kv_dtype="e4m3", q_dtype="bf16", kv_in_dtype="f32", num_q_heads=32, num_kv_heads=8,
                head_dim=64, block_size=16, seq_lens=[40, 70], q_lens=[1, 1]),  # 64-byte fp8 rows
        W.build("f32", seed=3, kv_dtype="f32", num_q_heads=8, num_kv_heads=4, head_dim=64, block_size=16,
                seq_lens=[40, 70], q_lens=[1, 1]),                           # fp32 kernel
        W.build("r12", seed=3, kv_dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                seq_lens=[40, 70], q_lens=[3, 1]),                           # a 12-row decode tile
    ]
    for bad in cases:
        with pytest.raises(api.PkvError):
            _plan(api, bad, heads_per_item=4)
        assert _plan(api, bad).info["heads_per_item"] == 1


def test_plan_tail_check_stays_cheap(api):
    """The tail check's schedule simulation is O(items log CTAs): the shared-prefix batch on 168
    decode CTAs (512 four-head items of 256 distinct lengths, just past three rounds, where no longer
    piece length changes the item count) plans in well under a millisecond (about 70 us on a
    desktop core; 580 us with a per-distinct-cost merge of all CTA loads)."""
    import time
    w = W.prefix_reuse_bf16()
    pl = api.Planner(w.cu_q_lens, w.seq_lens, w.block_tables, num_q_heads=w.num_q_heads,
                     num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, block_size=w.block_size, kv_dtype=w.kv_dtype,
                     causal=w.causal, num_ctas=168)
    p = pl.plan()
    assert p.info["heads_per_item"] == 4 and p.info["num_items"] == 640
    t0 = time.perf_counter()
    for _ in range(50):
        pl.plan()
    assert (time.perf_counter() - t0) / 50 < 1e-3


def _attention_status(api, w, plan_buf):
    """pkv_paged_attention's synchronous status for a (possibly edited) host plan, with placeholder
    device pointers: plan validation comes before any CUDA call."""
    c = _cache(num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, block_size=w.block_size,
               kv_dtype=api.DTYPE_CODES[w.kv_dtype], num_blocks=w.num_blocks)
    fake = 0x10000
    return api._lib.pkv_paged_attention(C.byref(c), fake, api.PKV_BF16, w.num_q_heads, fake, fake, fake,
                                        w.block_tables.shape[1], w.num_seqs, 0.1, int(w.causal),
                                        plan_buf.data_ptr(), fake, None, fake, 1 << 30, None, None)


def test_paged_attention_refuses_broken_four_head_plans(api):
    """A four-head plan is checked before anything is enqueued: a decode item whose first KV head is not a
    multiple of 4 or that carries more than 8 rows a head, and the four-head flag on a pool whose
    decode tiles run on a kernel without four-head items, return PKV_ERR_PLAN (5)."""
    w = W.llama3_8b_decode_bf16(batch=9, lo=10, hi=900)
    good = _plan(api, w, heads_per_item=4, num_ctas=40)
    base = good.buffer.clone()
    h = PD.decode(base)["header"]
    off = int(h["items_off"])
    for field, value in (("kv_head", 1), ("n_q", 3)):  # kv_head 1; 3 tokens x 4 heads = 12 rows
        bad = base.clone()
        items = np.frombuffer(bad.numpy(), dtype=PD.ITEM, count=int(h["n_items"]), offset=off).copy()
        items[0][field] = value
        bad[off:off + items.nbytes] = torch.from_numpy(items.view(np.uint8))
        assert _attention_status(api, w, bad) == 5, (field, api._lib.pkv_last_error())
    w4 = W.build("b4", seed=3, kv_dtype="bf16", num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=4,
                 seq_lens=[40, 70], q_lens=[1, 1])
    p4 = _plan(api, w4, num_ctas=40)
    assert p4.info["heads_per_item"] == 1
    flagged = p4.buffer.clone()
    hdr = np.frombuffer(flagged.numpy()[:128].tobytes(), PD.HEADER).copy()
    hdr["flags"] |= PD.PLAN_HEADS4
    flagged[:128] = torch.from_numpy(hdr.view(np.uint8).copy())
    assert _attention_status(api, w4, flagged) == 5
    assert b"four-head" in api._lib.pkv_last_error()
