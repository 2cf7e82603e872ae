"""Decode a plan buffer (host bytes) into numpy records, for tests."""
import numpy as np

HEADER = np.dtype([("magic", "<u4"), ("bytes", "<u4"), ("n_items", "<i4"), ("n_reduce", "<i4"), ("n_parts", "<i4"),
                   ("n_part_rows", "<i4"), ("num_seqs", "<i4"), ("total_q", "<i4"), ("num_q_heads", "<i4"),
                   ("num_kv_heads", "<i4"), ("head_dim", "<i4"), ("block_size", "<i4"), ("kv_dtype", "<i4"),
                   ("causal", "<i4"), ("num_ctas", "<i4"), ("n_groups", "<i4"), ("items_off", "<u4"),
                   ("reduce_off", "<u4"), ("parts_off", "<u4"), ("n_tc_items", "<i4"), ("tc_items_off", "<u4"),
                   ("tc_num_ctas", "<i4"), ("window", "<i4"), ("wait_limit_kcycles", "<i4"), ("debug_flags", "<i4"),
                   ("flags", "<i4"), ("rows_off", "<u4"), ("n_rows", "<i4"), ("pad", "<i4", 4)])
ITEM = np.dtype([("seq", "<i4"), ("kv_head", "<i4"), ("q_begin", "<i4"), ("n_q", "<i4"), ("k_begin", "<i4"),
                 ("k_end", "<i4"), ("pos0", "<i4"), ("part_row", "<i4")])
REDUCE = np.dtype([("q_begin", "<i4"), ("n_q", "<i4"), ("kv_head", "<i4"), ("parts_begin", "<i4"),
                   ("n_parts", "<i4"), ("pad", "<i4", 3)])
assert HEADER.itemsize == 128 and ITEM.itemsize == 32 and REDUCE.itemsize == 32


TILE_ROWS, DECODE_ROWS, TILE_ROWS_TC, TC_TILE_KEYS = 64, 16, 128, 128
PLAN_CORUN, PLAN_HEADS4, HEADS4_ROWS = 0x1, 0x2, 8


def decode(buf) -> dict:
    """Header, both item lists (items: register-tile list then tensor-memory list), merges, parts."""
    b = np.asarray(buf.cpu().numpy() if hasattr(buf, "cpu") else buf, dtype=np.uint8)
    h = np.frombuffer(b[:128].tobytes(), HEADER)[0]
    reg = np.frombuffer(b[h["items_off"]:h["items_off"] + 32 * h["n_items"]].tobytes(), ITEM)
    tc = np.frombuffer(b[h["tc_items_off"]:h["tc_items_off"] + 32 * h["n_tc_items"]].tobytes(), ITEM)
    if h["flags"] & PLAN_HEADS4:
        reg_heads = _expand_heads4(reg, int(h["num_q_heads"]) // int(h["num_kv_heads"]))
    else:
        reg_heads = reg
    items = np.concatenate([reg_heads, tc])
    reds = np.frombuffer(b[h["reduce_off"]:h["reduce_off"] + 32 * h["n_reduce"]].tobytes(), REDUCE)
    parts = np.frombuffer(b[h["parts_off"]:h["parts_off"] + 4 * h["n_parts"]].tobytes(), "<i4")
    rows = np.frombuffer(b[h["rows_off"]:h["rows_off"] + 4 * h["n_rows"]].tobytes(), "<i4")
    return {"header": h, "items": items, "reg_items": reg, "tc_items": tc, "reduces": reds, "parts": parts,
            "rows": rows}


def _expand_heads4(reg, g: int) -> np.ndarray:
    """The decode-tile items of a four-head plan as one record per KV head: item (kv_head h, part_row p)
    stands for heads h .. h + 3, head h + w writing partial rows p + w * n_q * g."""
    assert (reg["kv_head"] % 4 == 0).all() and (reg["n_q"] * g <= HEADS4_ROWS).all()
    out = np.repeat(reg, 4)
    w = np.tile(np.arange(4, dtype=np.int32), len(reg))
    out["kv_head"] += w
    part = out["part_row"] >= 0
    out["part_row"][part] += (w * out["n_q"] * g)[part]
    return out


def item_tokens(plan: dict, it) -> np.ndarray:
    """Query tokens of an item: the run q_begin .. q_begin + n_q, or its listed tokens (pos0 <= -2)."""
    if it["pos0"] <= -2:
        off = -2 - int(it["pos0"])
        return plan["rows"][off:off + int(it["n_q"])]
    return np.arange(int(it["q_begin"]), int(it["q_begin"]) + int(it["n_q"]))


def check_coverage(plan: dict, cu_q, seq_lens, num_q_heads: int, num_kv_heads: int, causal: bool, block_tables=None,
                   block_size=None, window: int = 0):
    """Every (query token, KV head) row group sees exactly its keys once, through one output path.

    Under a window the key ranges may start below a row's first visible key (the kernels mask
    per row) but not past it."""
    h, items, reds, parts = plan["header"], plan["items"], plan["reduces"], plan["parts"]
    g = num_q_heads // num_kv_heads
    # List membership: tensor-memory items carry more than 16 and at most 128 rows and
    # start their key range on a multiple of the 128-key tile (or of the block size when
    # smaller); register-tile items carry at most 64 rows.
    for it in plan["reg_items"]:
        assert it["n_q"] * g <= TILE_ROWS
    for it in plan["tc_items"]:
        assert DECODE_ROWS < it["n_q"] * g <= TILE_ROWS_TC
        if block_size is not None:
            assert it["k_begin"] % min(block_size, TC_TILE_KEYS) == 0
    S = len(seq_lens)
    tok_seq = np.repeat(np.arange(S), np.diff(cu_q))
    # Partial rows: map part_row -> item, and check items' partial rows don't overlap.
    used = np.zeros(max(1, int(h["n_part_rows"])), np.int32)
    by_part = {}
    for it in items:
        assert 1 <= it["n_q"] and it["k_begin"] < it["k_end"]
        if it["part_row"] >= 0:
            used[it["part_row"]:it["part_row"] + it["n_q"] * g] += 1
            by_part[int(it["part_row"])] = it
    assert (used <= 1).all()
    # Expected key set per (token, kv head): [0, limit).
    seen = {}

    def add(tok, kvh, a, b, via):
        seen.setdefault((tok, kvh), []).append((a, b, via))

    def group_source(p):
        """The item whose partial rows hold row p, and p's token offset inside it."""
        for row0, it in by_part.items():
            if row0 <= p < row0 + it["n_q"] * g:
                return it, (p - row0) // g
        raise AssertionError("part row without an item")

    def check_shared_blocks(tok, src):
        if block_tables is not None and src["seq"] != tok_seq[tok]:
            # Group tile: the keys it reads must be identical blocks in both tables.
            s_own, s_src = tok_seq[tok], int(src["seq"])
            nb = (int(src["k_end"]) + block_size - 1) // block_size
            assert (block_tables[s_own, :nb] == block_tables[s_src, :nb]).all()

    # Listed items: shared-prefix group tiles of the tensor-memory list, writing partial rows.
    listed = items[items["pos0"] <= -2]
    for it in listed:
        assert it["part_row"] >= 0 and it["n_q"] * g > 16 and it["k_begin"] == 0
        tok = item_tokens(plan, it)
        assert len(tok) == it["n_q"] and int(tok[0]) == int(it["q_begin"]) and (np.diff(tok) > 0).all()
    for it in plan["reg_items"]:
        assert it["pos0"] > -2
    assert (items["part_row"] >= -1).all() and h["flags"] in (0, 1, 2, 3)
    if h["flags"] & PLAN_CORUN:  # side by side: both lists run at once
        assert len(plan["reg_items"]) > 0 and len(plan["tc_items"]) > 0
    direct = items[items["part_row"] == -1]
    for it in direct:
        for i in range(it["n_q"]):
            add(int(it["q_begin"]) + i, int(it["kv_head"]), int(it["k_begin"]), int(it["k_end"]), "direct")
    for r in reds:
        for p in parts[r["parts_begin"]:r["parts_begin"] + r["n_parts"]]:
            # The part is either an item's first row or a row inside a group item.
            src, off = group_source(p)
            assert src["kv_head"] == r["kv_head"]
            src_tok = item_tokens(plan, src)
            for i in range(r["n_q"]):
                tok = int(r["q_begin"]) + i
                assert int(src_tok[off + i]) == tok
                add(tok, int(r["kv_head"]), int(src["k_begin"]), int(src["k_end"]), "part")
            check_shared_blocks(int(r["q_begin"]), src)
    for tok in range(int(cu_q[-1])):
        s = tok_seq[tok]
        j = tok - int(cu_q[s])
        ql, L = int(cu_q[s + 1] - cu_q[s]), int(seq_lens[s])
        lim = L - ql + j + 1 if causal else L
        for kvh in range(num_kv_heads):
            ranges = sorted(seen.pop((tok, kvh)))
            vias = {v for _, _, v in ranges}
            assert len(vias) == 1, "a row is both written directly and merged"
            start = max(0, L - ql + j + 1 - window) if window > 0 else 0
            cover = ranges[0][0]
            assert cover <= start and (window > 0 or cover == 0), (tok, kvh, ranges)
            for a, b, _ in ranges:
                assert a == cover, (tok, kvh, ranges)
                cover = b
            # Ranges may extend past a causal row's own limit (the kernel masks per row)
            # but must cover it and stop at the tile's last row limit.
            assert cover >= lim and cover <= (L if not causal else L)
    assert not seen
