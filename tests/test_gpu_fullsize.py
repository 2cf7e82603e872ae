"""Full-size workloads, in the launch configuration the benchmark times (needs a B200).

The GPU runs the whole batch; the oracle recomputes sampled sequences (every
query row and head of each), and kv_append is checked byte for byte on every
block those sequences own.
"""
import numpy as np
import pytest
import torch

from gpu_common import assert_close, gpu_out_f64, oracle_out, oracle_pool, oracle_pool_bytes
from paged_kv_attention_block_b200 import workloads as W

pytestmark = pytest.mark.gpu

SAMPLES = {
    "tiny_fp32": [0, 1, 2, 3],
    "llama3_8b_decode_bf16": [0, 17, 63],
    "mixed_bf16": [0, 3, 4, 123],
    "longctx_fp8": [5],
    "prefix_reuse_bf16": [0, 128, 255],
    "llama3_8b_decode_nvfp4": [0, 17, 63],
    "mixed_fp8": [0, 3, 4, 123],
}


@pytest.mark.parametrize("name", list(W.NAMED))
def test_fullsize_sampled(name):
    assert torch.cuda.is_available()
    from paged_kv_attention_block_b200 import build
    build.build()
    from paged_kv_attention_block_b200 import runner

    w = W.NAMED[name]()
    dw = runner.DeviceWorkload(w)
    dw.append_new()
    plan = dw.plan()
    out = dw.attention(plan)
    torch.cuda.synchronize()
    assert int(dw.status.item()) == 0
    seqs = SAMPLES[name]
    pool = oracle_pool(w, seqs)
    ref, _ = oracle_out(w, pool, seqs=seqs)
    rows = np.concatenate([np.arange(w.cu_q_lens[s], w.cu_q_lens[s + 1]) for s in seqs])
    assert_close(gpu_out_f64(out), ref, w.kv_dtype, rows=rows)
    # Pool bytes of the sampled sequences' blocks.
    got = dw.cache.pool
    for s in seqs:
        nb = (int(w.seq_lens[s]) + w.block_size - 1) // w.block_size
        ids = torch.from_numpy(w.block_tables[s, :nb].astype(np.int64)).cuda()
        g = got.index_select(0, ids)
        g = (g.view(torch.int16) if g.dtype in (torch.bfloat16, torch.float16) else g).cpu().numpy()
        want = oracle_pool_bytes(pool)[w.block_tables[s, :nb]]
        if w.kv_dtype == "f32":
            assert (g.view(np.uint32) == want.view(np.uint32)).all()
        else:
            assert (g.view(want.dtype) == want).all()
    w.release()
