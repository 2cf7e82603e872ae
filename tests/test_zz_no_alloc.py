"""pkv_paged_attention_noalloc against pkv_paged_attention (needs a B200).

The no-allocation entry point serves callers that are given only their input
and output buffers and may not allocate device memory (plug-ins inside a host
framework, allocator-free runtimes, fixed memory budgets).  It keeps its
scratch in an array built into the library, so two calls in a row must both
match the workspace-based entry point; a plan that needs more scratch than the
array holds must be refused before anything is launched.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from gpu_common import assert_close, gpu_out_f64
from paged_kv_attention_block_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_attention_block_b200 import build
    build.build()
    from paged_kv_attention_block_b200 import api, runner
    return api, runner


CASES = [
    ("decode_split", lambda: W.llama3_8b_decode_bf16(batch=9, lo=200, hi=3000), {"kv_split": 256, "num_ctas": 64}),
    ("mixed", lambda: W.mixed_bf16(n_decode=7, n_prefill=2, chunk=120, dec_lo=50, dec_hi=2000, cached_lo_blocks=1,
                                   cached_hi_blocks=5), {"num_ctas": 64}),
    ("fp8_split", lambda: W.longctx_fp8(batch=2, seq_len=5000), {"kv_split": 512}),
]


@pytest.mark.parametrize("name,make,opts", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry(pkv, name, make, opts):
    api, runner = pkv
    w = make()
    dw = runner.DeviceWorkload(w)
    dw.append_new()
    plan = dw.plan(**opts)
    ref_lse = torch.empty(w.total_q, w.num_q_heads, device="cuda")
    ref = dw.attention(plan, out_lse=ref_lse).clone()
    torch.cuda.synchronize()
    ref64 = gpu_out_f64(ref)
    for call in range(2):  # the built-in scratch keeps the previous call's contents
        out = torch.full_like(dw.q, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        api.paged_attention_noalloc(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, plan, w.softmax_scale,
                                    w.causal, out=out, out_lse=lse, status=dw.status)
        torch.cuda.synchronize()
        assert int(dw.status.item()) == 0
        assert_close(gpu_out_f64(out), ref64, w.kv_dtype, what=f"{name} call {call}")
        assert torch.allclose(lse, ref_lse, atol=1e-5, rtol=0), f"{name} call {call}: lse differs"


def test_noalloc_refuses_oversized_plan(pkv):
    api, _ = pkv
    S = 64
    cu = np.arange(S + 1, dtype=np.int32)
    lens = np.full(S, 4096, np.int32)
    plan = api.plan_attention(cu, lens, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=64,
                              kv_dtype="bf16", max_blocks=64, num_ctas=296, kv_split=64, pin=False)
    assert plan.workspace_bytes > 32 << 20
    cache = api.Cache.allocate(4, 1, 8, 64, 128, "bf16", device="cuda")
    c = cache._c()
    st = api._lib.pkv_paged_attention_noalloc(C.byref(c), 0x1000, api.PKV_BF16, 32, 0x1000, 0x1000, 0x1000, 64, S,
                                              0.1, 1, plan.buffer.data_ptr(), 0x1000, None, None, None)
    assert st == 4, api._lib.pkv_last_error()
    assert b"scratch" in api._lib.pkv_last_error()
