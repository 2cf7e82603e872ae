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
    """A plan whose scratch exceeds the built-in array is refused before any launch.  Every
    argument is a real device buffer of the right shape, so a regression that let the call
    through would show as a wrong status or output, not as a stray memory access."""
    api, runner = pkv
    w = W.llama3_8b_decode_bf16(batch=64, lo=4096, hi=4096)
    dw = runner.DeviceWorkload(w, history=False)
    plan = dw.plan(num_ctas=296, kv_split=64)
    assert plan.workspace_bytes > 32 << 20
    out = torch.full_like(dw.q, float("nan"))
    with pytest.raises(api.PkvError) as e:
        api.paged_attention_noalloc(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, plan, w.softmax_scale,
                                    w.causal, out=out, status=dw.status)
    assert e.value.status == 4 and "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert int(dw.status.item()) == 0 and torch.isnan(out.float()).all()  # nothing ran
