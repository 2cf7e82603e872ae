"""Stage a synthetic workload on the GPU and run steps through the binding.

A step is what an in-flight-batching runtime does per layer and iteration:
append this step's K/V (kv_append), plan the launch (host), and run
paged_attention (which merges split key ranges itself).  The history a step
attends over is appended once, up front, through the same kv_append kernel.
"""
from __future__ import annotations

import numpy as np
import torch

from . import api
from .workloads import Workload

_TORCH = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def to_device(x: np.ndarray, dtype: str, device) -> torch.Tensor:
    """Storage array from the generator (float32 or uint16 bits) -> device tensor of that dtype."""
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(device)
    t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device)
    return t.view(_TORCH[dtype])


class DeviceWorkload:
    def __init__(self, w: Workload, device="cuda", history: bool = True, seq_chunk_tokens: int = 1 << 21,
                 fill_byte: int | None = None):
        self.w = w
        self.device = torch.device(device)
        self.cache = api.Cache.allocate(w.num_blocks, w.num_layers, w.num_kv_heads, w.block_size, w.head_dim,
                                        w.kv_dtype, device=self.device, k_scale=w.k_scale, v_scale=w.v_scale,
                                        fill_byte=fill_byte)
        self.cache.layer = w.layer
        self.block_tables = torch.from_numpy(w.block_tables).to(self.device)
        self.seq_lens = torch.from_numpy(w.seq_lens).to(self.device)
        self.cu_q = torch.from_numpy(w.cu_q_lens).to(self.device)
        self.start_pos = torch.from_numpy(w.start_pos).to(self.device)
        self.q = to_device(w.q, w.q_dtype, self.device)
        k, v, _, _ = w.packed_kv("new")
        self.k_new = to_device(k, w.kv_in_dtype, self.device)
        self.v_new = to_device(v, w.kv_in_dtype, self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        # Pinned plan buffers reused round-robin; an event per slot marks when its upload was enqueued.
        self._plan_bufs = [None] * 4
        self._plan_events = [None] * 4
        self._plan_slot = 0
        if history:
            self.append_history(seq_chunk_tokens)

    def append_history(self, chunk_tokens: int = 1 << 21) -> None:
        """Append every sequence's cached tokens, a few sequences per call."""
        w = self.w
        s = 0
        while s < w.num_seqs:
            e, tok = s, 0
            while e < w.num_seqs and (e == s or tok + int(w.seq_lens[e] - w.q_lens[e]) <= chunk_tokens):
                tok += int(w.seq_lens[e] - w.q_lens[e])
                e += 1
            k, v, cu, sp = w.packed_kv("history", range(s, e))
            if len(k):
                bt = self.block_tables[s:e].contiguous()
                api.kv_append(self.cache, to_device(k, w.kv_in_dtype, self.device),
                              to_device(v, w.kv_in_dtype, self.device), torch.from_numpy(cu).to(self.device),
                              torch.from_numpy(sp).to(self.device), bt, status=self.status)
            s = e
        torch.cuda.synchronize(self.device)

    def append_new(self, stream=None) -> None:
        api.kv_append(self.cache, self.k_new, self.v_new, self.cu_q, self.start_pos, self.block_tables,
                      status=self.status, stream=stream)

    def plan(self, **opts) -> api.Plan:
        w = self.w
        i = self._plan_slot
        if self._plan_events[i] is not None:
            self._plan_events[i].synchronize()  # that buffer's upload has run
        p = api.plan_attention(w.cu_q_lens, w.seq_lens, num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                               head_dim=w.head_dim, block_size=w.block_size, kv_dtype=w.kv_dtype, causal=w.causal,
                               block_tables=w.block_tables, buffer=self._plan_bufs[i],
                               **({"window": w.window} if w.window else {}), **opts)
        self._plan_bufs[i] = p.buffer
        p.slot = i
        self._plan_slot = (i + 1) % len(self._plan_bufs)
        return p

    def attention(self, plan: api.Plan, out=None, out_lse=None, workspace=None, stream=None):
        w = self.w
        out = api.paged_attention(self.cache, self.q, self.cu_q, self.seq_lens, self.block_tables, plan,
                                  w.softmax_scale, w.causal, out=out, out_lse=out_lse, workspace=workspace,
                                  status=self.status, stream=stream)
        slot = getattr(plan, "slot", None)
        if slot is not None:
            ev = torch.cuda.Event()
            ev.record(torch.cuda.current_stream(self.device) if stream is None else stream)
            self._plan_events[slot] = ev
        return out

    def pool_bytes(self) -> np.ndarray:
        p = self.cache.pool
        if p.dtype in (torch.bfloat16, torch.float16):
            return p.view(torch.int16).cpu().numpy().view(np.uint16)
        return p.cpu().numpy()
