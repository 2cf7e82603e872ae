"""Shared pieces of the GPU parity tests: oracle runs and the comparison rule."""
from __future__ import annotations

import numpy as np
import torch

import oracle.pkv_oracle as O
from paged_kv_attention_block_b200 import workloads as W

# Tolerances on the attention output (relative to the output magnitude for
# 16-bit and fp8 pools, absolute for float32 pools).
# NVFP4 values are exact in f16 (an E2M1 value times an E4M3 scale), so after the shared stored
# codes its arithmetic is the fp8 path's: f16 operands rounded once (q, P), float32 sums.
TOL = {"f32": 1e-5, "bf16": 2e-2, "f16": 2e-2, "e4m3": 6e-2, "nvfp4": 2e-2}


def oracle_pool(w: W.Workload, seqs=None) -> O.OraclePool:
    pool = O.new_pool(w.num_blocks, w.num_layers, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype,
                      w.k_scale, w.v_scale)
    for which in ("history", "new"):
        k, v, cu, sp = w.packed_kv(which, seqs)
        rows = w.block_tables if seqs is None else w.block_tables[list(seqs)]
        O.kv_append(pool, w.layer, k, v, w.kv_in_dtype, cu, sp, rows)
    return pool


def oracle_pool_bytes(pool: O.OraclePool) -> np.ndarray:
    """The oracle pool as the device holds it (NVFP4: the packed byte image)."""
    return O.nvfp4_pool_bytes(pool) if pool.dtype == "nvfp4" else pool.bits


def oracle_out(w: W.Workload, pool: O.OraclePool, seqs=None):
    q = O.decode_bits(w.q, w.q_dtype) if w.q_dtype != "f32" else w.q.astype(np.float64)
    return O.paged_attention(pool, w.layer, q, w.cu_q_lens, w.seq_lens, w.block_tables, w.num_q_heads,
                             w.softmax_scale, w.causal, seqs=seqs, window=w.window)


def gpu_out_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, kv_dtype: str, rows=None, what="out"):
    """got/ref: [T][Hq][D]; rows: token indices to compare (default: all finite ref rows)."""
    if rows is not None:
        got, ref = got[rows], ref[rows]
    assert np.isfinite(got).all(), f"{what}: non-finite values in the GPU output"
    tol = TOL[kv_dtype]
    if kv_dtype == "f32":
        err = np.abs(got - ref).max()
        assert err <= tol, f"{what}: max abs err {err:.3g} > {tol}"
        return err
    mag = np.abs(ref).max(axis=-1)
    floor = 1e-3 * np.abs(ref).max()
    denom = np.maximum(mag, floor)
    err = (np.abs(got - ref).max(axis=-1) / denom).max()
    assert err <= tol, f"{what}: max row-relative err {err:.3g} > {tol}"
    return err
