"""ctypes binding of libpkv.so (declared in include/pkv.h).

Every function here only converts torch tensors and Python values into the
pointers and sizes of the C ABI, calls it, and raises ``PkvError`` on a
nonzero status.  All computation happens in the library's CUDA kernels; if the
library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.environ.get("PKV_LIBRARY", os.path.join(_HERE, "libpkv.so"))


if not os.path.exists(library_path()):
    raise ImportError(
        f"{library_path()} is missing: build it with `python -m paged_kv_attention_block_b200.build` "
        "(the CUDA library is the only implementation)")

_lib = C.CDLL(library_path())

PKV_F32, PKV_BF16, PKV_F16, PKV_FP8_E4M3, PKV_NVFP4 = 0, 1, 2, 3, 4
DTYPE_CODES = {"f32": PKV_F32, "bf16": PKV_BF16, "f16": PKV_F16, "e4m3": PKV_FP8_E4M3, "nvfp4": PKV_NVFP4}
_TORCH_CODES = {torch.float32: PKV_F32, torch.bfloat16: PKV_BF16, torch.float16: PKV_F16,
                torch.float8_e4m3fn: PKV_FP8_E4M3, torch.uint8: PKV_FP8_E4M3}
_CODE_TORCH = {PKV_F32: torch.float32, PKV_BF16: torch.bfloat16, PKV_F16: torch.float16,
               PKV_FP8_E4M3: torch.uint8, PKV_NVFP4: torch.uint8}


class PkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.pkv_last_error().decode()
        super().__init__(f"{where}: {_lib.pkv_status_string(status).decode()} ({status}): {msg}")


class _Cache(C.Structure):
    _fields_ = [("pool", C.c_void_p), ("num_blocks", C.c_int64), ("num_layers", C.c_int32), ("layer", C.c_int32),
                ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("block_size", C.c_int32),
                ("kv_dtype", C.c_int32), ("k_scale", C.c_void_p), ("v_scale", C.c_void_p)]


_WORKSPACE_TOO_SMALL = 4  # PKV_ERR_WORKSPACE


class _PlanRequest(C.Structure):
    _fields_ = [("num_seqs", C.c_int32), ("num_q_heads", C.c_int32), ("num_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("block_size", C.c_int32), ("kv_dtype", C.c_int32), ("causal", C.c_int32),
                ("num_ctas", C.c_int32), ("kv_split", C.c_int32), ("cascade", C.c_int32),
                ("min_shared_tokens", C.c_int32), ("max_blocks", C.c_int32), ("cu_q_lens", C.c_void_p),
                ("seq_lens", C.c_void_p), ("block_tables", C.c_void_p), ("window", C.c_int32),
                ("wait_limit_kcycles", C.c_int32), ("debug_flags", C.c_int32), ("tc_num_ctas", C.c_int32),
                ("heads_per_item", C.c_int32)]

PKV_DEBUG_WITHHOLD_LOADS = 0x1


class _PlanInfo(C.Structure):
    _fields_ = [("plan_bytes", C.c_size_t), ("workspace_bytes", C.c_size_t), ("num_items", C.c_int32),
                ("num_reduce", C.c_int32), ("num_parts", C.c_int32), ("num_partial_rows", C.c_int32),
                ("num_groups", C.c_int32), ("num_ctas", C.c_int32), ("num_tc_items", C.c_int32),
                ("tc_num_ctas", C.c_int32), ("side_by_side", C.c_int32), ("heads_per_item", C.c_int32)]


_P, _I32, _I64, _SZ, _F = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t, C.c_float
_lib.pkv_abi_version.restype = _I32
_lib.pkv_status_string.restype = C.c_char_p
_lib.pkv_status_string.argtypes = [_I32]
_lib.pkv_last_error.restype = C.c_char_p
_lib.pkv_copy_block_prefix.restype = _I32
_lib.pkv_copy_block_prefix.argtypes = [C.POINTER(_Cache), _P, _P, _P, _I32, _P, _P]
_lib.pkv_kv_append.restype = _I32
_lib.pkv_kv_append.argtypes = [C.POINTER(_Cache), _P, _P, _I32, _P, _P, _P, _I32, _I32, _I32, _P, _P]
_lib.pkv_attention_plan.restype = _I32
_lib.pkv_attention_plan.argtypes = [C.POINTER(_PlanRequest), _P, _SZ, C.POINTER(_PlanInfo)]
_lib.pkv_default_num_ctas.restype = _I32
_lib.pkv_default_num_ctas.argtypes = [_I32, _I32, _I32, C.POINTER(_I32)]
_lib.pkv_paged_attention.restype = _I32
_lib.pkv_paged_attention.argtypes = [C.POINTER(_Cache), _P, _I32, _I32, _P, _P, _P, _I32, _I32, _F, _I32, _P, _P, _P,
                                     _P, _SZ, _P, _P]
_lib.pkv_paged_attention_timed.restype = _I32
_lib.pkv_paged_attention_timed.argtypes = [C.POINTER(_Cache), _P, _I32, _I32, _P, _P, _P, _I32, _I32, _F, _I32, _P, _P,
                                           _P, _P, _SZ, _P, _P, _P, _P]
_lib.pkv_paged_attention_noalloc.restype = _I32
_lib.pkv_paged_attention_noalloc.argtypes = [C.POINTER(_Cache), _P, _I32, _I32, _P, _P, _P, _I32, _I32, _F, _I32, _P,
                                             _P, _P, _P, _P]
_lib.pkv_stream_read.restype = _I32
_lib.pkv_stream_read.argtypes = [_P, _SZ, _I32, _P, _P, _P]
_lib.pkv_split_kv_reduce.restype = _I32
_lib.pkv_split_kv_reduce.argtypes = [_P, _P, _I32, _I64, _I32, _P, _I32, _P, _P]


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PkvError(status, where)


def status_string(status: int) -> str:
    return _lib.pkv_status_string(status).decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    return _TORCH_CODES[t.dtype]


@dataclass
class Cache:
    """A paged KV pool ``[num_blocks][num_layers][2][Hkv][B][D]`` on the GPU and the layer a call uses.

    An NVFP4 pool is ``[num_blocks][num_layers][2][Hkv][B * D * 9 / 16]`` bytes: per run, B rows
    of D/2 bytes of E2M1 codes, then B rows of D/16 bytes of E4M3 block scales."""

    pool: torch.Tensor
    kv_dtype: int
    block_size: int
    layer: int = 0
    k_scale: torch.Tensor | None = None  # float32 [num_layers][Hkv], fp8 and NVFP4 pools
    v_scale: torch.Tensor | None = None

    @staticmethod
    def allocate(num_blocks: int, num_layers: int, num_kv_heads: int, block_size: int, head_dim: int, kv_dtype: str,
                 device="cuda", fill_nan: bool = True, k_scale=None, v_scale=None,
                 fill_byte: int | None = None) -> "Cache":
        """``fill_byte`` (0..255) fills every pool byte with that value instead of the NaN sentinels."""
        code = DTYPE_CODES[kv_dtype]
        shape = (num_blocks, num_layers, 2, num_kv_heads, block_size, head_dim)
        if code == PKV_NVFP4:
            shape = (num_blocks, num_layers, 2, num_kv_heads, block_size * (head_dim // 2 + head_dim // 16))
        tdt = _CODE_TORCH[code]
        pool = torch.empty(shape, dtype=tdt, device=device)
        if fill_byte is not None:
            pool.view(torch.uint8).fill_(int(fill_byte))
        elif fill_nan:  # sentinel NaNs in every slot no sequence owns (NVFP4: NaN block scales)
            if code in (PKV_FP8_E4M3, PKV_NVFP4):
                pool.fill_(0x7F)
            else:
                pool.fill_(float("nan"))
        to_dev = lambda s: None if s is None else torch.as_tensor(s, dtype=torch.float32).to(device).contiguous()  # noqa: E731
        return Cache(pool, code, block_size, 0, to_dev(k_scale), to_dev(v_scale))

    @property
    def num_kv_heads(self) -> int:
        return self.pool.shape[3]

    @property
    def head_dim(self) -> int:
        if self.kv_dtype == PKV_NVFP4:
            return self.pool.shape[4] // self.block_size * 16 // 9
        return self.pool.shape[5]

    def _c(self) -> _Cache:
        p = self.pool
        return _Cache(p.data_ptr(), p.shape[0], p.shape[1], self.layer, p.shape[3], self.head_dim, self.block_size,
                      self.kv_dtype, _ptr(self.k_scale), _ptr(self.v_scale))


def kv_append(cache: Cache, k_new: torch.Tensor, v_new: torch.Tensor, cu_new: torch.Tensor, start_pos: torch.Tensor,
              block_tables: torch.Tensor, total_new: int | None = None, status: torch.Tensor | None = None,
              stream=None) -> None:
    """Write packed new K/V rows ``[total_new][Hkv][D]`` into their pool slots (device tensors)."""
    num_seqs = start_pos.shape[0]
    if total_new is None:
        total_new = k_new.shape[0]
    c = cache._c()
    _check(_lib.pkv_kv_append(C.byref(c), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), _ptr(cu_new),
                              _ptr(start_pos), _ptr(block_tables), block_tables.shape[1], num_seqs, total_new,
                              _ptr(status), _stream(stream)), "kv_append")


def copy_block_prefix(cache: Cache, src_blocks: torch.Tensor, dst_blocks: torch.Tensor, n_tokens: torch.Tensor,
                      status: torch.Tensor | None = None, stream=None) -> None:
    """Copy slots [0, n_tokens[i]) of block src_blocks[i] into block dst_blocks[i] (device int32 tensors),
    every layer, K and V, every head (partial reuse of a cached block)."""
    c = cache._c()
    _check(_lib.pkv_copy_block_prefix(C.byref(c), _ptr(src_blocks), _ptr(dst_blocks), _ptr(n_tokens),
                                      src_blocks.shape[0], _ptr(status), _stream(stream)), "copy_block_prefix")


@dataclass
class Plan:
    """Host plan buffer (page-locked) and its sizes."""

    buffer: torch.Tensor
    info: dict

    @property
    def workspace_bytes(self) -> int:
        return self.info["workspace_bytes"]


def _host_i32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def plan_attention(cu_q_lens, seq_lens, *, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
                   kv_dtype: int | str, causal: bool = True, block_tables=None, max_blocks: int | None = None,
                   num_ctas: int = 0, kv_split: int = 0, cascade: bool = True, min_shared_tokens: int = 0,
                   pin: bool = True, buffer: torch.Tensor | None = None, window: int = 0,
                   wait_limit_kcycles: int = 0, debug_flags: int = 0, tc_num_ctas: int = 0,
                   heads_per_item: int = 0) -> Plan:
    """Build the work list for one paged_attention call from host copies of the lengths.

    ``tc_num_ctas`` > 0 runs the tcgen05 tiles side by side with the decode tiles on that many
    CTAs (``num_ctas`` > 0 then counts the decode-tile kernel's); 0 lets the planner decide
    (with ``num_ctas`` = 0); < 0 never.

    ``heads_per_item`` 4 makes every decode-sized item cover four consecutive KV heads (one per
    consumer warp of the TMA-fed decode kernel); 1 one head; 0 lets the planner decide.

    ``window`` > 0 limits every (causal) row to its ``window`` most recent positions; the
    plan carries it to ``paged_attention``, as it does ``wait_limit_kcycles`` (limit of every
    pipeline wait, thousands of SM cycles, 0 = default) and ``debug_flags``
    (``PKV_DEBUG_WITHHOLD_LOADS`` makes every wait run out, to test the timeout path).

    ``buffer`` (uint8, host) is reused when large enough; the caller must not
    reuse a buffer whose plan upload may still be pending on the GPU.
    """
    cu = _host_i32(cu_q_lens)
    sl = _host_i32(seq_lens)
    bt = None if block_tables is None else _host_i32(block_tables)
    if max_blocks is None:
        max_blocks = bt.shape[1] if bt is not None else 1
    code = DTYPE_CODES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    req = _PlanRequest(sl.shape[0], num_q_heads, num_kv_heads, head_dim, block_size, code, int(bool(causal)), num_ctas,
                       kv_split, int(bool(cascade)), min_shared_tokens, max_blocks, cu.ctypes.data, sl.ctypes.data,
                       None if bt is None else bt.ctypes.data, int(window), int(wait_limit_kcycles), int(debug_flags),
                       int(tc_num_ctas), int(heads_per_item))
    info = _PlanInfo()
    # With a buffer given, plan straight into it (one call); only a buffer too small costs a
    # size query and a new buffer.
    st = (_lib.pkv_attention_plan(C.byref(req), buffer.data_ptr(), buffer.numel(), C.byref(info))
          if buffer is not None else _WORKSPACE_TOO_SMALL)
    if st == 0:
        buf = buffer
    else:
        if st != _WORKSPACE_TOO_SMALL:
            _check(st, "attention_plan")
        _check(_lib.pkv_attention_plan(C.byref(req), None, 0, C.byref(info)), "attention_plan")
        buf = torch.empty(int(info.plan_bytes), dtype=torch.uint8, pin_memory=pin and torch.cuda.is_available())
        _check(_lib.pkv_attention_plan(C.byref(req), buf.data_ptr(), buf.numel(), C.byref(info)), "attention_plan")
    return Plan(buf, {f: getattr(info, f) for f, _ in _PlanInfo._fields_})


class Planner:
    """A reusable host planner for batches of one size: the planning request and the host int32
    arrays it points at are built once, so each :meth:`plan` is a single call into the library.

    ``cu_q_lens`` ``[num_seqs + 1]``, ``seq_lens`` ``[num_seqs]`` and ``block_tables``
    ``[num_seqs][max_blocks]`` are the host arrays the planner reads; contiguous int32 arrays
    given here (numpy, or CPU torch tensors, page-locked ones included) are used in place, so a
    caller that updates them between steps re-plans without any copy; others are copied once.
    ``block_tables`` may be None (no shared-prefix grouping).
    """

    def __init__(self, cu_q_lens, seq_lens, block_tables=None, *, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, kv_dtype: int | str, causal: bool = True, num_ctas: int = 0,
                 kv_split: int = 0, cascade: bool = True, min_shared_tokens: int = 0, window: int = 0,
                 max_blocks: int | None = None, wait_limit_kcycles: int = 0, debug_flags: int = 0,
                 tc_num_ctas: int = 0, heads_per_item: int = 0):
        self.cu_q_lens = self._host(cu_q_lens)
        self.seq_lens = self._host(seq_lens)
        self.block_tables = None if block_tables is None else self._host(block_tables)
        if max_blocks is None:
            max_blocks = self.block_tables.shape[1] if self.block_tables is not None else 1
        code = DTYPE_CODES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
        self._req = _PlanRequest(self.seq_lens.shape[0], num_q_heads, num_kv_heads, head_dim, block_size, code,
                                 int(bool(causal)), num_ctas, kv_split, int(bool(cascade)), min_shared_tokens,
                                 max_blocks, self.cu_q_lens.ctypes.data, self.seq_lens.ctypes.data,
                                 None if self.block_tables is None else self.block_tables.ctypes.data, int(window),
                                 int(wait_limit_kcycles), int(debug_flags), int(tc_num_ctas),
                                 int(heads_per_item))
        self._req_ref = C.byref(self._req)
        self._info = _PlanInfo()
        self._info_ref = C.byref(self._info)

    @staticmethod
    def _host(x) -> np.ndarray:
        if isinstance(x, torch.Tensor):
            if x.device.type != "cpu":
                raise ValueError("the planner reads host arrays")
            if x.dtype == torch.int32 and x.is_contiguous():
                return x.numpy()  # shares the tensor's memory
            x = x.numpy()
        return np.ascontiguousarray(x, dtype=np.int32)

    def plan(self, buffer: torch.Tensor | None = None, pin: bool = True) -> Plan:
        """Plan into ``buffer`` (uint8 host; a new page-locked one when missing or too small)."""
        st = (_lib.pkv_attention_plan(self._req_ref, buffer.data_ptr(), buffer.numel(), self._info_ref)
              if buffer is not None else _WORKSPACE_TOO_SMALL)
        if st != 0:
            if st != _WORKSPACE_TOO_SMALL:
                _check(st, "attention_plan")
            _check(_lib.pkv_attention_plan(self._req_ref, None, 0, self._info_ref), "attention_plan")
            buffer = torch.empty(int(self._info.plan_bytes), dtype=torch.uint8,
                                 pin_memory=pin and torch.cuda.is_available())
            _check(_lib.pkv_attention_plan(self._req_ref, buffer.data_ptr(), buffer.numel(), self._info_ref),
                   "attention_plan")
        return Plan(buffer, {f: getattr(self._info, f) for f, _ in _PlanInfo._fields_})

    def plan_into(self, buffer: torch.Tensor) -> int:
        """Plan into ``buffer`` (large enough, as a previous :meth:`plan` of these shapes returned it);
        returns the plan's bytes.  The cheapest form: one library call, no result dictionary."""
        _check(_lib.pkv_attention_plan(self._req_ref, buffer.data_ptr(), buffer.numel(), self._info_ref),
               "attention_plan")
        return self._info.plan_bytes


def attention_workspace_bytes(plan: Plan) -> int:
    return plan.workspace_bytes


def default_num_ctas(kv_dtype: int | str, head_dim: int, block_size: int) -> int:
    code = DTYPE_CODES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    n = C.c_int32(0)
    _check(_lib.pkv_default_num_ctas(code, head_dim, block_size, C.byref(n)), "default_num_ctas")
    return n.value


def paged_attention(cache: Cache, q: torch.Tensor, cu_q_lens: torch.Tensor, seq_lens: torch.Tensor,
                    block_tables: torch.Tensor, plan: Plan, softmax_scale: float, causal: bool = True,
                    out: torch.Tensor | None = None, out_lse: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None,
                    kernel_events=None):
    """out = softmax(scale q K^T) V over the paged cache; returns ``out``.

    ``kernel_events``: optional (begin, end) torch.cuda.Event pair recorded right
    before and right after the attention kernels (pkv_paged_attention_timed).
    """
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device=q.device)
    c = cache._c()
    # The library launches on (and sizes its grids for) the current device: make it q's.
    with torch.cuda.device(q.device):
        args = (C.byref(c), _ptr(q), _dtype_code(q), q.shape[1], _ptr(cu_q_lens), _ptr(seq_lens), _ptr(block_tables),
                block_tables.shape[1], seq_lens.shape[0], float(softmax_scale), int(bool(causal)),
                plan.buffer.data_ptr(), _ptr(out), _ptr(out_lse), _ptr(workspace), workspace.numel(), _ptr(status),
                _stream(stream))
        if kernel_events is None:
            _check(_lib.pkv_paged_attention(*args), "paged_attention")
        else:
            handles = [e.cuda_event for e in kernel_events]
            if not all(handles):
                raise ValueError("kernel_events: record each event once before use (torch creates CUDA events lazily)")
            _check(_lib.pkv_paged_attention_timed(*args, *handles), "paged_attention")
    return out


def paged_attention_noalloc(cache: Cache, q: torch.Tensor, cu_q_lens: torch.Tensor, seq_lens: torch.Tensor,
                            block_tables: torch.Tensor, plan: Plan, softmax_scale: float, causal: bool = True,
                            out: torch.Tensor | None = None, out_lse: torch.Tensor | None = None,
                            status: torch.Tensor | None = None, stream=None):
    """paged_attention using the library's built-in scratch array instead of a workspace.

    For callers that may not allocate device memory; see pkv_paged_attention_noalloc
    in include/pkv.h for the size limit and the sharing rules.  ``out`` must be
    given by such callers (a default is allocated here only for convenience).
    """
    if out is None:
        out = torch.empty_like(q)
    c = cache._c()
    # The built-in scratch array is chosen by the current device: make it q's.
    with torch.cuda.device(q.device):
        _check(_lib.pkv_paged_attention_noalloc(C.byref(c), _ptr(q), _dtype_code(q), q.shape[1], _ptr(cu_q_lens),
                                                _ptr(seq_lens), _ptr(block_tables), block_tables.shape[1],
                                                seq_lens.shape[0], float(softmax_scale), int(bool(causal)),
                                                plan.buffer.data_ptr(), _ptr(out), _ptr(out_lse), _ptr(status),
                                                _stream(stream)), "paged_attention_noalloc")
    return out


def split_kv_reduce(partial_o: torch.Tensor, partial_lse: torch.Tensor, out_dtype=torch.float32,
                    out: torch.Tensor | None = None, out_lse: torch.Tensor | None = None, stream=None):
    """Merge ``[n][rows][D]`` partial states into ``[rows][D]``; returns (out, out_lse)."""
    n, rows, d = partial_o.shape
    if out is None:
        out = torch.empty((rows, d), dtype=out_dtype, device=partial_o.device)
    _check(_lib.pkv_split_kv_reduce(_ptr(partial_o), _ptr(partial_lse), n, rows, d, _ptr(out), _dtype_code(out),
                                    _ptr(out_lse), _stream(stream)), "split_kv_reduce")
    return out, out_lse


def stream_read(buf: torch.Tensor, sink: torch.Tensor, mode: int = 0, status: torch.Tensor | None = None,
                stream=None) -> None:
    """Read every byte of device tensor ``buf`` once (pkv_stream_read); ``sink``: device int32 [1]."""
    _check(_lib.pkv_stream_read(buf.data_ptr(), buf.numel() * buf.element_size(), int(mode), sink.data_ptr(),
                                _ptr(status), _stream(stream)), "stream_read")


class GraphStep:
    """One serving step from page-locked host inputs, as three CUDA graphs per buffer slot.

    A step is: one host-to-device copy of the packed inputs (q, new K/V rows, cu_q_lens,
    seq_lens, start_pos, block tables); ``kv_append`` and ``paged_attention`` (which uploads
    the step's plan from its page-locked buffer); one device-to-host copy of the output.
    The copies run on their own streams, so with two slots the inputs of step i+1 travel
    while step i computes and the output of step i travels while step i+1 computes; the
    host plans step i+1 meanwhile.  Every call of :meth:`run` re-plans on the host into the
    slot's plan buffer; the slot's graphs are captured again whenever a new plan differs
    from the captured one in a launch-shaping field (item and merge counts, CTA counts).

    Callers write a step's inputs into :attr:`host` ``[slot]`` (named page-locked views of
    one buffer) before :meth:`run` takes that slot and after :meth:`wait` has returned for
    the slot's previous step, and read the output from the tensor that :meth:`wait` returns
    before the slot's next step is launched.
    """

    _FIELDS = ("q", "k_new", "v_new", "cu_q", "seq_lens", "start_pos", "block_tables")
    _SHAPE_KEYS = ("plan_bytes", "workspace_bytes", "num_items", "num_tc_items", "num_reduce", "num_parts",
                   "num_partial_rows", "num_ctas", "tc_num_ctas", "side_by_side", "heads_per_item")

    def __init__(self, cache: Cache, like: dict, plan_kwargs: dict, softmax_scale: float, causal: bool = True,
                 slots: int = 2, stream=None):
        self.cache, self.plan_kwargs, self.scale, self.causal = cache, dict(plan_kwargs), float(softmax_scale), causal
        self.stream = stream if stream is not None else torch.cuda.Stream()  # kernels
        dev = self.stream.device
        self.copy_in_stream = torch.cuda.Stream(dev)
        self.copy_out_stream = torch.cuda.Stream(dev)
        # One page-locked buffer and one device buffer per slot, each field 256-byte aligned.
        offs, total = {}, 0
        for name in self._FIELDS:
            t = like[name]
            offs[name] = (total, t.dtype, tuple(t.shape))
            total = (total + t.numel() * t.element_size() + 255) // 256 * 256

        def views(buf):
            return {n: buf[o:o + int(np.prod(sh)) * torch.empty((), dtype=dt).element_size()].view(dt).view(sh)
                    for n, (o, dt, sh) in offs.items()}

        self.h2d_bytes = total
        self._hbuf = [torch.empty(total, dtype=torch.uint8).pin_memory() for _ in range(slots)]
        self._dbuf = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(slots)]
        self.host = [views(b) for b in self._hbuf]
        self._dev = [views(b) for b in self._dbuf]
        q = like["q"]
        self._out_d = [torch.empty(q.shape, dtype=q.dtype, device=dev) for _ in range(slots)]
        self._out_h = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(slots)]
        self.d2h_bytes = q.numel() * q.element_size()
        self._plans = [None] * slots
        self._planners = [None] * slots
        self._graphs = [None] * slots  # (copy in, compute, copy out) per slot
        self._shape = [None] * slots
        self._ready = [torch.cuda.Event() for _ in range(slots)]     # inputs of the slot on the device
        self._consumed = [torch.cuda.Event() for _ in range(slots)]  # kernels done with inputs, plan, output buffer
        self._fetched = [torch.cuda.Event() for _ in range(slots)]   # output of the slot on the host
        self._pending = [False] * slots
        self._ws = None
        self._slot = 0

    def _plan_into(self, b: int) -> Plan:
        # One planner per slot reads the slot's page-locked lengths and tables in place.
        if self._planners[b] is None:
            h = self.host[b]
            self._planners[b] = Planner(h["cu_q"], h["seq_lens"], h["block_tables"], **self.plan_kwargs)
        buf = None if self._plans[b] is None else self._plans[b].buffer
        return self._planners[b].plan(buf)

    def _capture(self, b: int, plan: Plan) -> None:
        if self._ws is None or self._ws.numel() < plan.workspace_bytes:
            self._ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device=self.stream.device)
        d = self._dev[b]
        g_in, g_run, g_out = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_in, stream=self.copy_in_stream):
            self._dbuf[b].copy_(self._hbuf[b], non_blocking=True)
        with torch.cuda.graph(g_run, stream=self.stream):
            kv_append(self.cache, d["k_new"], d["v_new"], d["cu_q"], d["start_pos"], d["block_tables"])
            paged_attention(self.cache, d["q"], d["cu_q"], d["seq_lens"], d["block_tables"], plan, self.scale,
                            self.causal, out=self._out_d[b], workspace=self._ws)
        with torch.cuda.graph(g_out, stream=self.copy_out_stream):
            self._out_h[b].copy_(self._out_d[b], non_blocking=True)
        self._graphs[b] = (g_in, g_run, g_out)

    def run(self) -> int:
        """Plan and launch one step on the next slot; returns the slot (pass it to :meth:`wait`)."""
        b = self._slot
        self._slot = (b + 1) % len(self._graphs)
        if self._pending[b]:
            self._consumed[b].synchronize()  # the slot's last kernels have read its inputs and plan
        plan = self._plan_into(b)
        self._plans[b] = plan
        shape = tuple(plan.info[k] for k in self._SHAPE_KEYS)
        if self._graphs[b] is None or shape != self._shape[b]:
            torch.cuda.synchronize(self.stream.device)
            self._capture(b, plan)
            self._shape[b] = shape
        g_in, g_run, g_out = self._graphs[b]
        with torch.cuda.stream(self.copy_in_stream):
            self.copy_in_stream.wait_event(self._consumed[b])  # device inputs of the slot free
            g_in.replay()
            self._ready[b].record(self.copy_in_stream)
        with torch.cuda.stream(self.stream):
            self.stream.wait_event(self._ready[b])
            self.stream.wait_event(self._fetched[b])  # the slot's previous output has left
            g_run.replay()
            self._consumed[b].record(self.stream)
        with torch.cuda.stream(self.copy_out_stream):
            self.copy_out_stream.wait_event(self._consumed[b])
            g_out.replay()
            self._fetched[b].record(self.copy_out_stream)
        self._pending[b] = True
        return b

    def wait(self, slot: int) -> torch.Tensor:
        """Block until the slot's step has finished; returns its page-locked host output."""
        self._fetched[slot].synchronize()
        self._pending[slot] = False
        return self._out_h[slot]
