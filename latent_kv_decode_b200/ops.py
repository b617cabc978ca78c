"""ctypes binding of libmla.so (include/mla.h): argument marshalling only.

Every function takes torch CUDA tensors, passes their device pointers,
strides and the current CUDA stream to the C ABI, and raises on a non-zero
status. All arithmetic happens in the library's kernels; torch only
allocates outputs and workspace. When libmla.so is missing, every call
raises: there is no other implementation behind these names.

Calls (same names as the C ABI):

- ``mla_absorb_q(q_nope, wkv_b)``: blank [1], q_lat = q_nope . W_UK[h].
- ``mla_decode(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, ...)``:
  blanks [2]-[4] and step 5; returns a :class:`DecodeCall` whose ``x`` and
  ``lse`` are final when it used one split, else after ``mla_combine``.
- ``mla_combine(call)``: merges the split partials of a :class:`DecodeCall`.
- ``mla_up_proj(x, wkv_b, Dn)``: blank [5], out = W_UV[h] . x.
- ``mla_decode_step(q_nope, q_pe, kv_cache, pe_cache, wkv_b, softmax_scale,
  causal_mask)``: the four calls in a row with the signature of the 6547.cn
  question's ``mla_decode_step``.
- ``mla_cache_append(c_kv, k_pe, kv_cache, pe_cache, seq_lens, ...)``: the
  step before the decode, writing the new tokens' rows (or FP4 entries) into
  the cache.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")

MLA_F32, MLA_BF16, MLA_FP4 = 0, 1, 2
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_CUDA"}
DEVICE_ERR_BLOCK_TABLE = 1
DEVICE_ERR_TIMEOUT = 2

# every function the header declares, with its ctypes signature
_c = ctypes
_SIGS = {
    "mla_status_string": (_c.c_char_p, [_c.c_int]),
    "mla_last_cuda_error": (_c.c_int, []),
    "mla_version": (_c.c_char_p, []),
    "mla_absorb_q": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p] + [_c.c_int] * 6 +
                     [_c.c_int, _c.c_void_p]),
    "mla_up_proj": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p] + [_c.c_int] * 6 +
                    [_c.c_int, _c.c_void_p]),
    "mla_decode_num_splits": (_c.c_int, [_c.c_void_p]),
    "mla_decode_workspace_size": (_c.c_size_t, [_c.c_void_p]),
    "mla_decode": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "mla_combine": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
    "mla_decode_static_scratch": (_c.c_int, [_c.c_void_p, _c.c_void_p]),
    "mla_cache_append": (_c.c_int, [_c.c_void_p, _c.c_void_p]),
    "mla_group_wo_workspace_size": (_c.c_size_t, [_c.c_void_p]),
    "mla_group_wo": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_size_t, _c.c_void_p]),
}


class MlaError(RuntimeError):
    pass


class DecodeArgs(ctypes.Structure):
    """Mirror of ``mla_decode_args`` in include/mla.h (field order and types)."""

    _fields_ = [
        ("B", _c.c_int), ("H", _c.c_int), ("Q", _c.c_int), ("Ckv", _c.c_int), ("Dr", _c.c_int),
        ("q_dtype", _c.c_int), ("cache_dtype", _c.c_int),
        ("q_lat", _c.c_void_p), ("q_pe", _c.c_void_p), ("kv_cache", _c.c_void_p),
        ("pe_cache", _c.c_void_p),
        ("kv_row_stride", _c.c_int64), ("pe_row_stride", _c.c_int64),
        ("kv_batch_stride", _c.c_int64), ("pe_batch_stride", _c.c_int64),
        ("Lk", _c.c_int), ("seq_lens", _c.c_void_p), ("block_table", _c.c_void_p),
        ("max_pages", _c.c_int), ("page_size", _c.c_int), ("num_pages", _c.c_int),
        ("causal_mask", _c.c_void_p), ("causal", _c.c_int), ("softmax_scale", _c.c_float),
        ("sinks", _c.c_void_p), ("rope_tail", _c.c_int), ("rope_theta", _c.c_float),
        ("num_splits", _c.c_int), ("x", _c.c_void_p), ("lse", _c.c_void_p),
        ("err_flag", _c.c_void_p),
    ]


class AppendArgs(ctypes.Structure):
    """Mirror of ``mla_append_args`` in include/mla.h (field order and types)."""

    _fields_ = [
        ("B", _c.c_int), ("Q", _c.c_int), ("Ckv", _c.c_int), ("Dr", _c.c_int),
        ("src_dtype", _c.c_int), ("cache_dtype", _c.c_int),
        ("c_kv", _c.c_void_p), ("k_pe", _c.c_void_p), ("kv_cache", _c.c_void_p),
        ("pe_cache", _c.c_void_p),
        ("kv_row_stride", _c.c_int64), ("pe_row_stride", _c.c_int64),
        ("kv_batch_stride", _c.c_int64), ("pe_batch_stride", _c.c_int64),
        ("Lk", _c.c_int), ("seq_lens", _c.c_void_p), ("block_table", _c.c_void_p),
        ("max_pages", _c.c_int), ("page_size", _c.c_int), ("num_pages", _c.c_int),
        ("rope_tail", _c.c_int), ("rope_theta", _c.c_float), ("err_flag", _c.c_void_p),
    ]


class GroupWoArgs(ctypes.Structure):
    """Mirror of ``mla_group_wo_args`` in include/mla.h (field order and types)."""

    _fields_ = [
        ("B", _c.c_int), ("H", _c.c_int), ("Q", _c.c_int), ("Ckv", _c.c_int),
        ("G", _c.c_int), ("R", _c.c_int), ("D", _c.c_int), ("dtype", _c.c_int),
        ("x", _c.c_void_p), ("wo_a", _c.c_void_p), ("wo_b", _c.c_void_p), ("out", _c.c_void_p),
        ("err_flag", _c.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmla.so once; raise if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MlaError(f"{LIB_PATH} is missing; build it with `python -m latent_kv_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != 0:
        extra = ""
        if status == 4:
            extra = f" (cudaError {lib().mla_last_cuda_error()})"
        raise MlaError(f"{what} failed: {STATUS.get(status, status)}{extra}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _qdtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MLA_F32
    if t.dtype == torch.bfloat16:
        return MLA_BF16
    raise MlaError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise MlaError("libmla takes CUDA tensors only")


def mla_absorb_q(q_nope: torch.Tensor, wkv_b: torch.Tensor, q_lat: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    _need_cuda(q_nope, wkv_b)
    B, H, Q, Dn = q_nope.shape
    Ckv = wkv_b.shape[2]
    Vd = wkv_b.shape[1] - Dn
    if q_lat is None:
        q_lat = torch.empty((B, H, Q, Ckv), dtype=q_nope.dtype, device=q_nope.device)
    assert q_nope.is_contiguous() and wkv_b.is_contiguous() and q_lat.is_contiguous()
    _check(lib().mla_absorb_q(_ptr(q_nope), _ptr(wkv_b), _ptr(q_lat), B, H, Q, Dn, Vd, Ckv,
                              _qdtype(q_nope), _stream(stream)), "mla_absorb_q")
    return q_lat


def mla_up_proj(x: torch.Tensor, wkv_b: torch.Tensor, Dn: int, out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    _need_cuda(x, wkv_b)
    B, H, Q, Ckv = x.shape
    Vd = wkv_b.shape[1] - Dn
    if out is None:
        out = torch.empty((B, H, Q, Vd), dtype=x.dtype, device=x.device)
    assert x.is_contiguous() and wkv_b.is_contiguous() and out.is_contiguous()
    _check(lib().mla_up_proj(_ptr(x), _ptr(wkv_b), _ptr(out), B, H, Q, Dn, Vd, Ckv, _qdtype(x),
                             _stream(stream)), "mla_up_proj")
    return out


@dataclass
class DecodeCall:
    """One mla_decode call: its arguments, workspace and outputs.

    ``x``/``lse`` are final after the call when ``num_splits == 1``, and after
    :func:`mla_combine` otherwise.
    """

    args: DecodeArgs
    num_splits: int
    workspace: Optional[torch.Tensor]
    x: torch.Tensor
    lse: Optional[torch.Tensor]
    keep: list = field(default_factory=list)   # tensors the pointers in args refer to


def make_decode_args(q_lat, q_pe, kv_cache, pe_cache, softmax_scale: float, *, seq_lens=None,
                     block_table=None, page_size: int = 64, causal_mask=None, causal: bool = False,
                     sinks=None, rope_tail: int = 0, rope_theta: float = 10000.0,
                     num_splits: int = 0, x=None, lse=None, want_lse: bool = True,
                     err_flag=None, Lk: Optional[int] = None) -> DecodeCall:
    """Fill a DecodeArgs from tensors (no GPU work).

    kv_cache / pe_cache: (B, Lk, C) views (any row/batch stride) for a
    contiguous cache, or (num_pages, page_size, C) pools with ``block_table``
    (B, max_pages) int32. FP4 caches are uint8 tensors of 288-byte rows and
    take ``q_pe = pe_cache = None``.
    """
    _need_cuda(q_lat, q_pe, kv_cache, pe_cache, seq_lens, block_table, causal_mask, sinks)
    B, H, Q, Ckv = q_lat.shape
    assert q_lat.is_contiguous()
    Dr = 0 if q_pe is None else q_pe.shape[-1]
    if q_pe is not None:
        assert q_pe.is_contiguous()
    fp4 = kv_cache.dtype == torch.uint8
    a = DecodeArgs()
    a.B, a.H, a.Q, a.Ckv, a.Dr = B, H, Q, Ckv, Dr
    a.q_dtype = _qdtype(q_lat)
    a.cache_dtype = MLA_FP4 if fp4 else _qdtype(kv_cache)
    a.q_lat, a.q_pe = _ptr(q_lat), _ptr(q_pe)
    a.kv_cache, a.pe_cache = _ptr(kv_cache), _ptr(pe_cache)
    assert kv_cache.stride(-1) == 1
    a.kv_row_stride = kv_cache.stride(1)
    a.kv_batch_stride = kv_cache.stride(0)
    if pe_cache is not None:
        assert pe_cache.stride(-1) == 1
        a.pe_row_stride = pe_cache.stride(1)
        a.pe_batch_stride = pe_cache.stride(0)
    if block_table is not None:
        assert block_table.dtype == torch.int32 and block_table.is_contiguous()
        a.block_table = _ptr(block_table)
        a.max_pages = block_table.shape[1]
        a.page_size = page_size
        a.num_pages = kv_cache.shape[0]
        a.kv_batch_stride = a.pe_batch_stride = 0
        a.Lk = Lk if Lk is not None else a.max_pages * page_size
    else:
        a.Lk = Lk if Lk is not None else kv_cache.shape[1]
    if seq_lens is not None:
        assert seq_lens.dtype == torch.int32 and seq_lens.is_contiguous()
        a.seq_lens = _ptr(seq_lens)
    if causal_mask is not None:
        causal_mask = causal_mask.reshape(-1).to(torch.uint8).contiguous()
        a.causal_mask = _ptr(causal_mask)
    a.causal = int(bool(causal))
    a.softmax_scale = float(softmax_scale)
    if sinks is not None:
        assert sinks.dtype == torch.float32 and sinks.is_contiguous()
        a.sinks = _ptr(sinks)
    a.rope_tail, a.rope_theta = int(rope_tail), float(rope_theta)
    a.num_splits = int(num_splits)
    if x is None:
        x = torch.empty((B, H, Q, Ckv), dtype=q_lat.dtype, device=q_lat.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Q), dtype=torch.float32, device=q_lat.device)
    a.x, a.lse = _ptr(x), _ptr(lse)
    a.err_flag = _ptr(err_flag)
    S = lib().mla_decode_num_splits(ctypes.byref(a))
    if S < 0:
        raise MlaError("mla_decode arguments rejected (MLA_ERR_INVALID_ARG or MLA_ERR_UNSUPPORTED)")
    keep = [q_lat, q_pe, kv_cache, pe_cache, seq_lens, block_table, causal_mask, sinks, err_flag]
    return DecodeCall(args=a, num_splits=S, workspace=None, x=x, lse=lse, keep=keep)


def workspace_bytes(call: DecodeCall) -> int:
    return int(lib().mla_decode_workspace_size(ctypes.byref(call.args)))


def mla_decode(q_lat, q_pe, kv_cache, pe_cache, softmax_scale: float, *, workspace=None,
               stream=None, **kw) -> DecodeCall:
    """Enqueue mla_decode; returns the DecodeCall (see its docstring)."""
    call = make_decode_args(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, **kw)
    launch_decode(call, workspace=workspace, stream=stream)
    return call


def launch_decode(call: DecodeCall, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    need = workspace_bytes(call)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=call.x.device)
    call.workspace = workspace
    ws_ptr = _ptr(workspace) if need else None
    _check(lib().mla_decode(ctypes.byref(call.args), ws_ptr, need, _stream(stream)), "mla_decode")


def mla_combine(call: DecodeCall, stream=None) -> DecodeCall:
    """Enqueue mla_combine for a DecodeCall (no-op with one split)."""
    need = workspace_bytes(call)
    ws = call.workspace
    _check(lib().mla_combine(ctypes.byref(call.args), _ptr(ws) if need else None, need,
                             _stream(stream)), "mla_combine")
    return call


def mla_decode_static_scratch(call: DecodeCall, stream=None) -> DecodeCall:
    """Decode and combine with the library's own scratch array: no workspace, no allocation.

    For callers that may not allocate device memory at decode time. The
    call's ``x``/``lse`` are final once the enqueued work completes. Raises
    when the split count needs more than MLA_STATIC_SCRATCH_BYTES (32 MiB).
    All such calls share one array per device: keep them from overlapping
    on the GPU.
    """
    _check(lib().mla_decode_static_scratch(ctypes.byref(call.args), _stream(stream)),
           "mla_decode_static_scratch")
    return call


def decode(q_lat, q_pe, kv_cache, pe_cache, softmax_scale: float, **kw):
    """mla_decode followed by mla_combine; returns (x, lse)."""
    call = mla_decode(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, **kw)
    mla_combine(call, stream=kw.get("stream"))
    return call.x, call.lse


def mla_decode_step(q_nope, q_pe, kv_cache, pe_cache, wkv_b, softmax_scale, causal_mask=None,
                    **kw):
    """The whole absorbed decode step -> out (B,H,Q,Vd): absorb, decode, combine, up-project."""
    Dn = q_nope.shape[-1]
    q_lat = mla_absorb_q(q_nope, wkv_b, stream=kw.get("stream"))
    x, _ = decode(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, causal_mask=causal_mask, **kw)
    return mla_up_proj(x, wkv_b, Dn, stream=kw.get("stream"))


def make_append_args(c_kv, k_pe, kv_cache, pe_cache, seq_lens, *, block_table=None, page_size: int = 64,
                     rope_tail: int = 0, rope_theta: float = 10000.0, err_flag=None,
                     Lk: Optional[int] = None) -> AppendArgs:
    """Fill an AppendArgs from tensors (no GPU work).

    c_kv (B, Q, Ckv) / k_pe (B, Q, Dr) are the new tokens' rows; seq_lens
    (B) int32 are the lengths after the append. The cache tensors follow
    make_decode_args: (B, Lk, C) views or (num_pages, page_size, C) pools with
    ``block_table``; a uint8 kv_cache of 288-byte rows takes FP4 entries.
    """
    _need_cuda(c_kv, k_pe, kv_cache, pe_cache, seq_lens, block_table, err_flag)
    B, Q, Ckv = c_kv.shape
    assert c_kv.is_contiguous() and seq_lens.dtype == torch.int32 and seq_lens.is_contiguous()
    Dr = 0 if k_pe is None else k_pe.shape[-1]
    if k_pe is not None:
        assert k_pe.is_contiguous() and k_pe.dtype == c_kv.dtype
    a = AppendArgs()
    a.B, a.Q, a.Ckv, a.Dr = B, Q, Ckv, Dr
    a.src_dtype = _qdtype(c_kv)
    a.cache_dtype = MLA_FP4 if kv_cache.dtype == torch.uint8 else _qdtype(kv_cache)
    a.c_kv, a.k_pe = _ptr(c_kv), _ptr(k_pe)
    a.kv_cache, a.pe_cache = _ptr(kv_cache), _ptr(pe_cache)
    assert kv_cache.stride(-1) == 1
    a.kv_row_stride, a.kv_batch_stride = kv_cache.stride(1), kv_cache.stride(0)
    if pe_cache is not None:
        assert pe_cache.stride(-1) == 1
        a.pe_row_stride, a.pe_batch_stride = pe_cache.stride(1), pe_cache.stride(0)
    a.seq_lens = _ptr(seq_lens)
    if block_table is not None:
        assert block_table.dtype == torch.int32 and block_table.is_contiguous()
        a.block_table = _ptr(block_table)
        a.max_pages, a.page_size, a.num_pages = block_table.shape[1], page_size, kv_cache.shape[0]
        a.kv_batch_stride = a.pe_batch_stride = 0
        a.Lk = Lk if Lk is not None else a.max_pages * page_size
    else:
        a.Lk = Lk if Lk is not None else kv_cache.shape[1]
    a.rope_tail, a.rope_theta = int(rope_tail), float(rope_theta)
    a.err_flag = _ptr(err_flag)
    return a


def mla_cache_append(c_kv, k_pe, kv_cache, pe_cache, seq_lens, *, stream=None, **kw) -> None:
    """Enqueue mla_cache_append: write the new tokens into the cache in place."""
    a = make_append_args(c_kv, k_pe, kv_cache, pe_cache, seq_lens, **kw)
    _check(lib().mla_cache_append(ctypes.byref(a), _stream(stream)), "mla_cache_append")


class GroupWoCall:
    """Arguments and workspace of one mla_group_wo call (build once, launch many times)."""

    def __init__(self, args: GroupWoArgs, out: torch.Tensor, workspace: Optional[torch.Tensor], keep):
        self.args, self.out, self.workspace, self._keep = args, out, workspace, keep


def make_group_wo(x: torch.Tensor, wo_a: torch.Tensor, wo_b: Optional[torch.Tensor] = None, *,
                  out: Optional[torch.Tensor] = None, err_flag=None) -> GroupWoCall:
    """Prepare mla_group_wo: x (B,H,Q,Ckv), wo_a (G,R,(H/G)*Ckv), wo_b (D,G*R) or None, all bf16.

    Allocates ``out`` ((B,Q,D), or (B,Q,G*R) without wo_b) and the workspace
    when not given; no GPU work.
    """
    _need_cuda(x, wo_a, wo_b)
    for t in (x, wo_a, wo_b):
        if t is not None and not t.is_contiguous():
            raise MlaError("mla_group_wo: tensors must be contiguous")
    B, H, Q, C = x.shape
    G, R, _ = wo_a.shape
    a = GroupWoArgs()
    a.B, a.H, a.Q, a.Ckv, a.G, a.R = B, H, Q, C, G, R
    a.D = wo_b.shape[0] if wo_b is not None else 0
    a.dtype = _qdtype(x)
    width = a.D if wo_b is not None else G * R
    if out is None:
        out = torch.empty((B, Q, width), dtype=x.dtype, device=x.device)
    a.x, a.wo_a, a.wo_b, a.out = _ptr(x), _ptr(wo_a), _ptr(wo_b), _ptr(out)
    a.err_flag = _ptr(err_flag)
    need = lib().mla_group_wo_workspace_size(ctypes.byref(a))
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device) if need else None
    return GroupWoCall(a, out, ws, (x, wo_a, wo_b, err_flag))


def launch_group_wo(call: GroupWoCall, stream=None) -> torch.Tensor:
    """Enqueue mla_group_wo for a prepared call; returns its output tensor."""
    ws = call.workspace
    _check(lib().mla_group_wo(ctypes.byref(call.args), _ptr(ws), 0 if ws is None else ws.numel(),
                              _stream(stream)), "mla_group_wo")
    return call.out


def mla_group_wo(x, wo_a, wo_b=None, *, stream=None, **kw) -> torch.Tensor:
    """Grouped low-rank output projection after the inverse RoPE -> (B,Q,D) or (B,Q,G*R)."""
    return launch_group_wo(make_group_wo(x, wo_a, wo_b, **kw), stream=stream)
