"""Thin ctypes binding of libgqa_paged.so (include/gqa_paged.h).

Argument marshalling only: torch tensors are checked for device, dtype, shape and
contiguity and passed as raw device pointers with the current CUDA stream; every step of
the computation runs in the library's kernels.  There is no fallback: if the library is
missing or the tensors are not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgqa_paged.so")

GQA_OK = 0
GQA_KV_BF16 = 0
GQA_KV_FP8_E4M3 = 1
GQA_MAX_SPLITS = 64
GQA_SPLITS_BALANCED = -1

_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); the exported symbols of include/gqa_paged.h
SIGNATURES = {
    "gqa_paged_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "gqa_pick_splits": (_I, [_I, _I, _I, _I, _I]),
    "gqa_paged_decode": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                              ctypes.c_float, _I, _I, _P, _P, _P, _SZ, _P]),
    "gqa_paged_decode_partial": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                      ctypes.c_float, _I, _I, _P, _P, _P, _SZ, _P]),
    "gqa_paged_kt_build": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "gqa_paged_kt_append": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "gqa_paged_sparse_table_stride": (_I, [_I, _I, _I, _I]),
    "gqa_paged_sparse_select_workspace_size": (_SZ, [_I, _I, _I]),
    "gqa_paged_sparse_select": (_I, [_P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I,
                                     _P, _P, _P, _SZ, _P]),
    "gqa_paged_sparse_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "gqa_paged_sparse_decode": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                                     ctypes.c_float, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "gqa_paged_decode_static_scratch": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I,
                                             _I, _I, _I, ctypes.c_float, _I, _I, _P, _P, _P]),
    "gqa_paged_prefill_workspace_size": (_SZ, [_I, _I, _I]),
    "gqa_paged_decode_kernel_launches": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "gqa_paged_prefill": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I,
                               ctypes.c_float, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "lse_combine": (_I, [_P, _P, _I, _I, _I, _P, _P, _P]),
    "gqa_paged_gather": (_I, [_P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "gqa_paged_append_kv": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _I, _I,
                                 _P, _P]),
    "gqa_paged_append_decode": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I,
                                     _I, _I, _I, ctypes.c_float, _I, _I, _P, _P, _P, _SZ, _P]),
    "gqa_get_error": (_I, [_P, _P]),
    "gqa_status_string": (ctypes.c_char_p, [_I]),
}


class GQAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")


def load(path: Optional[str] = None):
    """Load the library (building it first if the sources are newer).  Raises when it
    cannot be built or loaded."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if path is None and (not os.path.exists(p) or _build._stale()):
        _build.build()
    if not os.path.exists(p):
        raise RuntimeError(f"libgqa_paged.so not found at {p}: the CUDA extension is required")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().gqa_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != GQA_OK:
        raise GQAError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


_KV_DTYPES = (torch.bfloat16, torch.uint8, torch.float8_e4m3fn)


def _kv_code(t: torch.Tensor) -> int:
    return GQA_KV_BF16 if t.dtype == torch.bfloat16 else GQA_KV_FP8_E4M3


# ------------------------------------------------------------------------ raw ABI names

def gqa_pick_splits(B: int, Hk: int, max_seq_len: int, page_size: int, kv_dtype: int = 0) -> int:
    return load().gqa_pick_splits(B, Hk, max_seq_len, page_size, kv_dtype)


def gqa_paged_decode_workspace_size(B, Hq, Hk, head_dim, page_size, max_seq_len, kv_dtype,
                                    num_splits) -> int:
    return load().gqa_paged_decode_workspace_size(B, Hq, Hk, head_dim, page_size, max_seq_len,
                                                  kv_dtype, num_splits)


def gqa_paged_decode_kernel_launches(B, Hq, Hk, head_dim, page_size, max_seq_len, kv_dtype,
                                     num_splits, pack_gqa=True) -> int:
    return load().gqa_paged_decode_kernel_launches(B, Hq, Hk, head_dim, page_size, max_seq_len,
                                                   kv_dtype, num_splits, 1 if pack_gqa else 0)


def gqa_paged_prefill_workspace_size(total_q, Hq, head_dim) -> int:
    return load().gqa_paged_prefill_workspace_size(total_q, Hq, head_dim)


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled, 256-byte aligned workspace of at least nbytes."""
    n = (max(int(nbytes), 256) + 255) // 256 * 256
    return torch.zeros(n, dtype=torch.uint8, device=device)


def gqa_paged_decode(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                     page_table: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                     num_splits: int = 0, pack_gqa: bool = True,
                     k_scale: Optional[torch.Tensor] = None,
                     v_scale: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, want_lse: bool = True,
                     stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Paged GQA decode.  q bf16 [B][Hq][D]; pools [num_pages][Hk][P][D] bf16 or e4m3
    (uint8/float8_e4m3fn with fp32 scales [num_pages][Hk]); page_table int32 [B][pt_stride];
    seq_lens int32 [B].  Returns (out bf16 [B][Hq][D], lse fp32 [B][Hq] or None)."""
    _need(q, "q", torch.bfloat16)
    B, Hq, D = q.shape
    _need(k_pages, "k_pages", _KV_DTYPES)
    _need(v_pages, "v_pages", k_pages.dtype, k_pages.shape)
    num_pages, Hk, P, D2 = k_pages.shape
    if D2 != D:
        raise ValueError("head_dim of q and the KV pools differ")
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B][pt_stride]")
    kv_dtype = _kv_code(k_pages)
    if kv_dtype == GQA_KV_FP8_E4M3:
        if k_scale is None or v_scale is None:
            raise ValueError("fp8 KV needs k_scale and v_scale")
        _need(k_scale, "k_scale", torch.float32, (num_pages, Hk))
        _need(v_scale, "v_scale", torch.float32, (num_pages, Hk))
    pt_stride = page_table.shape[1]
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq))
    need = gqa_paged_decode_workspace_size(B, Hq, Hk, D, P, pt_stride * P, kv_dtype, num_splits)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    _need(workspace, "workspace", torch.uint8)
    st = load().gqa_paged_decode(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale), _ptr(v_scale), kv_dtype,
        _ptr(page_table), pt_stride, _ptr(seq_lens), B, Hq, Hk, D, P, num_pages, float(scale),
        int(num_splits), int(bool(pack_gqa)), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check("gqa_paged_decode", st)
    return out, lse


def gqa_paged_decode_partial(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                             page_table: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                             num_splits: int = 0, pack_gqa: bool = True,
                             k_scale: Optional[torch.Tensor] = None,
                             v_scale: Optional[torch.Tensor] = None,
                             o_part: Optional[torch.Tensor] = None,
                             lse_part: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None,
                             stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode over the tokens page_table / seq_lens cover, as one split's fp32 partial
    result: (o_part fp32 [B][Hq][D] normalised, lse_part fp32 [B][Hq]), the inputs
    lse_combine merges."""
    _need(q, "q", torch.bfloat16)
    B, Hq, D = q.shape
    _need(k_pages, "k_pages", _KV_DTYPES)
    _need(v_pages, "v_pages", k_pages.dtype, k_pages.shape)
    num_pages, Hk, P, D2 = k_pages.shape
    if D2 != D:
        raise ValueError("head_dim of q and the KV pools differ")
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B][pt_stride]")
    kv_dtype = _kv_code(k_pages)
    if kv_dtype == GQA_KV_FP8_E4M3:
        if k_scale is None or v_scale is None:
            raise ValueError("fp8 KV needs k_scale and v_scale")
        _need(k_scale, "k_scale", torch.float32, (num_pages, Hk))
        _need(v_scale, "v_scale", torch.float32, (num_pages, Hk))
    pt_stride = page_table.shape[1]
    if o_part is None:
        o_part = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    _need(o_part, "o_part", torch.float32, (B, Hq, D))
    if lse_part is None:
        lse_part = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    _need(lse_part, "lse_part", torch.float32, (B, Hq))
    need = gqa_paged_decode_workspace_size(B, Hq, Hk, D, P, pt_stride * P, kv_dtype, num_splits)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    _need(workspace, "workspace", torch.uint8)
    st = load().gqa_paged_decode_partial(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale), _ptr(v_scale), kv_dtype,
        _ptr(page_table), pt_stride, _ptr(seq_lens), B, Hq, Hk, D, P, num_pages, float(scale),
        int(num_splits), int(bool(pack_gqa)), _ptr(o_part), _ptr(lse_part), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check("gqa_paged_decode_partial", st)
    return o_part, lse_part


def gqa_paged_decode_static_scratch(q: torch.Tensor, k_pages: torch.Tensor,
                                    v_pages: torch.Tensor, page_table: torch.Tensor,
                                    seq_lens: torch.Tensor, scale: float, num_splits: int = 0,
                                    pack_gqa: bool = True,
                                    k_scale: Optional[torch.Tensor] = None,
                                    v_scale: Optional[torch.Tensor] = None,
                                    out: Optional[torch.Tensor] = None,
                                    lse: Optional[torch.Tensor] = None,
                                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """gqa_paged_decode without a workspace: the library's fixed scratch array is used
    (for callers that cannot allocate device memory; see include/gqa_paged.h).  `out` and
    `lse` must be passed in by such callers; they are only created here for convenience."""
    _need(q, "q", torch.bfloat16)
    B, Hq, D = q.shape
    _need(k_pages, "k_pages", _KV_DTYPES)
    _need(v_pages, "v_pages", k_pages.dtype, k_pages.shape)
    num_pages, Hk, P, _ = k_pages.shape
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    kv_dtype = _kv_code(k_pages)
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    st = load().gqa_paged_decode_static_scratch(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale), _ptr(v_scale), kv_dtype,
        _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B, Hq, Hk, D, P, num_pages,
        float(scale), int(num_splits), int(bool(pack_gqa)), _ptr(out), _ptr(lse),
        _stream(stream))
    _check("gqa_paged_decode_static_scratch", st)
    return out, lse


def _append_args(k_new, v_new, k_pages, v_pages, page_table, seq_lens, k_scale, v_scale):
    _need(k_pages, "k_pages", _KV_DTYPES)
    _need(v_pages, "v_pages", k_pages.dtype, k_pages.shape)
    num_pages, Hk, P, D = k_pages.shape
    _need(seq_lens, "seq_lens", torch.int32)
    B = seq_lens.shape[0]
    _need(k_new, "k_new", torch.bfloat16, (B, Hk, D))
    _need(v_new, "v_new", torch.bfloat16, (B, Hk, D))
    _need(page_table, "page_table", torch.int32)
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B][pt_stride]")
    kv_dtype = _kv_code(k_pages)
    if kv_dtype == GQA_KV_FP8_E4M3:
        if k_scale is None or v_scale is None:
            raise ValueError("fp8 KV needs k_scale and v_scale")
        _need(k_scale, "k_scale", torch.float32, (num_pages, Hk))
        _need(v_scale, "v_scale", torch.float32, (num_pages, Hk))
    return B, Hk, D, P, num_pages, kv_dtype


def gqa_paged_append_kv(k_new: torch.Tensor, v_new: torch.Tensor, k_pages: torch.Tensor,
                        v_pages: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor,
                        k_scale: Optional[torch.Tensor] = None,
                        v_scale: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Write token seq_lens[b] - 1 of every sequence (k_new / v_new bf16 [B][Hk][D]) into
    the paged cache, in place (e4m3 pools quantise it; see include/gqa_paged.h).  Returns
    the workspace holding the error word."""
    B, Hk, D, P, num_pages, kv_dtype = _append_args(k_new, v_new, k_pages, v_pages, page_table,
                                                     seq_lens, k_scale, v_scale)
    if workspace is None:
        workspace = new_workspace(256, k_pages.device)
    _need(workspace, "workspace", torch.uint8)
    st = load().gqa_paged_append_kv(
        _ptr(k_new), _ptr(v_new), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale), _ptr(v_scale),
        kv_dtype, _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B, Hk, D, P, num_pages,
        _ptr(workspace), _stream(stream))
    _check("gqa_paged_append_kv", st)
    return workspace


def gqa_paged_append_decode(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                            k_pages: torch.Tensor, v_pages: torch.Tensor,
                            page_table: torch.Tensor, seq_lens: torch.Tensor, scale: float,
                            num_splits: int = 0, pack_gqa: bool = True,
                            k_scale: Optional[torch.Tensor] = None,
                            v_scale: Optional[torch.Tensor] = None,
                            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None, want_lse: bool = True,
                            stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """gqa_paged_append_kv then gqa_paged_decode on one stream."""
    _need(q, "q", torch.bfloat16)
    B, Hk, D, P, num_pages, kv_dtype = _append_args(k_new, v_new, k_pages, v_pages, page_table,
                                                     seq_lens, k_scale, v_scale)
    Bq, Hq, Dq = q.shape
    if Bq != B or Dq != D:
        raise ValueError("q must be [B][Hq][head_dim] with the pools' head_dim")
    pt_stride = page_table.shape[1]
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq))
    need = gqa_paged_decode_workspace_size(B, Hq, Hk, D, P, pt_stride * P, kv_dtype, num_splits)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    _need(workspace, "workspace", torch.uint8)
    st = load().gqa_paged_append_decode(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale),
        _ptr(v_scale), kv_dtype, _ptr(page_table), pt_stride, _ptr(seq_lens), B, Hq, Hk, D, P,
        num_pages, float(scale), int(num_splits), int(bool(pack_gqa)), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check("gqa_paged_append_decode", st)
    return out, lse


def gqa_paged_prefill(q: torch.Tensor, cu_q: torch.Tensor, k_pages: torch.Tensor,
                      v_pages: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor,
                      scale: float, max_q_len: int, causal: bool = True,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, want_lse: bool = True,
                      stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Causal chunked prefill.  q bf16 [total_q][Hq][D]; cu_q int32 [B+1]; bf16 pools."""
    _need(q, "q", torch.bfloat16)
    T, Hq, D = q.shape
    _need(k_pages, "k_pages", torch.bfloat16)
    _need(v_pages, "v_pages", torch.bfloat16, k_pages.shape)
    num_pages, Hk, P, D2 = k_pages.shape
    if D2 != D:
        raise ValueError("head_dim of q and the KV pools differ")
    B = seq_lens.shape[0]
    _need(cu_q, "cu_q", torch.int32, (B + 1,))
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    pt_stride = page_table.shape[1]
    if out is None:
        out = torch.empty(T, Hq, D, dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (T, Hq, D))
    if lse is None and want_lse:
        lse = torch.empty(T, Hq, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (T, Hq))
    if workspace is None:
        workspace = new_workspace(gqa_paged_prefill_workspace_size(T, Hq, D), q.device)
    st = load().gqa_paged_prefill(
        _ptr(q), _ptr(cu_q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), pt_stride,
        _ptr(seq_lens), B, Hq, Hk, D, P, num_pages, float(scale), int(bool(causal)), T,
        int(max_q_len), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream))
    _check("gqa_paged_prefill", st)
    return out, lse


def lse_combine(o_part: torch.Tensor, lse_part: torch.Tensor,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Merge split results: o_part fp32 [S][rows][D], lse_part fp32 [S][rows]."""
    _need(o_part, "o_part", torch.float32)
    S, rows, D = o_part.shape
    _need(lse_part, "lse_part", torch.float32, (S, rows))
    if out is None:
        out = torch.empty(rows, D, dtype=torch.bfloat16, device=o_part.device)
    _need(out, "out", torch.bfloat16, (rows, D))
    if lse is None:
        lse = torch.empty(rows, dtype=torch.float32, device=o_part.device)
    _need(lse, "lse", torch.float32, (rows,))
    st = load().lse_combine(_ptr(o_part), _ptr(lse_part), S, rows, D, _ptr(out), _ptr(lse),
                            _stream(stream))
    _check("lse_combine", st)
    return out, lse


def gqa_paged_gather(k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
                     seq_lens: torch.Tensor, cu_kv: torch.Tensor, total: int,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Bit-exact copy-out of the paged cache: returns (k, v) [total][Hk][D]."""
    _need(k_pages, "k_pages", _KV_DTYPES)
    _need(v_pages, "v_pages", k_pages.dtype, k_pages.shape)
    num_pages, Hk, P, D = k_pages.shape
    B = seq_lens.shape[0]
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(cu_kv, "cu_kv", torch.int64, (B + 1,))
    ko = torch.empty(total, Hk, D, dtype=k_pages.dtype, device=k_pages.device)
    vo = torch.empty_like(ko)
    st = load().gqa_paged_gather(_ptr(k_pages), _ptr(v_pages), _ptr(page_table),
                                 page_table.shape[1], _ptr(seq_lens), _ptr(cu_kv), B, Hk, D, P,
                                 num_pages, k_pages.element_size(), _ptr(ko), _ptr(vo),
                                 _stream(stream))
    _check("gqa_paged_gather", st)
    return ko, vo


def gqa_get_error(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream, return and clear the device error word of `workspace`."""
    _need(workspace, "workspace", torch.uint8)
    return load().gqa_get_error(_ptr(workspace), _stream(stream))


# ------------------------------------------------------------------------ sparse decode

def _sparse_common(q, k_pages, page_table, seq_lens):
    _need(q, "q", torch.bfloat16)
    B, Hq, D = q.shape
    _need(k_pages, "k_pages", torch.bfloat16)
    num_pages, Hk, P, D2 = k_pages.shape
    if D2 != D:
        raise ValueError("head_dim of q and the KV pools differ")
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B][pt_stride]")
    return B, Hq, Hk, D, P, num_pages, page_table.shape[1]


def new_kt_cache(k_pages: torch.Tensor) -> torch.Tensor:
    """An empty KT cache for a bf16 pool: bf16 [num_pages][Hk][D][2]."""
    num_pages, Hk, P, D = k_pages.shape
    return torch.zeros(num_pages, Hk, D, 2, dtype=torch.bfloat16, device=k_pages.device)


def gqa_paged_kt_build(k_pages: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor,
                       kt: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """KT entries (per page and kv head: min and max of the keys over the valid tokens)
    of every page the sequences reference; returns kt bf16 [num_pages][Hk][D][2]."""
    _need(k_pages, "k_pages", torch.bfloat16)
    num_pages, Hk, P, D = k_pages.shape
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32)
    B = seq_lens.shape[0]
    if kt is None:
        kt = new_kt_cache(k_pages)
    _need(kt, "kt", torch.bfloat16, (num_pages, Hk, D, 2))
    if workspace is None:
        workspace = new_workspace(256, k_pages.device)
    st = load().gqa_paged_kt_build(_ptr(k_pages), _ptr(page_table), page_table.shape[1],
                                   _ptr(seq_lens), B, Hk, D, P, num_pages, _ptr(kt),
                                   _ptr(workspace), _stream(stream))
    _check("gqa_paged_kt_build", st)
    return kt


def gqa_paged_kt_append(k_new: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor,
                        kt: torch.Tensor, page_size: int,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Update the KT entries with the token at position seq_lens[b] - 1 (k_new bf16
    [B][Hk][D]), in place."""
    _need(k_new, "k_new", torch.bfloat16)
    B, Hk, D = k_new.shape
    _need(kt, "kt", torch.bfloat16)
    num_pages = kt.shape[0]
    _need(page_table, "page_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if workspace is None:
        workspace = new_workspace(256, kt.device)
    st = load().gqa_paged_kt_append(_ptr(k_new), _ptr(page_table), page_table.shape[1],
                                    _ptr(seq_lens), B, Hk, D, int(page_size), num_pages, _ptr(kt),
                                    _ptr(workspace), _stream(stream))
    _check("gqa_paged_kt_append", st)
    return kt


def gqa_paged_sparse_table_stride(pt_stride: int, page_size: int, topk: int, window: int) -> int:
    return load().gqa_paged_sparse_table_stride(pt_stride, page_size, topk, window)


def gqa_paged_sparse_select(q: torch.Tensor, kt: torch.Tensor, k_pages: torch.Tensor,
                            page_table: torch.Tensor, seq_lens: torch.Tensor, topk: int,
                            window: int, workspace: Optional[torch.Tensor] = None,
                            stream=None):
    """The chosen pages: returns (sel_table int32 [B*Hk][ss] of physical*Hk + kv head,
    sel_lens int32 [B*Hk], sel_pages int32 [B*Hk][ss] logical pages)."""
    B, Hq, Hk, D, P, num_pages, pts = _sparse_common(q, k_pages, page_table, seq_lens)
    _need(kt, "kt", torch.bfloat16, (num_pages, Hk, D, 2))
    ss = gqa_paged_sparse_table_stride(pts, P, topk, window)
    dev = q.device
    sel_table = torch.full((B * Hk, max(ss, 1)), -1, dtype=torch.int32, device=dev)
    sel_pages = torch.full((B * Hk, max(ss, 1)), -1, dtype=torch.int32, device=dev)
    sel_lens = torch.zeros(B * Hk, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_workspace(load().gqa_paged_sparse_select_workspace_size(B, Hk, pts), dev)
    st = load().gqa_paged_sparse_select(_ptr(q), _ptr(kt), _ptr(page_table), pts, _ptr(seq_lens),
                                        B, Hq, Hk, D, P, num_pages, int(topk), int(window),
                                        _ptr(sel_table), max(ss, 1), _ptr(sel_lens),
                                        _ptr(sel_pages), _ptr(workspace), workspace.numel(),
                                        _stream(stream))
    _check("gqa_paged_sparse_select", st)
    return sel_table, sel_lens, sel_pages


def gqa_paged_sparse_decode_workspace_size(B, Hq, Hk, head_dim, page_size, pt_stride, topk,
                                           window, num_splits=0) -> int:
    return load().gqa_paged_sparse_decode_workspace_size(B, Hq, Hk, head_dim, page_size,
                                                         pt_stride, topk, window, num_splits)


def gqa_paged_sparse_decode(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                            kt: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor,
                            scale: float, topk: int, window: int, num_splits: int = 0,
                            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None, want_lse: bool = True,
                            stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Page-level top-K sparse decode (bf16 pools): the window pages plus the topk
    best-scoring earlier pages of every (sequence, kv head) are attended."""
    B, Hq, Hk, D, P, num_pages, pts = _sparse_common(q, k_pages, page_table, seq_lens)
    _need(v_pages, "v_pages", torch.bfloat16, k_pages.shape)
    _need(kt, "kt", torch.bfloat16, (num_pages, Hk, D, 2))
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq))
    need = gqa_paged_sparse_decode_workspace_size(B, Hq, Hk, D, P, pts, topk, window, num_splits)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    _need(workspace, "workspace", torch.uint8)
    st = load().gqa_paged_sparse_decode(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(kt), _ptr(page_table), pts, _ptr(seq_lens),
        B, Hq, Hk, D, P, num_pages, float(scale), int(topk), int(window), int(num_splits),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream))
    _check("gqa_paged_sparse_decode", st)
    return out, lse
