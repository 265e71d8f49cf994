"""ctypes binding over libattn.so: argument marshalling only.

torch is used here for device memory (output and workspace tensors) and for the current CUDA
stream; every step of the computation runs in the library's CUDA kernels. If the shared library has
not been built, the first call raises -- there is no other code path.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn.so")

STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_ALIGNMENT",
          4: "ATTN_ERR_WORKSPACE", 5: "ATTN_ERR_LAUNCH", 6: "ATTN_ERR_TIMEOUT"}

# (name, restype, argtypes) for every symbol include/attn.h declares
_P, _I, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_DIMS = [_I] * 6 + [_I, _F, _P]  # B, Hq, Hkv, Sq, Sk, D, causal, scale, stream
SIGNATURES = [
    ("attn_fwd", _I, [_P] * 5 + _DIMS),
    ("attn_fwd_f32", _I, [_P] * 5 + _DIMS),
    # q, k, v, o, lse, q_scale, k_scale, v_scale, B, Hq, Hkv, Sq, Sk, D, causal, scale, stream
    ("attn_fwd_fp8", _I, [_P] * 5 + [_F] * 3 + _DIMS),
    ("attn_bwd_workspace_size", _S, [_I] * 6),
    ("attn_bwd", _I, [_P] * 9 + [_P, _S] + _DIMS),
    ("attn_bwd_f32_workspace_size", _S, [_I] * 6),
    ("attn_bwd_f32", _I, [_P] * 9 + [_P, _S] + _DIMS),
    # q, k, v, o, lse, cu_q, cu_k, B, max_sq, max_sk, total_q, total_k, Hq, Hkv, D, causal, scale, stream
    ("attn_fwd_varlen", _I, [_P] * 7 + [_I] * 9 + [_F, _P]),
    ("attn_bwd_varlen_workspace_size", _S, [_I] * 6),
    # q, k, v, o, lse, dout, dq, dk, dv, cu_q, cu_k, B, max_sq, max_sk, total_q, total_k, Hq, Hkv, D,
    # causal, scale, workspace, workspace_bytes, stream
    ("attn_bwd_varlen", _I, [_P] * 11 + [_I] * 9 + [_F, _P, _S, _P]),
    ("attn_decode_workspace_size", _S, [_I] * 4),
    ("attn_decode_splitkv", _I, [_P] * 5 + [_I] + [_P, _P] + [_I] * 4 + [_F, _P, _S, _P]),
    ("attn_decode_splitkv_static", _I, [_P] * 5 + [_I] + [_P, _P] + [_I] * 4 + [_F, _P]),
    ("attn_decode_default_splits", _I, [_I, _I]),
    # q, k_pages, v_pages, block_table, max_pages, seq_lens, page_size, num_pages, num_splits,
    # max_splits, o, lse, N, Hq, Hkv, D, scale, workspace, workspace_bytes, stream
    ("attn_decode_paged", _I, [_P] * 4 + [_I, _P, _I, _I, _P, _I, _P, _P] + [_I] * 4 + [_F, _P, _S, _P]),
    # q, k, v, kv_offsets, num_splits, max_splits, o, lse, N, q_len, Hq, Hkv, D, scale, workspace,
    # workspace_bytes, stream
    ("attn_decode_splitkv_qlen", _I, [_P] * 5 + [_I] + [_P, _P] + [_I] * 5 + [_F, _P, _S, _P]),
    # as attn_decode_paged with q_len after N
    ("attn_decode_paged_qlen", _I, [_P] * 4 + [_I, _P, _I, _I, _P, _I, _P, _P] + [_I] * 5 + [_F, _P, _S, _P]),
    # o_acc, lse_acc, o_part, lse_part, o_out, B, S, H, D, stream
    ("attn_merge", _I, [_P] * 5 + [_I] * 4 + [_P]),
    ("attn_status_string", ctypes.c_char_p, [_I]),
    ("attn_get_device_status", _I, [_P]),
    ("attn_launch_count", ctypes.c_uint64, []),
    ("attn_last_path", ctypes.c_char_p, [_I]),
    ("attn_profile_start", _I, []),
    ("attn_profile_stop", _I, []),
    ("attn_profile_entries", _I, []),
    ("attn_profile_name", ctypes.c_char_p, [_I]),
    ("attn_profile_total_ms", ctypes.c_double, [_I]),
    ("attn_profile_launches", _I, [_I]),
]

_lib = None


class AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """Load libattn.so (once) and declare its C signatures."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libattn.so is not built ({LIB_PATH}); run "
                              f"`python -m online_softmax_attention_fwd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise AttnError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    # a plain int: ctypes passes it as the declared void* without building a c_void_p object
    return None if t is None else t.data_ptr()


# torch's raw current-stream query skips building a Stream object (about 3 us per call); the public
# call is the fallback where it is missing
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream():
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _expect(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-D tensor")


def _prefill_dims(q, k, v):
    B, Sq, Hq, D = q.shape
    Bk, Sk, Hkv, Dk = k.shape
    if Bk != B or Dk != D or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    return B, Hq, Hkv, Sq, Sk, D


def _fwd(fn, dtype, q, k, v, causal, scale, out, lse):
    for n, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, n, dtype, 4)
    B, Hq, Hkv, Sq, Sk, D = _prefill_dims(q, k, v)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(fn, getattr(lib(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
                                  int(bool(causal)), scale, _stream()))
    return o, lse


def fwd(q, k, v, causal: bool = False, scale: Optional[float] = None, out=None, lse=None):
    """bf16 forward: (O [B,Sq,Hq,D] bf16, lse [B,Hq,Sq] fp32) via attn_fwd (tcgen05 kernel)."""
    return _fwd("attn_fwd", torch.bfloat16, q, k, v, causal, scale, out, lse)


def fwd_f32(q, k, v, causal: bool = False, scale: Optional[float] = None, out=None, lse=None):
    """fp32 forward via attn_fwd_f32 (CUDA-core fp32 kernel, no TF32)."""
    return _fwd("attn_fwd_f32", torch.float32, q, k, v, causal, scale, out, lse)


def fwd_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float, causal: bool = False,
            scale: Optional[float] = None, out=None, lse=None):
    """FP8 forward via attn_fwd_fp8: q, k, v are E4M3 codes as uint8 tensors [B,S,H,128] (e.g.
    ``x.to(torch.float8_e4m3fn).view(torch.uint8)``) with per-tensor scales; returns
    (O [B,Sq,Hq,128] bf16, lse [B,Hq,Sq] fp32)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, n, torch.uint8, 4)
    B, Hq, Hkv, Sq, Sk, D = _prefill_dims(q, k, v)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check("attn_fwd_fp8", lib().attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), float(q_scale),
                                              float(k_scale), float(v_scale), B, Hq, Hkv, Sq, Sk, D,
                                              int(bool(causal)), scale, _stream()))
    return o, lse


def _bwd(fn, wsfn, dtype, q, k, v, o, lse, do, causal, scale, workspace, out=None):
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", do)):
        _expect(t, n, dtype, 4)
    _expect(lse, "lse", torch.float32, 3)
    B, Hq, Hkv, Sq, Sk, D = _prefill_dims(q, k, v)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq, dk, dv = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) if out is None else out
    need = getattr(lib(), wsfn)(B, Hq, Hkv, Sq, Sk, D)
    if workspace is None:
        workspace = torch.empty(max(int(need), 256), dtype=torch.uint8, device=q.device)
    _check(fn, getattr(lib(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _ptr(workspace), workspace.numel(), B, Hq, Hkv, Sq, Sk, D,
                                  int(bool(causal)), scale, _stream()))
    return dq, dk, dv


def bwd(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None, workspace=None, out=None):
    """bf16 backward via attn_bwd: returns (dQ, dK, dV) bf16 (written into `out` if given)."""
    return _bwd("attn_bwd", "attn_bwd_workspace_size", torch.bfloat16, q, k, v, o, lse, do, causal, scale,
                workspace, out)


def bwd_f32(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None, workspace=None,
            out=None):
    """fp32 backward via attn_bwd_f32: returns (dQ, dK, dV) fp32 (written into `out` if given)."""
    return _bwd("attn_bwd_f32", "attn_bwd_f32_workspace_size", torch.float32, q, k, v, o, lse, do, causal,
                scale, workspace, out)


def _varlen_dims(q, k, v, cu_q, cu_k, max_seqlen_q, max_seqlen_k):
    _expect(cu_q, "cu_seqlens_q", torch.int32, 1)
    _expect(cu_k, "cu_seqlens_k", torch.int32, 1)
    Tq, Hq, D = q.shape
    Tk, Hkv, Dk = k.shape
    if Dk != D or tuple(v.shape) != tuple(k.shape) or cu_q.numel() != cu_k.numel() or cu_q.numel() < 2:
        raise ValueError("shape mismatch in packed prefill arguments")
    B = cu_q.numel() - 1
    if max_seqlen_q is None or max_seqlen_k is None:
        # host-side bounds from the offsets (one device-to-host read); pass them to avoid it
        lq = torch.diff(cu_q).max().item()
        lk = torch.diff(cu_k).max().item()
        max_seqlen_q = int(lq) if max_seqlen_q is None else max_seqlen_q
        max_seqlen_k = int(lk) if max_seqlen_k is None else max_seqlen_k
    return B, Tq, Tk, Hq, Hkv, D, max(1, int(max_seqlen_q)), max(1, int(max_seqlen_k))


def fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q=None, max_seqlen_k=None, causal: bool = False,
               scale: Optional[float] = None, out=None, lse=None):
    """Packed variable-length forward via attn_fwd_varlen: q [Tq, Hq, D], k, v [Tk, Hkv, D] bf16,
    cu_seqlens [B+1] int32; returns (O [Tq, Hq, D] bf16, lse [Hq, Tq] fp32)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, n, torch.bfloat16, 3)
    B, Tq, Tk, Hq, Hkv, D, mq, mk = _varlen_dims(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((Hq, Tq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check("attn_fwd_varlen", lib().attn_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, mq, mk, Tq, Tk,
        Hq, Hkv, D, int(bool(causal)), scale, _stream()))
    return o, lse


def bwd_varlen(q, k, v, o, lse, do, cu_seqlens_q, cu_seqlens_k, max_seqlen_q=None, max_seqlen_k=None,
               causal: bool = False, scale: Optional[float] = None, workspace=None, out=None):
    """Packed variable-length backward via attn_bwd_varlen: returns (dQ, dK, dV) bf16."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", do)):
        _expect(t, n, torch.bfloat16, 3)
    _expect(lse, "lse", torch.float32, 2)
    B, Tq, Tk, Hq, Hkv, D, mq, mk = _varlen_dims(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq, dk, dv = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) if out is None else out
    need = int(lib().attn_bwd_varlen_workspace_size(B, Hq, Hkv, mq, mk, D))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check("attn_bwd_varlen", lib().attn_bwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(cu_seqlens_q),
        _ptr(cu_seqlens_k), B, mq, mk, Tq, Tk, Hq, Hkv, D, int(bool(causal)), scale, _ptr(workspace),
        workspace.numel(), _stream()))
    return dq, dk, dv


def bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D) -> int:
    return int(lib().attn_bwd_workspace_size(B, Hq, Hkv, Sq, Sk, D))


def decode_workspace_size(N, Hq, D, max_splits) -> int:
    return int(lib().attn_decode_workspace_size(N, Hq, D, max_splits))


def default_splits(L: int, max_splits: int = 16) -> int:
    return int(lib().attn_decode_default_splits(int(L), int(max_splits)))


def decode(q, k, v, kv_offsets, num_splits=None, max_splits: int = 16, scale: Optional[float] = None,
           want_lse: bool = True, out=None, lse=None, workspace=None):
    """Split-KV decode. q [N, Hq, D] (one query token per stream) calls attn_decode_splitkv and
    returns (O [N, Hq, D] bf16, lse [N, Hq] fp32 or None); q [N, q_len, Hq, D] (several tokens per
    stream, the newest q_len positions of each cache) calls attn_decode_splitkv_qlen and returns
    (O [N, q_len, Hq, D], lse [N, Hq, q_len] or None)."""
    multi = isinstance(q, torch.Tensor) and q.dim() == 4
    _expect(q, "q", torch.bfloat16, 4 if multi else 3)
    _expect(k, "k", torch.bfloat16, 3)
    _expect(v, "v", torch.bfloat16, 3)
    _expect(kv_offsets, "kv_offsets", torch.int32, 1)
    if num_splits is not None:
        _expect(num_splits, "num_splits", torch.int32, 1)
    if multi:
        N, q_len, Hq, D = q.shape
    else:
        (N, Hq, D), q_len = q.shape, 1
    Hkv = k.shape[1]
    if tuple(v.shape) != tuple(k.shape) or k.shape[2] != D or kv_offsets.numel() != N + 1:
        raise ValueError("shape mismatch in decode arguments")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    if want_lse and lse is None:
        shape = (N, Hq, q_len) if multi else (N, Hq)
        lse = torch.empty(shape, dtype=torch.float32, device=q.device)
    need = decode_workspace_size(N * q_len, Hq, D, max_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    L = lib()
    if multi:
        _check("attn_decode_splitkv_qlen", L.attn_decode_splitkv_qlen(
            _ptr(q), _ptr(k), _ptr(v), _ptr(kv_offsets), _ptr(num_splits), int(max_splits), _ptr(o),
            _ptr(lse) if want_lse else None, N, q_len, Hq, Hkv, D, scale, _ptr(workspace), workspace.numel(),
            _stream()))
    else:
        _check("attn_decode_splitkv", L.attn_decode_splitkv(
            _ptr(q), _ptr(k), _ptr(v), _ptr(kv_offsets), _ptr(num_splits), int(max_splits), _ptr(o),
            _ptr(lse) if want_lse else None, N, Hq, Hkv, D, scale, _ptr(workspace), workspace.numel(), _stream()))
    return o, (lse if want_lse else None)


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_splits=None, max_splits: int = 16,
                 scale: Optional[float] = None, want_lse: bool = True, out=None, lse=None, workspace=None):
    """Split-KV decode over a paged cache via attn_decode_paged (q [N, Hq, D]) or
    attn_decode_paged_qlen (q [N, q_len, Hq, D]); returns (O like q, lse or None).

    k_pages, v_pages [num_pages, page_size, Hkv, D] bf16; block_table [N, max_pages] int32 page ids;
    seq_lens [N] int32. Key t of stream n is k_pages[block_table[n, t // page_size], t % page_size].
    """
    multi = isinstance(q, torch.Tensor) and q.dim() == 4
    _expect(q, "q", torch.bfloat16, 4 if multi else 3)
    _expect(k_pages, "k_pages", torch.bfloat16, 4)
    _expect(v_pages, "v_pages", torch.bfloat16, 4)
    _expect(block_table, "block_table", torch.int32, 2)
    _expect(seq_lens, "seq_lens", torch.int32, 1)
    if num_splits is not None:
        _expect(num_splits, "num_splits", torch.int32, 1)
    if multi:
        N, q_len, Hq, D = q.shape
    else:
        (N, Hq, D), q_len = q.shape, 1
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    if (tuple(v_pages.shape) != tuple(k_pages.shape) or k_pages.shape[3] != D or block_table.shape[0] != N
            or seq_lens.numel() != N):
        raise ValueError("shape mismatch in paged decode arguments")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    if want_lse and lse is None:
        shape = (N, Hq, q_len) if multi else (N, Hq)
        lse = torch.empty(shape, dtype=torch.float32, device=q.device)
    need = decode_workspace_size(N * q_len, Hq, D, max_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    L = lib()
    common = (int(page_size), int(num_pages), _ptr(num_splits), int(max_splits), _ptr(o),
              _ptr(lse) if want_lse else None)
    if multi:
        _check("attn_decode_paged_qlen", L.attn_decode_paged_qlen(
            _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), int(block_table.shape[1]), _ptr(seq_lens),
            *common, N, q_len, Hq, Hkv, D, scale, _ptr(workspace), workspace.numel(), _stream()))
    else:
        _check("attn_decode_paged", L.attn_decode_paged(
            _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), int(block_table.shape[1]), _ptr(seq_lens),
            *common, N, Hq, Hkv, D, scale, _ptr(workspace), workspace.numel(), _stream()))
    return o, (lse if want_lse else None)


def merge(o_acc, lse_acc, o_part, lse_part, o_out=None):
    """Folds a partial attention (o_part [B,S,H,D] bf16, lse_part [B,H,S] fp32) into the running
    result (o_acc fp32, lse_acc fp32, updated in place) via attn_merge; writes the merged O in bf16
    into o_out when given. Returns (o_acc, lse_acc)."""
    _expect(o_acc, "o_acc", torch.float32, 4)
    _expect(lse_acc, "lse_acc", torch.float32, 3)
    _expect(o_part, "o_part", torch.bfloat16, 4)
    _expect(lse_part, "lse_part", torch.float32, 3)
    if o_out is not None:
        _expect(o_out, "o_out", torch.bfloat16, 4)
    B, S, H, D = o_acc.shape
    if tuple(o_part.shape) != (B, S, H, D) or tuple(lse_acc.shape) != (B, H, S) or tuple(lse_part.shape) != (B, H, S):
        raise ValueError("shape mismatch in merge arguments")
    _check("attn_merge", lib().attn_merge(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part), _ptr(o_out),
                                          B, S, H, D, _stream()))
    return o_acc, lse_acc


def device_status() -> int:
    """Wait for the current stream, then read and clear the device status word (0 = ok)."""
    return int(lib().attn_get_device_status(_stream()))


def launch_count() -> int:
    return int(lib().attn_launch_count())


def last_path(kind: int) -> str:
    return lib().attn_last_path(int(kind)).decode()


def profile_start() -> None:
    _check("attn_profile_start", lib().attn_profile_start())


def profile_stop() -> dict:
    """Stop the per-kernel profiler; returns {kernel family: (total ms, launches)}."""
    _check("attn_profile_stop", lib().attn_profile_stop())
    L = lib()
    return {L.attn_profile_name(i).decode(): (float(L.attn_profile_total_ms(i)), int(L.attn_profile_launches(i)))
            for i in range(L.attn_profile_entries())}
