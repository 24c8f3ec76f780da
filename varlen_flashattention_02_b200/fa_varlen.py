"""Python binding of libfa_varlen.so (include/fa_varlen.h).

Argument marshalling only: every step of the attention runs in the CUDA
kernels of the library. PyTorch provides device memory and the stream. If the
library is missing, importing this module raises; there is no fallback.

    out, lse = fa_varlen_fwd(q, k, v, cu_q, cu_k, max_q, max_k, scale, causal)
    dq, dk, dv = fa_varlen_bwd(dout, q, k, v, out, lse, cu_q, cu_k, max_q, max_k,
                               scale, causal)

q, k, v, dout: bf16 CUDA tensors [total_tokens, heads, head_dim], contiguous.
cu_q, cu_k: int32 CUDA tensors [batch + 1] of cumulative offsets.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_varlen.so")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK", 1: "FA_ERR_INVALID_ARGUMENT", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_WORKSPACE",
    4: "FA_ERR_CUDA", 5: "FA_ERR_BAD_SEQLENS", 6: "FA_ERR_DEVICE_TIMEOUT",
}


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class KvLayout(ctypes.Structure):
    """fa_kv_layout_t: where the keys and values of each sequence live."""
    _fields_ = [("cu_seqlens_k", ctypes.c_void_p), ("seqlens_k", ctypes.c_void_p), ("leftpad_k", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("cache_rows", ctypes.c_int), ("page_size", ctypes.c_int),
                ("max_pages_per_seq", ctypes.c_int), ("total_rows", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m varlen_flashattention_02_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.fa_varlen_fwd_workspace_size.argtypes = [I, I, I, I]
    lib.fa_varlen_fwd_workspace_size.restype = S
    lib.fa_varlen_bwd_workspace_size.argtypes = [I, I, I, I, I]
    lib.fa_varlen_bwd_workspace_size.restype = S
    lib.fa_varlen_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, ctypes.c_float, I, P, P, P, S, P]
    lib.fa_varlen_fwd.restype = I
    lib.fa_varlen_bwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, ctypes.c_float, I,
                                  P, P, P, P, S, P]
    lib.fa_varlen_bwd.restype = I
    lib.fa_varlen_fwd_gqa.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, ctypes.c_float, I, P, P, P, S, P]
    lib.fa_varlen_fwd_gqa.restype = I
    lib.fa_varlen_bwd_gqa.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, ctypes.c_float, I,
                                      P, P, P, P, S, P]
    lib.fa_varlen_bwd_gqa.restype = I
    lib.fa_varlen_bwd_deterministic.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, ctypes.c_float, I,
                                                P, P, P, P, S, P]
    lib.fa_varlen_bwd_deterministic.restype = I
    lib.fa_varlen_fwd_splitkv_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.fa_varlen_fwd_splitkv_workspace_size.restype = S
    lib.fa_varlen_fwd_splitkv.argtypes = [P, P, P, P, ctypes.POINTER(KvLayout), I, I, I, I, I, I, I,
                                          ctypes.c_float, I, I, P, P, P, S, P]
    lib.fa_varlen_fwd_splitkv.restype = I
    lib.fa_varlen_splitkv_num_splits.argtypes = [I, I, I, I, I, I]
    lib.fa_varlen_splitkv_num_splits.restype = I
    lib.fa_varlen_fwd_kvcache.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, ctypes.c_float, I, P, P, P, S, P]
    lib.fa_varlen_fwd_kvcache.restype = I
    lib.fa_varlen_fwd_paged.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, ctypes.c_float, I, P, P,
                                        P, S, P]
    lib.fa_varlen_fwd_paged.restype = I
    lib.fa_set_test_hooks.argtypes = [ctypes.c_uint64, I]
    lib.fa_set_test_hooks.restype = None
    lib.fa_get_device_status.argtypes = [P, P]
    lib.fa_get_device_status.restype = I
    lib.fa_varlen_fwd_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, ctypes.c_float, I, P, P, P]
    lib.fa_varlen_fwd_noalloc.restype = I
    lib.fa_set_kernel_events.argtypes = [P, I]
    lib.fa_set_kernel_events.restype = None
    lib.fa_status_string.argtypes = [I]
    lib.fa_status_string.restype = ctypes.c_char_p
    return lib


lib = _load()

EXPORTED = ("fa_varlen_fwd_workspace_size", "fa_varlen_bwd_workspace_size", "fa_varlen_fwd",
            "fa_varlen_bwd", "fa_varlen_fwd_gqa", "fa_varlen_bwd_gqa", "fa_varlen_fwd_kvcache",
            "fa_varlen_fwd_paged", "fa_varlen_bwd_deterministic", "fa_varlen_fwd_splitkv",
            "fa_varlen_fwd_splitkv_workspace_size", "fa_varlen_splitkv_num_splits", "fa_varlen_fwd_noalloc",
            "fa_get_device_status", "fa_set_kernel_events", "fa_status_string")


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(name, t, H=None, D=None):
    if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [tokens, heads, head_dim]")
    if H is not None and (t.shape[1] != H or t.shape[2] != D):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected [*, {H}, {D}]")


def _check_cu(name, t):
    if t.dtype != torch.int32 or t.dim() != 1 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor [batch + 1]")


def fwd_workspace_size(batch: int, total_q: int, heads: int, head_dim: int) -> int:
    return int(lib.fa_varlen_fwd_workspace_size(batch, total_q, heads, head_dim))


def bwd_workspace_size(batch: int, total_q: int, total_k: int, heads: int, head_dim: int) -> int:
    return int(lib.fa_varlen_bwd_workspace_size(batch, total_q, total_k, heads, head_dim))


def new_workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def fa_varlen_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                  softmax_scale: float, causal: bool, out=None, softmax_lse=None, workspace=None,
                  stream=None):
    """Forward. Returns (out bf16 [Tq,H,D], softmax_lse fp32 [H,Tq])."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    _check_qkv("k", k, H, D)
    _check_qkv("v", v, H, D)
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    _check_cu("cu_seqlens_k", cu_seqlens_k)
    batch = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if softmax_lse is None:
        softmax_lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    need = fwd_workspace_size(batch, Tq, H, D)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    rc = lib.fa_varlen_fwd(_p(q), _p(k), _p(v), _p(cu_seqlens_q), _p(cu_seqlens_k), batch, Tq,
                           k.shape[0], int(max_seqlen_q), int(max_seqlen_k), H, D,
                           float(softmax_scale), int(bool(causal)), _p(out), _p(softmax_lse),
                           _p(workspace), workspace.numel(), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_fwd")
    return out, softmax_lse


def fa_varlen_bwd(dout, q, k, v, out, softmax_lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                  max_seqlen_k: int, softmax_scale: float, causal: bool, dq=None, dk=None, dv=None,
                  workspace=None, stream=None):
    """Backward of sum(out * dout). Returns (dq, dk, dv), bf16, shaped like q, k, v."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    for name, t in (("k", k), ("v", v), ("dout", dout), ("out", out)):
        _check_qkv(name, t, H, D)
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    _check_cu("cu_seqlens_k", cu_seqlens_k)
    batch = cu_seqlens_q.numel() - 1
    Tk = k.shape[0]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_size(batch, Tq, Tk, H, D)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    rc = lib.fa_varlen_bwd(_p(dout), _p(q), _p(k), _p(v), _p(out), _p(softmax_lse), _p(cu_seqlens_q),
                           _p(cu_seqlens_k), batch, Tq, Tk, int(max_seqlen_q), int(max_seqlen_k), H, D,
                           float(softmax_scale), int(bool(causal)), _p(dq), _p(dk), _p(dv),
                           _p(workspace), workspace.numel(), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_bwd")
    return dq, dk, dv


def _kv_heads(H, k):
    Hk = k.shape[1]
    if Hk < 1 or H % Hk != 0:
        raise ValueError(f"query heads ({H}) must be a multiple of key/value heads ({Hk})")
    return Hk


def fa_varlen_fwd_gqa(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                      softmax_scale: float, causal: bool, out=None, softmax_lse=None, workspace=None,
                      stream=None):
    """Grouped-/multi-query forward: k and v have Hk heads, H a multiple of
    Hk; query head h reads key/value head h // (H // Hk). Returns (out,
    softmax_lse) as fa_varlen_fwd does."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    _check_qkv("k", k)
    Hk = _kv_heads(H, k)
    _check_qkv("k", k, Hk, D)
    _check_qkv("v", v, Hk, D)
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    _check_cu("cu_seqlens_k", cu_seqlens_k)
    batch = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if softmax_lse is None:
        softmax_lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    need = fwd_workspace_size(batch, Tq, H, D)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    rc = lib.fa_varlen_fwd_gqa(_p(q), _p(k), _p(v), _p(cu_seqlens_q), _p(cu_seqlens_k), batch, Tq,
                               k.shape[0], int(max_seqlen_q), int(max_seqlen_k), H, Hk, D,
                               float(softmax_scale), int(bool(causal)), _p(out), _p(softmax_lse),
                               _p(workspace), workspace.numel(), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_fwd_gqa")
    return out, softmax_lse


def fa_varlen_bwd_deterministic(dout, q, k, v, out, softmax_lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                                max_seqlen_k: int, softmax_scale: float, causal: bool, dq=None, dk=None, dv=None,
                                workspace=None, stream=None):
    """Backward whose results are bitwise identical from run to run (dQ
    contributions added in key-tile order). k, v may have fewer heads than q
    as in fa_varlen_bwd_gqa. Returns (dq, dk, dv)."""
    return fa_varlen_bwd_gqa(dout, q, k, v, out, softmax_lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                             max_seqlen_k, softmax_scale, causal, dq, dk, dv, workspace, stream, _deterministic=True)


def fa_varlen_bwd_gqa(dout, q, k, v, out, softmax_lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                      max_seqlen_k: int, softmax_scale: float, causal: bool, dq=None, dk=None, dv=None,
                      workspace=None, stream=None, _deterministic=False):
    """Grouped-/multi-query backward: dk, dv have Hk heads and hold the sums
    over each key/value head's query heads. Returns (dq, dk, dv)."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    _check_qkv("k", k)
    Hk = _kv_heads(H, k)
    for name, t in (("k", k), ("v", v)):
        _check_qkv(name, t, Hk, D)
    for name, t in (("dout", dout), ("out", out)):
        _check_qkv(name, t, H, D)
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    _check_cu("cu_seqlens_k", cu_seqlens_k)
    batch = cu_seqlens_q.numel() - 1
    Tk = k.shape[0]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_size(batch, Tq, Tk, H, D)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    fn = lib.fa_varlen_bwd_deterministic if _deterministic else lib.fa_varlen_bwd_gqa
    rc = fn(_p(dout), _p(q), _p(k), _p(v), _p(out), _p(softmax_lse), _p(cu_seqlens_q), _p(cu_seqlens_k), batch,
            Tq, Tk, int(max_seqlen_q), int(max_seqlen_k), H, Hk, D, float(softmax_scale), int(bool(causal)),
            _p(dq), _p(dk), _p(dv), _p(workspace), workspace.numel(), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_bwd_deterministic" if _deterministic else "fa_varlen_bwd_gqa")
    return dq, dk, dv


def fa_varlen_fwd_kvcache(q, k_cache, v_cache, cu_seqlens_q, seqlens_k, leftpad_k, max_seqlen_q: int,
                          softmax_scale: float, causal: bool, out=None, softmax_lse=None, workspace=None,
                          stream=None):
    """Forward over a key/value cache [batch, cache_rows, Hk, D]: sequence b's
    keys are rows leftpad_k[b] .. seqlens_k[b]-1 of slot b (leftpad_k may be
    None). Returns (out, softmax_lse) as fa_varlen_fwd does."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [batch, cache_rows, heads_k, head_dim]")
    batch, rows, Hk, Dk = k_cache.shape
    if tuple(v_cache.shape) != (batch, rows, Hk, Dk) or Dk != D:
        raise ValueError("k_cache and v_cache must both be [batch, cache_rows, heads_k, head_dim]")
    _kv_heads(H, k_cache[0])
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    for name, t in (("seqlens_k", seqlens_k), ("leftpad_k", leftpad_k)):
        if t is not None and (t.dtype != torch.int32 or t.dim() != 1 or t.numel() != batch or not t.is_cuda):
            raise ValueError(f"{name} must be an int32 CUDA tensor [batch]")
    if cu_seqlens_q.numel() - 1 != batch:
        raise ValueError("cu_seqlens_q must have batch + 1 entries")
    if out is None:
        out = torch.empty_like(q)
    if softmax_lse is None:
        softmax_lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    need = fwd_workspace_size(batch, Tq, H, D)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    rc = lib.fa_varlen_fwd_kvcache(_p(q), _p(k_cache), _p(v_cache), _p(cu_seqlens_q), _p(seqlens_k),
                                   _p(leftpad_k), batch, Tq, rows, int(max_seqlen_q), H, Hk, D,
                                   float(softmax_scale), int(bool(causal)), _p(out), _p(softmax_lse),
                                   _p(workspace), workspace.numel(), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_fwd_kvcache")
    return out, softmax_lse


def fa_varlen_fwd_paged(q, k_pages, v_pages, cu_seqlens_q, seqlens_k, block_table, max_seqlen_q: int,
                        max_seqlen_k: int, softmax_scale: float, causal: bool, out=None, softmax_lse=None,
                        workspace=None, stream=None):
    """Forward over a paged key/value cache: pools [num_pages, page_size, Hk,
    D] (page_size a multiple of 128), block_table int32 [batch, max_pages],
    seqlens_k int32 [batch]. Returns (out, softmax_lse) as fa_varlen_fwd."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    for name, t in (("k_pages", k_pages), ("v_pages", v_pages)):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [num_pages, page_size, heads_k, head_dim]")
    num_pages, page_size, Hk, Dk = k_pages.shape
    if tuple(v_pages.shape) != tuple(k_pages.shape) or Dk != D:
        raise ValueError("k_pages and v_pages must both be [num_pages, page_size, heads_k, head_dim]")
    _kv_heads(H, k_pages[0])
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    batch = cu_seqlens_q.numel() - 1
    if seqlens_k.dtype != torch.int32 or seqlens_k.numel() != batch or not seqlens_k.is_cuda:
        raise ValueError("seqlens_k must be an int32 CUDA tensor [batch]")
    if (block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != batch
            or not block_table.is_contiguous() or not block_table.is_cuda):
        raise ValueError("block_table must be a contiguous int32 CUDA tensor [batch, max_pages]")
    if out is None:
        out = torch.empty_like(q)
    if softmax_lse is None:
        softmax_lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    need = fwd_workspace_size(batch, Tq, H, D)
    if workspace is None:
        workspace = new_workspace(need, q.device)
    rc = lib.fa_varlen_fwd_paged(_p(q), _p(k_pages), _p(v_pages), _p(cu_seqlens_q), _p(seqlens_k),
                                 _p(block_table), batch, Tq, num_pages, page_size, block_table.shape[1],
                                 int(max_seqlen_q), int(max_seqlen_k), H, Hk, D, float(softmax_scale),
                                 int(bool(causal)), _p(out), _p(softmax_lse), _p(workspace), workspace.numel(),
                                 _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_fwd_paged")
    return out, softmax_lse


def fa_varlen_splitkv_num_splits(batch: int, max_seqlen_q: int, num_heads: int, num_heads_k: int,
                                 max_seqlen_k: int, sm_count: int = 0) -> int:
    """Advisory split count for :func:`fa_varlen_fwd_splitkv` (same name in
    the C ABI): the smallest count whose work units fill the SMs in nearly
    whole waves. ``sm_count`` 0 queries the current device."""
    return int(lib.fa_varlen_splitkv_num_splits(int(batch), int(max_seqlen_q), int(num_heads), int(num_heads_k),
                                                int(max_seqlen_k), int(sm_count)))


def fa_varlen_fwd_splitkv(q, k, v, cu_seqlens_q, max_seqlen_q: int, max_seqlen_k: int, softmax_scale: float,
                          causal: bool, num_splits: int, cu_seqlens_k=None, seqlens_k=None, leftpad_k=None,
                          block_table=None, out=None, softmax_lse=None, workspace=None, stream=None):
    """Split-KV forward with the query heads of a key/value group packed into
    one tile (decoding). Keys are packed (cu_seqlens_k; k, v [Tk, Hk, D]),
    in cache slots (seqlens_k, optional leftpad_k; k, v [batch, rows, Hk,
    D]) or paged (seqlens_k, block_table; k, v [pages, page_size, Hk, D]).
    Returns (out, softmax_lse) as fa_varlen_fwd does."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    batch = cu_seqlens_q.numel() - 1
    lay = KvLayout()
    if block_table is not None:
        num_pages, page_size, Hk = k.shape[0], k.shape[1], k.shape[2]
        lay.seqlens_k, lay.block_table = seqlens_k.data_ptr(), block_table.data_ptr()
        lay.page_size, lay.max_pages_per_seq, lay.total_rows = page_size, block_table.shape[1], num_pages * page_size
    elif seqlens_k is not None:
        rows, Hk = k.shape[1], k.shape[2]
        lay.seqlens_k = seqlens_k.data_ptr()
        lay.leftpad_k = leftpad_k.data_ptr() if leftpad_k is not None else None
        lay.cache_rows, lay.total_rows = rows, batch * rows
    else:
        _check_cu("cu_seqlens_k", cu_seqlens_k)
        Hk = k.shape[1]
        lay.cu_seqlens_k, lay.total_rows = cu_seqlens_k.data_ptr(), k.shape[0]
    for name, t in (("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda or t.shape[-1] != D:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor with head_dim {D}")
    if H % Hk != 0:
        raise ValueError(f"query heads ({H}) must be a multiple of key/value heads ({Hk})")
    if out is None:
        out = torch.empty_like(q)
    if softmax_lse is None:
        softmax_lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    need = int(lib.fa_varlen_fwd_splitkv_workspace_size(batch, Tq, H, Hk, D, int(num_splits)))
    if workspace is None:
        workspace = new_workspace(need, q.device)
    rc = lib.fa_varlen_fwd_splitkv(_p(q), _p(k), _p(v), _p(cu_seqlens_q), ctypes.byref(lay), batch, Tq,
                                   int(max_seqlen_q), int(max_seqlen_k), H, Hk, D, float(softmax_scale),
                                   int(bool(causal)), int(num_splits), _p(out), _p(softmax_lse), _p(workspace),
                                   workspace.numel(), _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_fwd_splitkv")
    return out, softmax_lse


def fa_varlen_fwd_noalloc(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                          softmax_scale: float, causal: bool, out=None, softmax_lse=None, stream=None):
    """Forward without a workspace, for callers that cannot allocate device
    memory: the library's own device buffer serves as scratch. Calls that can
    overlap on the GPU must be serialised by the caller (they share it)."""
    _check_qkv("q", q)
    Tq, H, D = q.shape
    _check_qkv("k", k, H, D)
    _check_qkv("v", v, H, D)
    _check_cu("cu_seqlens_q", cu_seqlens_q)
    _check_cu("cu_seqlens_k", cu_seqlens_k)
    batch = cu_seqlens_q.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if softmax_lse is None:
        softmax_lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    rc = lib.fa_varlen_fwd_noalloc(_p(q), _p(k), _p(v), _p(cu_seqlens_q), _p(cu_seqlens_k), batch, Tq,
                                   k.shape[0], int(max_seqlen_q), int(max_seqlen_k), H, D,
                                   float(softmax_scale), int(bool(causal)), _p(out), _p(softmax_lse),
                                   _stream(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_varlen_fwd_noalloc")
    return out, softmax_lse


def device_status(workspace, stream=None) -> int:
    """Synchronise the stream and return the device status word of the last
    call that used this workspace."""
    return int(lib.fa_get_device_status(_p(workspace), _stream(stream)))
