"""TEST INFRASTRUCTURE ONLY: ctypes front end of the fp64 CPU oracle.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. The product path (the CUDA library and its
binding) never calls it and shares no code with it.

The arithmetic lives in ``fa_oracle.c`` (plain C, fp64, OpenMP over
(sequence, head) units); this module only builds it, marshals numpy arrays
and returns numpy results. Inputs are numpy arrays of float64 or raw bf16 bit
patterns (uint16), laid out [tokens, heads, head_dim].

Every function is pinned by ``tests/test_oracle_pins.py`` to closed forms,
invariants, a library routine (torch's fp64 CPU attention and autograd),
finite differences and brute force on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libfa_oracle.so")
_lock = threading.Lock()
_lib = None

IN_F64 = 0
IN_BF16 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class OracleLib:
    """One loaded build of the oracle (the default one, or a test's mutant)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.fa_oracle_fwd.argtypes = [P, P, P, I, P, P, I, I, I, I, ctypes.c_double, I, I, P, I, P, P]
        lib.fa_oracle_fwd.restype = I
        lib.fa_oracle_bwd.argtypes = [P, P, P, P, I, P, P, I, I, I, I, ctypes.c_double, I, I, P, P, P, P]
        lib.fa_oracle_bwd.restype = I
        lib.fa_oracle_seqlens.argtypes = [P, I, P]
        lib.fa_oracle_seqlens.restype = I
        lib.fa_oracle_elem_offset.argtypes = [P, I, ctypes.c_int64, I, I, I]
        lib.fa_oracle_elem_offset.restype = ctypes.c_int64
        lib.fa_oracle_num_threads.argtypes = []
        lib.fa_oracle_num_threads.restype = I
        self.lib = lib
        self.path = path

    def num_threads(self) -> int:
        return self.lib.fa_oracle_num_threads()

    def seqlens(self, cu) -> np.ndarray:
        """Lengths from cumulative offsets (cu[b+1] - cu[b])."""
        cu = np.ascontiguousarray(cu, dtype=np.int32)
        out = np.zeros(max(len(cu) - 1, 0), dtype=np.int32)
        if self.lib.fa_oracle_seqlens(_ptr(cu), len(cu) - 1, _ptr(out)) != 0:
            raise ValueError("cumulative offsets must start at 0 and be non-decreasing")
        return out

    def elem_offset(self, cu, b: int, r: int, heads: int, h: int, d: int) -> int:
        cu = np.ascontiguousarray(cu, dtype=np.int32)
        return int(self.lib.fa_oracle_elem_offset(_ptr(cu), b, r, heads, h, d))

    def fwd(self, q, k, v, cu_q, cu_k, scale: float, causal: bool, units=None, row_step: int = 1):
        """Returns (out [Tq,H,d] f64, lse [H,Tq] f64). k and v may have fewer
        heads than q (grouped-query attention: query head h uses key/value
        head h // (H // Hk)). With ``units`` (list of (b, h), h a query head),
        only those units are computed; with ``row_step`` > 1 only query rows
        i % row_step == 0 of each unit. Other entries are NaN."""
        q, dt = _as_input(q)
        k, dtk = _as_input(k)
        v, dtv = _as_input(v)
        assert dt == dtk == dtv
        cu_q = np.ascontiguousarray(cu_q, dtype=np.int32)
        cu_k = np.ascontiguousarray(cu_k, dtype=np.int32)
        Tq, H, d = q.shape
        Hk = _kv_heads(H, k, v)
        out = np.full((Tq, H, d), np.nan)
        lse = np.full((H, Tq), np.nan)
        n, _keep, up = _units_arg(units)
        rc = self.lib.fa_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(cu_q), _ptr(cu_k),
                                    len(cu_q) - 1, H, Hk, d, float(scale), int(bool(causal)), n, up,
                                    int(row_step), _ptr(out), _ptr(lse))
        if rc != 0:
            raise MemoryError("oracle forward failed to allocate")
        return out, lse

    def bwd(self, q, k, v, dout, cu_q, cu_k, scale: float, causal: bool, units=None):
        """Returns (dq, dk, dv) as f64 arrays shaped like q, k, v. With
        ``units`` (list of (b, hk), hk a key/value head), only those units
        are computed: dk, dv of head hk and dq of the query heads it serves."""
        q, dt = _as_input(q)
        k, _ = _as_input(k)
        v, _ = _as_input(v)
        dout, _ = _as_input(dout)
        cu_q = np.ascontiguousarray(cu_q, dtype=np.int32)
        cu_k = np.ascontiguousarray(cu_k, dtype=np.int32)
        Tq, H, d = q.shape
        Hk = _kv_heads(H, k, v)
        Tk = k.shape[0]
        dq = np.full((Tq, H, d), np.nan)
        dk = np.full((Tk, Hk, d), np.nan)
        dv = np.full((Tk, Hk, d), np.nan)
        n, _keep, up = _units_arg(units)
        rc = self.lib.fa_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), dt, _ptr(cu_q),
                                    _ptr(cu_k), len(cu_q) - 1, H, Hk, d, float(scale),
                                    int(bool(causal)), n, up, _ptr(dq), _ptr(dk), _ptr(dv))
        if rc != 0:
            raise MemoryError("oracle backward failed to allocate")
        return dq, dk, dv


def kvcache_to_packed(k_cache, v_cache, seqlens_k, leftpad_k=None):
    """Key/value cache layout -> packed layout (page "Mecanismo cu_seqlens en
    FlashAttention", "Lógica de cálculo de longitud": with non-cumulative key
    lengths, sequence b has seqlens_k[b] - leftpad_k[b] keys). Slot b of the
    [batch, rows, Hk, d] cache holds them at rows leftpad_k[b] ..
    seqlens_k[b]-1. Returns (k, v, cu_k) packed back to back."""
    seqlens_k = np.asarray(seqlens_k, dtype=np.int64)
    batch, rows = k_cache.shape[:2]
    leftpad_k = np.zeros(batch, dtype=np.int64) if leftpad_k is None else np.asarray(leftpad_k, dtype=np.int64)
    if np.any(leftpad_k < 0) or np.any(seqlens_k < leftpad_k) or np.any(seqlens_k > rows):
        raise ValueError("need 0 <= leftpad_k <= seqlens_k <= cache rows")
    lk = seqlens_k - leftpad_k
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    k = np.concatenate([k_cache[b, leftpad_k[b]:seqlens_k[b]] for b in range(batch)], axis=0)
    v = np.concatenate([v_cache[b, leftpad_k[b]:seqlens_k[b]] for b in range(batch)], axis=0)
    return np.ascontiguousarray(k), np.ascontiguousarray(v), cu_k


def paged_to_packed(k_pages, v_pages, seqlens_k, block_table):
    """Paged key/value cache -> packed layout: sequence b has seqlens_k[b]
    keys; key position p lives in page block_table[b][p // page_size] at row
    p % page_size of the [num_pages, page_size, Hk, d] pools. Returns
    (k, v, cu_k) packed back to back."""
    seqlens_k = np.asarray(seqlens_k, dtype=np.int64)
    block_table = np.asarray(block_table, dtype=np.int64)
    num_pages, page_size = k_pages.shape[:2]
    ks, vs = [], []
    for b, lk in enumerate(seqlens_k):
        pos = np.arange(lk)
        if lk > block_table.shape[1] * page_size:
            raise ValueError("sequence longer than its block table")
        pages = block_table[b, pos // page_size]
        if np.any(pages < 0) or np.any(pages >= num_pages):
            raise ValueError("page index outside the pool")
        ks.append(k_pages[pages, pos % page_size])
        vs.append(v_pages[pages, pos % page_size])
    cu_k = np.concatenate([[0], np.cumsum(seqlens_k)]).astype(np.int32)
    return np.ascontiguousarray(np.concatenate(ks)), np.ascontiguousarray(np.concatenate(vs)), cu_k


def fwd_paged(q, k_pages, v_pages, cu_q, seqlens_k, block_table, scale: float, causal: bool, units=None,
              row_step: int = 1):
    """The forward over a paged key/value cache: the plain varlen forward on
    each sequence's keys gathered from its pages."""
    k, v, cu_k = paged_to_packed(k_pages, v_pages, seqlens_k, block_table)
    return fwd(q, k, v, cu_q, cu_k, scale, causal, units, row_step)


def fwd_kvcache(q, k_cache, v_cache, cu_q, seqlens_k, leftpad_k, scale: float, causal: bool, units=None,
                row_step: int = 1):
    """The forward over a key/value cache: the plain varlen forward on the
    keys the cache holds for each sequence."""
    k, v, cu_k = kvcache_to_packed(k_cache, v_cache, seqlens_k, leftpad_k)
    return fwd(q, k, v, cu_q, cu_k, scale, causal, units, row_step)


def _load() -> OracleLib:
    global _lib
    with _lock:
        if _lib is None:
            _lib = OracleLib(build())
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _as_input(x: np.ndarray):
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), IN_BF16
    return np.ascontiguousarray(x, dtype=np.float64), IN_F64


def _kv_heads(H: int, k: np.ndarray, v: np.ndarray) -> int:
    Hk = k.shape[1]
    if v.shape[1] != Hk or Hk < 1 or H % Hk != 0:
        raise ValueError(f"query heads ({H}) must be a multiple of key/value heads ({Hk})")
    return Hk


def _units_arg(units):
    if units is None:
        return 0, None, None
    u = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 2))
    return len(u), u, _ptr(u)


def num_threads() -> int:
    return _load().num_threads()


def seqlens(cu) -> np.ndarray:
    return _load().seqlens(cu)


def elem_offset(cu, b: int, r: int, heads: int, h: int, d: int) -> int:
    return _load().elem_offset(cu, b, r, heads, h, d)


def fwd(q, k, v, cu_q, cu_k, scale: float, causal: bool, units=None, row_step: int = 1):
    return _load().fwd(q, k, v, cu_q, cu_k, scale, causal, units, row_step)


def bwd(q, k, v, dout, cu_q, cu_k, scale: float, causal: bool, units=None):
    return _load().bwd(q, k, v, dout, cu_q, cu_k, scale, causal, units)
