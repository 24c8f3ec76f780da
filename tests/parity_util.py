"""Helpers for the GPU parity tests: move seeded inputs to the device, run
the library, and compare with the fp64 oracle under the stated tolerances.

Tolerances (fixed before any kernel ran):
  forward out: max |gpu - oracle| <= 1e-2 and ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3
  forward lse: max |gpu - oracle| <= 1e-3 (rows with no visible key: both -inf)
  backward dq, dk, dv: relative L2 error <= 2e-2
"""
from __future__ import annotations

import numpy as np

OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 2e-2


def to_dev(bits: np.ndarray):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def cu_dev(cu: np.ndarray):
    import torch

    return torch.from_numpy(np.ascontiguousarray(cu, dtype=np.int32)).cuda()


def bf16_dev_to_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    den = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (den if den > 0 else 1.0)


def run_fwd(w, **kw):
    """Runs the library forward on workload ``w``; returns (out, lse) torch tensors."""
    from varlen_flashattention_02_b200 import fa_varlen

    t = w.tensors()
    q, k, v = to_dev(t["q"]), to_dev(t["k"]), to_dev(t["v"])
    out, lse = fa_varlen.fa_varlen_fwd(q, k, v, cu_dev(w.cu_q), cu_dev(w.cu_k), w.max_seqlen_q,
                                       w.max_seqlen_k, w.scale, w.causal, **kw)
    return (q, k, v), out, lse


def rows_of_units(w, units, row_step=1):
    """Packed query row indices (and their heads) covered by ``units``."""
    rows, heads = [], []
    for b, h in units:
        for i in range(0, int(w.cu_q[b + 1] - w.cu_q[b]), row_step):
            rows.append(int(w.cu_q[b]) + i)
            heads.append(h)
    return np.array(rows, dtype=np.int64), np.array(heads, dtype=np.int64)


def check_fwd(w, out, lse, ref_out, ref_lse, rows, heads):
    """Compare on the given (row, head) entries; returns the error figures."""
    got = bf16_dev_to_f64(out)[rows, heads]
    want = ref_out[rows, heads]
    gl = lse.cpu().numpy().astype(np.float64)[heads, rows]
    wl = ref_lse[heads, rows]
    assert np.all(np.isfinite(got)), "non-finite output"
    empty = ~np.isfinite(wl)
    assert np.all(gl[empty] == -np.inf), "rows with no visible key must have lse = -inf"
    assert np.all(got[empty] == 0.0), "rows with no visible key must be zero"
    max_abs = float(np.max(np.abs(got - want))) if got.size else 0.0
    rl2 = rel_l2(got, want) if got.size else 0.0
    lse_err = float(np.max(np.abs(gl[~empty] - wl[~empty]))) if np.any(~empty) else 0.0
    assert max_abs <= OUT_MAX_ABS, f"out max-abs {max_abs:.3e} > {OUT_MAX_ABS}"
    assert rl2 <= OUT_REL_L2, f"out rel-L2 {rl2:.3e} > {OUT_REL_L2}"
    assert lse_err <= LSE_MAX_ABS, f"lse max-abs {lse_err:.3e} > {LSE_MAX_ABS}"
    return {"out_max_abs": max_abs, "out_rel_l2": rl2, "lse_max_abs": lse_err}
