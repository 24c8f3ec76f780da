"""Degenerate batches as a whole: queries but no keys at all (total_k = 0),
keys but no queries (total_q = 0), and neither. The pages define the output
of a query row as an average over the keys it sees ("Flash-Atención y
Flash-Atención-2"; "Mecanismo cu_seqlens en FlashAttention", "Lógica de
cálculo de longitud": a sequence's rows are cu[b] .. cu[b+1]-1, so a zero
length owns none); over an empty set the library returns a zero row and a
logsumexp of -inf, and every gradient that no attention term reaches is
exactly zero. The outputs are first filled with NaN so that a row the
library fails to write shows up."""
import math

import pytest

from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

# Every case runs through the grouped-query entry points (plain multi-head
# attention is the case Hk = H), at every head_dim, with both backwards.
CASES = [
    ("no-keys", [3, 0, 130], [0, 0, 0]),
    ("no-queries", [0, 0], [5, 200]),
    ("nothing", [0], [0]),
]


@pytest.mark.parametrize("deterministic", [False, True], ids=["bwd", "bwd-det"])
@pytest.mark.parametrize("heads", [(2, 2), (4, 1)], ids=["mha", "mqa"])
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_whole_batch_degenerate(case, causal, D, heads, deterministic):
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    name, lq, lk = case
    H, Hk = heads
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=D, causal=causal, seed=77, heads_k=Hk)
    t = w.tensors()
    q, k, v, do = (pu.to_dev(t[n]) for n in ("q", "k", "v", "dout"))
    cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
    out = torch.full_like(q, float("nan"))
    lse = torch.full((H, q.shape[0]), float("nan"), dtype=torch.float32, device="cuda")
    out, lse = fa_varlen.fa_varlen_fwd_gqa(q, k, v, cq, ck, max(lq), max(lk), w.scale, causal, out=out,
                                           softmax_lse=lse)
    torch.cuda.synchronize()
    if sum(lk) == 0:
        assert bool((out == 0).all()), "rows with no key at all must be zero"
        assert bool((lse == -math.inf).all()), "rows with no key at all must have lse = -inf"
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    args = (do, q, k, v, out, lse, cq, ck, max(lq), max(lk), w.scale, causal)
    if deterministic:
        dq, dk, dv = fa_varlen.fa_varlen_bwd_deterministic(*args, dq=dq, dk=dk, dv=dv)
    else:
        dq, dk, dv = fa_varlen.fa_varlen_bwd_gqa(*args, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    if sum(lk) == 0:
        assert bool((dq == 0).all()), "dq of rows that see no key must be zero"
    if sum(lq) == 0:
        assert bool((dk == 0).all()) and bool((dv == 0).all()), "dk, dv of keys no query sees must be zero"


@pytest.mark.parametrize("splits", [1, 3])
@pytest.mark.parametrize("case", [("empty-caches", [1, 1, 1], [0, 0, 0]), ("no-queries", [0, 0], [5, 200])],
                         ids=["empty-caches", "no-queries"])
def test_splitkv_whole_batch_degenerate(case, splits):
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    name, lq, lk = case
    w = synth.make_workload(name, lq, lk, heads=8, head_dim=128, causal=True, seed=78, heads_k=2)
    t = w.tensors()
    q, k, v = (pu.to_dev(t[n]) for n in ("q", "k", "v"))
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.heads, q.shape[0]), float("nan"), dtype=torch.float32, device="cuda")
    out, lse = fa_varlen.fa_varlen_fwd_splitkv(q, k, v, pu.cu_dev(w.cu_q), max(lq), max(lk), w.scale, True, splits,
                                               cu_seqlens_k=pu.cu_dev(w.cu_k), out=out, softmax_lse=lse)
    torch.cuda.synchronize()
    if sum(lk) == 0:
        assert bool((out == 0).all()) and bool((lse == -math.inf).all())
