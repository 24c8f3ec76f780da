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

CASES = [
    ("no-keys", [3, 0, 130], [0, 0, 0]),
    ("no-queries", [0, 0], [5, 200]),
    ("nothing", [0], [0]),
]


@pytest.mark.parametrize("deterministic", [False, True], ids=["bwd", "bwd-det"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_whole_batch_degenerate(case, causal, D, deterministic):
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    name, lq, lk = case
    H = 2
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=D, causal=causal, seed=77)
    t = w.tensors()
    q, k, v, do = (pu.to_dev(t[n]) for n in ("q", "k", "v", "dout"))
    cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
    scale = w.scale
    out = torch.full_like(q, float("nan"))
    lse = torch.full((H, q.shape[0]), float("nan"), dtype=torch.float32, device="cuda")
    out, lse = fa_varlen.fa_varlen_fwd(q, k, v, cq, ck, max(lq), max(lk), scale, causal, out=out, softmax_lse=lse)
    torch.cuda.synchronize()
    if sum(lk) == 0:
        assert bool((out == 0).all()), "rows with no key at all must be zero"
        assert bool((lse == -math.inf).all()), "rows with no key at all must have lse = -inf"
    bwd = fa_varlen.fa_varlen_bwd_deterministic if deterministic else fa_varlen.fa_varlen_bwd
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    dq, dk, dv = bwd(do, q, k, v, out, lse, cq, ck, max(lq), max(lk), scale, causal, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    if sum(lk) == 0:
        assert bool((dq == 0).all()), "dq of rows that see no key must be zero"
    if sum(lq) == 0:
        assert bool((dk == 0).all()) and bool((dv == 0).all()), "dk, dv of keys no query sees must be zero"
