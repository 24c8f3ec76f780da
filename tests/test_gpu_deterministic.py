"""GPU checks of the deterministic backward (fa_varlen_bwd_deterministic):
parity with the fp64 oracle, and bitwise-identical gradients across repeated
runs (the ordinary backward's bulk fp32 dQ additions land in varying
order)."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    ("ragged", [513, 260, 1, 384], [513, 260, 1, 384], 2, 2, 128),
    ("lq-ne-lk-gqa", [200, 64, 300, 17], [300, 64, 130, 250], 4, 2, 64),
    ("long", [3000, 45], [3000, 45], 2, 1, 128),
]


def _grads(w, det):
    from varlen_flashattention_02_b200 import fa_varlen

    t = w.tensors()
    q, k, v, do = (pu.to_dev(t[n]) for n in ("q", "k", "v", "dout"))
    cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
    fwd = fa_varlen.fa_varlen_fwd_gqa if w.kv_heads != w.heads else fa_varlen.fa_varlen_fwd
    out, lse = fwd(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal)
    bwd = fa_varlen.fa_varlen_bwd_deterministic if det else fa_varlen.fa_varlen_bwd_gqa
    ws = fa_varlen.new_workspace(fa_varlen.bwd_workspace_size(w.batch, w.total_q, w.total_k, w.heads, w.head_dim),
                                 q.device)
    grads = bwd(do, q, k, v, out, lse, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal, workspace=ws)
    assert fa_varlen.device_status(ws) == 0
    return grads


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_deterministic_parity_and_repeatability(case, causal):
    import torch

    name, lq, lk, H, Hk, D = case
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=D, causal=causal, seed=701 + len(lq), heads_k=Hk)
    first = _grads(w, True)
    t = w.tensors()
    ref = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, w.causal)
    for name_, g, r in zip(("dq", "dk", "dv"), first, ref):
        err = pu.rel_l2(pu.bf16_dev_to_f64(g), r)
        assert err <= pu.GRAD_REL_L2, f"{name_} rel-L2 {err:.3e}"
    for _ in range(3):
        again = _grads(w, True)
        for a, b in zip(first, again):
            assert torch.equal(a, b), "deterministic backward changed between runs"


def test_deterministic_full_size_repeatable():
    """The fwd+bwd benchmark workload (16384 tokens, lengths U{512..8192},
    16 heads, d=128, causal): two deterministic runs agree bit for bit and
    agree with the ordinary backward within the gradient tolerance."""
    import torch

    w = synth.standard_workload(5)
    a = _grads(w, True)
    b = _grads(w, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = _grads(w, False)
    for x, y in zip(a, c):
        xd, yd = x.double(), y.double()
        assert float((xd - yd).norm() / yd.norm()) < 1e-2
