"""Maximum sizes: the packed tensors of one call hold more than 2^31
elements, so every offset past that point needs 64-bit address arithmetic
(page "Mecanismo cu_seqlens en FlashAttention", "Optimización de acceso a
memoria": sequence b's rows start at cu_seqlens[b], an offset that grows with
the whole batch, and each row holds heads x head_dim elements).

520 causal sequences of 2048 tokens, 16 heads, head_dim 128: 1,064,960
packed rows, 2.18e9 elements per tensor (4.4 GB in bf16); the backward's fp32
dQ accumulator holds as many. The sequences repeat four seeded blocks, so
every sequence has a twin among the first four. For the last four sequences
(element offsets above 2^31) the forward output and logsumexp and the dK, dV
gradients must equal their twins' bit for bit: each comes from the same
inputs through the same per-tile computation, wherever it sits in the batch.
dQ, which is added from several key tiles in no fixed order, must agree with
its twin's within a relative L2 of 1e-3. One head of two far sequences is also
checked against the oracle."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

L, NSEQ, H, D, NBLK = 2048, 520, 16, 128, 4


def test_offsets_beyond_2_31_elements():
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    total = L * NSEQ
    assert total * H * D > 2**31
    blocks = [synth.make_workload(f"large-block{i}", [L], heads=H, head_dim=D, causal=True, seed=900 + i)
              for i in range(NBLK)]
    names = ("q", "k", "v", "dout")
    big = {n: torch.empty((total, H, D), dtype=torch.bfloat16, device="cuda") for n in names}
    for i, w in enumerate(blocks):
        t = w.tensors()
        for n in names:
            src = pu.to_dev(t[n])
            # Sequences i, i + 4, i + 8, ... hold block i.
            big[n].view(NSEQ // NBLK, NBLK, L, H, D)[:, i].copy_(src.unsqueeze(0).expand(NSEQ // NBLK, L, H, D))
    cu = pu.cu_dev(np.arange(0, total + 1, L, dtype=np.int32))
    scale = blocks[0].scale
    out, lse = fa_varlen.fa_varlen_fwd(big["q"], big["k"], big["v"], cu, cu, L, L, scale, True)
    dq, dk, dv = fa_varlen.fa_varlen_bwd(big["dout"], big["q"], big["k"], big["v"], out, lse, cu, cu, L, L, scale,
                                         True)
    torch.cuda.synchronize()

    def seq(x, s):
        return x[s * L:(s + 1) * L]

    for s in range(NSEQ - NBLK, NSEQ):
        twin = s % NBLK
        assert torch.equal(seq(out, s), seq(out, twin)), f"out of sequence {s}"
        assert torch.equal(lse[:, s * L:(s + 1) * L], lse[:, twin * L:(twin + 1) * L]), f"lse of sequence {s}"
        assert torch.equal(seq(dk, s), seq(dk, twin)), f"dk of sequence {s}"
        assert torch.equal(seq(dv, s), seq(dv, twin)), f"dv of sequence {s}"
        a, b = seq(dq, s).double(), seq(dq, twin).double()
        assert float((a - b).norm() / b.norm()) <= 1e-3, f"dq of sequence {s}"
    for x in (out, dq, dk, dv):
        assert bool(torch.isfinite(x.float()).all())

    for s, h in ((NSEQ - 1, H - 1), (NSEQ - 3, 0)):
        w = blocks[s % NBLK]
        t = w.tensors()
        ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True, units=[(0, h)])
        got = pu.bf16_dev_to_f64(seq(out, s)[:, h])
        assert float(np.max(np.abs(got - ref_out[:, h]))) <= pu.OUT_MAX_ABS
        assert pu.rel_l2(got, ref_out[:, h]) <= pu.OUT_REL_L2
        gl = lse[h, s * L:(s + 1) * L].cpu().numpy().astype(np.float64)
        assert float(np.max(np.abs(gl - ref_lse[h]))) <= pu.LSE_MAX_ABS
        rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, True, units=[(0, h)])
        for name, x, want in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            err = pu.rel_l2(pu.bf16_dev_to_f64(seq(x, s)[:, h]), want[:, h])
            assert err <= pu.GRAD_REL_L2, f"{name}[{s},{h}] rel-L2 {err:.3e}"
    del big, out, lse, dq, dk, dv
    torch.cuda.empty_cache()


def test_single_sequence_of_262144_tokens():
    """One causal sequence of 262,144 tokens (2048 tiles of 128: the work
    list's cost histogram clamps the longest items, and key tile 0's item has
    2048 steps). The forward is checked against the oracle on sampled rows of
    both heads; the backward, too long for the fp64 oracle, against what holds
    at any size: every row of P sums to one, so sum_j dV_j = sum_i dO_i, and
    every row of dS sums to zero, so sum_j dK_j = 0 (up to rounding)."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    n = 262144
    w = synth.make_workload("one-long", [n], heads=2, head_dim=64, causal=True, seed=910)
    t = w.tensors()
    q, k, v, do = (pu.to_dev(t[x]) for x in ("q", "k", "v", "dout"))
    cu = pu.cu_dev(w.cu_q)
    out, lse = fa_varlen.fa_varlen_fwd(q, k, v, cu, cu, n, n, w.scale, True)
    dq, dk, dv = fa_varlen.fa_varlen_bwd(do, q, k, v, out, lse, cu, cu, n, n, w.scale, True)
    torch.cuda.synchronize()
    step = 8191  # rows 0, 8191, ... : both ends of tiles, early and late in the sequence
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_q, w.scale, True, row_step=step)
    rows = np.arange(0, n, step)
    rows_dev = torch.as_tensor(rows, device="cuda")
    for h in range(w.heads):
        got = pu.bf16_dev_to_f64(out[rows_dev, h])
        assert float(np.max(np.abs(got - ref_out[rows, h]))) <= pu.OUT_MAX_ABS
        assert pu.rel_l2(got, ref_out[rows, h]) <= pu.OUT_REL_L2
        gl = lse[h, rows_dev].cpu().numpy().astype(np.float64)
        assert float(np.max(np.abs(gl - ref_lse[h, rows]))) <= pu.LSE_MAX_ABS
    for x in (out, dq, dk, dv):
        assert bool(torch.isfinite(x.float()).all())
    dvs, dos = dv.double().sum(0), do.double().sum(0)
    assert float((dvs - dos).norm() / dos.norm()) < 2e-2
    assert float(dk.double().sum(0).norm() / dk.double().norm()) < 5e-2
    del q, k, v, do, out, lse, dq, dk, dv
    torch.cuda.empty_cache()
