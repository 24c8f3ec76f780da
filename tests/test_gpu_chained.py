"""Stream ordering of the library's calls. Inside a call every kernel after
the work-list kernel is launched as a programmatic dependent of the one
before it; the call as a whole must still start after the caller's previous
work on the stream and finish before the caller's next work. Here a torch
kernel overwrites the inputs immediately before each call, on the same
stream and into the same buffers, and another copies the outputs right
after it, with no synchronisation between the rounds. Every round must give
exactly what the same call gives in isolation (synchronised before and
after): bitwise for the forward, the split-KV forward and the deterministic
backward, within a tight relative bound for the backward whose dQ additions
race. A round that read the previous round's inputs, or whose outputs were
copied before they were complete, would differ at order one. Each round is
also checked against the oracle on its own inputs (relative L2)."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

LQ = [300, 700, 150, 900]
LK = [500, 700, 40, 1200]
ROUNDS = (401, 402, 403)


def _run_rounds(srcs, bufs, call):
    """call() -> tuple of output tensors. Returns (isolated, back_to_back)."""
    import torch

    def one(src):
        for n, b in bufs.items():
            b.copy_(src[n])
        return tuple(o.clone() for o in call())

    iso = []
    for src in srcs:
        torch.cuda.synchronize()
        iso.append(one(src))
        torch.cuda.synchronize()
    b2b = [one(src) for src in srcs]  # no synchronisation between the rounds
    torch.cuda.synchronize()
    return iso, b2b


def _oracle_fwd_rel(w, out):
    t = w.tensors()
    ref_out, _ = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal)
    got = pu.bf16_dev_to_f64(out)
    assert np.all(np.isfinite(got))
    assert pu.rel_l2(got, ref_out) <= pu.OUT_REL_L2


def test_forward_between_torch_kernels():
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    ws = [synth.make_workload("chain", LQ, LK, heads=4, head_dim=128, causal=True, seed=s) for s in ROUNDS]
    w0 = ws[0]
    srcs = [{n: pu.to_dev(w.tensors()[n]) for n in ("q", "k", "v")} for w in ws]
    bufs = {n: torch.empty_like(srcs[0][n]) for n in ("q", "k", "v")}
    cq, ck = pu.cu_dev(w0.cu_q), pu.cu_dev(w0.cu_k)
    out = torch.empty_like(bufs["q"])
    lse = torch.empty((w0.heads, w0.total_q), dtype=torch.float32, device="cuda")
    work = fa_varlen.new_workspace(int(fa_varlen.lib.fa_varlen_fwd_workspace_size(w0.batch, w0.total_q, w0.heads, 128)),
                                   "cuda")

    def call():
        return fa_varlen.fa_varlen_fwd(bufs["q"], bufs["k"], bufs["v"], cq, ck, w0.max_seqlen_q, w0.max_seqlen_k,
                                       w0.scale, True, out=out, softmax_lse=lse, workspace=work)

    iso, b2b = _run_rounds(srcs, bufs, call)
    assert fa_varlen.device_status(work) == 0
    for w, a, b in zip(ws, iso, b2b):
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
        _oracle_fwd_rel(w, a[0])
    assert not torch.equal(iso[0][0], iso[1][0])  # the rounds do differ


@pytest.mark.parametrize("deterministic", [False, True], ids=["atomic", "deterministic"])
def test_backward_between_torch_kernels(deterministic):
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    ws = [synth.make_workload("chain", LQ, LK, heads=4, head_dim=128, causal=True, seed=s) for s in ROUNDS]
    w0 = ws[0]
    srcs = [{n: pu.to_dev(w.tensors()[n]) for n in ("q", "k", "v", "dout")} for w in ws]
    bufs = {n: torch.empty_like(srcs[0][n]) for n in ("q", "k", "v", "dout")}
    cq, ck = pu.cu_dev(w0.cu_q), pu.cu_dev(w0.cu_k)
    bwd = fa_varlen.fa_varlen_bwd_deterministic if deterministic else fa_varlen.fa_varlen_bwd

    def call():
        q, k, v, do = bufs["q"], bufs["k"], bufs["v"], bufs["dout"]
        out, lse = fa_varlen.fa_varlen_fwd(q, k, v, cq, ck, w0.max_seqlen_q, w0.max_seqlen_k, w0.scale, True)
        return bwd(do, q, k, v, out, lse, cq, ck, w0.max_seqlen_q, w0.max_seqlen_k, w0.scale, True)

    iso, b2b = _run_rounds(srcs, bufs, call)
    for w, a, b in zip(ws, iso, b2b):
        t = w.tensors()
        refs = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, True)
        for name, x, y, want in zip(("dq", "dk", "dv"), a, b, refs):
            if deterministic:
                assert torch.equal(x, y), name
            else:
                assert pu.rel_l2(pu.bf16_dev_to_f64(y), pu.bf16_dev_to_f64(x)) <= 1e-3, name
            g = pu.bf16_dev_to_f64(x)
            assert np.all(np.isfinite(g)), name
            assert pu.rel_l2(g, want) <= pu.GRAD_REL_L2, name


def test_splitkv_between_torch_kernels():
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    lq, lk, H, Hk = [1, 1, 2, 1], [3000, 700, 2048, 1], 16, 4
    ws = [synth.make_workload("chain-dec", lq, lk, heads=H, head_dim=128, causal=True, seed=s, heads_k=Hk)
          for s in ROUNDS]
    w0 = ws[0]
    srcs = [{n: pu.to_dev(w.tensors()[n]) for n in ("q", "k", "v")} for w in ws]
    bufs = {n: torch.empty_like(srcs[0][n]) for n in ("q", "k", "v")}
    cq, ck = pu.cu_dev(w0.cu_q), pu.cu_dev(w0.cu_k)
    out = torch.empty_like(bufs["q"])
    lse = torch.empty((H, w0.total_q), dtype=torch.float32, device="cuda")

    def call():
        return fa_varlen.fa_varlen_fwd_splitkv(bufs["q"], bufs["k"], bufs["v"], cq, w0.max_seqlen_q, w0.max_seqlen_k,
                                               w0.scale, True, 5, cu_seqlens_k=ck, out=out, softmax_lse=lse)

    iso, b2b = _run_rounds(srcs, bufs, call)
    for w, a, b in zip(ws, iso, b2b):
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
        _oracle_fwd_rel(w, a[0])
