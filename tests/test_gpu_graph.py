"""The library's calls under CUDA graph capture. Every call only enqueues
work on its stream (kernels chained as programmatic dependents), so a
forward and backward captured once into a graph must, when the graph is
replayed with new inputs copied into the captured buffers, give exactly what
the same calls give eagerly on those inputs: bitwise for out, lse, dK and dV
(each computed by one CTA in a fixed order), within a relative L2 of 1e-3 for
dQ (added from several key tiles in no fixed order). Each replay is also
checked against the oracle (relative L2)."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

LQ = [300, 700, 150, 1200]
LK = [500, 700, 40, 1200]
ROUNDS = (501, 502, 503)


@pytest.mark.parametrize("D", [64, 128])
def test_fwd_bwd_graph_replay(D):
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    ws = [synth.make_workload("graph", LQ, LK, heads=4, head_dim=D, causal=True, seed=s) for s in ROUNDS]
    w0 = ws[0]
    names = ("q", "k", "v", "dout")
    srcs = [{n: pu.to_dev(w.tensors()[n]) for n in names} for w in ws]
    bufs = {n: torch.empty_like(srcs[0][n]) for n in names}
    cq, ck = pu.cu_dev(w0.cu_q), pu.cu_dev(w0.cu_k)
    mq, mk = w0.max_seqlen_q, w0.max_seqlen_k

    def step():
        out, lse = fa_varlen.fa_varlen_fwd(bufs["q"], bufs["k"], bufs["v"], cq, ck, mq, mk, w0.scale, True)
        dq, dk, dv = fa_varlen.fa_varlen_bwd(bufs["dout"], bufs["q"], bufs["k"], bufs["v"], out, lse, cq, ck, mq, mk,
                                             w0.scale, True)
        return out, lse, dq, dk, dv

    # Eager results first (also the warm-up that loads every kernel).
    eager = []
    for src in srcs:
        for n in names:
            bufs[n].copy_(src[n])
        eager.append(tuple(x.clone() for x in step()))
    torch.cuda.synchronize()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # a warm-up on the capture stream, as torch recommends
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        captured = step()

    for w, src, want in zip(ws, srcs, eager):
        for n in names:
            bufs[n].copy_(src[n])
        g.replay()
        torch.cuda.synchronize()
        got = tuple(x.clone() for x in captured)
        for name, a, b in zip(("out", "lse", "dk", "dv"), (got[0], got[1], got[3], got[4]),
                              (want[0], want[1], want[3], want[4])):
            assert torch.equal(a, b), f"{name}: replay differs from the eager call"
        a, b = got[2].double(), want[2].double()
        assert float((a - b).norm() / b.norm()) <= 1e-3, "dq: replay differs from the eager call"
        t = w.tensors()
        ref_out, _ = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True)
        assert pu.rel_l2(pu.bf16_dev_to_f64(got[0]), ref_out) <= pu.OUT_REL_L2
        refs = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, True)
        for name, x, ref in zip(("dq", "dk", "dv"), got[2:], refs):
            assert pu.rel_l2(pu.bf16_dev_to_f64(x), ref) <= pu.GRAD_REL_L2, name
    assert not torch.equal(eager[0][0], eager[1][0])  # the rounds do differ
    del g


def test_splitkv_decode_graph_replay():
    """A decoding step (split-KV forward, one query token per sequence,
    grouped heads) captured once and replayed with new query and cache
    contents: bitwise equal to the eager call, and oracle-checked."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    lq, lk, H, Hk = [1, 1, 1, 1], [3000, 700, 2048, 1], 16, 4
    ws = [synth.make_workload("graph-dec", lq, lk, heads=H, head_dim=128, causal=True, seed=s, heads_k=Hk)
          for s in ROUNDS]
    w0 = ws[0]
    names = ("q", "k", "v")
    srcs = [{n: pu.to_dev(w.tensors()[n]) for n in names} for w in ws]
    bufs = {n: torch.empty_like(srcs[0][n]) for n in names}
    cq, ck = pu.cu_dev(w0.cu_q), pu.cu_dev(w0.cu_k)
    splits = fa_varlen.fa_varlen_splitkv_num_splits(w0.batch, 1, H, Hk, w0.max_seqlen_k)

    def step():
        return fa_varlen.fa_varlen_fwd_splitkv(bufs["q"], bufs["k"], bufs["v"], cq, 1, w0.max_seqlen_k, w0.scale,
                                               True, splits, cu_seqlens_k=ck)

    eager = []
    for src in srcs:
        for n in names:
            bufs[n].copy_(src[n])
        eager.append(tuple(x.clone() for x in step()))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        captured = step()
    for w, src, want in zip(ws, srcs, eager):
        for n in names:
            bufs[n].copy_(src[n])
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(captured[0], want[0]) and torch.equal(captured[1], want[1])
        t = w.tensors()
        ref_out, _ = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True)
        assert pu.rel_l2(pu.bf16_dev_to_f64(captured[0]), ref_out) <= pu.OUT_REL_L2
    del g


def test_two_streams_concurrently():
    """Two independent fwd+bwd calls on two streams at once, each with its
    own inputs and workspaces: the library keeps no state between calls
    beyond the caller's buffers, so each gives exactly what it gives alone
    (dQ within 1e-3)."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    w1 = synth.make_workload("two-a", [900, 300, 1500], heads=4, head_dim=128, causal=True, seed=601)
    w2 = synth.make_workload("two-b", [128, 2000, 64, 700], [400, 2000, 64, 900], heads=2, head_dim=64,
                             causal=False, seed=602)

    def run(w):
        t = w.tensors()
        q, k, v, do = (pu.to_dev(t[n]) for n in ("q", "k", "v", "dout"))
        cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)

        def call():
            out, lse = fa_varlen.fa_varlen_fwd(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal)
            grads = fa_varlen.fa_varlen_bwd(do, q, k, v, out, lse, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale,
                                            w.causal)
            return (out, lse) + tuple(grads)
        return call

    c1, c2 = run(w1), run(w2)
    alone = [c1(), c2()]
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    together = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            r1 = c1()
        with torch.cuda.stream(s2):
            r2 = c2()
        together.append((r1, r2))
    torch.cuda.synchronize()
    for r1, r2 in together:
        for got, want in ((r1, alone[0]), (r2, alone[1])):
            for name, a, b in zip(("out", "lse", "dk", "dv"), (got[0], got[1], got[3], got[4]),
                                  (want[0], want[1], want[3], want[4])):
                assert torch.equal(a, b), name
            a, b = got[2].double(), want[2].double()
            assert float((a - b).norm() / b.norm()) <= 1e-3
