"""GPU parity of grouped- and multi-query attention (k, v with fewer heads
than q; page "Flash-Atención y Flash-Atención-2", FlashAttention-2 section)
against the fp64 oracle, forward and backward, through the *_gqa entry
points of the C ABI."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

# (name, query lengths, key lengths, query heads, key/value heads, head_dim)
CASES = [
    ("gqa2-ragged", [300, 129, 1, 640], [300, 129, 1, 640], 4, 2, 128),
    ("mqa-lq-ne-lk", [200, 64, 300, 17], [300, 64, 130, 250], 4, 1, 64),
    ("gqa3-empty", [0, 5, 260, 0, 131], [3, 0, 257, 0, 300], 6, 2, 128),
    ("gqa4-d64-long", [1000, 45], [1000, 45], 8, 2, 64),
]


def _run(w):
    from varlen_flashattention_02_b200 import fa_varlen

    t = w.tensors()
    q, k, v, do = (pu.to_dev(t[n]) for n in ("q", "k", "v", "dout"))
    cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
    out, lse = fa_varlen.fa_varlen_fwd_gqa(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal)
    dq, dk, dv = fa_varlen.fa_varlen_bwd_gqa(do, q, k, v, out, lse, cq, ck, w.max_seqlen_q, w.max_seqlen_k,
                                             w.scale, w.causal)
    return out, lse, dq, dk, dv


def _grad_ok(name, got, want):
    g = pu.bf16_dev_to_f64(got)
    assert np.all(np.isfinite(g)), f"{name}: non-finite"
    err = pu.rel_l2(g, want)
    assert err <= pu.GRAD_REL_L2, f"{name} rel-L2 {err:.3e} > {pu.GRAD_REL_L2}"


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gqa_small(case, causal):
    name, lq, lk, H, Hk, D = case
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=D, causal=causal, seed=301 + len(lq), heads_k=Hk)
    out, lse, dq, dk, dv = _run(w)
    t = w.tensors()
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal)
    rows = np.repeat(np.arange(w.total_q), H)
    heads = np.tile(np.arange(H), w.total_q)
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, w.causal)
    _grad_ok("dq", dq, rq)
    _grad_ok("dk", dk, rk)
    _grad_ok("dv", dv, rv)
    # Keys of sequences without queries get exactly zero gradient.
    gk, gv = pu.bf16_dev_to_f64(dk), pu.bf16_dev_to_f64(dv)
    for b in range(w.batch):
        if w.cu_q[b + 1] == w.cu_q[b]:
            sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
            assert np.all(gk[sk] == 0.0) and np.all(gv[sk] == 0.0)


def test_gqa_equals_repeated_heads_on_gpu():
    """The GPU forward with shared key/value heads gives the same bits as the
    multi-head forward on the key/value heads repeated over each group (same
    tiles, same arithmetic), and dq matches too; dk, dv are the group sums
    (checked against the oracle above)."""
    import torch
    from varlen_flashattention_02_b200 import fa_varlen

    w = synth.make_workload("gqa-vs-mha", [700, 300, 1024], heads=8, head_dim=128, causal=True, seed=311,
                            heads_k=2)
    t = w.tensors()
    q, k, v = (pu.to_dev(t[n]) for n in ("q", "k", "v"))
    cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
    out, lse = fa_varlen.fa_varlen_fwd_gqa(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, True)
    kr = torch.repeat_interleave(k, 4, dim=1).contiguous()
    vr = torch.repeat_interleave(v, 4, dim=1).contiguous()
    out_r, lse_r = fa_varlen.fa_varlen_fwd(q, kr, vr, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, True)
    assert torch.equal(out, out_r) and torch.equal(lse, lse_r)


def test_gqa_full_size_sampled():
    """A Llama-style grouping at the benchmark's size: 16384 tokens, lengths
    U{512..8192} (seed 5), 32 query heads over 8 key/value heads, d=128,
    causal. Sampled forward rows and whole backward units (sequence,
    key/value head) of the two shortest sequences are checked against the
    oracle; every output and gradient is checked to be finite."""
    import torch

    lens = synth.lengths_uniform(5, synth.TOTAL_TOKENS, 512, 8192)
    w = synth.make_workload("varlen-16k-h32-kv8-d128-causal", lens, heads=32, head_dim=128, causal=True, seed=5,
                            heads_k=8)
    out, lse, dq, dk, dv = _run(w)
    t = w.tensors()
    order = np.argsort(np.diff(w.cu_q), kind="stable")
    short = [int(b) for b in order[:2]]
    units = [(b, h) for b in short for h in (0, 13, 31)]
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True, units=units, row_step=16)
    rows, heads = pu.rows_of_units(w, units, 16)
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)
    kv_units = [(b, hk) for b in short for hk in (0, 7)]
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, True, units=kv_units)
    for b, hk in kv_units:
        sq = slice(int(w.cu_q[b]), int(w.cu_q[b + 1]))
        sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
        for h in range(hk * 4, hk * 4 + 4):
            _grad_ok(f"dq[{b},{h}]", dq[sq, h], rq[sq, h])
        _grad_ok(f"dk[{b},{hk}]", dk[sk, hk], rk[sk, hk])
        _grad_ok(f"dv[{b},{hk}]", dv[sk, hk], rv[sk, hk])
    for x in (out, dq, dk, dv):
        assert bool(torch.isfinite(x.float()).all())
