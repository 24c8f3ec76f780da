"""GPU parity of head_dim 256 (page "Flash-Atención y Flash-Atención-2":
FlashAttention-2 supports head dimensions up to 256) against the fp64
oracle, forward and backward: ragged varlen batches, causal and not, grouped
heads, the key/value cache layouts (forward), the deterministic backward, and
sampled full-size cases."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

# (name, query lengths, key lengths, heads, key/value heads)
CASES = [
    ("tails", [63, 64, 65, 127, 128, 129, 1], [63, 64, 65, 127, 128, 129, 1], 2, 2),
    ("lq-ne-lk", [200, 64, 300, 17], [300, 64, 130, 250], 2, 1),
    ("empty-and-one", [0, 5, 1, 0, 130, 3], [3, 0, 1, 0, 257, 300], 4, 2),
    ("multi-tile", [700, 260], [700, 260], 2, 2),
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_d256_small(case, causal):
    from varlen_flashattention_02_b200 import fa_varlen

    name, lq, lk, H, Hk = case
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=256, causal=causal, seed=601 + len(lq), heads_k=Hk)
    t = w.tensors()
    q, k, v = (pu.to_dev(t[n]) for n in ("q", "k", "v"))
    fn = fa_varlen.fa_varlen_fwd_gqa if Hk != H else fa_varlen.fa_varlen_fwd
    out, lse = fn(q, k, v, pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k), w.max_seqlen_q, w.max_seqlen_k, w.scale, causal)
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, causal)
    rows = np.repeat(np.arange(w.total_q), H)
    heads = np.tile(np.arange(H), w.total_q)
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)


def test_d256_paged_equals_packed():
    """Pages (of 128 rows) hold d = 256 keys too; the result is the packed
    forward's, bit for bit, and matches the oracle."""
    import torch
    from varlen_flashattention_02_b200 import fa_varlen

    rng = np.random.default_rng(611)
    lq, lk, ps, H, Hk = [3, 200, 1], [600, 129, 1], 128, 4, 2
    pages_per = [-(-n // ps) for n in lk]
    n_pages = sum(pages_per) + 2
    perm = rng.permutation(n_pages).astype(np.int32)
    bt = np.zeros((3, max(pages_per)), dtype=np.int32)
    nxt = 0
    for b in range(3):
        bt[b, :pages_per[b]] = perm[nxt:nxt + pages_per[b]]
        nxt += pages_per[b]
    cu_q = synth.cu_from_lengths(lq)
    q = synth.bf16_normal(rng, (int(cu_q[-1]), H, 256))
    kp = synth.bf16_normal(rng, (n_pages, ps, Hk, 256))
    vp = synth.bf16_normal(rng, (n_pages, ps, Hk, 256))
    lk_a = np.array(lk, dtype=np.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    scale = 1.0 / 16.0
    out, lse = fa_varlen.fa_varlen_fwd_paged(pu.to_dev(q), pu.to_dev(kp), pu.to_dev(vp), dev(cu_q), dev(lk_a), dev(bt),
                                             max(lq), max(lk), scale, True)
    k, v, cu_k = oracle.paged_to_packed(kp, vp, lk_a, bt)
    out_p, lse_p = fa_varlen.fa_varlen_fwd_gqa(pu.to_dev(q), pu.to_dev(k), pu.to_dev(v), dev(cu_q), dev(cu_k),
                                               max(lq), max(lk), scale, True)
    assert torch.equal(out, out_p) and torch.equal(lse, lse_p)
    ref_out, ref_lse = oracle.fwd(q, k, v, cu_q, cu_k, scale, True)
    w = synth.make_workload("paged-d256", lq, heads=H, head_dim=256, causal=True)
    rows = np.repeat(np.arange(int(cu_q[-1])), H)
    heads = np.tile(np.arange(H), int(cu_q[-1]))
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)


def test_d256_full_size_sampled():
    """16384 tokens, lengths U{512..8192} (seed 5), 16 heads, d = 256,
    causal: sampled (sequence, head) rows against the oracle, every output
    finite."""
    import torch

    lens = synth.lengths_uniform(5, synth.TOTAL_TOKENS, 512, 8192)
    w = synth.make_workload("varlen-16k-h16-d256-causal", lens, heads=16, head_dim=256, causal=True, seed=5)
    _, out, lse = pu.run_fwd(w)
    order = np.argsort(np.diff(w.cu_q), kind="stable")
    units = [(int(b), h) for b in (order[0], order[-1]) for h in (0, 15)]
    t = w.tensors()
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True, units=units, row_step=32)
    rows, heads = pu.rows_of_units(w, units, 32)
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)
    assert bool(torch.isfinite(out.float()).all())


def _bwd(w, deterministic=False):
    from varlen_flashattention_02_b200 import fa_varlen

    t = w.tensors()
    q, k, v, do = (pu.to_dev(t[n]) for n in ("q", "k", "v", "dout"))
    cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
    fwd = fa_varlen.fa_varlen_fwd_gqa if w.kv_heads != w.heads else fa_varlen.fa_varlen_fwd
    out, lse = fwd(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal)
    if deterministic:
        bwd = fa_varlen.fa_varlen_bwd_deterministic
    else:
        bwd = fa_varlen.fa_varlen_bwd_gqa if w.kv_heads != w.heads else fa_varlen.fa_varlen_bwd
    return bwd(do, q, k, v, out, lse, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal)


def _check_grad(name, got, want):
    g = pu.bf16_dev_to_f64(got)
    assert np.all(np.isfinite(g)), f"{name}: non-finite"
    err = pu.rel_l2(g, want)
    assert err <= pu.GRAD_REL_L2, f"{name} rel-L2 {err:.3e} > {pu.GRAD_REL_L2}"


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_d256_backward_small(case, causal):
    """dq, dk, dv at d = 256 (a dV pass and a dK/dQ pass over the same work
    list) against the oracle, on ragged batches with tails at 63/64/65 and
    127/128/129 rows (both passes' query tile sizes), lq != lk, empty
    sequences and grouped heads."""
    name, lq, lk, H, Hk = case
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=256, causal=causal, seed=621 + len(lq), heads_k=Hk)
    dq, dk, dv = _bwd(w)
    t = w.tensors()
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, causal)
    _check_grad("dq", dq, rq)
    _check_grad("dk", dk, rk)
    _check_grad("dv", dv, rv)
    gk, gv = pu.bf16_dev_to_f64(dk), pu.bf16_dev_to_f64(dv)
    for b in range(w.batch):
        if w.cu_q[b + 1] == w.cu_q[b]:  # keys no query sees get exactly zero gradient
            sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
            assert np.all(gk[sk] == 0.0) and np.all(gv[sk] == 0.0)


def test_d256_backward_deterministic_repeats():
    """The deterministic backward at d = 256: parity, and the same bits on
    every run."""
    import torch

    w = synth.make_workload("det-d256", [700, 300, 1], heads=4, head_dim=256, causal=True, seed=631, heads_k=2)
    runs = [_bwd(w, deterministic=True) for _ in range(3)]
    for r in runs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(runs[0], r))
    t = w.tensors()
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, True)
    for n, g, r in zip(("dq", "dk", "dv"), runs[0], (rq, rk, rv)):
        _check_grad(n, g, r)


def test_d256_backward_full_size_sampled():
    """16384 tokens, lengths U{512..8192} (seed 5), 16 heads, d = 256,
    causal, in the benchmark's launch configuration: whole (sequence, head)
    units of the shortest and the longest sequence at the first and last
    head against the oracle; every gradient finite."""
    import torch

    lens = synth.lengths_uniform(5, synth.TOTAL_TOKENS, 512, 8192)
    w = synth.make_workload("varlen-16k-h16-d256-causal", lens, heads=16, head_dim=256, causal=True, seed=5)
    dq, dk, dv = _bwd(w)
    order = np.argsort(np.diff(w.cu_q), kind="stable")
    units = [(int(b), h) for b in (order[0], order[-1]) for h in (0, 15)]
    t = w.tensors()
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, True, units=units)
    for b, h in units:
        sq = slice(int(w.cu_q[b]), int(w.cu_q[b + 1]))
        sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
        _check_grad(f"dq[{b},{h}]", dq[sq, h], rq[sq, h])
        _check_grad(f"dk[{b},{h}]", dk[sk, h], rk[sk, h])
        _check_grad(f"dv[{b},{h}]", dv[sk, h], rv[sk, h])
    for x in (dq, dk, dv):
        assert bool(torch.isfinite(x.float()).all())
