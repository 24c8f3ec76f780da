"""GPU parity of the backward against the fp64 oracle. The GPU backward is fed
the GPU forward's own out and logsumexp (as a training step would); the
oracle recomputes everything from the bf16 inputs alone."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

SMALL = [
    ("one-tile", [100], [100], 2, 128),
    ("tails-63-64-65-127-128-129-1", [63, 64, 65, 127, 128, 129, 1], [63, 64, 65, 127, 128, 129, 1], 2, 128),
    ("lq-ne-lk", [200, 64, 300, 17], [300, 64, 130, 250], 2, 64),
    ("empty-and-one", [0, 5, 1, 0, 130, 3], [3, 0, 1, 0, 257, 300], 2, 128),
    ("multi-tile-ragged", [513, 260, 384], [513, 260, 384], 2, 64),
    ("long-ragged", [1000, 45], [1000, 45], 1, 128),
    ("long-d64", [2000, 130], [2000, 130], 2, 64),
]


def _run_bwd(w):
    from varlen_flashattention_02_b200 import fa_varlen

    (q, k, v), out, lse = pu.run_fwd(w)
    do = pu.to_dev(w.tensors()["dout"])
    dq, dk, dv = fa_varlen.fa_varlen_bwd(do, q, k, v, out, lse, pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k),
                                         w.max_seqlen_q, w.max_seqlen_k, w.scale, w.causal)
    return dq, dk, dv


def _check(name, got, want, mask=None):
    g = pu.bf16_dev_to_f64(got)
    if mask is not None:
        g, want = g[mask], want[mask]
    assert np.all(np.isfinite(g)), f"{name}: non-finite"
    err = pu.rel_l2(g, want)
    assert err <= pu.GRAD_REL_L2, f"{name} rel-L2 {err:.3e} > {pu.GRAD_REL_L2}"
    return err


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_bwd_small(case, causal):
    name, lq, lk, H, D = case
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=D, causal=causal, seed=201 + len(lq))
    dq, dk, dv = _run_bwd(w)
    t = w.tensors()
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, w.causal)
    _check("dq", dq, rq)
    _check("dk", dk, rk)
    _check("dv", dv, rv)
    # Structural zeros: query rows that see no key and keys of sequences with
    # no query get exactly zero gradient.
    g = pu.bf16_dev_to_f64(dq)
    gk, gv = pu.bf16_dev_to_f64(dk), pu.bf16_dev_to_f64(dv)
    for b in range(w.batch):
        lqb, lkb = int(w.cu_q[b + 1] - w.cu_q[b]), int(w.cu_k[b + 1] - w.cu_k[b])
        empty_rows = lqb if lkb == 0 else (max(0, lqb - lkb) if causal else 0)
        assert np.all(g[w.cu_q[b]:w.cu_q[b] + empty_rows] == 0.0)
        if lqb == 0:
            assert np.all(gk[w.cu_k[b]:w.cu_k[b + 1]] == 0.0) and np.all(gv[w.cu_k[b]:w.cu_k[b + 1]] == 0.0)


@pytest.mark.parametrize("D", [64, 128])
def test_bwd_full_size_sampled(D):
    """The fwd+bwd workload (16384 tokens, lengths U{512..8192}, 16 heads,
    causal) at full size in the benchmark's launch configuration; whole
    (sequence, head) units of the two shortest, the median and the longest
    sequence (for this seed: all four, 685 to 6695 tokens; the longest key
    tiles loop over the most query tiles) at the first and last head are
    checked against the oracle, and every gradient is checked to be finite."""
    import torch

    w = synth.standard_workload(5)
    if D != w.head_dim:
        w = synth.make_workload(w.name + f"-d{D}", np.diff(w.cu_q), heads=w.heads, head_dim=D, causal=True,
                                seed=w.seed)
    dq, dk, dv = _run_bwd(w)
    lens = np.diff(w.cu_q)
    order = [int(b) for b in np.argsort(lens, kind="stable")]
    picked = sorted({order[0], order[1], order[len(order) // 2], order[-1]})
    units = [(b, h) for b in picked for h in (0, w.heads - 1)]
    t = w.tensors()
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, w.causal, units=units)
    for b, h in units:
        sq = slice(int(w.cu_q[b]), int(w.cu_q[b + 1]))
        sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
        _check(f"dq[{b},{h}]", dq[sq, h], rq[sq, h])
        _check(f"dk[{b},{h}]", dk[sk, h], rk[sk, h])
        _check(f"dv[{b},{h}]", dv[sk, h], rv[sk, h])
    for x in (dq, dk, dv):
        assert bool(torch.isfinite(x.float()).all())


def test_bwd_gradient_sums():
    """Properties that hold at any size: per (sequence, head), the rows of dS
    sum to zero so sum_j dK_j = 0, and the rows of P sum to one so
    sum_j dV_j = sum_i dO_i (every query row of a causal lq == lk sequence
    sees at least one key)."""
    import torch

    w = synth.make_workload("sums", [700, 300, 1024], heads=2, head_dim=128, causal=True, seed=9)
    dq, dk, dv = _run_bwd(w)
    do = torch.from_numpy(synth.bf16_bits_to_f32(w.tensors()["dout"])).double()
    for b in range(w.batch):
        sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
        sq = slice(int(w.cu_q[b]), int(w.cu_q[b + 1]))
        dvs = dv[sk].double().sum(0).cpu()
        dos = do[sq].sum(0)
        assert float((dvs - dos).norm() / dos.norm()) < 2e-2
        dks = dk[sk].double().sum(0).cpu()
        assert float(dks.norm() / dk[sk].double().norm().cpu()) < 5e-2


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_bwd_many_short_sequences(causal):
    """2000 sequences of 1 to 64 queries and 1 to 96 keys (seeded): thousands
    of one-tile backward items. Every gradient against the oracle."""
    rng = np.random.default_rng(13)
    lq = rng.integers(1, 65, 2000).tolist()
    lk = rng.integers(1, 97, 2000).tolist()
    w = synth.make_workload("many-short", lq, lk, heads=2, head_dim=128, causal=causal, seed=14)
    dq, dk, dv = _run_bwd(w)
    t = w.tensors()
    rq, rk, rv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, w.causal)
    _check("dq", dq, rq)
    _check("dk", dk, rk)
    _check("dv", dv, rv)


@pytest.mark.parametrize("D", [64, 128])
def test_bwd_varlen_equals_per_sequence(D):
    """A packed batch's gradients equal each sequence's run alone: dK and dV
    bit for bit (each key tile's are formed by one CTA in a fixed order from
    that sequence's rows only), dQ within a relative L2 of 1e-3 (its
    additions from several key tiles land in no fixed order). Catches any
    leak across sequence boundaries that a whole-batch tolerance could hide."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    w = synth.make_workload("pack-bwd", [300, 129, 64, 700], [200, 129, 400, 700], heads=2, head_dim=D,
                            causal=True, seed=15)
    t = w.tensors()
    q, k, v, do = (pu.to_dev(t[n]) for n in ("q", "k", "v", "dout"))
    cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
    out, lse = fa_varlen.fa_varlen_fwd(q, k, v, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale, True)
    dq, dk, dv = fa_varlen.fa_varlen_bwd(do, q, k, v, out, lse, cq, ck, w.max_seqlen_q, w.max_seqlen_k, w.scale,
                                         True)
    for b in range(w.batch):
        sq = slice(int(w.cu_q[b]), int(w.cu_q[b + 1]))
        sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
        nq, nk = sq.stop - sq.start, sk.stop - sk.start
        c1q = torch.tensor([0, nq], dtype=torch.int32, device="cuda")
        c1k = torch.tensor([0, nk], dtype=torch.int32, device="cuda")
        qb, kb, vb, dob = (x.contiguous() for x in (q[sq], k[sk], v[sk], do[sq]))
        ob, lb = fa_varlen.fa_varlen_fwd(qb, kb, vb, c1q, c1k, nq, nk, w.scale, True)
        assert torch.equal(ob, out[sq]) and torch.equal(lb, lse[:, sq])
        gq, gk, gv = fa_varlen.fa_varlen_bwd(dob, qb, kb, vb, ob, lb, c1q, c1k, nq, nk, w.scale, True)
        assert torch.equal(gk, dk[sk]) and torch.equal(gv, dv[sk]), f"dk/dv of sequence {b}"
        a, r = gq.double(), dq[sq].double()
        assert float((a - r).norm() / r.norm()) <= 1e-3, f"dq of sequence {b}"
