"""GPU parity of the forward (through the C ABI via the thin binding) against
the fp64 oracle on the same seeded bf16 inputs."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

# (name, query lengths, key lengths, heads, head_dim)
SMALL = [
    ("one-tile", [100], [100], 2, 128),
    ("tails-127-128-129-1", [127, 128, 129, 1], [127, 128, 129, 1], 3, 128),
    ("lq-ne-lk", [200, 64, 300, 17], [300, 64, 130, 250], 2, 64),
    ("empty-and-one", [0, 5, 1, 0, 130, 3], [3, 0, 1, 0, 257, 300], 2, 128),
    ("multi-tile-ragged", [513, 260, 384], [513, 260, 384], 2, 64),
    ("long-ragged", [1000, 45], [1000, 45], 1, 128),
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_fwd_small(case, causal):
    name, lq, lk, H, D = case
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=D, causal=causal, seed=101 + len(lq))
    _, out, lse = pu.run_fwd(w)
    t = w.tensors()
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal)
    rows = np.repeat(np.arange(w.total_q), H)
    heads = np.tile(np.arange(H), w.total_q)
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)


def test_fwd_workload1_full():
    """Two sequences, cu_q=[0,200,1024], cu_k=[0,300,1024], 12 heads, d=64,
    scale 1/8, non-causal: every output checked."""
    w = synth.standard_workload(1)
    _, out, lse = pu.run_fwd(w)
    t = w.tensors()
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal)
    rows = np.repeat(np.arange(w.total_q), w.heads)
    heads = np.tile(np.arange(w.heads), w.total_q)
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)


def _sampled_units(w, n_seq=3, heads=(0,)):
    lens = np.diff(w.cu_q)
    order = np.argsort(lens, kind="stable")
    picks = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})[:n_seq]
    return [(b, h) for b in picks for h in heads]


FULL = [
    ("fixed-8x2048-full", lambda: synth.standard_workload(2, causal=False), 16),
    ("fixed-8x2048-causal", lambda: synth.standard_workload(2, causal=True), 16),
    ("packed-16k-h32", lambda: synth.standard_workload(3), 8),
    ("long-16k-d64", lambda: synth.standard_workload(4, head_dim=64), 64),
    ("long-16k-d128", lambda: synth.standard_workload(4, head_dim=128), 64),
    ("varlen-16k-h16", lambda: synth.standard_workload(5), 8),
]


@pytest.mark.parametrize("case", FULL, ids=[c[0] for c in FULL])
def test_fwd_full_size_sampled(case):
    """Full-size workloads in the benchmark's launch configuration; sampled
    (sequence, head) units and query rows are checked against the oracle,
    and every output is checked to be finite."""
    _, make, row_step = case
    w = make()
    _, out, lse = pu.run_fwd(w)
    H = w.heads
    units = _sampled_units(w, heads=(0, H // 2, H - 1))
    t = w.tensors()
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal,
                                  units=units, row_step=row_step)
    rows, heads = pu.rows_of_units(w, units, row_step)
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)
    import torch

    assert bool(torch.isfinite(out.float()).all())
    assert bool(torch.isfinite(lse).all())  # every row sees at least one key here


def test_fwd_deterministic():
    w = synth.standard_workload(1)
    _, o1, l1 = pu.run_fwd(w)
    _, o2, l2 = pu.run_fwd(w)
    assert bool(o1.equal(o2)) and bool(l1.equal(l2))


def test_fwd_varlen_equals_per_sequence():
    """A packed batch gives the same result as each sequence run alone."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    w = synth.make_workload("pack", [300, 129, 64], [200, 129, 400], heads=2, head_dim=128,
                            causal=True, seed=7)
    (q, k, v), out, lse = pu.run_fwd(w)
    for b in range(w.batch):
        sq = slice(int(w.cu_q[b]), int(w.cu_q[b + 1]))
        sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
        cq = torch.tensor([0, sq.stop - sq.start], dtype=torch.int32, device="cuda")
        ck = torch.tensor([0, sk.stop - sk.start], dtype=torch.int32, device="cuda")
        o1, l1 = fa_varlen.fa_varlen_fwd(q[sq].contiguous(), k[sk].contiguous(), v[sk].contiguous(), cq, ck,
                                         sq.stop - sq.start, sk.stop - sk.start, w.scale, True)
        assert torch.equal(o1, out[sq]) and torch.equal(l1, lse[:, sq])


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_many_short_sequences(causal):
    """2000 sequences of 1 to 64 queries and 1 to 96 keys (seeded): the
    single-CTA work-list kernel loops over thousands of sequences and the
    forward takes thousands of one-tile items. Every output row and LSE
    against the oracle."""
    rng = np.random.default_rng(11)
    lq = rng.integers(1, 65, 2000).tolist()
    lk = rng.integers(1, 97, 2000).tolist()
    w = synth.make_workload("many-short", lq, lk, heads=2, head_dim=64, causal=causal, seed=12)
    (q, k, v), out, lse = pu.run_fwd(w)
    t = w.tensors()
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal)
    got = pu.bf16_dev_to_f64(out)
    gl = lse.cpu().numpy().astype(np.float64)
    empty = ~np.isfinite(ref_lse)  # [H, rows]
    assert np.all(gl[empty] == -np.inf) and np.all(got.transpose(1, 0, 2)[empty] == 0.0)
    assert float(np.max(np.abs(gl[~empty] - ref_lse[~empty]))) <= pu.LSE_MAX_ABS
    assert pu.rel_l2(got, ref_out) <= pu.OUT_REL_L2
    # Rows that see one to a few keys output a mix of a few N(0,1) values,
    # up to |out| of about 5, where the bf16 rounding of the stored output
    # (2^-9 |out|) and of P in the P V product (at most 2^-9 max|v|) exceed
    # the suite's 1e-2 on their own: each element is held to 1e-2 + 2^-7 |ref|.
    err = np.abs(got - ref_out)
    assert np.all(err <= 1e-2 + 2.0 ** -7 * np.abs(ref_out)), float(np.max(err - 2.0 ** -7 * np.abs(ref_out)))
