"""GPU parity of the forward over a paged key/value cache (the cu_seqlens
page, "Integración con máscaras causales y caché paginada": keys in a pool of
fixed-size pages, a block table per sequence) against the fp64 oracle,
through fa_varlen_fwd_paged."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

# (name, query lengths, key lengths, page size, spare pages, H, Hk, D)
CASES = [
    ("p128-ragged", [5, 128, 1, 300], [700, 100, 1, 300], 128, 5, 4, 2, 128),
    ("p256-decode", [1, 2, 1, 16, 1], [1000, 1, 0, 513, 257], 256, 3, 8, 1, 64),
    ("p128-prefill", [640, 129], [640, 129], 128, 0, 2, 2, 128),
]


def _make(case, seed):
    name, lq, lk, ps, spare, H, Hk, D = case
    rng = np.random.default_rng(seed)
    batch = len(lq)
    pages_per = [-(-n // ps) for n in lk]
    n_pages = sum(pages_per) + spare
    max_pages = max(max(pages_per), 1) + 1
    perm = rng.permutation(n_pages).astype(np.int32)
    bt = np.zeros((batch, max_pages), dtype=np.int32)
    nxt = 0
    for b in range(batch):
        bt[b, :pages_per[b]] = perm[nxt:nxt + pages_per[b]]
        nxt += pages_per[b]
    cu_q = synth.cu_from_lengths(lq)
    q = synth.bf16_normal(rng, (int(cu_q[-1]), H, D))
    kp = synth.bf16_normal(rng, (n_pages, ps, Hk, D))
    vp = synth.bf16_normal(rng, (n_pages, ps, Hk, D))
    return cu_q, q, kp, vp, np.array(lk, dtype=np.int32), bt, 1.0 / np.sqrt(D)


def _dev(a):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(cu_q, q, kp, vp, lk, bt, scale, causal, **kw):
    from varlen_flashattention_02_b200 import fa_varlen

    return fa_varlen.fa_varlen_fwd_paged(pu.to_dev(q), pu.to_dev(kp), pu.to_dev(vp), _dev(cu_q), _dev(lk), _dev(bt),
                                         int(np.max(np.diff(cu_q))), max(int(np.max(lk)), 1), scale, causal, **kw)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_paged_small(case, causal):
    cu_q, q, kp, vp, lk, bt, scale = _make(case, 501 + len(case[1]))
    out, lse = _run(cu_q, q, kp, vp, lk, bt, scale, causal)
    ref_out, ref_lse = oracle.fwd_paged(q, kp, vp, cu_q, lk, bt, scale, causal)
    H = q.shape[1]
    w = synth.make_workload("paged", np.diff(cu_q), heads=H, head_dim=q.shape[2], causal=causal)
    rows = np.repeat(np.arange(int(cu_q[-1])), H)
    heads = np.tile(np.arange(H), int(cu_q[-1]))
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)


def test_paged_equals_packed_forward():
    """Pages change only where the keys are read from: the same keys packed
    with cumulative offsets give the same bits."""
    import torch
    from varlen_flashattention_02_b200 import fa_varlen

    cu_q, q, kp, vp, lk, bt, scale = _make(CASES[0], 511)
    out, lse = _run(cu_q, q, kp, vp, lk, bt, scale, True)
    k, v, cu_k = oracle.paged_to_packed(kp, vp, lk, bt)
    out_p, lse_p = fa_varlen.fa_varlen_fwd_gqa(pu.to_dev(q), pu.to_dev(k), pu.to_dev(v), _dev(cu_q), _dev(cu_k),
                                               int(np.max(np.diff(cu_q))), int(np.max(lk)), scale, True)
    assert torch.equal(out, out_p) and torch.equal(lse, lse_p)


def test_paged_rejects_page_outside_pool():
    """A block-table entry outside the pool is reported by the device check
    (FA_ERR_BAD_SEQLENS in the workspace status), not read."""
    from varlen_flashattention_02_b200 import fa_varlen

    cu_q, q, kp, vp, lk, bt, scale = _make(CASES[2], 521)
    bad = bt.copy()
    bad[1, 0] = kp.shape[0]
    ws = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(2, int(cu_q[-1]), q.shape[1], q.shape[2]), "cuda")
    _run(cu_q, q, kp, vp, lk, bad, scale, False, workspace=ws)
    assert fa_varlen.device_status(ws) == 5  # FA_ERR_BAD_SEQLENS
