"""GPU parity of the split-KV forward (fa_varlen_fwd_splitkv: query heads of
a key/value group packed into one tile, key tiles split across CTAs and
merged by logsumexp) against the fp64 oracle, for the packed, cache-slot and
paged key layouts, including decode-like calls with one query token."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu


def _dev(a):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check(q, cu_q, out, lse, ref_out, ref_lse, H, D, causal):
    w = synth.make_workload("splitkv", np.diff(cu_q), heads=H, head_dim=D, causal=causal)
    T = int(cu_q[-1])
    pu.check_fwd(w, out, lse, ref_out, ref_lse, np.repeat(np.arange(T), H), np.tile(np.arange(H), T))


# (name, query lengths, key lengths, H, Hk, D, splits)
PACKED = [
    ("decode-gqa8", [1, 1, 1, 1], [1500, 700, 4096, 1], 32, 4, 128, 6),
    ("decode-mha", [1, 2, 1], [3000, 900, 129], 4, 4, 64, 4),
    ("chunk-gqa4", [16, 5, 40], [2000, 600, 40], 8, 2, 128, 3),
    ("prefill-nosplit", [300, 128], [300, 700], 4, 1, 128, 1),
    ("group6", [3, 1], [1000, 250], 12, 2, 64, 5),
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", PACKED, ids=[c[0] for c in PACKED])
def test_splitkv_packed(case, causal):
    from varlen_flashattention_02_b200 import fa_varlen

    name, lq, lk, H, Hk, D, S = case
    w = synth.make_workload(name, lq, lk, heads=H, head_dim=D, causal=causal, seed=801 + len(lq), heads_k=Hk)
    t = w.tensors()
    q, k, v = (pu.to_dev(t[n]) for n in ("q", "k", "v"))
    out, lse = fa_varlen.fa_varlen_fwd_splitkv(q, k, v, pu.cu_dev(w.cu_q), w.max_seqlen_q, w.max_seqlen_k, w.scale,
                                               causal, S, cu_seqlens_k=pu.cu_dev(w.cu_k))
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, causal)
    _check(t["q"], w.cu_q, out, lse, ref_out, ref_lse, H, D, causal)


@pytest.mark.parametrize("splits", [1, 4])
def test_splitkv_cache_slots(splits):
    """Key/value cache slots with left padding, one query token per sequence
    (decoding), 32 query heads over 8 key/value heads."""
    from varlen_flashattention_02_b200 import fa_varlen

    rng = np.random.default_rng(811)
    batch, rows, H, Hk, D = 5, 2048, 32, 8, 128
    lk = np.array([2048, 17, 1000, 0, 1300], dtype=np.int32)
    pad = np.array([0, 3, 40, 5, 700], dtype=np.int32)
    seqlens = np.minimum(pad + lk, rows).astype(np.int32)
    cu_q = synth.cu_from_lengths([1] * batch)
    q = synth.bf16_normal(rng, (batch, H, D))
    kc = synth.bf16_normal(rng, (batch, rows, Hk, D))
    vc = synth.bf16_normal(rng, (batch, rows, Hk, D))
    scale = 1.0 / np.sqrt(D)
    for causal in (False, True):
        out, lse = fa_varlen.fa_varlen_fwd_splitkv(pu.to_dev(q), pu.to_dev(kc), pu.to_dev(vc), _dev(cu_q), 1, rows,
                                                   scale, causal, splits, seqlens_k=_dev(seqlens), leftpad_k=_dev(pad))
        ref_out, ref_lse = oracle.fwd_kvcache(q, kc, vc, cu_q, seqlens, pad, scale, causal)
        _check(q, cu_q, out, lse, ref_out, ref_lse, H, D, causal)


def test_splitkv_paged_decode():
    """Paged cache (pages of 256 rows, shuffled pool), one query token per
    sequence, 16 query heads over 2 key/value heads, 8 splits."""
    from varlen_flashattention_02_b200 import fa_varlen

    rng = np.random.default_rng(821)
    ps, H, Hk, D = 256, 16, 2, 128
    lk = [3000, 1, 700, 256]
    pages_per = [-(-n // ps) for n in lk]
    n_pages = sum(pages_per) + 3
    perm = rng.permutation(n_pages).astype(np.int32)
    bt = np.zeros((len(lk), max(pages_per)), dtype=np.int32)
    nxt = 0
    for b, npg in enumerate(pages_per):
        bt[b, :npg] = perm[nxt:nxt + npg]
        nxt += npg
    cu_q = synth.cu_from_lengths([1] * len(lk))
    q = synth.bf16_normal(rng, (len(lk), H, D))
    kp = synth.bf16_normal(rng, (n_pages, ps, Hk, D))
    vp = synth.bf16_normal(rng, (n_pages, ps, Hk, D))
    lk_a = np.array(lk, dtype=np.int32)
    scale = 1.0 / np.sqrt(D)
    out, lse = fa_varlen.fa_varlen_fwd_splitkv(pu.to_dev(q), pu.to_dev(kp), pu.to_dev(vp), _dev(cu_q), 1, max(lk),
                                               scale, True, 8, seqlens_k=_dev(lk_a), block_table=_dev(bt))
    ref_out, ref_lse = oracle.fwd_paged(q, kp, vp, cu_q, lk_a, bt, scale, True)
    _check(q, cu_q, out, lse, ref_out, ref_lse, H, D, True)


def test_splitkv_split_count_invariance():
    """Different split counts give the same attention within rounding."""
    import torch
    from varlen_flashattention_02_b200 import fa_varlen

    w = synth.make_workload("inv", [4, 1], [5000, 3000], heads=16, head_dim=128, causal=True, seed=831, heads_k=4)
    t = w.tensors()
    q, k, v = (pu.to_dev(t[n]) for n in ("q", "k", "v"))
    outs = [fa_varlen.fa_varlen_fwd_splitkv(q, k, v, pu.cu_dev(w.cu_q), w.max_seqlen_q, w.max_seqlen_k, w.scale,
                                            True, s, cu_seqlens_k=pu.cu_dev(w.cu_k)) for s in (1, 2, 7, 40)]
    for o, l in outs[1:]:
        assert float((o.float() - outs[0][0].float()).abs().max()) < 1e-2
        assert float((l - outs[0][1]).abs().max()) < 1e-3


@pytest.mark.parametrize("batch,keys,splits", [(64, 8192, 2), (4, 32768, 9)],
                         ids=["64x8192-2splits", "4x32768-9splits"])
def test_splitkv_decode_bench_shapes(batch, keys, splits):
    """The benchmark's decode lines at full size, on the same seeded inputs:
    one query token per sequence, 32 query heads over 8 key/value heads,
    d=128, with the split counts the advisor picks for 148 SMs. Every output
    row is compared with the oracle."""
    from varlen_flashattention_02_b200 import fa_varlen

    assert fa_varlen.fa_varlen_splitkv_num_splits(batch, 1, 32, 8, keys, 148) == splits
    w = synth.decode_workload(batch, keys)
    t = w.tensors()
    q, k, v = (pu.to_dev(t[n]) for n in ("q", "k", "v"))
    out, lse = fa_varlen.fa_varlen_fwd_splitkv(q, k, v, pu.cu_dev(w.cu_q), w.max_seqlen_q, w.max_seqlen_k, w.scale,
                                               True, splits, cu_seqlens_k=pu.cu_dev(w.cu_k))
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True)
    _check(t["q"], w.cu_q, out, lse, ref_out, ref_lse, w.heads, w.head_dim, True)


def test_splitkv_workspace_reused():
    """The CTA that finishes a unit's last split merges the partials, counted
    in the workspace; the work-list kernel zeroes the counts at every call, so
    calls that reuse one workspace (different inputs, different split counts)
    each match the oracle."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    lq, lk, H, Hk, D = [1, 2, 1], [3000, 777, 4096], 16, 4, 128
    ws = fa_varlen.new_workspace(int(fa_varlen.lib.fa_varlen_fwd_splitkv_workspace_size(3, 4, H, Hk, D, 8)), "cuda")
    for seed, splits in ((851, 8), (852, 3), (853, 8)):
        w = synth.make_workload("reuse", lq, lk, heads=H, head_dim=D, causal=True, seed=seed, heads_k=Hk)
        t = w.tensors()
        q, k, v = (pu.to_dev(t[n]) for n in ("q", "k", "v"))
        out, lse = fa_varlen.fa_varlen_fwd_splitkv(q, k, v, pu.cu_dev(w.cu_q), w.max_seqlen_q, w.max_seqlen_k,
                                                   w.scale, True, splits, cu_seqlens_k=pu.cu_dev(w.cu_k),
                                                   workspace=ws)
        torch.cuda.synchronize()
        ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True)
        _check(t["q"], w.cu_q, out, lse, ref_out, ref_lse, H, D, True)
