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


# Decode calls (at most one query tile per sequence) run without a work list:
# the decode kernel checks every sequence itself. Each case breaks one check.
# (name, layout, cu_q, max_seqlen_q, key description)
BAD = [
    ("cu_q-decreasing", "packed", [0, 2, 1, 3], 4, None),
    ("cu_q-end", "packed", [0, 1, 2, 2], 4, None),
    ("lq-over-max", "packed", [0, 3, 4, 5], 2, None),
    ("cu_k-end", "packed", [0, 1, 2, 3], 4, "cu_k_end"),
    ("slots-leftpad", "slots", [0, 1, 2, 3], 4, "leftpad"),
    ("slots-rows", "slots", [0, 1, 2, 3], 4, "rows"),
    ("paged-page", "paged", [0, 1, 2, 3], 4, "page"),
    ("paged-len", "paged", [0, 1, 2, 3], 4, "len"),
]


@pytest.mark.parametrize("case", BAD, ids=[c[0] for c in BAD])
def test_splitkv_bad_sequences_reported(case):
    """A malformed sequence is reported as FA_ERR_BAD_SEQLENS; the same
    workspace then serves a well-formed call, which matches the oracle."""
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    name, layout, cu_q, max_q, kind = case
    rng = np.random.default_rng(861)
    H, Hk, D, batch, Tq = 8, 2, 128, 3, cu_q[-1] if name != "cu_q-end" else 3
    q = pu.to_dev(synth.bf16_normal(rng, (Tq, H, D)))
    cq = _dev(np.array(cu_q, dtype=np.int32))
    scale = 1.0 / np.sqrt(D)
    ws = fa_varlen.new_workspace(int(fa_varlen.lib.fa_varlen_fwd_splitkv_workspace_size(batch, Tq, H, Hk, D, 4)), "cuda")
    if layout == "packed":
        ck_np = np.array([0, 300, 500, 900], dtype=np.int32)
        if kind == "cu_k_end":
            ck_np[-1] = 800  # the keys' offsets end short of total_k (900 rows)
        k = pu.to_dev(synth.bf16_normal(rng, (900, Hk, D)))
        v = pu.to_dev(synth.bf16_normal(rng, (900, Hk, D)))
        kw = dict(cu_seqlens_k=_dev(ck_np))
        max_k = 400
    elif layout == "slots":
        rows = 512
        k = pu.to_dev(synth.bf16_normal(rng, (batch, rows, Hk, D)))
        v = pu.to_dev(synth.bf16_normal(rng, (batch, rows, Hk, D)))
        sl = np.array([300, 200, 512], dtype=np.int32)
        lp = np.array([0, 10, 5], dtype=np.int32)
        if kind == "leftpad":
            lp[1] = 250  # left padding past the sequence end
        else:
            sl[2] = 600  # more rows than the cache slot has
        kw = dict(seqlens_k=_dev(sl), leftpad_k=_dev(lp))
        max_k = 1024
    else:
        ps, n_pages = 256, 6
        k = pu.to_dev(synth.bf16_normal(rng, (n_pages, ps, Hk, D)))
        v = pu.to_dev(synth.bf16_normal(rng, (n_pages, ps, Hk, D)))
        bt = np.array([[0, 1], [2, 3], [4, 5]], dtype=np.int32)
        sl = np.array([300, 256, 400], dtype=np.int32)
        if kind == "page":
            bt[2, 1] = 7  # a page outside the 6-page pool
        else:
            sl[1] = 600  # more keys than two pages hold
        kw = dict(seqlens_k=_dev(sl), block_table=_dev(bt))
        max_k = 1024
    fa_varlen.fa_varlen_fwd_splitkv(q, k, v, cq, max_q, max_k, scale, True, 4, workspace=ws, **kw)
    assert fa_varlen.device_status(ws) == 5  # FA_ERR_BAD_SEQLENS
    # A well-formed call on the same workspace.
    good = synth.make_workload("bad-then-good", [1, 1, 1], [300, 200, 400], heads=H, head_dim=D, causal=True,
                               seed=862, heads_k=Hk)
    t = good.tensors()
    out, lse = fa_varlen.fa_varlen_fwd_splitkv(pu.to_dev(t["q"]), pu.to_dev(t["k"]), pu.to_dev(t["v"]),
                                               pu.cu_dev(good.cu_q), 1, 400, good.scale, True, 4,
                                               cu_seqlens_k=pu.cu_dev(good.cu_k), workspace=ws)
    assert fa_varlen.device_status(ws) == 0
    ref_out, ref_lse = oracle.fwd(t["q"], t["k"], t["v"], good.cu_q, good.cu_k, good.scale, True)
    _check(t["q"], good.cu_q, out, lse, ref_out, ref_lse, H, D, True)
