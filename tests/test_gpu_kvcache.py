"""GPU parity of the forward over a key/value cache (per-sequence key
lengths with left padding, keys in fixed-size slots; page "Mecanismo
cu_seqlens en FlashAttention", "Lógica de cálculo de longitud") against the
fp64 oracle, through fa_varlen_fwd_kvcache."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu

# (name, query lengths, key lengths kept, left padding, slot rows, H, Hk, D)
CASES = [
    ("prefill-chunks", [5, 128, 1, 300], [600, 100, 1, 177], [0, 30, 0, 200], 600, 4, 2, 128),
    ("decode-like", [1, 1, 2, 1, 1, 16], [513, 1, 1000, 64, 0, 250], [7, 0, 24, 0, 3, 130], 1100, 8, 1, 64),
    ("no-padding", [260, 70], [700, 129], [0, 0], 700, 2, 2, 128),
]


def _make(case, causal, seed):
    name, lq, lk, pad, rows, H, Hk, D = case
    rng = np.random.default_rng(seed)
    batch = len(lq)
    cu_q = synth.cu_from_lengths(lq)
    q = synth.bf16_normal(rng, (int(cu_q[-1]), H, D))
    kc = synth.bf16_normal(rng, (batch, rows, Hk, D))
    vc = synth.bf16_normal(rng, (batch, rows, Hk, D))
    seqlens_k = np.array(pad, dtype=np.int32) + np.array(lk, dtype=np.int32)
    return cu_q, q, kc, vc, seqlens_k, np.array(pad, dtype=np.int32), 1.0 / np.sqrt(D)


def _run(cu_q, q, kc, vc, seqlens_k, pad, scale, causal, use_pad=True):
    import torch
    from varlen_flashattention_02_b200 import fa_varlen

    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return fa_varlen.fa_varlen_fwd_kvcache(pu.to_dev(q), pu.to_dev(kc), pu.to_dev(vc), dev(cu_q), dev(seqlens_k),
                                           dev(pad) if use_pad else None, int(np.max(np.diff(cu_q))), scale,
                                           causal)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_kvcache_small(case, causal):
    cu_q, q, kc, vc, seqlens_k, pad, scale = _make(case, causal, 401 + len(case[1]))
    use_pad = bool(np.any(pad))
    out, lse = _run(cu_q, q, kc, vc, seqlens_k, pad, scale, causal, use_pad)
    ref_out, ref_lse = oracle.fwd_kvcache(q, kc, vc, cu_q, seqlens_k, pad if use_pad else None, scale, causal)
    H = q.shape[1]
    w = synth.make_workload("kv", np.diff(cu_q), heads=H, head_dim=q.shape[2], causal=causal)
    rows = np.repeat(np.arange(int(cu_q[-1])), H)
    heads = np.tile(np.arange(H), int(cu_q[-1]))
    pu.check_fwd(w, out, lse, ref_out, ref_lse, rows, heads)


def test_kvcache_equals_packed_forward():
    """The cache layout changes only where the keys are read from: the same
    keys packed with cumulative offsets give the same bits."""
    import torch
    from varlen_flashattention_02_b200 import fa_varlen

    case = CASES[0]
    cu_q, q, kc, vc, seqlens_k, pad, scale = _make(case, True, 411)
    out, lse = _run(cu_q, q, kc, vc, seqlens_k, pad, scale, True)
    k, v, cu_k = oracle.kvcache_to_packed(kc, vc, seqlens_k, pad)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out_p, lse_p = fa_varlen.fa_varlen_fwd_gqa(pu.to_dev(q), pu.to_dev(k), pu.to_dev(v), dev(cu_q), dev(cu_k),
                                               int(np.max(np.diff(cu_q))), int(np.max(np.diff(cu_k))), scale, True)
    assert torch.equal(out, out_p) and torch.equal(lse, lse_p)


def test_kvcache_rejects_padding_beyond_length():
    """leftpad_k[b] > seqlens_k[b] is a malformed cache description: the
    device check records FA_ERR_BAD_SEQLENS in the workspace status."""
    import torch
    from varlen_flashattention_02_b200 import fa_varlen

    case = CASES[2]
    cu_q, q, kc, vc, seqlens_k, pad, scale = _make(case, False, 421)
    bad_pad = pad.copy()
    bad_pad[1] = seqlens_k[1] + 1
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ws = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(2, int(cu_q[-1]), q.shape[1], q.shape[2]), "cuda")
    fa_varlen.fa_varlen_fwd_kvcache(pu.to_dev(q), pu.to_dev(kc), pu.to_dev(vc), dev(cu_q), dev(seqlens_k),
                                    dev(bad_pad), int(np.max(np.diff(cu_q))), scale, False, workspace=ws)
    assert fa_varlen.device_status(ws) == 5  # FA_ERR_BAD_SEQLENS
