"""The fp64 oracle against facts fixed outside it (closed forms, invariants,
torch's fp64 attention and autograd, finite differences, brute force and the
pages' worked examples). CPU only."""
import math

import numpy as np
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return oracle._load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_blockwise_normalisation_is_not_attention(orc):
    """Page 2, "Bloques pequeños, normalización global": normalising each key
    block separately and summing is not the same computation. A two-block
    split of one row must differ from the oracle by far more than any
    tolerance used against the GPU."""
    rng = np.random.default_rng(30)
    lq, lk, d = 4, 256, 16
    q = rng.standard_normal((lq, 1, d))
    k = rng.standard_normal((lk, 1, d))
    v = rng.standard_normal((lk, 1, d))
    cu_q = np.array([0, lq], dtype=np.int32)
    cu_k = np.array([0, lk], dtype=np.int32)
    scale = 1.0 / math.sqrt(d)
    out, _ = orc.fwd(q, k, v, cu_q, cu_k, scale, False)
    s = scale * q[:, 0] @ k[:, 0].T
    naive = np.zeros((lq, d))
    for blk in (slice(0, 128), slice(128, 256)):
        p = np.exp(s[:, blk] - s[:, blk].max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        naive += p @ v[blk, 0]
    assert np.max(np.abs(naive - out[:, 0])) > 0.1


def test_seqlens_rejects_bad_offsets(orc):
    with pytest.raises(ValueError):
        orc.seqlens([1, 4, 6])
    with pytest.raises(ValueError):
        orc.seqlens([0, 4, 3])


def test_kvcache_layout_is_the_packed_definition():
    """Key/value cache layout (page 1, "Lógica de cálculo de longitud":
    non-cumulative key lengths with left padding): sequence b has
    seqlens_k[b] - leftpad_k[b] keys at slot rows leftpad_k[b] ..
    seqlens_k[b]-1. A cache built here by scattering packed keys into slots
    (garbage everywhere else) must give exactly the packed forward."""
    rng = np.random.default_rng(31)
    H, Hk, d, rows = 4, 2, 6, 40
    lk = np.array([12, 0, 25, 1])
    pad = np.array([3, 7, 15, 0])
    lq = [5, 3, 9, 1]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    q = rng.standard_normal((cu_q[-1], H, d))
    k = rng.standard_normal((cu_k[-1], Hk, d))
    v = rng.standard_normal((cu_k[-1], Hk, d))
    kc = rng.standard_normal((4, rows, Hk, d)) * 50.0
    vc = rng.standard_normal((4, rows, Hk, d)) * 50.0
    for b in range(4):
        kc[b, pad[b]:pad[b] + lk[b]] = k[cu_k[b]:cu_k[b + 1]]
        vc[b, pad[b]:pad[b] + lk[b]] = v[cu_k[b]:cu_k[b + 1]]
    seqlens_k = pad + lk
    kp, vp, ck = oracle.kvcache_to_packed(kc, vc, seqlens_k, pad)
    assert list(np.diff(ck)) == list(seqlens_k - pad)
    assert np.array_equal(kp, k) and np.array_equal(vp, v)
    for causal in (False, True):
        a = oracle.fwd_kvcache(q, kc, vc, cu_q, seqlens_k, pad, 0.4, causal)
        b_ = oracle.fwd(q, k, v, cu_q, cu_k, 0.4, causal)
        assert np.array_equal(a[0], b_[0]) and np.array_equal(a[1], b_[1])
    with pytest.raises(ValueError):
        oracle.kvcache_to_packed(kc, vc, np.array([5, 5, 5, 5]), np.array([6, 0, 0, 0]))
    with pytest.raises(ValueError):
        oracle.kvcache_to_packed(kc, vc, np.array([5, 5, rows + 1, 5]), None)


def test_paged_layout_is_the_packed_definition():
    """Paged key/value cache (the cu_seqlens page, "Integración con máscaras
    causales y caché paginada"): key position p of sequence b lives in page
    block_table[b][p // page_size], row p % page_size. Packed keys scattered
    into a shuffled page pool (garbage in unused pages and rows) must give
    exactly the packed forward."""
    rng = np.random.default_rng(32)
    H, Hk, d, ps = 2, 1, 5, 4
    lk = np.array([9, 0, 4, 13])
    lq = [3, 2, 4, 6]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    q = rng.standard_normal((cu_q[-1], H, d))
    k = rng.standard_normal((cu_k[-1], Hk, d))
    v = rng.standard_normal((cu_k[-1], Hk, d))
    n_pages, max_pages = 12, 5
    kp = rng.standard_normal((n_pages, ps, Hk, d)) * 40.0
    vp = rng.standard_normal((n_pages, ps, Hk, d)) * 40.0
    perm = rng.permutation(n_pages)
    bt = np.full((4, max_pages), -7, dtype=np.int32)  # unused entries are never read
    nxt = 0
    for b in range(4):
        for i in range(-(-lk[b] // ps)):
            bt[b, i] = perm[nxt]
            nxt += 1
        for pos in range(lk[b]):
            kp[bt[b, pos // ps], pos % ps] = k[cu_k[b] + pos]
            vp[bt[b, pos // ps], pos % ps] = v[cu_k[b] + pos]
    k2, v2, ck = oracle.paged_to_packed(kp, vp, lk, bt)
    assert np.array_equal(ck, cu_k) and np.array_equal(k2, k) and np.array_equal(v2, v)
    for causal in (False, True):
        a = oracle.fwd_paged(q, kp, vp, cu_q, lk, bt, 0.45, causal)
        b_ = oracle.fwd(q, k, v, cu_q, cu_k, 0.45, causal)
        assert np.array_equal(a[0], b_[0]) and np.array_equal(a[1], b_[1])
    bad = bt.copy()
    bad[0, 1] = n_pages
    with pytest.raises(ValueError):
        oracle.paged_to_packed(kp, vp, lk, bad)
