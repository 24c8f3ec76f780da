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
