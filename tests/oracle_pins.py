"""Pins of the fp64 oracle to facts fixed outside the oracle itself.

Each ``pin_*`` function takes a loaded oracle build (``oracle.OracleLib``) and
raises AssertionError if the build disagrees with: a closed form, an
invariant of softmax attention, a library routine (torch's fp64 CPU attention
and autograd), finite differences, a pure-Python brute force, or the worked
examples printed on the pages. ``test_oracle_pins.py`` runs them on the real
oracle; ``test_oracle_mutants.py`` runs them on deliberately broken copies to
show that each plausible mistake is caught.
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(rng, T, H, d):
    return rng.standard_normal((T, H, d))


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def _visible(i, j, lq, lk, causal):
    return (not causal) or (j <= i + (lk - lq))


# A small varlen batch covering lq < lk, lq > lk, lq == lk and a one-token sequence.
LQ = [5, 9, 1, 7]
LK = [8, 6, 1, 7]


def _batch(seed, H=2, d=4, lq=LQ, lk=LK):
    rng = np.random.default_rng(seed)
    cu_q, cu_k = _cu(lq), _cu(lk)
    q = _rand(rng, cu_q[-1], H, d)
    k = _rand(rng, cu_k[-1], H, d)
    v = _rand(rng, cu_k[-1], H, d)
    do = _rand(rng, cu_q[-1], H, d)
    return q, k, v, do, cu_q, cu_k


def pin_seqlens_golden(orc):
    """Worked examples of page 1 ("Estructuras de datos clave", "Ejemplo de uso
    con PyTorch"): [0,128,300] -> 128, 172 and [0,200,1024] -> 200, 824."""
    with open(os.path.join(GOLDEN, "cu_seqlens_examples.txt")) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 2
    for ln in rows:
        cu_s, len_s, _ = ln.split(";")
        cu = [int(x) for x in cu_s.split(",")]
        lens = [int(x) for x in len_s.split(",")]
        assert list(orc.seqlens(cu)) == lens


def pin_elem_offset(orc):
    """Page 1, "Optimización de acceso a memoria": in varlen mode the offset of
    a sequence is cu[b] times the row stride. Also checked against numpy's own
    index arithmetic for every (row, head) of a packed [T, H, d] tensor."""
    cu = np.array([0, 128, 300, 1000], dtype=np.int32)
    H, d = 12, 64
    for b in range(3):
        assert orc.elem_offset(cu, b, 0, H, 0, d) == int(cu[b]) * H * d
        for r in (0, 1, int(cu[b + 1] - cu[b]) - 1):
            for h in (0, 5, H - 1):
                want = int(np.ravel_multi_index((int(cu[b]) + r, h, 0), (int(cu[-1]), H, d)))
                assert orc.elem_offset(cu, b, r, H, h, d) == want
    # 64-bit: a packed tensor past 2^32 elements.
    big = np.array([0, 3_000_000, 6_000_000], dtype=np.int32)
    assert orc.elem_offset(big, 1, 5, 32, 31, 128) == (3_000_005 * 32 + 31) * 128


def pin_rows_sum_to_one(orc):
    """Softmax rows sum to 1: with V channel 0 set to 1, output channel 0 is
    the row sum of P (1 for rows with a visible key, 0 for rows without)."""
    for causal in (False, True):
        q, k, v, _, cu_q, cu_k = _batch(11)
        v[:, :, 0] = 1.0
        out, _ = orc.fwd(q, k, v, cu_q, cu_k, 0.7, causal)
        for b in range(len(LQ)):
            for i in range(LQ[b]):
                nvis = sum(_visible(i, j, LQ[b], LK[b], causal) for j in range(LK[b]))
                want = 1.0 if nvis else 0.0
                assert np.all(np.abs(out[cu_q[b] + i, :, 0] - want) < 1e-12)


def pin_lse_bounds(orc):
    """max_j S_ij <= LSE_i <= max_j S_ij + ln(#visible), S = scale q.k."""
    scale = 0.9
    for causal in (False, True):
        q, k, v, _, cu_q, cu_k = _batch(12)
        _, lse = orc.fwd(q, k, v, cu_q, cu_k, scale, causal)
        for b in range(len(LQ)):
            for h in range(q.shape[1]):
                S = scale * q[cu_q[b]:cu_q[b + 1], h] @ k[cu_k[b]:cu_k[b + 1], h].T
                for i in range(LQ[b]):
                    vis = [j for j in range(LK[b]) if _visible(i, j, LQ[b], LK[b], causal)]
                    l = lse[h, cu_q[b] + i]
                    if not vis:
                        assert l == -np.inf
                        continue
                    mx = max(S[i, j] for j in vis)
                    assert mx - 1e-12 <= l <= mx + math.log(len(vis)) + 1e-12


def pin_varlen_independence(orc):
    """The varlen result equals each sequence run alone (bitwise in fp64)."""
    for causal in (False, True):
        q, k, v, do, cu_q, cu_k = _batch(13)
        out, lse = orc.fwd(q, k, v, cu_q, cu_k, 0.5, causal)
        dq, dk, dv = orc.bwd(q, k, v, do, cu_q, cu_k, 0.5, causal)
        for b in range(len(LQ)):
            sq = slice(cu_q[b], cu_q[b + 1])
            sk = slice(cu_k[b], cu_k[b + 1])
            one_q = np.array([0, LQ[b]], dtype=np.int32)
            one_k = np.array([0, LK[b]], dtype=np.int32)
            o1, l1 = orc.fwd(q[sq], k[sk], v[sk], one_q, one_k, 0.5, causal)
            g = orc.bwd(q[sq], k[sk], v[sk], do[sq], one_q, one_k, 0.5, causal)
            assert np.array_equal(o1, out[sq]) and np.array_equal(l1, lse[:, sq])
            assert np.array_equal(g[0], dq[sq]) and np.array_equal(g[1], dk[sk])
            assert np.array_equal(g[2], dv[sk])


def pin_single_key(orc):
    """One visible key: the output is that V row and LSE = scale q.k."""
    rng = np.random.default_rng(14)
    H, d = 3, 5
    q, k, v = _rand(rng, 4, H, d), _rand(rng, 1, H, d), _rand(rng, 1, H, d)
    cu_q, cu_k = _cu([4]), _cu([1])
    out, lse = orc.fwd(q, k, v, cu_q, cu_k, 0.3, False)
    for i in range(4):
        for h in range(H):
            assert np.allclose(out[i, h], v[0, h], rtol=0, atol=1e-14)
            assert abs(lse[h, i] - 0.3 * float(np.dot(q[i, h], k[0, h]))) < 1e-12


def pin_causal_row0(orc):
    """Causal with lq == lk: row 0 sees only key 0, so out[0] = v[0] and
    LSE[0] = scale q0.k0; row 1 is the two-key closed form."""
    rng = np.random.default_rng(15)
    H, d, n = 2, 6, 5
    q, k, v = _rand(rng, n, H, d), _rand(rng, n, H, d), _rand(rng, n, H, d)
    cu = _cu([n])
    out, lse = orc.fwd(q, k, v, cu, cu, 0.4, True)
    for h in range(H):
        assert np.allclose(out[0, h], v[0, h], rtol=0, atol=1e-14)
        assert abs(lse[h, 0] - 0.4 * float(np.dot(q[0, h], k[0, h]))) < 1e-12
        s0 = 0.4 * float(np.dot(q[1, h], k[0, h]))
        s1 = 0.4 * float(np.dot(q[1, h], k[1, h]))
        w1 = 1.0 / (1.0 + math.exp(s0 - s1))  # logistic of the score gap
        assert np.allclose(out[1, h], (1 - w1) * v[0, h] + w1 * v[1, h], rtol=0, atol=1e-13)


def pin_constant_v(orc):
    """A constant V row vector c gives out = c on visible rows, and then
    dQ = dK = 0 while dV sums dO over the rows that see each key."""
    q, k, v, do, cu_q, cu_k = _batch(16)
    c = np.array([0.25, -1.5, 2.0, 0.125])
    v[:] = c
    for causal in (False, True):
        out, _ = orc.fwd(q, k, v, cu_q, cu_k, 1.1, causal)
        dq, dk, _ = orc.bwd(q, k, v, do, cu_q, cu_k, 1.1, causal)
        for b in range(len(LQ)):
            for i in range(LQ[b]):
                if any(_visible(i, j, LQ[b], LK[b], causal) for j in range(LK[b])):
                    assert np.allclose(out[cu_q[b] + i], c, rtol=0, atol=1e-13)
        assert np.max(np.abs(dq)) < 1e-12 and np.max(np.abs(dk)) < 1e-12


def _brute(q, k, v, do, cu_q, cu_k, scale, causal):
    """Pure-Python definition with math.fsum, row by row (no numpy math).
    k and v may have fewer heads than q: query head h reads key/value head
    h // (H // Hk)."""
    T, H, d = q.shape
    g = H // k.shape[1]
    out = [[[0.0] * d for _ in range(H)] for _ in range(T)]
    lse = [[0.0] * T for _ in range(H)]
    for b in range(len(cu_q) - 1):
        lq, lk = int(cu_q[b + 1] - cu_q[b]), int(cu_k[b + 1] - cu_k[b])
        for h in range(H):
            hk = h // g
            for i in range(lq):
                qi = [float(x) for x in q[cu_q[b] + i, h]]
                vis = [j for j in range(lk) if _visible(i, j, lq, lk, causal)]
                if not vis:
                    lse[h][cu_q[b] + i] = -math.inf
                    continue
                s = {j: scale * math.fsum(qi[c] * float(k[cu_k[b] + j, hk, c]) for c in range(d))
                     for j in vis}
                mx = max(s.values())
                z = math.fsum(math.exp(s[j] - mx) for j in vis)
                lse[h][cu_q[b] + i] = mx + math.log(z)
                for c in range(d):
                    out[cu_q[b] + i][h][c] = math.fsum(
                        math.exp(s[j] - mx) / z * float(v[cu_k[b] + j, hk, c]) for j in vis)
    return np.array(out), np.array(lse)


def pin_bruteforce(orc):
    """Tiny inputs (lq, lk <= 4, d <= 4) against the pure-Python brute force,
    with as many key/value heads as query heads and with 2 query heads per
    key/value head."""
    for causal in (False, True):
        for lq, lk, Hk in (([3, 4, 1], [4, 2, 3], 2), ([3, 4, 1], [4, 2, 3], 1)):
            q, k, v, do, cu_q, cu_k = _batch(17, H=2, d=3, lq=lq, lk=lk)
            k, v = k[:, :Hk], v[:, :Hk]
            out, lse = orc.fwd(q, k, v, cu_q, cu_k, 0.8, causal)
            bo, bl = _brute(q, k, v, do, cu_q, cu_k, 0.8, causal)
            assert np.allclose(out, bo, rtol=0, atol=1e-13)
            fin = np.isfinite(bl)
            assert np.array_equal(fin, np.isfinite(lse))
            assert np.allclose(lse[fin], bl[fin], rtol=0, atol=1e-13)


def pin_torch_sdpa(orc):
    """Per sequence, the definition is what torch's fp64 CPU
    scaled_dot_product_attention computes with the same boolean mask, and its
    autograd gives the gradients of sum(out * dout)."""
    import torch

    for causal in (False, True):
        q, k, v, do, cu_q, cu_k = _batch(18, H=3, d=8, lq=[6, 9, 7], lk=[9, 4, 7])
        out, lse = orc.fwd(q, k, v, cu_q, cu_k, 0.6, causal)
        dq, dk, dv = orc.bwd(q, k, v, do, cu_q, cu_k, 0.6, causal)
        for b in range(3):
            sq, sk = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
            lq, lk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
            mask = torch.tensor([[_visible(i, j, lq, lk, causal) for j in range(lk)] for i in range(lq)])
            rows_ok = mask.any(dim=1)
            # torch gives NaN for a row with nothing visible: let such rows see
            # every key and zero their dout, so they add no gradient anywhere.
            tmask = mask | ~rows_ok[:, None]
            tq = torch.tensor(q[sq]).transpose(0, 1).requires_grad_(True)
            tk = torch.tensor(k[sk]).transpose(0, 1).requires_grad_(True)
            tv = torch.tensor(v[sk]).transpose(0, 1).requires_grad_(True)
            to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tmask, scale=0.6)
            tdo = torch.tensor(do[sq]).transpose(0, 1) * rows_ok[None, :, None]
            (to * tdo).sum().backward()
            got = torch.tensor(out[sq]).transpose(0, 1)
            assert torch.allclose(got[:, rows_ok], to.detach()[:, rows_ok], rtol=0, atol=1e-12)
            sc = (tq.detach() @ tk.detach().transpose(1, 2)) * 0.6
            tl = torch.logsumexp(sc.masked_fill(~mask, -math.inf), dim=-1)
            gl = torch.tensor(lse[:, sq])
            assert torch.allclose(gl[:, rows_ok], tl[:, rows_ok], rtol=0, atol=1e-12)
            assert torch.allclose(torch.tensor(dq[sq]).transpose(0, 1)[:, rows_ok],
                                  tq.grad[:, rows_ok], rtol=0, atol=1e-11)
            assert torch.allclose(torch.tensor(dk[sk]).transpose(0, 1), tk.grad, rtol=0, atol=1e-11)
            assert torch.allclose(torch.tensor(dv[sk]).transpose(0, 1), tv.grad, rtol=0, atol=1e-11)


def pin_finite_differences(orc):
    """Central differences of L = sum(out * dout) w.r.t. q, k and v."""
    lq, lk = [3, 2], [4, 3]
    for causal in (False, True):
        q, k, v, do, cu_q, cu_k = _batch(19, H=1, d=3, lq=lq, lk=lk)
        grads = orc.bwd(q, k, v, do, cu_q, cu_k, 0.7, causal)

        def loss(q_, k_, v_):
            o, _ = orc.fwd(q_, k_, v_, cu_q, cu_k, 0.7, causal)
            return float(np.sum(o * do))

        eps = 1e-6
        for which, arr in enumerate((q, k, v)):
            num = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += eps
                lp = loss(*args)
                args[which][idx] -= 2 * eps
                lm = loss(*args)
                num[idx] = (lp - lm) / (2 * eps)
            err = np.linalg.norm(num - grads[which]) / max(np.linalg.norm(num), 1e-30)
            assert err <= 1e-6, (which, err)


def pin_grad_invariants(orc):
    """Rows of P sum to 1, so sum_j dV_j = sum of dO over rows with a visible
    key; rows of dS sum to 0, so sum_j dK_j = 0 (per sequence and head)."""
    for causal in (False, True):
        q, k, v, do, cu_q, cu_k = _batch(20)
        _, dk, dv = orc.bwd(q, k, v, do, cu_q, cu_k, 0.9, causal)
        for b in range(len(LQ)):
            sk = slice(cu_k[b], cu_k[b + 1])
            rows = [cu_q[b] + i for i in range(LQ[b])
                    if any(_visible(i, j, LQ[b], LK[b], causal) for j in range(LK[b]))]
            want = do[rows].sum(axis=0) if rows else np.zeros(do.shape[1:])
            assert np.allclose(dv[sk].sum(axis=0), want, rtol=0, atol=1e-12)
            assert np.allclose(dk[sk].sum(axis=0), 0.0, rtol=0, atol=1e-12)


def pin_empty_rows(orc):
    """Rows with no visible key (causal with lq > lk; lk = 0): out 0, LSE -inf,
    no gradient; an empty query sequence contributes nothing."""
    q, k, v, do, cu_q, cu_k = _batch(21, H=2, d=4, lq=[6, 3, 0], lk=[2, 0, 3])
    out, lse = orc.fwd(q, k, v, cu_q, cu_k, 1.0, True)
    dq, dk, dv = orc.bwd(q, k, v, do, cu_q, cu_k, 1.0, True)
    # sequence 0: lq=6, lk=2 -> row i sees keys j <= i - 4: rows 0..3 see nothing.
    assert np.all(out[0:4] == 0.0) and np.all(lse[:, 0:4] == -np.inf)
    assert np.all(dq[0:4] == 0.0)
    assert np.all(np.isfinite(lse[:, 4:6]))
    # sequence 1: no keys at all.
    assert np.all(out[6:9] == 0.0) and np.all(lse[:, 6:9] == -np.inf) and np.all(dq[6:9] == 0.0)
    # sequence 2: no queries; its keys get zero gradients.
    assert np.all(dk[2:5] == 0.0) and np.all(dv[2:5] == 0.0)


def pin_bf16_path(orc):
    """bf16 bit-pattern inputs give exactly the fp64 result of the widened values."""
    from varlen_flashattention_02_b200 import synth

    rng = np.random.default_rng(22)
    cu_q, cu_k = _cu([5, 3]), _cu([4, 6])
    qb = synth.bf16_normal(rng, (8, 2, 8))
    kb = synth.bf16_normal(rng, (10, 2, 8))
    vb = synth.bf16_normal(rng, (10, 2, 8))
    dob = synth.bf16_normal(rng, (8, 2, 8))
    wide = [synth.bf16_bits_to_f32(x).astype(np.float64) for x in (qb, kb, vb, dob)]
    for causal in (False, True):
        a = orc.fwd(qb, kb, vb, cu_q, cu_k, 0.35, causal)
        b = orc.fwd(*wide[:3], cu_q, cu_k, 0.35, causal)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
        ga = orc.bwd(qb, kb, vb, dob, cu_q, cu_k, 0.35, causal)
        gb = orc.bwd(*wide, cu_q, cu_k, 0.35, causal)
        assert all(np.array_equal(x, y) for x, y in zip(ga, gb))


def pin_row_and_unit_sampling(orc):
    """A sample of units or of query rows is exactly the full result on the
    sampled entries (rows of the forward are independent)."""
    q, k, v, do, cu_q, cu_k = _batch(23, H=3, d=4, lq=[9, 12], lk=[7, 12])
    for causal in (False, True):
        full_o, full_l = orc.fwd(q, k, v, cu_q, cu_k, 0.45, causal)
        o, l = orc.fwd(q, k, v, cu_q, cu_k, 0.45, causal, units=[(1, 2), (0, 0)], row_step=4)
        for b, h in ((1, 2), (0, 0)):
            rows = [cu_q[b] + i for i in range(0, cu_q[b + 1] - cu_q[b], 4)]
            assert np.array_equal(o[rows, h], full_o[rows, h])
            assert np.array_equal(l[h, rows], full_l[h, rows])
        assert np.isnan(o[cu_q[0] + 1, 0, 0]) and np.isnan(o[0, 1, 0])
        g_full = orc.bwd(q, k, v, do, cu_q, cu_k, 0.45, causal)
        g = orc.bwd(q, k, v, do, cu_q, cu_k, 0.45, causal, units=[(1, 1)])
        sq, sk = slice(cu_q[1], cu_q[2]), slice(cu_k[1], cu_k[2])
        assert np.array_equal(g[0][sq, 1], g_full[0][sq, 1])
        assert np.array_equal(g[1][sk, 1], g_full[1][sk, 1])
        assert np.array_equal(g[2][sk, 1], g_full[2][sk, 1])


def _repeat_heads(x, g):
    """[T, Hk, d] -> [T, Hk * g, d], each key/value head repeated g times in a
    row (query heads h = hk*g .. hk*g + g - 1 read head hk)."""
    return np.repeat(x, g, axis=1)


def pin_gqa_is_repeated_heads(orc):
    """Grouped-query attention is multi-head attention on key/value heads
    repeated across their group (page "Flash-Atención y Flash-Atención-2",
    FlashAttention-2 section: several query heads attend to one key/value
    head): out, lse and dq equal those of the repeated-head inputs exactly,
    and dk, dv of a shared head are the sums over its group."""
    for H, Hk in ((6, 2), (6, 3), (4, 1)):
        g = H // Hk
        # d >= H keeps a planted head-stride mistake in bounds (see the mutants).
        q, k, v, do, cu_q, cu_k = _batch(24, H=H, d=6, lq=[7, 4, 9], lk=[6, 8, 9])
        k, v = k[:, :Hk].copy(), v[:, :Hk].copy()
        kr, vr = _repeat_heads(k, g), _repeat_heads(v, g)
        for causal in (False, True):
            o, l = orc.fwd(q, k, v, cu_q, cu_k, 0.55, causal)
            ro, rl = orc.fwd(q, kr, vr, cu_q, cu_k, 0.55, causal)
            assert np.array_equal(o, ro) and np.array_equal(l, rl)
            dq, dk, dv = orc.bwd(q, k, v, do, cu_q, cu_k, 0.55, causal)
            rq, rk, rv = orc.bwd(q, kr, vr, do, cu_q, cu_k, 0.55, causal)
            assert np.array_equal(dq, rq)
            T = k.shape[0]
            assert np.allclose(dk, rk.reshape(T, Hk, g, -1).sum(axis=2), rtol=0, atol=1e-12)
            assert np.allclose(dv, rv.reshape(T, Hk, g, -1).sum(axis=2), rtol=0, atol=1e-12)


def pin_gqa_torch_sdpa(orc):
    """Grouped-query attention against torch's fp64 CPU
    scaled_dot_product_attention with enable_gqa (which maps query head h to
    key/value head h // (H // Hk)) and its autograd."""
    import torch

    H, Hk = 4, 2
    for causal in (False, True):
        q, k, v, do, cu_q, cu_k = _batch(25, H=H, d=6, lq=[5, 8], lk=[8, 5])
        k, v = k[:, :Hk].copy(), v[:, :Hk].copy()
        out, lse = orc.fwd(q, k, v, cu_q, cu_k, 0.5, causal)
        dq, dk, dv = orc.bwd(q, k, v, do, cu_q, cu_k, 0.5, causal)
        for b in range(2):
            sq, sk = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
            lq, lk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
            mask = torch.tensor([[_visible(i, j, lq, lk, causal) for j in range(lk)] for i in range(lq)])
            rows_ok = mask.any(dim=1)
            tmask = mask | ~rows_ok[:, None]
            tq = torch.tensor(q[sq]).transpose(0, 1).requires_grad_(True)
            tk = torch.tensor(k[sk]).transpose(0, 1).requires_grad_(True)
            tv = torch.tensor(v[sk]).transpose(0, 1).requires_grad_(True)
            to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tmask, scale=0.5,
                                                                  enable_gqa=True)
            tdo = torch.tensor(do[sq]).transpose(0, 1) * rows_ok[None, :, None]
            (to * tdo).sum().backward()
            got = torch.tensor(out[sq]).transpose(0, 1)
            assert torch.allclose(got[:, rows_ok], to.detach()[:, rows_ok], rtol=0, atol=1e-12)
            assert torch.allclose(torch.tensor(dq[sq]).transpose(0, 1)[:, rows_ok],
                                  tq.grad[:, rows_ok], rtol=0, atol=1e-11)
            assert torch.allclose(torch.tensor(dk[sk]).transpose(0, 1), tk.grad, rtol=0, atol=1e-11)
            assert torch.allclose(torch.tensor(dv[sk]).transpose(0, 1), tv.grad, rtol=0, atol=1e-11)


ALL_PINS = [
    pin_seqlens_golden, pin_elem_offset, pin_rows_sum_to_one, pin_lse_bounds,
    pin_varlen_independence, pin_single_key, pin_causal_row0, pin_constant_v,
    pin_bruteforce, pin_torch_sdpa, pin_finite_differences, pin_grad_invariants,
    pin_empty_rows, pin_bf16_path, pin_row_and_unit_sampling, pin_gqa_is_repeated_heads,
    pin_gqa_torch_sdpa,
]
