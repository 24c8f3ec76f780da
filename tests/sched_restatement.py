"""CPU restatement of the work-list preparation, for checking the device
scheduler bit for bit (as a multiset, plus the longest-first order).

Tile counts follow page "Mecanismo cu_seqlens en FlashAttention",
"Lógica de cálculo de longitud": sequence b has cu[b+1] - cu[b] rows, so it
contributes ceil(len / 256) forward items (query blocks of 256 rows) and
ceil(len_k / 128) backward items (key tiles); the cost of an item is the
number of 128-row tiles on the other side that it must visit under the
(bottom-right) causal rule.
"""
from __future__ import annotations

FWD_BM = FWD_BN = 128
FWD_ITEM_ROWS = 256
BWD_BN, BWD_BM = 128, 128
HEADER = 256
BINS = 2048


def align(x, a):
    return (x + a - 1) // a * a


def fwd_cost(t, lq, lk, causal):
    if lk <= 0 or lq <= 0:
        return 0
    nk = -(-lk // FWD_BN)
    if not causal:
        return nk
    rmax = min((t + 1) * FWD_ITEM_ROWS, lq) - 1
    last = rmax + lk - lq
    if last < 0:
        return 0
    return min(nk, last // FWD_BN + 1)


def bwd_cost(j, lq, lk, causal):
    nq = -(-lq // BWD_BM)
    if lk <= 0 or lq <= 0:
        return 0
    if not causal:
        return nq
    first = max(j * BWD_BN - (lk - lq), 0)
    begin = nq if first >= lq else first // BWD_BM
    return nq - begin


def work_list(cu_q, cu_k, causal, backward=False):
    """All (sequence, tile, cost) triples."""
    out = []
    for b in range(len(cu_q) - 1):
        lq, lk = int(cu_q[b + 1] - cu_q[b]), int(cu_k[b + 1] - cu_k[b])
        n = -(-(lk if backward else lq) // (BWD_BN if backward else FWD_ITEM_ROWS))
        for t in range(n):
            c = bwd_cost(t, lq, lk, causal) if backward else fwd_cost(t, lq, lk, causal)
            out.append((b, t, min(c, BINS - 1)))
    return out


def layout(batch, total_q, total_k, backward=False):
    seq_off = HEADER
    pairs = align(seq_off + 4 * (batch + 1), 256)
    max_pairs = (total_k // BWD_BN if backward else total_q // FWD_ITEM_ROWS) + batch + 1
    return {"seq_off": seq_off, "pairs": pairs, "max_pairs": max_pairs}
