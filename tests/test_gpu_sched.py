"""The device work-list preparation against its CPU restatement, and the
device-side rejection of malformed cumulative offsets."""
import numpy as np
import pytest

from tests import parity_util as pu
from tests import sched_restatement as sr
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu


def _read_pairs(ws, backward, batch, total_q, total_k, with_classes=False):
    lay = sr.layout(batch, total_q, total_k, backward)
    raw = ws.cpu().numpy()
    status, n_pairs = (int(x) for x in raw[:8].view(np.uint32))
    pairs = raw[lay["pairs"]:lay["pairs"] + 8 * n_pairs].view(np.int32).reshape(-1, 2)
    if with_classes:
        # header words 4..15: number of pairs of cost >= 2^k, k = 0..11
        return status, pairs, raw[16:64].view(np.uint32).astype(np.int64)
    return status, pairs


def _check_order(pairs, want, class_end):
    cost = {(b, t): c for b, t, c in want}
    got = [(int(b), int(t)) for b, t in pairs]
    assert sorted(got) == sorted(cost)  # same multiset, no padding tiles
    costs = [cost[p] for p in got]
    assert all(costs[i] >= costs[i + 1] for i in range(len(costs) - 1))  # longest first
    clamped = np.minimum(np.array(costs, dtype=np.int64), 2047)
    assert [int(x) for x in class_end] == [int(np.sum(clamped >= (1 << k))) for k in range(12)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("wl", [1, 3, 5])
def test_fwd_work_list(wl, causal):
    from varlen_flashattention_02_b200 import fa_varlen

    w = synth.standard_workload(wl)
    w.causal = causal
    ws = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(w.batch, w.total_q, w.heads, w.head_dim), "cuda")
    pu.run_fwd(w, workspace=ws)
    status, pairs, class_end = _read_pairs(ws, False, w.batch, w.total_q, w.total_k, with_classes=True)
    assert status == 0
    _check_order(pairs, sr.work_list(w.cu_q, w.cu_k, causal), class_end)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("wl", [3, 5])
def test_bwd_work_list(wl, causal):
    """The backward's list (key tiles, ordered by the query tiles that see
    them) and its cost-class boundaries, which set the backward's work
    order."""
    from varlen_flashattention_02_b200 import fa_varlen

    w = synth.standard_workload(wl)
    w.causal = causal
    (q, k, v), out, lse = pu.run_fwd(w)
    ws = fa_varlen.new_workspace(fa_varlen.bwd_workspace_size(w.batch, w.total_q, w.total_k, w.heads, w.head_dim),
                                 "cuda")
    do = pu.to_dev(w.tensors()["dout"])
    fa_varlen.fa_varlen_bwd(do, q, k, v, out, lse, pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k), w.max_seqlen_q,
                            w.max_seqlen_k, w.scale, causal, workspace=ws)
    status, pairs, class_end = _read_pairs(ws, True, w.batch, w.total_q, w.total_k, with_classes=True)
    assert status == 0
    _check_order(pairs, sr.work_list(w.cu_q, w.cu_k, causal, backward=True), class_end)


@pytest.mark.parametrize("cu_q,cu_k,max_q", [
    ([0, 10, 5, 20], [0, 10, 15, 20], 64),   # decreasing
    ([1, 10, 20], [0, 10, 20], 64),          # does not start at 0
    ([0, 10, 20], [0, 10, 20], 8),           # longer than max_seqlen
], ids=["decreasing", "nonzero-start", "over-max"])
def test_bad_seqlens_reported(cu_q, cu_k, max_q):
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    H, D = 2, 64
    Tq, Tk = 20, 20
    q = torch.randn(Tq, H, D, device="cuda").bfloat16()
    k = torch.randn(Tk, H, D, device="cuda").bfloat16()
    v = torch.randn(Tk, H, D, device="cuda").bfloat16()
    ws = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(2, Tq, H, D), "cuda")
    cq = torch.tensor(cu_q, dtype=torch.int32, device="cuda")
    ck = torch.tensor(cu_k, dtype=torch.int32, device="cuda")
    fa_varlen.fa_varlen_fwd(q, k, v, cq, ck, max_q, 64, 0.125, False, workspace=ws)
    assert fa_varlen.device_status(ws) == 5  # FA_ERR_BAD_SEQLENS
    # The same workspace is usable again afterwards.
    good = torch.tensor([0, 10, 20], dtype=torch.int32, device="cuda")
    fa_varlen.fa_varlen_fwd(q, k, v, good, good, 10, 10, 0.125, False, workspace=ws)
    assert fa_varlen.device_status(ws) == 0


@pytest.mark.parametrize("D", [64, 128])
def test_device_timeout_reported(D):
    """Failure detection on the device without any fault: with a 10 ms wait
    limit and the test hook that withholds the first value-tile load of work
    item 0, the MMA warp's bounded wait for that tile runs out; the CTA stops,
    the workspace status reads FA_ERR_DEVICE_TIMEOUT, and the context stays
    usable: the next ordinary call on the same workspace returns FA_OK with
    parity."""
    import torch

    import oracle
    from varlen_flashattention_02_b200 import fa_varlen

    w = synth.make_workload("timeout", [700, 300, 129], heads=2, head_dim=D, causal=True, seed=61)
    ws = fa_varlen.new_workspace(fa_varlen.fwd_workspace_size(w.batch, w.total_q, w.heads, w.head_dim), "cuda")
    lib = fa_varlen.lib
    lib.fa_set_test_hooks(10_000_000, 1)
    try:
        pu.run_fwd(w, workspace=ws)
        assert fa_varlen.device_status(ws) == 6  # FA_ERR_DEVICE_TIMEOUT
    finally:
        lib.fa_set_test_hooks(0, 0)
    (_, _, _), out, lse = pu.run_fwd(w, workspace=ws)
    torch.cuda.synchronize()
    assert fa_varlen.device_status(ws) == 0
    t = w.tensors()
    ro, rl = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal)
    rows = np.repeat(np.arange(w.total_q), w.heads)
    heads = np.tile(np.arange(w.heads), w.total_q)
    pu.check_fwd(w, out, lse, ro, rl, rows, heads)
