"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, timing
aggregated as the max over ranks, whole-job weak-scaling value."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank  # rank 1 is the slow one
        out[rank] = bench.max_over_ranks(mine)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 15.0


def test_max_over_ranks_without_group():
    import bench

    assert bench.max_over_ranks(3.25) == 3.25


def test_weak_scaling_value():
    import bench

    # 2 ranks, 1e12 FLOP each per step, slowest step 2 ms -> 1000 TFLOP/s whole job.
    assert bench.weak_scaling_value(2, 1e12, 2.0) == pytest.approx(1000.0)
    assert bench.weak_scaling_value(1, 3.5e11, 1.0) == pytest.approx(350.0)


def _head_split_worker(rank, world, port, out):
    """One rank of a head-split problem: its slice of a small workload through
    the oracle, then the slices gathered over gloo and reassembled on rank 0."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    from varlen_flashattention_02_b200 import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.make_workload("split", [70, 130, 1], [90, 130, 4], heads=6, head_dim=64, causal=True, seed=77)
        h0, h1 = bench.head_range(w.heads, world, rank)
        t = bench.shard_heads(w.tensors(), h0, h1)
        o, l = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, True)
        dq, dk, dv = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], w.cu_q, w.cu_k, w.scale, True)
        mine = [torch.from_numpy(np.ascontiguousarray(x)) for x in (o, l, dq, dk, dv)]
        gathered = []
        for x in mine:
            parts = [torch.empty_like(x) for _ in range(world)]
            dist.all_gather(parts, x)
            gathered.append(parts)
        if rank == 0:
            full_o, full_l = oracle.fwd(*(w.tensors()[n] for n in ("q", "k", "v")), w.cu_q, w.cu_k, w.scale, True)
            full_g = oracle.bwd(*(w.tensors()[n] for n in ("q", "k", "v", "dout")), w.cu_q, w.cu_k, w.scale, True)
            # out, dq, dk, dv: [tokens, heads, d] -> concatenate along heads;
            # lse: [heads, tokens] -> along its first axis.
            ok = [np.array_equal(torch.cat(gathered[0], 1).numpy(), full_o),
                  np.array_equal(torch.cat(gathered[1], 0).numpy(), full_l)]
            ok += [np.array_equal(torch.cat(g, 1).numpy(), f) for g, f in zip(gathered[2:], full_g)]
            out["ok"] = ok
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_split_reassembles_bitwise_gloo():
    """Two gloo ranks split the heads of one problem (bench.py --split heads):
    the per-rank results, gathered, equal the whole problem's bit for bit (no
    exchange is needed because every (sequence, head) unit is independent)."""
    import oracle

    oracle.build()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_head_split_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert out["ok"] == [True] * 5


def _seq_split_worker(rank, world, port, out):
    """One rank of a sequence-split problem: its sequences, repacked, through
    the oracle; the pieces gathered over gloo and put back in place on rank 0."""
    import numpy as np
    import torch.distributed as dist

    import bench
    import oracle
    from varlen_flashattention_02_b200 import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.make_workload("seqsplit", [70, 130, 1, 45, 200], [90, 130, 4, 45, 150], heads=2, head_dim=64,
                                causal=True, seed=78)
        seqs = bench.sequence_split(w.cu_q, w.cu_k, world)[rank]
        t, cq, ck = bench.shard_sequences(w.tensors(), w.cu_q, w.cu_k, seqs)
        o, l = oracle.fwd(t["q"], t["k"], t["v"], cq, ck, w.scale, True)
        g = oracle.bwd(t["q"], t["k"], t["v"], t["dout"], cq, ck, w.scale, True)
        pieces = [None] * world
        dist.all_gather_object(pieces, (seqs, o, l) + tuple(g))
        if rank == 0:
            full_o, full_l = oracle.fwd(*(w.tensors()[n] for n in ("q", "k", "v")), w.cu_q, w.cu_k, w.scale, True)
            full_g = oracle.bwd(*(w.tensors()[n] for n in ("q", "k", "v", "dout")), w.cu_q, w.cu_k, w.scale, True)
            got = [np.full_like(x, np.nan) for x in (full_o, full_l) + tuple(full_g)]
            for seq_list, po, pl, pdq, pdk, pdv in pieces:
                rq = rk = 0
                for b in seq_list:
                    nq = int(w.cu_q[b + 1] - w.cu_q[b])
                    nk = int(w.cu_k[b + 1] - w.cu_k[b])
                    sq = slice(int(w.cu_q[b]), int(w.cu_q[b + 1]))
                    sk = slice(int(w.cu_k[b]), int(w.cu_k[b + 1]))
                    got[0][sq], got[1][:, sq], got[2][sq] = po[rq:rq + nq], pl[:, rq:rq + nq], pdq[rq:rq + nq]
                    got[3][sk], got[4][sk] = pdk[rk:rk + nk], pdv[rk:rk + nk]
                    rq, rk = rq + nq, rk + nk
            want = (full_o, full_l) + tuple(full_g)
            out["ok"] = [np.array_equal(a, b) for a, b in zip(got, want)]
            out["parts"] = [list(p[0]) for p in pieces]
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sequence_split_reassembles_bitwise_gloo():
    """Two gloo ranks split the sequences of one problem (bench.py --split
    sequences), balanced by lq*lk: each rank's repacked problem, gathered and
    put back at the original offsets, equals the whole problem bit for bit."""
    import oracle

    oracle.build()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_seq_split_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert out["ok"] == [True] * 5
    assert sorted(sum(out["parts"], [])) == [0, 1, 2, 3, 4]  # every sequence exactly once


def test_sequence_split_balance():
    import numpy as np

    import bench

    cu = np.array([0, 5664, 12359, 13044, 16384], dtype=np.int32)  # the fwd+bwd workload's lengths
    assert bench.sequence_split(cu, cu, 2) == [[1], [0, 2, 3]]  # 44.8M vs 43.7M of lq*lk
    assert bench.sequence_split(cu, cu, 1) == [[0, 1, 2, 3]]
    assert bench.sequence_split(cu, cu, 4) == [[1], [0], [3], [2]]
    lq = np.array([5, 4, 3, 3, 3, 2])
    cq = np.concatenate([[0], np.cumsum(lq)])
    parts = bench.sequence_split(cq, cq, 2)  # greedy by lq^2: 25 | 16 9 | 9 (to 25) ...
    loads = [sum(int(lq[b]) ** 2 for b in p) for p in parts]
    assert sorted(sum(parts, [])) == list(range(6)) and abs(loads[0] - loads[1]) <= 9
    with pytest.raises(ValueError):
        bench.sequence_split(cu, cu, 5)


def test_shard_sequences():
    import numpy as np

    import bench

    cq = np.array([0, 2, 5, 6])
    ck = np.array([0, 1, 4, 8])
    q = np.arange(6 * 2).reshape(6, 1, 2)
    k = np.arange(8 * 2).reshape(8, 1, 2) + 100
    t, nq, nk = bench.shard_sequences({"q": q, "k": k, "v": k, "dout": q}, cq, ck, [0, 2])
    assert np.array_equal(t["q"], q[[0, 1, 5]]) and np.array_equal(t["k"], k[[0, 4, 5, 6, 7]])
    assert list(nq) == [0, 2, 3] and list(nk) == [0, 1, 5]


def test_head_range():
    import bench

    assert [bench.head_range(16, 4, r) for r in range(4)] == [(0, 4), (4, 8), (8, 12), (12, 16)]
    # Uneven: the first 16 % 3 = 1 rank takes one more head; the ranges tile [0, 16).
    assert [bench.head_range(16, 3, r) for r in range(3)] == [(0, 6), (6, 11), (11, 16)]
    assert bench.head_range(5, 1, 0) == (0, 5)
    for bad in ((2, 4, 0), (16, 0, 0), (16, 2, 2)):
        with pytest.raises(ValueError):
            bench.head_range(*bad)


def test_shard_heads_grouped():
    import numpy as np

    import bench

    q = np.arange(3 * 8 * 2, dtype=np.uint16).reshape(3, 8, 2)
    k = np.arange(3 * 2 * 2, dtype=np.uint16).reshape(3, 2, 2) + 1000
    s = bench.shard_heads({"q": q, "k": k, "v": k, "dout": q}, 4, 8, kv_group=4)
    assert np.array_equal(s["q"], q[:, 4:8]) and np.array_equal(s["k"], k[:, 1:2])
    assert s["q"].flags.c_contiguous and s["k"].flags.c_contiguous
    with pytest.raises(ValueError):
        bench.shard_heads({"q": q}, 2, 6, kv_group=4)
