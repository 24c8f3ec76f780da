"""CPU-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_varlen.h")


@pytest.fixture(scope="module")
def lib():
    from varlen_flashattention_02_b200 import fa_varlen

    return fa_varlen.lib


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fa_varlen_fwd", "fa_varlen_bwd", "fa_varlen_fwd_workspace_size",
              "fa_varlen_bwd_workspace_size", "fa_get_device_status", "fa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in the header but not exported"


def test_status_strings(lib):
    assert lib.fa_status_string(0) == b"FA_OK"
    assert lib.fa_status_string(5) == b"FA_ERR_BAD_SEQLENS"
    assert lib.fa_status_string(6) == b"FA_ERR_DEVICE_TIMEOUT"


def test_workspace_sizes(lib):
    f = lib.fa_varlen_fwd_workspace_size(2, 1024, 12, 64)
    assert f >= 256 + 4 * 3 + 8 * (1024 // 128 + 3)
    b = lib.fa_varlen_bwd_workspace_size(2, 1024, 1024, 12, 64)
    assert b >= 12 * 1024 * 64 * 4  # holds the fp32 dQ accumulator
    assert lib.fa_varlen_fwd_workspace_size(0, 10, 1, 64) == 0


FAKE = 0x10000  # never dereferenced: validation fails first


def _fwd(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cu_q=FAKE, cu_k=FAKE, batch=2, total_q=1024, total_k=1024, max_q=824,
             max_k=724, H=12, D=64, scale=0.125, causal=0, out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=1 << 30,
             stream=None)
    a.update(over)
    return lib.fa_varlen_fwd(a["q"], a["k"], a["v"], a["cu_q"], a["cu_k"], a["batch"], a["total_q"],
                             a["total_k"], a["max_q"], a["max_k"], a["H"], a["D"], a["scale"], a["causal"],
                             a["out"], a["lse"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(D=96), 2), (dict(D=192), 2), (dict(D=512), 2), (dict(D=256, ws_bytes=64), 3), (dict(batch=0), 1), (dict(H=0), 1), (dict(total_q=-1), 1),
    (dict(scale=0.0), 1), (dict(scale=float("inf")), 1), (dict(scale=-1.0), 1), (dict(q=None), 1),
    (dict(cu_q=None), 1), (dict(q=FAKE + 8), 1), (dict(out=FAKE + 2), 1), (dict(ws=None), 3),
    (dict(ws=FAKE + 16), 3), (dict(ws_bytes=64), 3),
], ids=lambda x: str(x))
def test_fwd_rejects(lib, over, code):
    assert _fwd(lib, **over) == code


def _bwd(lib, **over):
    a = dict(do=FAKE, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cu_q=FAKE, cu_k=FAKE, batch=2, total_q=1024,
             total_k=1024, max_q=824, max_k=724, H=12, D=64, scale=0.125, causal=1, dq=FAKE, dk=FAKE, dv=FAKE,
             ws=FAKE, ws_bytes=1 << 34, stream=None)
    a.update(over)
    return lib.fa_varlen_bwd(a["do"], a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu_q"], a["cu_k"], a["batch"],
                             a["total_q"], a["total_k"], a["max_q"], a["max_k"], a["H"], a["D"], a["scale"],
                             a["causal"], a["dq"], a["dk"], a["dv"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(D=32), 2), (dict(D=192), 2), (dict(D=256, ws_bytes=1024), 3), (dict(batch=-3), 1), (dict(scale=float("nan")), 1), (dict(do=None), 1), (dict(dk=None), 1),
    (dict(dv=FAKE + 4), 1), (dict(ws_bytes=1024), 3),
], ids=lambda x: str(x))
def test_bwd_rejects(lib, over, code):
    assert _bwd(lib, **over) == code


def test_no_cpu_fallback_in_binding():
    """The binding only marshals arguments: it must not import the oracle or
    compute attention itself."""
    src = open(os.path.join(ROOT, "varlen_flashattention_02_b200", "fa_varlen.py")).read()
    assert "oracle" not in src
    for forbidden in ("softmax(", "matmul", "einsum", "@ "):
        assert forbidden not in src


def _fwd_gqa(lib, Hk, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, cu_q=FAKE, cu_k=FAKE, batch=2, total_q=1024, total_k=1024, max_q=824,
             max_k=724, H=12, D=64, scale=0.125, causal=0, out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=64,
             stream=None)
    a.update(over)
    return lib.fa_varlen_fwd_gqa(a["q"], a["k"], a["v"], a["cu_q"], a["cu_k"], a["batch"], a["total_q"],
                                 a["total_k"], a["max_q"], a["max_k"], a["H"], Hk, a["D"], a["scale"], a["causal"],
                                 a["out"], a["lse"], a["ws"], a["ws_bytes"], a["stream"])


def _bwd_gqa(lib, Hk, **over):
    a = dict(do=FAKE, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cu_q=FAKE, cu_k=FAKE, batch=2, total_q=1024,
             total_k=1024, max_q=824, max_k=724, H=12, D=64, scale=0.125, causal=1, dq=FAKE, dk=FAKE, dv=FAKE,
             ws=FAKE, ws_bytes=1024, stream=None)
    a.update(over)
    return lib.fa_varlen_bwd_gqa(a["do"], a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu_q"], a["cu_k"],
                                 a["batch"], a["total_q"], a["total_k"], a["max_q"], a["max_k"], a["H"], Hk, a["D"],
                                 a["scale"], a["causal"], a["dq"], a["dk"], a["dv"], a["ws"], a["ws_bytes"],
                                 a["stream"])


@pytest.mark.parametrize("Hk,code", [(0, 1), (-1, 1), (5, 1), (24, 1), (13, 1), (1, 3), (4, 3), (12, 3)])
def test_gqa_head_counts(lib, Hk, code):
    """num_heads must be a positive multiple of num_heads_k (invalid argument,
    1); valid counts get as far as the too-small workspace (3)."""
    assert _fwd_gqa(lib, Hk) == code
    assert _bwd_gqa(lib, Hk) == code


def test_paged_rejects_page_size_not_multiple_of_tile(lib):
    """Pages must hold whole 128-key tiles (FA_ERR_UNSUPPORTED), checked before
    anything touches the GPU."""
    rc = lib.fa_varlen_fwd_paged(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 64, 8, 64, 4, 32, 256, 4, 4, 128,
                                 0.1, 1, FAKE, FAKE, FAKE, 1 << 20, None)
    assert rc == 2
    rc = lib.fa_varlen_fwd_paged(FAKE, FAKE, FAKE, FAKE, None, FAKE, 2, 64, 8, 128, 4, 32, 256, 4, 4, 128,
                                 0.1, 1, FAKE, FAKE, FAKE, 1 << 20, None)
    assert rc == 1


def test_splitkv_rejects(lib):
    """Split-KV forward: a null layout or a split count below 1 is an invalid
    argument; more than 128 query heads per key/value head is unsupported."""
    from varlen_flashattention_02_b200 import fa_varlen

    lay = fa_varlen.KvLayout()
    lay.cu_seqlens_k = FAKE
    lay.total_rows = 64
    args = lambda lay_ptr, splits, H, Hk: lib.fa_varlen_fwd_splitkv(
        FAKE, FAKE, FAKE, FAKE, lay_ptr, 2, 64, 32, 32, H, Hk, 128, 0.1, 1, splits, FAKE, FAKE, FAKE, 1 << 20, None)
    assert args(None, 2, 8, 1) == 1
    assert args(ctypes.byref(lay), 0, 8, 1) == 1
    assert args(ctypes.byref(lay), 2, 256, 1) == 2
    # head_dim 256 is refused by the split-KV forward (the other forwards and
    # the backwards accept it).
    assert lib.fa_varlen_fwd_splitkv(FAKE, FAKE, FAKE, FAKE, ctypes.byref(lay), 2, 64, 32, 32, 8, 1, 256, 0.1, 1, 2,
                                     FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert lib.fa_varlen_fwd_splitkv_workspace_size(2, 64, 8, 3, 128, 2) == 0
    assert lib.fa_varlen_fwd_splitkv_workspace_size(2, 64, 8, 2, 128, 4) > 4 * 64 * 8 * 128 * 4


def test_splitkv_num_splits(lib):
    """The advisory split count: smallest count whose equal-sized units keep
    at least 95% of the (SM x wave) slots busy, at least two 128-key tiles per
    range; if that leaves fewer than 8 key tiles per range, the smallest
    smaller count whose units occupy 85% of the SMs at once; 1 for invalid
    arguments. Values worked by hand for 148 SMs."""
    f = lib.fa_varlen_splitkv_num_splits
    # 64 sequences x 8 kv heads = 512 units: 1 split fills 512/592 = 86%,
    # 2 splits fill 1024/1036 = 98.8%.
    assert f(64, 1, 32, 8, 8192, 148) == 2
    # 4 x 8 = 32 units per split: 9 splits give 288 units in two waves
    # (288/296 = 97.3%); 1..8 stay below 95%.
    assert f(4, 1, 32, 8, 32768, 148) == 9
    # A large batch already fills the SMs without splitting.
    assert f(148 * 4, 1, 8, 8, 4096, 148) == 1
    # Two key tiles per range at most: 300 keys = 3 tiles -> 1 split only.
    assert f(1, 1, 8, 8, 300, 148) == 1
    # Query tiles count: 64 tokens x group 4 = 2 tiles per sequence.
    assert f(74, 64, 32, 8, 8192, 148) == f(148, 1, 32, 8, 8192, 148)
    # A group that does not divide 128: g = 3 packs floor(128/3) = 42 tokens
    # per tile, so 128 tokens need 4 tiles (not ceil(3*128/128) = 3). With 2
    # sequences x 8 kv heads that is 64 units per split; 9 splits fill
    # 576/592 = 97.3% (3 tiles per sequence would have given 3 splits:
    # 144/148); ceil(64/9) = 8 key tiles per range, not fewer than 8, so 9
    # stays. g = 6 packs 21 tokens: 64 tokens need 4 tiles, 3
    # sequences x 8 x 4 = 96 units, 3 splits fill 288/296 = 97.3%.
    assert f(2, 128, 24, 8, 8192, 148) == 9
    assert f(3, 64, 48, 8, 8192, 148) == 3
    assert f(74, 42, 24, 8, 8192, 148) == f(74, 1, 24, 8, 8192, 148)  # 42 tokens: still one tile
    # Short ranges: 16 sequences x 8 kv heads = 128 units per split, 4096
    # keys = 32 tiles. 8 splits fill 1024/1036 = 98.8% but leave 4 tiles per
    # range; 1 split already occupies 128/148 = 86% of the SMs.
    assert f(16, 1, 32, 8, 4096, 148) == 1
    # 8 x 8 = 64 units, 16384 keys = 128 tiles: 9 splits give 15 tiles per
    # range, long enough, so the fill rule's choice stays.
    assert f(8, 1, 32, 8, 16384, 148) == 9
    # Invalid arguments.
    assert f(0, 1, 32, 8, 8192, 148) == 1
    assert f(4, 1, 32, 7, 8192, 148) == 1
    assert f(4, 1, 32, 8, 0, 148) == 1
    # Exhaustive restatement over a grid of shapes.
    for batch in (1, 3, 16):
        for hk in (1, 2, 8):
            for lk in (128, 1000, 20000):
                for sms in (7, 148):
                    per = batch * hk
                    tiles = -(-lk // 128)
                    cap = min(1024, max(1, tiles // 2))
                    want, best = None, (0.0, 1)
                    for s in range(1, cap + 1):
                        u = per * s
                        fill = u / (-(-u // sms) * sms)
                        if fill >= 0.95:
                            want = s
                            break
                        if fill > best[0]:
                            best = (fill, s)
                    got = want if want is not None else best[1]
                    if -(-tiles // got) < 8:
                        got = next((s for s in range(1, got) if per * s * 100 >= 85 * sms), got)
                    assert f(batch, 1, hk, hk, lk, sms) == got

