"""The forward entry point that allocates nothing (fa_varlen_fwd_noalloc),
for callers that cannot call cudaMalloc (code inside another framework's
plugin interface that is handed only input and output pointers, or paths
where an allocation could synchronise the device). It is called here through
the C ABI (ctypes, raw device pointers) on two different problems in a row
(the second call reuses the library's buffer as the first left it) and must
give exactly the results of fa_varlen_fwd with a caller-provided workspace:
both run the same kernel on the same inputs, and each output row is written
by one CTA in a fixed order, so any difference, even in the last bit, would
point at stale scratch. The outputs are also checked against the fp64
oracle within the parity tolerances. This file is collected last on
purpose."""
import ctypes

import numpy as np
import pytest

import oracle
from tests import parity_util as pu
from varlen_flashattention_02_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc_call(lib, q, k, v, cq, ck, w, out, lse, stream):
    P = ctypes.c_void_p
    return lib.fa_varlen_fwd_noalloc(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(cq.data_ptr()),
                                     P(ck.data_ptr()), w.batch, w.total_q, w.total_k, w.max_seqlen_q,
                                     w.max_seqlen_k, w.heads, w.head_dim, ctypes.c_float(w.scale), int(w.causal),
                                     P(out.data_ptr()), P(lse.data_ptr()), P(stream.cuda_stream))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_noalloc_matches_workspace_entry_point(causal):
    import torch

    from varlen_flashattention_02_b200 import fa_varlen

    lib = fa_varlen.lib
    # Two different problems in a row, so the second call must not depend on
    # what the first one left in the shared buffer.
    cases = [synth.make_workload("a", [300, 129, 1, 700], [260, 129, 5, 700], heads=3, head_dim=128,
                                 causal=causal, seed=41),
             synth.make_workload("b", [64, 1000], [900, 1000], heads=2, head_dim=64, causal=causal, seed=42)]
    stream = torch.cuda.current_stream()
    for w in cases:
        (q, k, v), ref_out, ref_lse = pu.run_fwd(w)
        cq, ck = pu.cu_dev(w.cu_q), pu.cu_dev(w.cu_k)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((w.heads, w.total_q), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_call(lib, q, k, v, cq, ck, w, out, lse, stream) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), "out differs from the workspace forward"
        assert torch.equal(lse, ref_lse), "lse differs from the workspace forward"
        t = w.tensors()
        o_or, l_or = oracle.fwd(t["q"], t["k"], t["v"], w.cu_q, w.cu_k, w.scale, w.causal)
        rows = np.repeat(np.arange(w.total_q), w.heads)
        heads = np.tile(np.arange(w.heads), w.total_q)
        pu.check_fwd(w, out, lse, o_or, l_or, rows, heads)


def test_noalloc_rejects_sizes_beyond_its_buffer():
    from varlen_flashattention_02_b200 import fa_varlen

    lib = fa_varlen.lib
    fake = ctypes.c_void_p(0x10000)
    # 2^23 tokens in one sequence need 256 + 8 * (2^16 + 2) bytes of list: more than 256 KiB.
    rc = lib.fa_varlen_fwd_noalloc(fake, fake, fake, fake, fake, 1, 1 << 23, 1 << 23, 1 << 23, 1 << 23, 1, 64,
                                   ctypes.c_float(0.125), 0, fake, fake, None)
    assert rc == 3  # FA_ERR_WORKSPACE
