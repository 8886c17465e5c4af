"""hs2_sparse_attn_static -- the sparse layer for callers that cannot allocate device memory at
the point of the call (its scratch is a fixed device array inside the library).

Its results must match hs2_sparse_attn, the workspace entry point, on the same inputs, on two
calls in a row (the second call runs over scratch the first one left behind), and the fp64
oracle on the same index sets; shapes range from split rows to one block per row at the size
limit.  This file is
collected last so that a failure here cannot hide any other test's result; it also passes on
its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_hs2_b200 import hs2
from long_context_sparse_hs2_b200.inputs import make_inputs
from tests import parity
import oracle.hs2_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_hs2_b200 import build

    build.build()


def _selection(g, k, W):
    """The library's own full layer and selection (KV Reuse: the sparse layer reuses them)."""
    _, lse = hs2.full_attn(g["Q_full"], g["K"], g["V"], g["pos"], k=k, W=W)
    return hs2.select(g["Q_full"], g["K"], lse, g["pos"], k=k, W=W)


def _check_against_oracle(inp, idx, cnt, O_s, L_s, rows, what):
    """O_sparse / LSE_sparse of the given rows against the fp64 oracle on the same index sets."""
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    sets = {(b, h, t): np.sort(idx[b, h, t][:cnt[b, h, t]]) for b, h, t in rows}
    for (b, h, t), r in O.step_rows(inp, rows, selected_override=sets).items():
        parity.assert_close_o(O_s[b, r.heads, t], r.o_sparse, f"{what} O_sparse {(b, h, t)}")
        parity.assert_close_lse(L_s[b, r.heads, t], r.lse_sparse, f"{what} LSE_sparse {(b, h, t)}")


def _static_twice_matches(inp, g, idx, cnt, k, W, rows):
    O_ref, L_ref = hs2.sparse_attn(g["Q_sparse"], g["K"], g["V"], g["pos"], idx, cnt, k=k, W=W)
    torch.cuda.synchronize()
    O_ref = O_ref.float().cpu().numpy()
    L_ref = L_ref.cpu().numpy()
    for call in range(2):  # the second call starts from the scratch the first one left
        O_s, L_s = hs2.sparse_attn_static(g["Q_sparse"], g["K"], g["V"], g["pos"], idx, cnt, k=k, W=W)
        torch.cuda.synchronize()
        O_s, L_s = O_s.float().cpu().numpy(), L_s.cpu().numpy()
        parity.assert_close_o(O_s, O_ref, f"O_sparse (static scratch, call {call})")
        parity.assert_close_lse(L_s, L_ref, f"LSE_sparse (static scratch, call {call})")
        _check_against_oracle(inp, idx, cnt, O_s, L_s, rows, f"static call {call}")


@pytest.mark.parametrize("shape", [(2, 16, 2, 128, 3000, 1, 256, 64), (1, 8, 1, 64, 1500, 3, 100, 16)],
                         ids=["decode_d128", "three_queries_d64"])
def test_static_scratch_matches_workspace_entry_point(shape):
    B, Hq, Hkv, d, N, T, k, W = shape
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=77, needles=4)
    g = parity.gpu_inputs(inp)
    idx, cnt = _selection(g, k, W)
    rows = [(b, h, t) for b in range(B) for h in range(Hkv) for t in range(T)]
    _static_twice_matches(inp, g, idx, cnt, k, W, rows)


# Many selection rows (one CTA per row, no split partials) at the size limit: the scratch this
# shape needs -- 256 B status + 7597 rows x (32 B counters + 8 B (m, l) + 512 B O), each region
# rounded up to 256 B -- is 4 194 048 bytes, 256 short of the 4 MiB array; one more query row
# (7598) needs 4 194 560 and must be refused.
AT_LIMIT = (1, 1, 1, 128, 8000, 7597, 64, 16)


def test_static_scratch_at_its_size_limit_with_many_rows():
    B, Hq, Hkv, d, N, T, k, W = AT_LIMIT
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=78, needles=4)
    g = parity.gpu_inputs(inp)
    idx, cnt = _selection(g, k, W)
    _static_twice_matches(inp, g, idx, cnt, k, W, [(0, 0, t) for t in (0, 1, 2500, 5001, 7595, 7596)])


def test_static_scratch_rejects_shapes_beyond_its_size():
    L = hs2.lib()
    fake = 1 << 20
    B, Hq, Hkv, d, N, T, k, W = AT_LIMIT
    # one query row past the limit, and a chunked-prefill shape far beyond it: refused before
    # any launch (the pointers are never dereferenced)
    for dims in (hs2.make_dims(B, Hq, Hkv, T + 1, N, d, k, W), hs2.make_dims(1, 32, 4, 4096, 131072, 128, 2048, 128)):
        st = L.hs2_sparse_attn_static(ctypes.byref(dims), fake, fake, fake, fake, fake, fake, fake, fake, None)
        assert st == hs2.HS2_ERR_WORKSPACE
