"""hs2_sparse_attn_static -- the sparse layer for callers that cannot allocate device memory at
the point of the call (its scratch is a fixed device array inside the library).

Its results must match hs2_sparse_attn, the workspace entry point, on the same inputs, on two
calls in a row (the second call runs over scratch the first one left behind).  This file is
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

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_hs2_b200 import build

    build.build()


@pytest.mark.parametrize("shape", [(2, 16, 2, 128, 3000, 1, 256, 64), (1, 8, 1, 64, 1500, 3, 100, 16)],
                         ids=["decode_d128", "three_queries_d64"])
def test_static_scratch_matches_workspace_entry_point(shape):
    B, Hq, Hkv, d, N, T, k, W = shape
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=77, needles=4)
    g = parity.gpu_inputs(inp)
    # the selection comes from the library's own full layer (KV Reuse: the sparse layer reuses it)
    _, lse = hs2.full_attn(g["Q_full"], g["K"], g["V"], g["pos"], k=k, W=W)
    idx, cnt = hs2.select(g["Q_full"], g["K"], lse, g["pos"], k=k, W=W)
    O_ref, L_ref = hs2.sparse_attn(g["Q_sparse"], g["K"], g["V"], g["pos"], idx, cnt, k=k, W=W)
    torch.cuda.synchronize()
    O_ref = O_ref.float().cpu().numpy()
    L_ref = L_ref.cpu().numpy()
    for call in range(2):  # the second call starts from the scratch the first one left
        O_s, L_s = hs2.sparse_attn_static(g["Q_sparse"], g["K"], g["V"], g["pos"], idx, cnt, k=k, W=W)
        torch.cuda.synchronize()
        parity.assert_close_o(O_s.float().cpu().numpy(), O_ref, f"O_sparse (static scratch, call {call})")
        parity.assert_close_lse(L_s.cpu().numpy(), L_ref, f"LSE_sparse (static scratch, call {call})")


def test_static_scratch_rejects_shapes_beyond_its_size():
    # a chunked-prefill shape needs far more than the fixed scratch: refused before any launch
    dims = hs2.make_dims(1, 32, 4, 4096, 131072, 128, 2048, 128)
    L = hs2.lib()
    fake = 1 << 20
    st = L.hs2_sparse_attn_static(ctypes.byref(dims), fake, fake, fake, fake, fake, fake, fake, fake, None)
    assert st == hs2.HS2_ERR_WORKSPACE
