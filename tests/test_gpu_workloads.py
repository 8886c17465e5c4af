"""hs2_step at the five benchmark workloads' full sizes, checked on sampled rows.

The GPU runs the whole step exactly as bench.py launches it; the fp64 oracle then
recomputes the sampled (b, kv head, t) rows one by one: O_full and LSE_full of the
row's G query heads, the selection (near-tie rule), and the sparse outputs on the
GPU's validated index set.  Every row's index list is also checked for the
invariants that hold at any size (count formula, window present, no duplicates,
range, -1 padding).
"""
import numpy as np
import pytest
import torch

from long_context_sparse_hs2_b200 import hs2
from long_context_sparse_hs2_b200.inputs import WORKLOADS, generate
from tests import parity
from tests.test_gpu_parity import compare_step

pytestmark = pytest.mark.gpu

SAMPLES = {
    "tiny": [(0, 0, 0)],
    "batched": [(0, 0, 0), (3, 2, 0), (7, 3, 0)],
    "long": [(0, 0, 0), (0, 5, 0), (0, 7, 0)],
    "1m_t1": [(0, 0, 0), (0, 3, 0)],
    "1m_t16": [(0, 1, 0), (0, 2, 9), (0, 3, 15)],
    "prefill": [(0, 0, 0), (0, 1, 1000), (0, 2, 2047), (0, 3, 4095)],
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_hs2_b200 import build

    build.build()


def check_all_rows(inp, idx, cnt):
    """Invariants every selection row satisfies, checked for all rows."""
    B, Hkv, T, kw = idx.shape
    pos = inp.pos[:, None, :].repeat(Hkv, axis=1)             # [B, Hkv, T]
    pool = np.maximum(0, pos - inp.W + 1)
    want = np.minimum(inp.k, pool) + np.minimum(inp.W, pos + 1)
    np.testing.assert_array_equal(cnt, want)
    slot = np.arange(kw)[None, None, None, :]
    valid = slot < cnt[..., None]
    assert np.all(idx[~valid] == -1)
    assert np.all(idx[valid] >= 0)
    assert np.all(np.where(valid, idx, 0) <= pos[..., None])
    srt = np.sort(np.where(valid, idx, -1), axis=-1)
    dup = (srt[..., 1:] == srt[..., :-1]) & (srt[..., 1:] >= 0)
    assert not dup.any(), "duplicate indices"
    # the window is written in the first min(W, pos+1) slots
    wc = np.minimum(inp.W, pos + 1)
    first = idx[..., 0]
    np.testing.assert_array_equal(np.where(wc > 0, first, 0), np.where(wc > 0, pos - wc + 1, 0))


@pytest.mark.parametrize("fused", [False, True], ids=["chain", "fused"])
@pytest.mark.parametrize("name", list(SAMPLES))
def test_workload_full_size(name, fused, monkeypatch):
    w = WORKLOADS[name]
    if fused:
        if w.T != 1:
            pytest.skip("the single-kernel step is for T = 1")
        monkeypatch.setenv("HS2_FUSED_DECODE", "1")
    inp = generate(w)
    g = parity.gpu_inputs(inp)
    ws = hs2.alloc_workspace(hs2.dims_of(g["Q_full"], g["K"], w.k, w.W), "cuda")
    out = hs2.step(g["Q_full"], g["Q_sparse"], g["K"], g["V"], g["pos"], k=w.k, W=w.W, ws=ws)
    bits = hs2.read_device_status(ws)
    assert bits & ~hs2.DEV_CAND_OVERFLOW == 0, f"device status {bits:#x}"
    del g
    res = {}
    for key, t in out.as_dict().items():
        res[key] = t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()
    del out, ws
    torch.cuda.empty_cache()
    check_all_rows(inp, res["idx"], res["cnt"])
    compare_step(inp, res, rows=SAMPLES[name])
