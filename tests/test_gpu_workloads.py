"""hs2_step at the five benchmark workloads' full sizes, checked against the oracle.

The GPU runs the whole step exactly as bench.py launches it; the fp64 oracle then
recomputes (b, kv head, t) rows one by one: O_full and LSE_full of the row's G query
heads, the selection (near-tie rule), and the sparse outputs on the GPU's validated
index set.  Every row is recomputed for the decode workloads; 64 rows spread over kv
heads and query tiles for the 4096-query prefill.  Every row's index list is also
checked for the invariants that hold at any size (count formula, window present, no
duplicates, range, -1 padding).  The same runs with the cache stored as FP8 E4M3 or in
a paged pool check hs2_step_kv at full size.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_hs2_b200 import hs2
from dataclasses import replace

from long_context_sparse_hs2_b200.inputs import WORKLOADS, bf16_cache, fp8_e4m3_cache, generate, paged_cache
from tests import parity
from tests.test_gpu_parity import compare_step

pytestmark = pytest.mark.gpu

def _spread_prefill_rows():
    """64 prefill rows over every kv head, both query tiles of a CTA pair, and the first, middle
    and last 128-row query tiles (16 queries per tile at G = 8)."""
    rows = []
    for h in range(4):
        for t in (0, 1, 15, 16, 17, 31, 2040, 2047, 2048, 2063, 2064, 2079, 4064, 4079, 4080, 4095):
            rows.append((0, h, t))
    return rows


ALL = None  # every (b, kv head, t) row
SAMPLES = {
    "tiny": ALL,
    "batched": ALL,
    "long": ALL,
    "1m_t1": ALL,
    "1m_t16": ALL,
    "prefill": _spread_prefill_rows(),
}
# the cache in other formats/layouts, at full size: fp8 E4M3 (per-head scales) and a paged pool
VARIANTS = {
    "long_fp8": ("long", "fp8_e4m3", 0),
    "1m_t1_fp8": ("1m_t1", "fp8_e4m3", 0),
    "long_paged": ("long", "bf16", 64),
    "batched_fp8_paged": ("batched", "fp8_e4m3", 16),
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


def _run(inp, w, kv=None):
    g = parity.gpu_inputs(inp)
    if kv is None:
        ws = hs2.alloc_workspace(hs2.dims_of(g["Q_full"], g["K"], w.k, w.W), "cuda")
        out = hs2.step(g["Q_full"], g["Q_sparse"], g["K"], g["V"], g["pos"], k=w.k, W=w.W, ws=ws)
    else:
        del g["K"], g["V"]
        ws = hs2.alloc_workspace_kv(hs2.dims_kv(g["Q_full"], kv, w.k, w.W), kv, "cuda")
        out = hs2.step_kv(g["Q_full"], g["Q_sparse"], kv, g["pos"], k=w.k, W=w.W, ws=ws)
    bits = hs2.read_device_status(ws)
    assert bits & ~hs2.DEV_CAND_OVERFLOW == 0, f"device status {bits:#x}"
    del g
    res = {}
    for key, t in out.as_dict().items():
        res[key] = t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()
    del out, ws
    torch.cuda.empty_cache()
    return res


@pytest.mark.parametrize("name", list(SAMPLES))
def test_workload_full_size(name):
    w = WORKLOADS[name]
    inp = generate(w)
    res = _run(inp, w)
    check_all_rows(inp, res["idx"], res["cnt"])
    compare_step(inp, res, rows=SAMPLES[name])


@pytest.mark.parametrize("name", ["long", "1m_t1"])
def test_workload_full_size_one_launch_decode(name, monkeypatch):
    # the whole decode step in one cooperative launch (opt-in), at full size: every row's
    # selection invariants and the sampled rows against the oracle
    monkeypatch.setenv("HS2_FUSED_DECODE", "1")
    w = WORKLOADS[name]
    inp = generate(w)
    hs2.trace_enable(True)
    res = _run(inp, w)
    kernels = hs2.trace_collect()
    hs2.trace_enable(False)
    assert "decode_fused" in kernels, kernels
    check_all_rows(inp, res["idx"], res["cnt"])
    compare_step(inp, res, rows=SAMPLES[name])


@pytest.mark.parametrize("name", list(VARIANTS))
def test_workload_cache_variant_full_size(name):
    base, dtype, page_size = VARIANTS[name]
    w = WORKLOADS[base]
    inp = generate(w)
    c = fp8_e4m3_cache(inp.K, inp.V) if dtype == "fp8_e4m3" else bf16_cache(inp)
    if page_size:
        c = paged_cache(c, page_size, seed=w.seed)
    inp = replace(inp, cache=c)
    kv = parity.gpu_cache(c)
    res = _run(inp, w, kv)
    del kv
    torch.cuda.empty_cache()
    check_all_rows(inp, res["idx"], res["cnt"])
    compare_step(inp, res)
