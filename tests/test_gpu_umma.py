"""The tcgen05 full-attention sweep (128-row query tiles) against the fp64 oracle.

Shapes with T * G > 64 run the full layer on the Blackwell tensor cores.  These cases cover
both CTA modes (two query tiles sharing the K/V stream; one query tile whose two streams split
the key range), d = 64 and 128, G = 1, 8 and 16 (128, 16 and 8 queries per tile), an odd
number of query tiles (the last CTA's second tile is padding), key counts that are not a
multiple of the 128-key tile, and scattered positions (rows of one tile ending in different
key tiles, rows whose whole range lies in the first tile).  Every row's O_full and LSE_full is
checked; the mma.sync sweep (HS2_UMMA=0) is checked on the same inputs.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_hs2_b200 import hs2
from long_context_sparse_hs2_b200.inputs import f32_to_bf16_bits, make_inputs
import oracle.hs2_oracle as O
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_hs2_b200 import build

    build.build()
    hs2.lib()


CASES = [
    # B, Hq, Hkv, d, N, T, scattered positions
    (1, 8, 1, 128, 5000, 16, False),    # one query tile per kv head: split-key streams, several splits
    (2, 16, 2, 128, 3000, 40, False),   # three query tiles: pair mode, last pair half padding
    (1, 8, 1, 64, 3000, 40, False),     # d = 64
    (1, 4, 4, 128, 1200, 300, False),   # G = 1: 128 queries per tile
    (1, 32, 2, 128, 2000, 20, False),   # G = 16: 8 queries per tile
    (1, 8, 1, 128, 4100, 64, True),     # positions scattered over the whole key range
    (2, 8, 2, 64, 700, 17, True),       # ragged: 17 queries (two tiles, second nearly empty)
]


def scattered_positions(B, T, N, seed):
    rng = np.random.default_rng(seed)
    pos = np.sort(rng.integers(0, N, size=(B, T)), axis=1).astype(np.int32)
    pos[:, 0] = 0              # one visible key
    pos[:, 1 % T] = min(5, N - 1)
    pos[:, -1] = N - 1
    return pos


def full_rows_vs_oracle(inp, O_full, LSE_full):
    B, Hq, T, d = inp.Qf.shape
    Hkv = inp.K.shape[1]
    G = Hq // Hkv
    scale = O.softmax_scale(d)
    Qf, K, V = O.bf16_to_f64(inp.Qf), O.bf16_to_f64(inp.K), O.bf16_to_f64(inp.V)
    for b in range(B):
        for h in range(Hkv):
            hs = slice(h * G, (h + 1) * G)
            for t in range(T):
                p = int(inp.pos[b, t])
                o, lse, _ = O.full_attention_row(Qf[b, hs, t], K[b, h], V[b, h], p, scale)
                parity.assert_close_o(O_full[b, hs, t], o, f"O_full {(b, h, t)}")
                parity.assert_close_lse(LSE_full[b, hs, t], lse, f"LSE_full {(b, h, t)}")


@pytest.mark.parametrize("umma", ["1", "0"], ids=["tcgen05", "mma_sync"])
@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_full_attention_128_row_tiles(case, umma, monkeypatch):
    monkeypatch.setenv("HS2_UMMA", umma)
    B, Hq, Hkv, d, N, T, scattered = case
    pos = scattered_positions(B, T, N, seed=T) if scattered else None
    inp = make_inputs(B, Hq, Hkv, d, N, T, 16, 8, seed=N % 97, needles=4, pos=pos)
    g = parity.gpu_inputs(inp)
    hs2.trace_enable(True)
    O_full, LSE_full = hs2.full_attn(g["Q_full"], g["K"], g["V"], g["pos"])
    torch.cuda.synchronize()
    kernels = hs2.trace_collect()
    hs2.trace_enable(False)
    assert ("umma_attn" in kernels) == (umma == "1"), kernels
    full_rows_vs_oracle(inp, O_full.float().cpu().numpy(), LSE_full.cpu().numpy())


STEP_CASES = [
    # B, Hq, Hkv, d, N, T, k, W, scattered positions
    (1, 16, 2, 128, 2500, 24, 100, 32, False),   # G = 8, pair mode
    (2, 16, 2, 128, 3000, 16, 64, 16, False),    # split mode, two batch rows
    (1, 4, 4, 128, 1200, 300, 50, 16, False),    # G = 1
    (1, 32, 2, 64, 2000, 20, 64, 8, False),      # G = 16, d = 64
    (1, 8, 1, 128, 4100, 64, 300, 64, True),     # scattered: unranked rows (pos < W, k >= pool)
]


@pytest.mark.parametrize("case", STEP_CASES, ids=[str(c) for c in STEP_CASES])
def test_step_on_tcgen05_sweeps_matches_oracle(case):
    # the whole step on the tcgen05 full and score sweeps, then top-k and the sparse layer
    from tests.test_gpu_parity import compare_step, run_step

    B, Hq, Hkv, d, N, T, k, W, scattered = case
    pos = scattered_positions(B, T, N, seed=T + 1) if scattered else None
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=T + N % 31, needles=6, pos=pos)
    hs2.trace_enable(True)
    res = run_step(inp)
    kernels = hs2.trace_collect()
    hs2.trace_enable(False)
    assert "umma_attn" in kernels and "umma_score" in kernels, kernels
    compare_step(inp, res)


def test_many_rows_one_cta_per_row_topk():
    # >= 592 selection rows: the top-k runs one CTA per row (histogram, threshold, emit, radix)
    from tests.test_gpu_parity import compare_step, run_step

    inp = make_inputs(1, 32, 4, 128, 3000, 160, 64, 16, seed=21, needles=8)
    hs2.trace_enable(True)
    res = run_step(inp)
    kernels = hs2.trace_collect()
    hs2.trace_enable(False)
    assert "topk_rows" in kernels, kernels
    compare_step(inp, res)


def test_many_rows_all_scores_equal():
    # Q = 0: every pool key ties, far more candidates than shared memory holds (key re-scan
    # path); the k lowest indices must win in every row
    from tests.test_gpu_parity import compare_step, run_step

    inp = make_inputs(1, 16, 2, 128, 6000, 320, 100, 10, seed=22)
    inp.Qf = np.zeros_like(inp.Qf)
    res = run_step(inp)
    ref = compare_step(inp, res)
    for (b, h, t), r in ref.items():
        np.testing.assert_array_equal(np.sort(res["idx"][b, h, t][:res["cnt"][b, h, t]]), r.selected)


@pytest.mark.parametrize("bracket", ["1", "0"], ids=["unstored_keys", "stored_keys"])
def test_many_rows_large_pools_sample_bracket(bracket, monkeypatch):
    # pools >= 32768 keys and >= 592 rows.  Default: the keys are never stored -- a 1/16 tile
    # sample brackets each row's threshold, a filtering sweep keeps the candidates, and the
    # exact top-k is taken among them.  HS2_PREFILL_BRACKET=0 stores every key and brackets
    # inside the one-CTA-per-row top-k.  Sampled rows against the oracle, every row's invariants.
    from tests.test_gpu_parity import compare_step, run_step
    from tests.test_gpu_workloads import check_all_rows

    monkeypatch.setenv("HS2_PREFILL_BRACKET", bracket)
    inp = make_inputs(1, 8, 1, 128, 40000, 600, 2048, 128, seed=23, needles=32)
    g = parity.gpu_inputs(inp)
    ws = hs2.alloc_workspace(hs2.dims_of(g["Q_full"], g["K"], inp.k, inp.W), "cuda")
    hs2.trace_enable(True)
    res = run_step(inp, ws)
    kernels = hs2.trace_collect()
    hs2.trace_enable(False)
    if bracket == "1":
        assert "topk_bracket" in kernels and "topk_finalize" in kernels and "topk_rows" not in kernels, kernels
        # N(0, 1) scores: the sample brackets every row, no row is rescored
        assert hs2.read_device_status(ws) == 0
    else:
        assert "topk_rows" in kernels and "topk_bracket" not in kernels, kernels
    check_all_rows(inp, res["idx"], res["cnt"])
    compare_step(inp, res, rows=[(0, 0, t) for t in (0, 1, 77, 300, 301, 598, 599)])


def test_many_rows_large_pools_all_ties_fall_back():
    # every score equal: all pool keys share one bucket, the candidate list overflows, and each
    # row is rescored on the CUDA cores with the exact two-pass method (recomputing the tied
    # bucket's keys on every radix pass); flagged HS2_DEV_CAND_OVERFLOW
    from tests.test_gpu_parity import compare_step, run_step

    inp = make_inputs(1, 8, 1, 128, 40000, 600, 500, 64, seed=24)
    inp.Qf = np.zeros_like(inp.Qf)
    g = parity.gpu_inputs(inp)
    ws = hs2.alloc_workspace(hs2.dims_of(g["Q_full"], g["K"], inp.k, inp.W), "cuda")
    res = run_step(inp, ws)
    assert hs2.read_device_status(ws) == hs2.DEV_CAND_OVERFLOW
    rows = [(0, 0, t) for t in (0, 299, 599)]
    ref = compare_step(inp, res, rows=rows)
    for (b, h, t), r in ref.items():
        np.testing.assert_array_equal(np.sort(res["idx"][b, h, t][:res["cnt"][b, h, t]]), r.selected)


@pytest.mark.parametrize("factor", [3.0, 0.25], ids=["sample_too_strict", "sample_too_loose"])
def test_many_rows_large_pools_misleading_sample(factor):
    # K scaled by `factor` in exactly the sampled 128-key tiles (every 16th): the sample's
    # estimate of each row's k-th best score is far off, so the candidate list holds fewer
    # than k keys (factor 3) or overflows (factor 1/4), and every ranked row is rescored
    # exactly.  Sampled rows against the oracle, every row's invariants.
    from tests.test_gpu_parity import compare_step, run_step
    from tests.test_gpu_workloads import check_all_rows
    from long_context_sparse_hs2_b200.inputs import bf16_bits_to_f32

    inp = make_inputs(1, 8, 1, 128, 40000, 600, 2048, 128, seed=26)
    kk = bf16_bits_to_f32(inp.K)
    tiles = (np.arange(kk.shape[2]) // 128) % 16 == 0
    kk[:, :, tiles] *= np.float32(factor)
    inp.K = f32_to_bf16_bits(kk)
    g = parity.gpu_inputs(inp)
    ws = hs2.alloc_workspace(hs2.dims_of(g["Q_full"], g["K"], inp.k, inp.W), "cuda")
    res = run_step(inp, ws)
    assert hs2.read_device_status(ws) == hs2.DEV_CAND_OVERFLOW
    check_all_rows(inp, res["idx"], res["cnt"])
    compare_step(inp, res, rows=[(0, 0, t) for t in (0, 150, 599)])


def test_multi_cta_topk_with_several_chunks_per_cta():
    # 400 selection rows of ~40 K keys: the multi-CTA top-k gives each CTA several 4096-key
    # chunks (fewer CTAs than chunks per row); sampled rows against the oracle, every row's
    # invariants
    from tests.test_gpu_parity import compare_step, run_step
    from tests.test_gpu_workloads import check_all_rows

    inp = make_inputs(1, 8, 1, 128, 40000, 400, 2048, 128, seed=25, needles=32)
    hs2.trace_enable(True)
    res = run_step(inp)
    kernels = hs2.trace_collect()
    hs2.trace_enable(False)
    assert "topk_select" in kernels and "topk_rows" not in kernels, kernels
    check_all_rows(inp, res["idx"], res["cnt"])
    compare_step(inp, res, rows=[(0, 0, t) for t in (0, 133, 200, 399)])
