"""CUDA path vs the fp64 oracle on small seeded inputs (several tiles, ragged tails, edge cases).

Every call goes through the C ABI (via the ctypes binding).  Tolerances: see tests/parity.py.
"""
import numpy as np
import pytest
import torch

from long_context_sparse_hs2_b200 import hs2
from long_context_sparse_hs2_b200.inputs import f32_to_bf16_bits, make_inputs
import oracle.hs2_oracle as O
from tests import parity
from tests.oracle_pins import hand8_expected, hand8_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_hs2_b200 import build

    build.build()
    hs2.lib()


def run_step(inp, ws=None):
    g = parity.gpu_inputs(inp)
    out = hs2.step(g["Q_full"], g["Q_sparse"], g["K"], g["V"], g["pos"], k=inp.k, W=inp.W, ws=ws)
    torch.cuda.synchronize()
    return {k: v.float().cpu().numpy() if v.dtype == torch.bfloat16 else v.cpu().numpy()
            for k, v in out.as_dict().items()}


def compare_step(inp, res, rows=None):
    """Check every (or the given) row of a GPU step result against the oracle."""
    B, Hq, T, d = inp.Qf.shape
    Hkv = inp.K.shape[1]
    G = Hq // Hkv
    if rows is None:
        rows = [(b, h, t) for b in range(B) for h in range(Hkv) for t in range(T)]
    ref = O.step_rows(inp, rows)
    sets = {}
    for (b, h, t), r in ref.items():
        hs = r.heads
        parity.assert_close_o(res["O_full"][b, hs, t], r.o_full, f"O_full {(b, h, t)}")
        parity.assert_close_lse(res["LSE_full"][b, hs, t], r.lse_full, f"LSE_full {(b, h, t)}")
        sets[(b, h, t)] = parity.check_selection(res["idx"][b, h, t], res["cnt"][b, h, t], r)
    ref_sp = O.step_rows(inp, rows, selected_override=sets)
    for (b, h, t), r in ref_sp.items():
        hs = r.heads
        parity.assert_close_o(res["O_sparse"][b, hs, t], r.o_sparse, f"O_sparse {(b, h, t)}")
        parity.assert_close_lse(res["LSE_sparse"][b, hs, t], r.lse_sparse, f"LSE_sparse {(b, h, t)}")
    return ref


def test_hand8_exact():
    inp = hand8_inputs()
    res = run_step(inp)
    want = hand8_expected()
    for t in (0, 1):
        np.testing.assert_array_equal(np.sort(res["idx"][0, 0, t][:res["cnt"][0, 0, t]]), want[t]["selected"])
        assert np.all(res["idx"][0, 0, t][res["cnt"][0, 0, t]:] == -1)
        parity.assert_close_lse(res["LSE_full"][0, :, t], want[t]["lse_full"], "hand8 LSE_full")
        parity.assert_close_o(res["O_full"][0, :, t, :8], want[t]["o_full"], "hand8 O_full")
        parity.assert_close_lse(res["LSE_sparse"][0, :, t], want[t]["lse_sparse"], "hand8 LSE_sparse")
        parity.assert_close_o(res["O_sparse"][0, :, t, :8], want[t]["o_sparse"], "hand8 O_sparse")


CASES = [
    # B, Hq, Hkv, d, N, T, k, W
    (1, 4, 1, 64, 2048, 1, 64, 64),       # tiny decode shape
    (2, 8, 1, 128, 1000, 1, 37, 16),      # ragged N, G = 8
    (1, 16, 16, 128, 777, 3, 50, 5),      # G = 1, T = 3
    (1, 4, 2, 64, 640, 4, 20, 0),         # W = 0
    (1, 32, 2, 128, 3000, 2, 300, 100),   # G = 16, T = 2
    (2, 8, 4, 128, 1500, 5, 100, 64),     # G = 2
    (1, 8, 1, 128, 5000, 16, 256, 128),   # T*G = 128: one full row block, score re-sweep
    (1, 8, 1, 64, 3000, 40, 64, 32),      # several row blocks with a ragged last block
    (1, 4, 1, 128, 300, 1, 0, 16),        # k = 0: window only
    (1, 4, 1, 128, 300, 2, 10000, 16),    # k >= pool: collapses to full attention
    (1, 4, 1, 128, 300, 1, 10000, 16),    # k >= pool at T = 1: the whole pool in index order
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_step_matches_oracle(case):
    B, Hq, Hkv, d, N, T, k, W = case
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=hash(case) % 1000, needles=4)
    res = run_step(inp)
    compare_step(inp, res)


DYN_CASES = [c for c in CASES if c[5] * (c[1] // c[2]) <= 64][:5]


@pytest.mark.parametrize("case", DYN_CASES, ids=[str(c) for c in DYN_CASES])
def test_step_with_dynamically_scheduled_sweep(case, monkeypatch):
    # the full sweep's CTAs taking their key tiles in chunks from a per-row-block counter (the
    # default only for very long caches) must give the same results
    monkeypatch.setenv("HS2_DYN_SWEEP", "1")
    monkeypatch.setenv("HS2_FUSED_DECODE", "0")
    B, Hq, Hkv, d, N, T, k, W = case
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=hash(case) % 1000 + 3, needles=4)
    compare_step(inp, run_step(inp))


def test_positions_before_the_window_and_first_token():
    # pos < W (empty pool), pos = 0 (one visible key), and arbitrary positions per batch row
    pos = np.array([[0, 3, 10, 700], [5, 64, 65, 999]], np.int32)
    inp = make_inputs(2, 8, 2, 128, 1000, 4, 16, 64, seed=5, pos=pos)
    res = run_step(inp)
    compare_step(inp, res)
    inp.k, inp.W = 3, 0
    res = run_step(inp)
    compare_step(inp, res)


def test_decode_rows_at_scattered_positions():
    # T = 1 (the one-launch decode step): per batch row the first token, an empty pool (pos < W),
    # the pool's first key, and deep positions
    pos = np.array([[0], [3], [63], [64], [999], [517]], np.int32)
    inp = make_inputs(6, 8, 2, 128, 1000, 1, 16, 64, seed=15, needles=3, pos=pos)
    compare_step(inp, run_step(inp))


def test_empty_selection_gives_zero_output():
    inp = make_inputs(1, 4, 1, 64, 200, 1, 0, 0, seed=2)
    res = run_step(inp)
    assert res["cnt"][0, 0, 0] == 0
    assert np.all(res["O_sparse"] == 0) and np.all(np.isneginf(res["LSE_sparse"]))
    compare_step(inp, res)


def test_exact_ties_take_the_lower_index():
    inp = make_inputs(1, 8, 1, 128, 2000, 1, 8, 16, seed=9)
    K = inp.K.copy()
    q = O.bf16_to_f64(inp.Qf[0, 0, 0])
    unit = q / np.linalg.norm(q)
    groups = [np.array([100, 400, 900, 1500, 1600, 1700]), np.arange(1800, 1812)]
    for grp, boost in zip(groups, (5.0, 3.5)):
        row = f32_to_bf16_bits((O.bf16_to_f64(K[0, 0, grp[0]]) + boost * unit).astype(np.float32))
        for j in grp:
            K[0, 0, j] = row   # identical key rows: bit-identical scores on both sides
    inp.K = K
    res = run_step(inp)
    r = compare_step(inp, res)[(0, 0, 0)]
    assert r.scores[100] == r.scores[1700] and r.scores[1800] == r.scores[1811]
    S = set(res["idx"][0, 0, 0][:res["cnt"][0, 0, 0]].tolist())
    for grp in groups:
        taken = np.array([j in S for j in grp])
        # within a group of exact ties, the selected members are the lowest indices
        assert not np.any(~taken[:-1] & taken[1:]), f"tie group {grp} selected as {taken}"
        np.testing.assert_array_equal(taken, np.isin(grp, r.selected))


def test_all_scores_equal():
    # Q = 0 makes every logit 0, so every pool key has the same score: the k lowest indices win
    inp = make_inputs(1, 8, 2, 128, 3000, 2, 100, 10, seed=4)
    inp.Qf = np.zeros_like(inp.Qf)
    res = run_step(inp)
    ref = compare_step(inp, res)
    for key, r in ref.items():
        b, h, t = key
        np.testing.assert_array_equal(np.sort(res["idx"][b, h, t][:res["cnt"][b, h, t]]), r.selected)


def test_component_entry_points_and_kv_reuse():
    inp = make_inputs(2, 16, 2, 128, 2500, 3, 200, 50, seed=12)
    g = parity.gpu_inputs(inp)
    O_full, LSE_full = hs2.full_attn(g["Q_full"], g["K"], g["V"], g["pos"], k=inp.k, W=inp.W)
    idx, cnt = hs2.select(g["Q_full"], g["K"], LSE_full, g["pos"], k=inp.k, W=inp.W)
    # KV Reuse: two sparse layers with different queries reuse the same cache and the same indices
    Qs2 = torch.flip(g["Q_sparse"], dims=[1]).contiguous()
    O_sp1, L1 = hs2.sparse_attn(g["Q_sparse"], g["K"], g["V"], g["pos"], idx, cnt, k=inp.k, W=inp.W)
    O_sp2, L2 = hs2.sparse_attn(Qs2, g["K"], g["V"], g["pos"], idx, cnt, k=inp.k, W=inp.W)
    torch.cuda.synchronize()
    res = dict(O_full=O_full.float().cpu().numpy(), LSE_full=LSE_full.cpu().numpy(), idx=idx.cpu().numpy(),
               cnt=cnt.cpu().numpy(), O_sparse=O_sp1.float().cpu().numpy(), LSE_sparse=L1.cpu().numpy())
    compare_step(inp, res)
    inp2 = make_inputs(2, 16, 2, 128, 2500, 3, 200, 50, seed=12)
    inp2.Qs = np.ascontiguousarray(inp.Qs[:, ::-1])
    sets = {(b, h, t): np.sort(res["idx"][b, h, t][:res["cnt"][b, h, t]])
            for b in range(2) for h in range(2) for t in range(3)}
    ref2 = O.step_rows(inp2, selected_override=sets)
    O2 = O_sp2.float().cpu().numpy()
    for (b, h, t), r in ref2.items():
        parity.assert_close_o(O2[b, r.heads, t], r.o_sparse, "second sparse layer")


def test_sparse_attn_with_caller_indices_and_bad_entries():
    inp = make_inputs(1, 8, 1, 128, 1200, 2, 40, 8, seed=21)
    g = parity.gpu_inputs(inp)
    rng = np.random.default_rng(0)
    kw = inp.k + inp.W
    idx = np.full((1, 1, 2, kw), -1, np.int32)
    cnt = np.zeros((1, 1, 2), np.int32)
    sets = {}
    for t in range(2):
        p = int(inp.pos[0, t])
        sel = np.sort(rng.choice(p + 1, size=30, replace=False))
        idx[0, 0, t, :30] = rng.permutation(sel)
        cnt[0, 0, t] = 30
        sets[(0, 0, t)] = sel
    ws = hs2.alloc_workspace(hs2.dims_of(g["Q_sparse"], g["K"], inp.k, inp.W), "cuda")
    O_sp, L_sp = hs2.sparse_attn(g["Q_sparse"], g["K"], g["V"], g["pos"], torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(cnt).cuda(), k=inp.k, W=inp.W, ws=ws)
    assert hs2.read_device_status(ws) == 0
    ref = O.step_rows(inp, selected_override=sets)
    for (b, h, t), r in ref.items():
        parity.assert_close_o(O_sp[b, r.heads, t].float().cpu().numpy(), r.o_sparse, "caller indices")
    # out-of-range entries are skipped and flagged
    idx_bad = idx.copy()
    idx_bad[0, 0, 0, 0] = 5000
    idx_bad[0, 0, 1, 1] = -7
    hs2.sparse_attn(g["Q_sparse"], g["K"], g["V"], g["pos"], torch.from_numpy(idx_bad).cuda(),
                    torch.from_numpy(cnt).cuda(), k=inp.k, W=inp.W, ws=ws)
    assert hs2.read_device_status(ws) & hs2.DEV_BAD_INDEX


def test_device_status_bits():
    inp = make_inputs(1, 4, 1, 64, 512, 1, 16, 8, seed=3)
    g = parity.gpu_inputs(inp)
    ws = hs2.alloc_workspace(hs2.dims_of(g["Q_full"], g["K"], inp.k, inp.W), "cuda")
    hs2.step(g["Q_full"], g["Q_sparse"], g["K"], g["V"], g["pos"], k=inp.k, W=inp.W, ws=ws)
    assert hs2.read_device_status(ws) == 0
    bad_pos = torch.tensor([[600]], dtype=torch.int32, device="cuda")
    hs2.step(g["Q_full"], g["Q_sparse"], g["K"], g["V"], bad_pos, k=inp.k, W=inp.W, ws=ws)
    assert hs2.read_device_status(ws) & hs2.DEV_BAD_POS
    qnan = g["Q_full"].clone()
    qnan[0, 0, 0, 0] = float("nan")
    hs2.step(qnan, g["Q_sparse"], g["K"], g["V"], g["pos"], k=inp.k, W=inp.W, ws=ws)
    assert hs2.read_device_status(ws) & hs2.DEV_NONFINITE


def test_repeated_calls_reuse_workspace():
    inp = make_inputs(1, 8, 2, 128, 4000, 1, 128, 64, seed=33)
    g = parity.gpu_inputs(inp)
    ws = hs2.alloc_workspace(hs2.dims_of(g["Q_full"], g["K"], inp.k, inp.W), "cuda")
    ws.fill_(0xAB)   # garbage workspace must not matter
    a = run_step(inp, ws=ws)
    b = run_step(inp, ws=ws)
    np.testing.assert_array_equal(a["O_full"], b["O_full"])
    np.testing.assert_array_equal(a["cnt"], b["cnt"])
    for h in range(2):
        np.testing.assert_array_equal(np.sort(a["idx"][0, h, 0]), np.sort(b["idx"][0, h, 0]))
    compare_step(inp, b)


TAIL_CASES = [c for c in CASES if c[5] * (c[1] // c[2]) <= 16]


@pytest.mark.parametrize("path", ["fused", "chain"])
@pytest.mark.parametrize("case", TAIL_CASES, ids=[str(c) for c in TAIL_CASES])
def test_decode_tail_paths_match_oracle(case, path, monkeypatch):
    # the decode tail after the sweep: the kernel chain (score_hist -> topk_select ->
    # sparse_attn), and, for T = 1, the whole step in one cooperative launch
    # (HS2_FUSED_DECODE=1; the default for short caches)
    monkeypatch.setenv("HS2_FUSED_DECODE", "1" if path == "fused" else "0")
    B, Hq, Hkv, d, N, T, k, W = case
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=hash(case) % 1000 + 7, needles=4)
    hs2.trace_enable(True)
    res = run_step(inp)
    kernels = hs2.trace_collect()
    hs2.trace_enable(False)
    if path == "fused":
        assert ("decode_fused" in kernels) == (T == 1), kernels
    else:
        assert "decode_fused" not in kernels and "topk_select" in kernels, kernels
    compare_step(inp, res)


def test_bounded_wait_runs_out_and_the_device_stays_usable():
    # a pipeline wait that nothing completes gives up after its bound, sets DEV_TIMEOUT and lets
    # the kernel return; the next call on the same device works
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    hs2.selftest_wait_bound(ws, 2_000_000)  # 2 ms
    e1.record()
    assert hs2.read_device_status(ws) == hs2.DEV_TIMEOUT
    assert 2.0 <= e0.elapsed_time(e1) < 200.0
    inp = make_inputs(1, 8, 1, 128, 1000, 1, 37, 16, seed=9, needles=2)
    compare_step(inp, run_step(inp))
