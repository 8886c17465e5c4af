"""The KV cache in other formats and layouts, and the decode loop, on the GPU against the oracle.

* FP8 E4M3 caches (per-(b, kv head) scales) and paged pools (shuffled pages, junk in unmapped
  slots) through hs2_step_kv: every row against the fp64 oracle, which reads the stored codes
  back to exact values; paged and contiguous runs of the same data must give a bit-identical
  full layer and the same selected sets.
* hs2_kv_append: the stored bytes must equal the oracle's (bf16 copies, E4M3 codes rounded from
  the fp32 quotient, saturation), in every layout.
* hs2_decode_step: runs of consecutive steps (each appends one token and advances pos on the
  device), eagerly and replayed from one captured CUDA graph; every step against the oracle's
  decode loop, the final cache bit for bit.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from long_context_sparse_hs2_b200 import hs2
from long_context_sparse_hs2_b200.inputs import (bf16_cache, f32_to_bf16_bits, fp8_e4m3_cache, make_decode_steps,
                                                  make_inputs, paged_cache)
import oracle.hs2_oracle as O
from tests import parity
from tests.test_gpu_parity import compare_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_hs2_b200 import build

    build.build()


def _res(out):
    return {k: v.float().cpu().numpy() if v.dtype == torch.bfloat16 else v.cpu().numpy()
            for k, v in out.as_dict().items()}


def run_step_kv(inp, ws=None):
    g = parity.gpu_inputs(inp)
    cache = parity.gpu_cache(inp.cache)
    dm = hs2.dims_kv(g["Q_full"], cache, inp.k, inp.W)
    ws = hs2.alloc_workspace_kv(dm, cache, "cuda") if ws is None else ws
    out = hs2.step_kv(g["Q_full"], g["Q_sparse"], cache, g["pos"], k=inp.k, W=inp.W, ws=ws)
    bits = hs2.read_device_status(ws)
    return _res(out), bits


def with_cache(inp, dtype, page_size=0, seed=0):
    c = fp8_e4m3_cache(inp.K, inp.V) if dtype == "fp8_e4m3" else bf16_cache(inp)
    if page_size:
        c = paged_cache(c, page_size, seed=seed)
    return replace(inp, cache=c)


CASES = [
    # B, Hq, Hkv, d, N, T, k, W
    (1, 4, 1, 64, 2048, 1, 64, 64),       # tiny decode shape
    (2, 8, 1, 128, 1000, 1, 37, 16),      # ragged N, G = 8
    (1, 16, 16, 128, 777, 3, 50, 5),      # G = 1, T = 3
    (1, 32, 2, 128, 3000, 2, 300, 100),   # G = 16, T = 2
    (2, 8, 4, 64, 1500, 5, 100, 64),      # G = 2, d = 64
    (1, 8, 1, 128, 5000, 16, 256, 128),   # T*G = 128: score re-sweep on 128-row tiles
    (1, 8, 1, 64, 3000, 40, 64, 32),      # several row blocks, ragged last block
    (1, 4, 1, 128, 300, 2, 10000, 16),    # k >= pool
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_fp8_cache_step_matches_oracle(case):
    B, Hq, Hkv, d, N, T, k, W = case
    inp = with_cache(make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=hash(case) % 997, needles=4), "fp8_e4m3")
    res, bits = run_step_kv(inp)
    assert bits == 0, hex(bits)
    compare_step(inp, res)


@pytest.mark.parametrize("dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("page_size", [8, 16, 64, 256])
def test_paged_cache_step_matches_oracle_and_contiguous(dtype, page_size):
    case = (2, 16, 2, 128, 1700, 3, 120, 40)
    B, Hq, Hkv, d, N, T, k, W = case
    pos = np.array([[900, 1500, 1699], [63, 700, 1699]], np.int32)
    base = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=page_size, needles=4, pos=pos)
    paged = with_cache(base, dtype, page_size, seed=page_size)
    res, bits = run_step_kv(paged)
    assert bits == 0, hex(bits)
    compare_step(paged, res)
    flat, _ = run_step_kv(with_cache(base, dtype))
    # same data, same kernels: the full layer is bit-identical and the selected sets are equal (the
    # order inside an index row, and so the sparse layer's summation order, is not fixed)
    for key in ("O_full", "LSE_full", "cnt"):
        np.testing.assert_array_equal(res[key], flat[key], err_msg=key)
    np.testing.assert_array_equal(np.sort(res["idx"], axis=-1), np.sort(flat["idx"], axis=-1))
    parity.assert_close_o(res["O_sparse"], flat["O_sparse"], "O_sparse paged vs contiguous")
    parity.assert_close_lse(res["LSE_sparse"], flat["LSE_sparse"], "LSE_sparse paged vs contiguous")


def test_unmapped_page_is_flagged_and_reads_as_zeros():
    inp = with_cache(make_inputs(1, 8, 1, 128, 512, 1, 32, 16, seed=3, needles=2), "bf16", 64, seed=3)
    inp.cache.page_table[0, 2] = 10_000  # tokens 128..191 are visible but their page does not exist
    res, bits = run_step_kv(inp)
    assert bits & hs2.DEV_BAD_PAGE
    # the oracle on a cache whose page holds zeros gives the full layer's result
    z = inp.cache.copy()
    z.K = np.concatenate([z.K, np.zeros_like(z.K[:1])])
    z.V = np.concatenate([z.V, np.zeros_like(z.V[:1])])
    z.page_table[0, 2] = z.K.shape[0] - 1
    ref = O.step_rows(replace(inp, cache=z))[(0, 0, 0)]
    parity.assert_close_o(res["O_full"][0, :, 0], ref.o_full, "O_full with a zero page")
    parity.assert_close_lse(res["LSE_full"][0, :, 0], ref.lse_full, "LSE_full with a zero page")


def _append_case(dtype, page_size, seed):
    inp = make_inputs(2, 4, 2, 128, 300, 1, 8, 8, seed=seed)
    c = fp8_e4m3_cache(inp.K, inp.V) if dtype == "fp8_e4m3" else bf16_cache(inp)
    if page_size:
        c = paged_cache(c, page_size, seed=seed)
    rng = np.random.default_rng(seed)
    T = 5
    pos = np.stack([rng.choice(300, T, replace=False) for _ in range(2)]).astype(np.int32)
    x = rng.standard_normal((2, 2, T, 128)).astype(np.float32)
    if dtype == "fp8_e4m3":  # exact ties, subnormal codes and saturation, in units of the scale
        sc = c.k_scale[:, :, None, None]
        x[..., :8] = np.array([1.0625, 1.1875, 2 ** -10, 3 * 2 ** -11, 460.0, -1e6, 447.9, 0.0]) * sc
    k_new = f32_to_bf16_bits(x)
    v_new = f32_to_bf16_bits(rng.standard_normal((2, 2, T, 128)).astype(np.float32) * 3)
    return c, k_new, v_new, pos


@pytest.mark.parametrize("dtype,page_size", [("bf16", 0), ("fp8_e4m3", 0), ("bf16", 16), ("fp8_e4m3", 64)])
def test_kv_append_bytes_match_oracle(dtype, page_size):
    c, k_new, v_new, pos = _append_case(dtype, page_size, seed=11)
    want = c.copy()
    for b in range(2):
        for t in range(pos.shape[1]):
            O.append_token(want, b, int(pos[b, t]), k_new[b, :, t], v_new[b, :, t])
    cache = parity.gpu_cache(c)
    ws = hs2.kv_append(cache, parity.to_torch_bf16(k_new, "cuda"), parity.to_torch_bf16(v_new, "cuda"),
                       torch.from_numpy(pos).cuda())
    assert hs2.read_device_status(ws) == 0
    K, V = parity.cache_to_numpy(cache)
    np.testing.assert_array_equal(K, want.K)
    np.testing.assert_array_equal(V, want.V)


def _decode_run(dtype, page_size, seed, steps=5, graph=False, B=2, N=700, k=48, W=16):
    start = make_inputs(B, 16, 2, 128, N, 1, k, W, seed=seed, needles=3,
                        pos=np.array([[N - steps - 1 - 40 * b] for b in range(B)], np.int32))
    c = fp8_e4m3_cache(start.K, start.V) if dtype == "fp8_e4m3" else bf16_cache(start)
    if page_size:
        c = paged_cache(c, page_size, seed=seed)
    st = make_decode_steps(start, steps, seed=seed + 1, drift=0.3)
    want, final = O.decode_loop(st, c)
    cache = parity.gpu_cache(c)
    pos = torch.from_numpy(start.pos[:, 0].copy()).cuda()
    dev = "cuda"
    Qf = torch.empty((B, 16, 1, 128), dtype=torch.bfloat16, device=dev)
    Qs, Kn, Vn = torch.empty_like(Qf), torch.empty((B, 2, 1, 128), dtype=torch.bfloat16, device=dev), None
    Vn = torch.empty_like(Kn)
    dm = hs2.dims_kv(Qf, cache, k, W)
    ws = hs2.alloc_workspace_kv(dm, cache, dev)
    out = hs2.alloc_step_outputs(dm, dev)

    def load(s):
        Qf.copy_(parity.to_torch_bf16(st.Qf[s], dev))
        Qs.copy_(parity.to_torch_bf16(st.Qs[s], dev))
        Kn.copy_(parity.to_torch_bf16(st.K_new[s][:, :, None], dev))
        Vn.copy_(parity.to_torch_bf16(st.V_new[s][:, :, None], dev))

    def one():
        hs2.decode_step(Qf, Qs, cache, Kn, Vn, pos, k=k, W=W, out=out, ws=ws)

    g = None
    if graph:
        # one eager call on scratch copies first (the library sets kernel attributes on first use),
        # then capture one call on the real state: capturing runs nothing
        load(0)
        scratch = hs2.KVCache(K=cache.K.clone(), V=cache.V.clone(), N=cache.N, dtype=cache.dtype,
                              k_scale=cache.k_scale, v_scale=cache.v_scale, page_size=cache.page_size,
                              page_table=cache.page_table)
        hs2.decode_step(Qf, Qs, scratch, Kn, Vn, pos.clone(), k=k, W=W, ws=ws)
        torch.cuda.synchronize()
        del scratch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one()
    for s in range(steps):
        load(s)
        if g is not None:
            g.replay()
        else:
            one()
        torch.cuda.synchronize()
        assert hs2.read_device_status(ws) == 0
        res = _res(out)
        assert np.array_equal(pos.cpu().numpy(), start.pos[:, 0] + s + 1)
        sets = {}
        for (b, h, t), r in want[s].items():
            parity.assert_close_o(res["O_full"][b, r.heads, 0], r.o_full, f"step {s} O_full {(b, h)}")
            parity.assert_close_lse(res["LSE_full"][b, r.heads, 0], r.lse_full, f"step {s} LSE_full {(b, h)}")
            sets[(b, h, 0)] = parity.check_selection(res["idx"][b, h, 0], res["cnt"][b, h, 0], r)
        inp_s = replace(start, Qf=st.Qf[s], Qs=st.Qs[s], cache=final,
                        pos=(start.pos[:, 0] + s + 1)[:, None].astype(np.int32))
        for (b, h, t), r in O.step_rows(inp_s, selected_override=sets).items():
            parity.assert_close_o(res["O_sparse"][b, r.heads, 0], r.o_sparse, f"step {s} O_sparse {(b, h)}")
            parity.assert_close_lse(res["LSE_sparse"][b, r.heads, 0], r.lse_sparse, f"step {s} LSE_sparse {(b, h)}")
    K, V = parity.cache_to_numpy(cache)
    np.testing.assert_array_equal(K, final.K)
    np.testing.assert_array_equal(V, final.V)


@pytest.mark.parametrize("dtype,page_size", [("bf16", 0), ("fp8_e4m3", 0), ("bf16", 16), ("fp8_e4m3", 32)])
def test_decode_loop_matches_oracle(dtype, page_size):
    _decode_run(dtype, page_size, seed=21 + page_size)


@pytest.mark.parametrize("dtype,page_size", [("bf16", 0), ("fp8_e4m3", 16)])
def test_decode_loop_replayed_from_one_cuda_graph(dtype, page_size):
    _decode_run(dtype, page_size, seed=31 + page_size, graph=True)


@pytest.mark.parametrize("dtype,page_size,graph", [("bf16", 0, False), ("fp8_e4m3", 16, False), ("bf16", 16, True)])
def test_decode_loop_in_one_launch_per_step(dtype, page_size, graph, monkeypatch):
    # the decode loop with each step in one cooperative launch (HS2_FUSED_DECODE=1): FP8 and paged
    # caches, eager and replayed from one CUDA graph
    monkeypatch.setenv("HS2_FUSED_DECODE", "1")
    _decode_run(dtype, page_size, seed=41 + page_size, graph=graph)


def test_decode_step_on_a_full_cache_keeps_its_position():
    # pos[b] + 1 == N: nothing is appended, pos stays, the bit is set and the step runs at N - 1
    inp = make_inputs(1, 8, 1, 128, 256, 1, 16, 8, seed=4, pos=np.array([[255]], np.int32))
    cache = parity.gpu_cache(bf16_cache(inp))
    g = parity.gpu_inputs(inp)
    pos = torch.tensor([255], dtype=torch.int32, device="cuda")
    kn = torch.ones((1, 1, 1, 128), dtype=torch.bfloat16, device="cuda")
    dm = hs2.dims_kv(g["Q_full"], cache, 16, 8)
    ws = hs2.alloc_workspace_kv(dm, cache, "cuda")
    out = hs2.decode_step(g["Q_full"], g["Q_sparse"], cache, kn, kn, pos, k=16, W=8, ws=ws)
    assert hs2.read_device_status(ws) & hs2.DEV_BAD_POS
    assert int(pos.item()) == 255
    K, _ = parity.cache_to_numpy(cache)
    np.testing.assert_array_equal(K, inp.K)
    compare_step(inp, _res(out))


GARBAGE_CASES = [
    # B, Hq, Hkv, d, N, T, k, W, last position: slots past it hold NaN bit patterns
    (1, 4, 1, 64, 2048, 1, 64, 64, 1000),       # decode, kept logits
    (2, 16, 2, 128, 3000, 3, 100, 16, 2100),    # 16-row tiles, score re-sweep
    (1, 8, 1, 128, 5000, 16, 256, 128, 3001),   # 128-row tiles (tcgen05 sweeps for bf16)
    (1, 8, 1, 128, 6000, 40, 64, 32, 4444),     # two tcgen05 query tiles per CTA
]


@pytest.mark.parametrize("dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("case", GARBAGE_CASES, ids=[str(c) for c in GARBAGE_CASES])
def test_unwritten_cache_slots_past_the_positions_are_never_used(case, dtype):
    # a cache allocated for N tokens but written only up to the last query position: whatever its
    # other slots hold (here NaN in every byte pattern of the format) must not reach the outputs
    B, Hq, Hkv, d, N, T, k, W, last = case
    pos = np.broadcast_to(np.arange(last - T + 1, last + 1, dtype=np.int32), (B, T)).copy()
    inp = make_inputs(B, Hq, Hkv, d, N, T, k, W, seed=last, needles=3, pos=pos)
    inp = with_cache(inp, dtype)
    nan = 0xFFFF if dtype == "bf16" else 0xFF
    inp.cache.K[:, :, last + 1:] = nan
    inp.cache.V[:, :, last + 1:] = nan
    res, bits = run_step_kv(inp)
    assert bits == 0, hex(bits)
    compare_step(inp, res)
