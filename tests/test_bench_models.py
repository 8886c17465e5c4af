"""The bench's roofline numerators, checked on the CPU against closed forms.

`bench.py` divides algorithmic bytes (or FLOPs) per launch by the live CUDA-event time of the
dominant kernel.  These tests pin those numerators for every benchmark shape:
* K and V read once: 2 * B * Hkv * N * d * e bytes (e = 2 for bf16, 1 for FP8 E4M3);
* the metric's literal bytes: K once plus the gathered K and V rows of every selection row,
  min(k, pool) + min(W, pos + 1) rows each -- 290, 274, 1042 and 1312 MiB at the four decode
  shapes;
* the full layer's tensor FLOPs: 4 * B * Hq * d per visible (query, key) pair, causal inside a
  prefill chunk: T (N - T) + T (T + 1) / 2 pairs per head;
and that `roofline()` picks the bound by the ridge (prefill tensor-bound, 16 decode queries
HBM-bound) and reports achieved / peak.
"""
import pytest

import bench

MIB = 1 << 20


@pytest.mark.parametrize("name,mib", [("batched", 290), ("long", 274), ("1m_t1", 1042), ("1m_t16", 1312)])
def test_literal_bytes_of_the_decode_shapes(name, mib):
    w = bench.workload(name)
    bm = bench.byte_model(w)
    assert bm["literal"] / MIB == pytest.approx(mib, abs=0.5)


@pytest.mark.parametrize("name", ["tiny", "batched", "long", "1m_t1", "1m_t16", "prefill"])
@pytest.mark.parametrize("dtype,e", [("bf16", 2), ("fp8_e4m3", 1)])
def test_kv_once_and_gathered_rows(name, dtype, e):
    w = bench.workload(name)
    bm = bench.byte_model(w, dtype)
    assert bm["kv_once"] == 2 * w.B * w.Hkv * w.N * w.d * e
    rows = 0
    for t in range(w.T):
        pos = w.N - w.T + t
        pool = max(0, pos + 1 - w.W)
        rows += min(w.k, pool) + min(w.W, pos + 1)
    assert bm["gathered"] == w.B * w.Hkv * rows * 2 * w.d * e
    assert bm["literal"] == bm["kv_once"] // 2 + bm["gathered"]


def test_long_decode_numbers_by_hand():
    # B=1, Hkv=8, N=131072, d=128, k=4096, W=512, one query: 4608 rows per kv head
    bm = bench.byte_model(bench.workload("long"))
    assert bm["kv_once"] == 536870912
    assert bm["gathered"] == 8 * 4608 * 512
    assert bm["literal"] == 268435456 + 18874368


def test_prefill_flops_closed_form():
    w = bench.workload("prefill")
    pairs = w.T * (w.N - w.T) + w.T * (w.T + 1) // 2
    assert bench.flop_model(w) == 4 * w.B * w.Hq * w.d * pairs
    assert bench.flop_model(w) == pytest.approx(8.6587e12, rel=1e-4)


PEAKS = {"hbm_gbs": 6545.9, "bf16_tflops": 1609.7, "bf16_tflops_sustained": 1345.1}


def _kern(name, us):
    return {name: {"avg_us": us, "launches": 1, "share": 1.0}}


def test_roofline_prefill_is_tensor_bound():
    w = bench.workload("prefill")
    r = bench.roofline(w, "bf16", _kern("umma_attn", 8736.0), PEAKS, "measured", "prefill")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(bench.flop_model(w) / 8736e-6 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops"])


def test_roofline_sixteen_decode_queries_are_hbm_bound():
    w = bench.workload("1m_t16")
    r = bench.roofline(w, "bf16", _kern("umma_attn", 338.8), PEAKS, "measured", "1m_t16")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(2147483648 / 338.8e-6 / 1e9)
    assert r["tensor"]["achieved_tflops"] == pytest.approx(bench.flop_model(w) / 338.8e-6 / 1e12)


def test_roofline_decode_sweep_and_one_launch_step():
    w = bench.workload("long")
    r = bench.roofline(w, "bf16", _kern("full_attn_keep_logits", 92.0), PEAKS, "measured", "long")
    assert r["bound"] == "hbm" and r["algorithmic_bytes_per_launch"] == 536870912
    assert r["frac"] == pytest.approx(536870912 / 92e-6 / 1e9 / PEAKS["hbm_gbs"])
    t = bench.workload("tiny")
    bm = bench.byte_model(t)
    r = bench.roofline(t, "bf16", _kern("decode_fused", 60.0), PEAKS, "measured", "tiny")
    assert r["algorithmic_bytes_per_launch"] == bm["kv_once"] + bm["gathered"]
