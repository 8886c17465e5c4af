"""The C ABI without a GPU: the library loads, exports every declared entry point, and
rejects bad arguments with the documented status before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

from long_context_sparse_hs2_b200 import build as hs2_build
from long_context_sparse_hs2_b200 import hs2
from tests import parity
from tests.oracle_pins import hand8_inputs
import oracle.hs2_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "hs2.h")


@pytest.fixture(scope="module")
def L():
    hs2_build.build()
    return hs2.lib()


def declared_entry_points():
    text = open(HEADER).read()
    return re.findall(r"HS2_API\s+[\w\s\*]+?\b(hs2_\w+)\s*\(", text)


def test_exports_every_declared_symbol(L):
    names = declared_entry_points()
    assert set(names) == set(hs2.ENTRY_POINTS)
    for n in names:
        assert getattr(L, n) is not None


def test_version_and_status_strings(L):
    assert hs2.version() == "1.1"
    for s in range(6):
        assert isinstance(hs2.status_string(s), str) and hs2.status_string(s)


def _dims(**kw):
    base = dict(B=1, Hq=8, Hkv=1, T=1, N=4096, d=128, k=64, W=64)
    base.update(kw)
    return hs2.make_dims(**base)


def test_workspace_size(L):
    ok = hs2.workspace_size(_dims())
    assert ok > 0 and ok % 256 == 0
    assert hs2.workspace_size(_dims(N=8192)) > ok
    for bad in (dict(d=96), dict(Hq=12, Hkv=4), dict(Hq=7, Hkv=2), dict(T=0), dict(N=0), dict(k=-1),
                dict(W=-1), dict(T=5000), dict(B=0)):
        assert hs2.workspace_size(_dims(**bad)) == 0, bad
    assert L.hs2_workspace_size(None) == 0


def test_workspace_follows_the_execution_plan(L, monkeypatch):
    # 128-row query tiles (T*G > 64) run on the tcgen05 sweeps unless HS2_UMMA=0; the split
    # partials, and so the workspace, depend on the plan.  Every supported shape has a size.
    prefill = _dims(Hq=32, Hkv=4, T=4096, N=131072, k=2048, W=128)
    t16 = _dims(Hq=32, Hkv=4, T=16, N=1 << 20, k=8192, W=1024)
    sizes = {}
    for umma in ("1", "0"):
        monkeypatch.setenv("HS2_UMMA", umma)
        sizes[umma] = (hs2.workspace_size(prefill), hs2.workspace_size(t16))
        assert all(v > 0 and v % 256 == 0 for v in sizes[umma])
    assert sizes["1"] != sizes["0"]
    monkeypatch.delenv("HS2_UMMA")
    assert (hs2.workspace_size(prefill), hs2.workspace_size(t16)) == sizes["1"]  # the default is tcgen05
    for G in (1, 2, 4, 8, 16):
        for d in (64, 128):
            assert hs2.workspace_size(_dims(Hq=G, Hkv=1, T=max(1, 200 // G), N=5000, d=d)) > 0, (G, d)


def test_prefill_selection_does_not_store_every_score_key(L, monkeypatch):
    # chunked prefill (16384 selection rows over a 128K cache): the bracketed selection keeps a
    # 1/16 sample and candidate lists, well under 2 GB of workspace; storing every score key
    # (HS2_PREFILL_BRACKET=0) needs the 8.6 GB key matrix
    prefill = _dims(Hq=32, Hkv=4, T=4096, N=131072, k=2048, W=128)
    monkeypatch.delenv("HS2_PREFILL_BRACKET", raising=False)
    bracketed = hs2.workspace_size(prefill)
    monkeypatch.setenv("HS2_PREFILL_BRACKET", "0")
    stored = hs2.workspace_size(prefill)
    assert 0 < bracketed < 2e9 and stored > 8.5e9, (bracketed, stored)


def test_one_launch_decode_plan(L, monkeypatch):
    # the one-launch decode step keeps one sparse partial per sweep split, so its plan needs more
    # workspace than the kernel chain's; it is the default for short caches only
    tiny = _dims(B=1, Hq=4, Hkv=1, d=64, N=2048, T=1, k=64, W=64)
    long = _dims(B=1, Hq=64, Hkv=8, d=128, N=131072, T=1, k=4096, W=512)
    sizes = {}
    for env in (None, "0", "1"):
        if env is None:
            monkeypatch.delenv("HS2_FUSED_DECODE", raising=False)
        else:
            monkeypatch.setenv("HS2_FUSED_DECODE", env)
        sizes[env] = (hs2.workspace_size(tiny), hs2.workspace_size(long))
    assert sizes[None][0] == sizes["1"][0] > sizes["0"][0]      # tiny: one launch by default
    assert sizes[None][1] == sizes["0"][1] < sizes["1"][1]      # 128K: the chain by default


FAKE = 1 << 20  # a 256-byte-aligned non-null address; never dereferenced (checks fail first)


def _full(L, dims, q=FAKE, k=FAKE, v=FAKE, pos=FAKE, o=FAKE, lse=FAKE, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = hs2.workspace_size(dims)
    return L.hs2_full_attn(ctypes.byref(dims), q, k, v, pos, o, lse, ws, ws_bytes, None)


def test_rejects_bad_arguments_without_launching(L):
    d = _dims()
    assert _full(L, d, q=None) == hs2.HS2_ERR_INVALID_ARG
    assert _full(L, d, pos=None) == hs2.HS2_ERR_INVALID_ARG
    assert _full(L, d, k=FAKE + 8) == hs2.HS2_ERR_INVALID_ARG          # misaligned bf16 pointer
    assert _full(L, d, lse=FAKE + 2) == hs2.HS2_ERR_INVALID_ARG        # misaligned fp32 pointer
    assert _full(L, d, ws=None) == hs2.HS2_ERR_WORKSPACE
    assert _full(L, d, ws=FAKE + 16) == hs2.HS2_ERR_WORKSPACE          # ws must be 256-byte aligned
    assert _full(L, d, ws_bytes=hs2.workspace_size(d) - 1) == hs2.HS2_ERR_WORKSPACE
    assert _full(L, _dims(d=96)) == hs2.HS2_ERR_UNSUPPORTED
    assert _full(L, _dims(Hq=24, Hkv=8)) == hs2.HS2_ERR_UNSUPPORTED   # G = 3
    assert _full(L, _dims(Hq=7, Hkv=2)) == hs2.HS2_ERR_INVALID_ARG
    assert _full(L, _dims(T=4097, N=4096)) == hs2.HS2_ERR_INVALID_ARG
    assert L.hs2_full_attn(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == hs2.HS2_ERR_INVALID_ARG
    n = hs2.workspace_size(d)
    assert L.hs2_select(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, n, None) == hs2.HS2_ERR_INVALID_ARG
    assert L.hs2_sparse_attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, n, None) \
        == hs2.HS2_ERR_INVALID_ARG
    assert L.hs2_step(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                      n - 256, None) == hs2.HS2_ERR_WORKSPACE
    bits = ctypes.c_uint32()
    assert L.hs2_read_device_status(None, None, ctypes.byref(bits)) == hs2.HS2_ERR_INVALID_ARG


def test_python_binding_refuses_cpu_tensors():
    import torch

    x = torch.zeros(1, 4, 1, 64, dtype=torch.bfloat16)
    kv = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    pos = torch.zeros(1, 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        hs2.step(x, x, kv, kv, pos, k=1, W=1)


def test_selection_checker_accepts_oracle_and_rejects_wrong_sets():
    inp = hand8_inputs()
    r = O.step_rows(inp)[(0, 0, 1)]
    kw = inp.k + inp.W
    good = np.full(kw, -1)
    good[:4] = [7, 1, 6, 4]
    parity.check_selection(good, 4, r)
    swapped = good.copy()
    swapped[1] = 5   # 5 ties 1 exactly, so swapping them is allowed
    parity.check_selection(swapped, 4, r)
    for bad, cnt in (([7, 0, 6, 4], 4), ([7, 1, 6, 6], 4), ([7, 1, 6, -1], 3), ([1, 4, 6, 5], 4)):
        row = np.full(kw, -1)
        row[:len(bad)] = bad
        with pytest.raises(AssertionError):
            parity.check_selection(row, cnt, r)


def test_python_binding_refuses_tensors_on_two_devices():
    # the library launches on the current device and dereferences every pointer there, so the
    # binding must refuse a call whose tensors sit on two GPUs before anything is launched
    import types

    import torch

    on = lambda i: types.SimpleNamespace(device=torch.device("cuda", i))  # noqa: E731
    assert hs2.device_of("t", Q=on(1), K=on(1), ws=None) == torch.device("cuda", 1)
    with pytest.raises(ValueError, match="one CUDA device"):
        hs2.device_of("t", Q=on(0), K=on(1))
    with pytest.raises(ValueError, match="one CUDA device"):
        hs2.device_of("t", Q=on(0), K=on(0), ws=on(1))


def _desc(**kw):
    base = dict(dtype=hs2.KV_BF16, page_size=0, num_pages=0, max_pages=0, K=FAKE, V=FAKE, page_table=None,
                k_scale=None, v_scale=None)
    base.update(kw)
    return hs2.KvCacheDesc(**base)


def test_cache_descriptor_workspace_and_rejections(L):
    d = _dims(N=4096)
    ws_bf16 = L.hs2_workspace_size_kv(ctypes.byref(d), ctypes.byref(_desc()))
    assert ws_bf16 == hs2.workspace_size(d)           # a contiguous bf16 descriptor is the plain call
    paged = _desc(page_size=16, num_pages=300, max_pages=256, page_table=FAKE)
    fp8 = _desc(dtype=hs2.KV_FP8_E4M3, k_scale=FAKE, v_scale=FAKE)
    for desc in (paged, fp8, _desc(dtype=hs2.KV_FP8_E4M3, page_size=64, num_pages=70, max_pages=64,
                                   page_table=FAKE, k_scale=FAKE, v_scale=FAKE)):
        assert L.hs2_workspace_size_kv(ctypes.byref(d), ctypes.byref(desc)) > 0
    # 128-row query tiles: fp8 and paged caches take the warp-level MMA sweeps (another plan)
    pre = _dims(Hq=32, Hkv=4, T=4096, N=131072, k=2048, W=128)
    assert L.hs2_workspace_size_kv(ctypes.byref(pre), ctypes.byref(fp8)) == \
        L.hs2_workspace_size_kv(ctypes.byref(pre), ctypes.byref(_desc(page_size=64, num_pages=2048, max_pages=2048,
                                                                       page_table=FAKE)))
    bad_shapes = [_desc(page_size=24, num_pages=300, max_pages=256, page_table=FAKE),   # not a power of two
                  _desc(page_size=4, num_pages=2000, max_pages=1024, page_table=FAKE),  # below 8
                  _desc(page_size=16, num_pages=300, max_pages=255, page_table=FAKE),   # table too short
                  _desc(page_size=16, num_pages=0, max_pages=256, page_table=FAKE),
                  _desc(dtype=7)]
    for desc in bad_shapes:
        assert L.hs2_workspace_size_kv(ctypes.byref(d), ctypes.byref(desc)) == 0
    assert L.hs2_workspace_size_kv(ctypes.byref(d), None) == 0
    n = hs2.workspace_size(d) * 4
    def step(desc, dims=d, ws_bytes=n):
        return L.hs2_step_kv(ctypes.byref(dims), FAKE, FAKE, ctypes.byref(desc), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                             FAKE, FAKE, ws_bytes, None)
    assert step(bad_shapes[0]) == hs2.HS2_ERR_INVALID_ARG
    assert step(_desc(page_size=16, num_pages=300, max_pages=256)) == hs2.HS2_ERR_INVALID_ARG   # no page table
    assert step(_desc(dtype=hs2.KV_FP8_E4M3)) == hs2.HS2_ERR_INVALID_ARG                        # no scales
    assert step(_desc(K=FAKE + 8)) == hs2.HS2_ERR_INVALID_ARG                                   # misaligned cache
    assert step(_desc(), ws_bytes=16) == hs2.HS2_ERR_WORKSPACE
    assert step(_desc(), dims=_dims(d=96)) == hs2.HS2_ERR_UNSUPPORTED
    # the decode step takes one query per batch row
    t2 = _dims(T=2)
    assert L.hs2_decode_step(ctypes.byref(t2), ctypes.byref(_desc()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                             FAKE, FAKE, FAKE, FAKE, FAKE, n, None) == hs2.HS2_ERR_INVALID_ARG
    # the append needs the 256-byte status word
    assert L.hs2_kv_append(ctypes.byref(d), ctypes.byref(_desc()), FAKE, FAKE, FAKE, FAKE, 128, None) == \
        hs2.HS2_ERR_WORKSPACE


def test_parity_checker_rejects_nan():
    # a non-finite kernel output must fail the comparison, not slip through it
    with pytest.raises(AssertionError):
        parity.assert_close_o(np.array([0.5, np.nan]), np.array([0.5, 0.25]), "nan")
    with pytest.raises(AssertionError):
        parity.assert_close_lse(np.array([1.0, np.nan]), np.array([1.0, 2.0]), "nan")
    parity.assert_close_o(np.array([0.5, 0.251]), np.array([0.5, 0.25]), "close")


def test_wait_bound_selftest_argument_checks(L):
    assert L.hs2_selftest_wait_bound(None, 256, 10_000, None) == hs2.HS2_ERR_WORKSPACE
    assert L.hs2_selftest_wait_bound(FAKE, 128, 10_000, None) == hs2.HS2_ERR_WORKSPACE
    assert L.hs2_selftest_wait_bound(FAKE, 256, 10, None) == hs2.HS2_ERR_INVALID_ARG            # below 1 us
    assert L.hs2_selftest_wait_bound(FAKE, 256, 3_000_000_000, None) == hs2.HS2_ERR_INVALID_ARG  # above 2 s
