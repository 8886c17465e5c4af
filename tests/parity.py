"""Comparison rules between the CUDA path and the fp64 oracle.

* O (full and sparse): |o - o_ref| <= 1e-2 + 1e-2 * |o_ref| element-wise.
* LSE (full and sparse): |lse - lse_ref| <= 1e-3.
* Selection: the GPU's set must have the oracle's size, no duplicates, contain the
  forced window, stay inside [0, pos], and may differ from the oracle's set only by
  swapping pool keys whose oracle scores lie within 1e-4 of the oracle's k-th best
  pool score (several answers are then correct).  Sparse attention is compared with
  the oracle evaluated on the GPU's own (validated) set.
"""
from __future__ import annotations

import numpy as np
import torch

O_ATOL = 1e-2
O_RTOL = 1e-2
LSE_ATOL = 1e-3
SCORE_TIE_TOL = 1e-4


def to_torch_bf16(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def gpu_inputs(inp, device="cuda"):
    return dict(Q_full=to_torch_bf16(inp.Qf, device), Q_sparse=to_torch_bf16(inp.Qs, device),
                K=to_torch_bf16(inp.K, device), V=to_torch_bf16(inp.V, device),
                pos=torch.from_numpy(np.ascontiguousarray(inp.pos, dtype=np.int32)).to(device))


def assert_close_o(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    bound = O_ATOL + O_RTOL * np.abs(want)
    bad = ~(err <= bound)  # NaN anywhere fails
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(np.isnan(err), np.inf, err - bound)), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements off; worst at {i}: got {got[i]} want {want[i]}")


def assert_close_lse(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    both_inf = np.isneginf(got) & np.isneginf(want)
    err = np.where(both_inf, 0.0, np.abs(got - want))
    if not (err <= LSE_ATOL).all():
        i = np.unravel_index(np.nanargmax(np.where(np.isnan(err), np.inf, err)), err.shape)
        raise AssertionError(f"{what}: LSE off by {err[i]} at {i}: got {got[i]} want {want[i]}")


def check_selection(idx_row: np.ndarray, cnt: int, row, tol: float = SCORE_TIE_TOL) -> np.ndarray:
    """Validate one GPU index row against the oracle's RowResult; return the sorted GPU set."""
    idx_row = np.asarray(idx_row, dtype=np.int64)
    cnt = int(cnt)
    assert 0 <= cnt <= idx_row.shape[0], f"cnt {cnt} out of range"
    assert np.all(idx_row[cnt:] == -1), "padding after cnt must be -1"
    S = np.sort(idx_row[:cnt])
    assert len(np.unique(S)) == len(S), "duplicate indices"
    want = row.selected
    assert len(S) == len(want), f"size {len(S)} != oracle {len(want)}"
    if len(S):
        assert S[0] >= 0 and S[-1] <= row.pos, "index outside [0, pos]"
    win = np.arange(max(0, row.pos - row.W + 1), row.pos + 1)
    assert np.isin(win, S).all(), "forced window not fully selected"
    extra = np.setdiff1d(S, want)
    missing = np.setdiff1d(want, S)
    if len(extra) or len(missing):
        sk = row.kth_score
        P = row.scores.shape[0]
        assert np.all(extra < P), "a non-pool key was selected"
        assert np.all(row.scores[extra] >= sk - tol), \
            f"selected keys {extra[row.scores[extra] < sk - tol][:5]} are not near-ties of the k-th score {sk}"
        assert np.all(row.scores[missing] <= sk + tol), \
            f"dropped keys {missing[row.scores[missing] > sk + tol][:5]} beat the k-th score {sk}"
    return S


def gpu_cache(c, device="cuda"):
    """A generator-side KVCache (numpy) as the binding's KVCache (device tensors)."""
    from long_context_sparse_hs2_b200 import hs2

    def dev(a, dtype=None):
        if a is None:
            return None
        t = torch.from_numpy(np.ascontiguousarray(a))
        return t.to(device) if dtype is None else t.view(dtype).to(device)

    kv_dtype = torch.bfloat16 if c.dtype == "bf16" else None
    K = dev(c.K.view(np.int16) if c.dtype == "bf16" else c.K, kv_dtype)
    V = dev(c.V.view(np.int16) if c.dtype == "bf16" else c.V, kv_dtype)
    return hs2.KVCache(K=K, V=V, N=c.N, dtype=c.dtype, k_scale=dev(c.k_scale), v_scale=dev(c.v_scale),
                       page_size=c.page_size, page_table=dev(c.page_table))


def cache_to_numpy(cache):
    """The binding's KVCache contents back as numpy code arrays (uint16 for bf16, uint8 for fp8)."""
    if cache.dtype == "bf16":
        return cache.K.view(torch.int16).cpu().numpy().view(np.uint16), cache.V.view(torch.int16).cpu().numpy().view(np.uint16)
    return cache.K.view(torch.uint8).cpu().numpy(), cache.V.view(torch.uint8).cpu().numpy()
