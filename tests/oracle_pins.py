"""Pins that tie the fp64 oracle to facts outside itself.

Each ``pin_*`` function raises ``AssertionError`` when the oracle disagrees with
something the pages or the mathematics fix independently of the oracle's code:

* a hand-computed 8-token example whose expected values are closed forms
  (``tests/golden/hand8.json``);
* PyTorch's scaled-dot-product attention (a different implementation of full
  attention) on random GQA inputs with per-query causal limits;
* the attention weights of that library routine (read out by attending over an
  identity value matrix), whose per-key max over the GQA heads is exp(score);
* brute force over every k-subset of tiny pools for the top-k with the
  lower-index tie rule;
* invariants: weights sum to one, a single visible key, a constant query,
  window always present, the selection count formula, and the collapse of the
  sparse layer to full attention when k covers the pool.

The mutation test runs every pin against deliberately broken copies of the
oracle and requires each break to trip at least one pin.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

from long_context_sparse_hs2_b200.inputs import Inputs, f32_to_bf16_bits, make_inputs
import oracle.hs2_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- hand example

def _closed_form(expr: str) -> float:
    """Evaluate a closed form written with e, ln and + - * / ** (golden fixtures)."""
    return float(eval(expr, {"__builtins__": {}}, {"e": math.e, "ln": math.log}))


def hand8_inputs() -> Inputs:
    """The constructed inputs of the hand-computed example."""
    spec = json.load(open(os.path.join(GOLDEN, "hand8.json")))["construction"]
    B, Hq, Hkv, d, N, T = (spec[x] for x in ("B", "Hq", "Hkv", "d", "N", "T"))
    qf = np.zeros((B, Hq, T, d), np.float32)
    qs = np.zeros((B, Hq, T, d), np.float32)
    for t in range(T):
        qf[0, 0, t, 0] = 8.0
        qf[0, 1, t, 1] = 8.0
        qs[0, 0, t, 2] = 8.0
        qs[0, 1, t, 3] = 8.0
    k = np.zeros((B, Hkv, N, d), np.float32)
    for col, vals in spec["K_columns"].items():
        k[0, 0, :, int(col)] = vals
    v = np.zeros((B, Hkv, N, d), np.float32)
    for j in range(N):
        v[0, 0, j, j] = 1.0
    return Inputs(Qf=f32_to_bf16_bits(qf), Qs=f32_to_bf16_bits(qs), K=f32_to_bf16_bits(k),
                  V=f32_to_bf16_bits(v), pos=np.array(spec["pos"], np.int32),
                  k=spec["k"], W=spec["W"])


def hand8_expected():
    exp = json.load(open(os.path.join(GOLDEN, "hand8.json")))["expected"]
    out = {}
    for key, t in (("t0", 0), ("t1", 1)):
        e = exp[key]
        out[t] = dict(
            lse_full=np.array([_closed_form(x) for x in e["lse_full"]]),
            o_full=np.array([[_closed_form(x) for x in row] for row in e["o_full_dims0to7"]]),
            scores=np.array([_closed_form(x) for x in e["scores"]]),
            selected=np.array(e["selected"], np.int64),
            lse_sparse=np.array([_closed_form(x) for x in e["lse_sparse"]]),
            o_sparse=np.array([[_closed_form(x) for x in row] for row in e["o_sparse_dims0to7"]]),
        )
    return out


def pin_hand8():
    inp = hand8_inputs()
    res = O.step_rows(inp)
    want = hand8_expected()
    for t in (0, 1):
        r, w = res[(0, 0, t)], want[t]
        np.testing.assert_allclose(r.lse_full, w["lse_full"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.o_full[:, :8], w["o_full"], rtol=0, atol=1e-12)
        assert np.all(r.o_full[:, 8:] == 0)
        np.testing.assert_allclose(r.scores, w["scores"], rtol=0, atol=1e-12)
        np.testing.assert_array_equal(r.selected, w["selected"])
        np.testing.assert_allclose(r.lse_sparse, w["lse_sparse"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.o_sparse[:, :8], w["o_sparse"], rtol=0, atol=1e-12)
        assert np.all(r.o_sparse[:, 8:] == 0)


# ----------------------------------------------------------------------------- library routine

def _random_case(seed, B=2, Hq=4, Hkv=2, d=64, N=40, T=3, k=5, W=4):
    rng = np.random.default_rng(seed + 1000)
    pos = np.sort(rng.integers(0, N, size=(B, T)), axis=1).astype(np.int32)
    pos[:, -1] = N - 1
    return make_inputs(B, Hq, Hkv, d, N, T, k, W, seed, pos=pos)


def _sdpa_f64(q_bits, K_bits, V, pos_row, G):
    """torch SDPA in float64 for one (b, t): q [Hq, d], K/V [Hkv, N, d]."""
    q = torch.from_numpy(O.bf16_to_f64(q_bits))[None, :, None, :]           # [1,Hq,1,d]
    k = torch.from_numpy(O.bf16_to_f64(K_bits)).repeat_interleave(G, dim=0)[None]  # [1,Hq,N,d]
    v = torch.from_numpy(V).repeat_interleave(G, dim=0)[None]
    N = k.shape[2]
    mask = (torch.arange(N) <= int(pos_row))[None, None, None, :]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)[0, :, 0]


def pin_full_attention_matches_sdpa():
    for seed in range(3):
        inp = _random_case(seed)
        B, Hq, T, d = inp.Qf.shape
        Hkv = inp.K.shape[1]
        G = Hq // Hkv
        res = O.step(inp)
        for b in range(B):
            for t in range(T):
                ref = _sdpa_f64(inp.Qf[b, :, t], inp.K[b], O.bf16_to_f64(inp.V[b]), inp.pos[b, t], G)
                np.testing.assert_allclose(res.O_full[b, :, t], ref.numpy(), rtol=1e-10, atol=1e-12)


def pin_scores_match_sdpa_weights():
    """exp(score_j) equals the max over the GQA heads of SDPA's weight on key j."""
    for seed in range(3):
        inp = _random_case(seed)
        B, Hq, T, d = inp.Qf.shape
        Hkv, N = inp.K.shape[1], inp.K.shape[2]
        G = Hq // Hkv
        eye = np.broadcast_to(np.eye(N), (Hkv, N, N)).copy()
        res = O.step(inp)
        for b in range(B):
            for t in range(T):
                w = _sdpa_f64(inp.Qf[b, :, t], inp.K[b], eye, inp.pos[b, t], G).numpy()  # [Hq, N]
                pos = int(inp.pos[b, t])
                P = max(0, pos - inp.W + 1)
                for h in range(Hkv):
                    want = np.log(w[h * G:(h + 1) * G, :P].max(axis=0))
                    np.testing.assert_allclose(res.scores[(b, h, t)], want, rtol=0, atol=1e-10)


def pin_sparse_attention_matches_masked_sdpa():
    """Sparse attention equals SDPA over all keys with a mask that keeps only the selection."""
    for seed in range(3):
        inp = _random_case(seed, N=48, k=6, W=3)
        B, Hq, T, d = inp.Qf.shape
        Hkv, N = inp.K.shape[1], inp.K.shape[2]
        G = Hq // Hkv
        res = O.step(inp)
        for b in range(B):
            for t in range(T):
                for h in range(Hkv):
                    sel = res.selected[(b, h, t)]
                    q = torch.from_numpy(O.bf16_to_f64(inp.Qs[b, h * G:(h + 1) * G, t]))[None, :, None]
                    k = torch.from_numpy(O.bf16_to_f64(inp.K[b, h]))[None, None].expand(1, G, N, d)
                    v = torch.from_numpy(O.bf16_to_f64(inp.V[b, h]))[None, None].expand(1, G, N, d)
                    mask = torch.zeros(N, dtype=torch.bool)
                    mask[torch.from_numpy(sel)] = True
                    ref = torch.nn.functional.scaled_dot_product_attention(
                        q, k, v, attn_mask=mask[None, None, None, :])[0, :, 0].numpy()
                    np.testing.assert_allclose(res.O_sparse[b, h * G:(h + 1) * G, t], ref,
                                               rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- brute force

def _brute_topk(s, k):
    """The k-subset in which every member beats every non-member under (score desc, index asc)."""
    P = len(s)
    k = min(k, P)
    beats = lambda a, b: s[a] > s[b] or (s[a] == s[b] and a < b)
    found = []
    for sub in itertools.combinations(range(P), k):
        inside = set(sub)
        if all(beats(a, b) for a in inside for b in range(P) if b not in inside):
            found.append(sub)
    assert len(found) == 1
    best_sum = max(sum(s[list(c)]) for c in itertools.combinations(range(P), k)) if k else 0.0
    assert abs(sum(s[list(found[0])]) - best_sum) < 1e-12
    return np.array(found[0], np.int64)


def pin_topk_bruteforce():
    rng = np.random.default_rng(7)
    for trial in range(200):
        P = int(rng.integers(0, 9))
        k = int(rng.integers(0, 6))
        # scores from a small alphabet so that exact ties are common
        s = rng.choice(np.array([-3.0, -2.5, -2.0, -1.0, -0.5]), size=P)
        np.testing.assert_array_equal(O.topk_pool(s, k), _brute_topk(s, k))


def pin_topk_bruteforce_through_step():
    """Whole-step selection on tiny random inputs equals brute force on the pin-derived scores."""
    for seed in range(4):
        inp = make_inputs(1, 2, 1, 64, 12, 2, 3, 2, seed, pos=np.array([[7, 11]]), q_scale=0.5)
        res = O.step_rows(inp)
        for t in range(2):
            r = res[(0, 0, t)]
            top = _brute_topk(r.scores, inp.k)
            want = np.union1d(top, np.arange(max(0, r.pos - inp.W + 1), r.pos + 1))
            np.testing.assert_array_equal(r.selected, want)


def pin_exact_ties_take_lower_index():
    """Duplicated key rows give bit-identical scores; the lower index must win."""
    inp = make_inputs(1, 2, 1, 64, 16, 1, 1, 2, seed=11)
    K = inp.K.copy()
    # make keys 3 and 9 identical and clearly the best: boost them along q of head 0
    q = O.bf16_to_f64(inp.Qf[0, 0, 0])
    row = O.bf16_to_f64(K[0, 0, 3]) + 4.0 * q / np.linalg.norm(q)
    K[0, 0, 3] = f32_to_bf16_bits(row.astype(np.float32))
    K[0, 0, 9] = K[0, 0, 3]
    inp.K = K
    r = O.step_rows(inp)[(0, 0, 0)]
    assert r.scores[3] == r.scores[9] == r.scores.max()
    np.testing.assert_array_equal(r.selected, [3, 14, 15])


# ----------------------------------------------------------------------------- invariants

def pin_weights_sum_to_one():
    """With V = 1 everywhere, both attention outputs are exactly 1 (weights sum to 1)."""
    inp = _random_case(3)
    inp.V = np.full_like(inp.V, f32_to_bf16_bits(np.array([1.0], np.float32))[0])
    res = O.step(inp)
    np.testing.assert_allclose(res.O_full, 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res.O_sparse, 1.0, rtol=0, atol=1e-12)


def pin_single_key_and_constant_query():
    """pos = 0: O = v_0 and LSE = l_0.  Q = 0: LSE = ln(pos + 1) and O = mean of V[0..pos]."""
    inp = make_inputs(1, 2, 1, 64, 10, 2, 4, 2, seed=5, pos=np.array([[0, 9]]))
    res = O.step_rows(inp)
    r0 = res[(0, 0, 0)]
    v0 = O.bf16_to_f64(inp.V[0, 0, 0])
    np.testing.assert_allclose(r0.o_full, np.stack([v0, v0]), rtol=0, atol=1e-12)
    l0 = (O.bf16_to_f64(inp.Qf[0, :, 0]) @ O.bf16_to_f64(inp.K[0, 0, 0])) / 8.0
    np.testing.assert_allclose(r0.lse_full, l0, rtol=0, atol=1e-12)
    inp.Qf = np.zeros_like(inp.Qf)
    r1 = O.step_rows(inp)[(0, 0, 1)]
    np.testing.assert_allclose(r1.lse_full, math.log(10.0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r1.o_full[0], O.bf16_to_f64(inp.V[0, 0]).mean(axis=0), atol=1e-12)


def pin_window_and_count():
    """Window always selected; |selected| = min(k, |pool|) + min(W, pos + 1); all <= pos."""
    rng = np.random.default_rng(3)
    for trial in range(40):
        N = int(rng.integers(1, 30))
        W = int(rng.integers(0, 8))
        k = int(rng.integers(0, 10))
        pos = int(rng.integers(0, N))
        inp = make_inputs(1, 2, 1, 64, N, 1, k, W, seed=trial, pos=np.array([[pos]]))
        r = O.step_rows(inp)[(0, 0, 0)]
        pool = max(0, pos - W + 1)
        win = np.arange(max(0, pos - W + 1), pos + 1)
        assert set(win.tolist()) <= set(r.selected.tolist())
        assert len(r.selected) == min(k, pool) + min(W, pos + 1)
        assert len(set(r.selected.tolist())) == len(r.selected)
        assert r.selected.min(initial=0) >= 0 and r.selected.max(initial=0) <= pos
        assert r.scores.shape[0] == pool


def pin_collapse_to_full_attention():
    """k >= |pool| selects every visible key; with Q_sparse = Q_full the layers agree."""
    inp = _random_case(4, k=10 ** 6)
    inp.Qs = inp.Qf.copy()
    res = O.step(inp)
    np.testing.assert_allclose(res.O_sparse, res.O_full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(res.LSE_sparse, res.LSE_full, rtol=0, atol=1e-12)
    for (b, h, t), sel in res.selected.items():
        np.testing.assert_array_equal(sel, np.arange(int(inp.pos[b, t]) + 1))


ALL_PINS = [
    pin_hand8,
    pin_full_attention_matches_sdpa,
    pin_scores_match_sdpa_weights,
    pin_sparse_attention_matches_masked_sdpa,
    pin_topk_bruteforce,
    pin_topk_bruteforce_through_step,
    pin_exact_ties_take_lower_index,
    pin_weights_sum_to_one,
    pin_single_key_and_constant_query,
    pin_window_and_count,
    pin_collapse_to_full_attention,
]


# the stored-cache readers (fp8, paged, decode loop) have their own pins
from tests.cache_pins import CACHE_PINS  # noqa: E402

ALL_PINS = ALL_PINS + CACHE_PINS
