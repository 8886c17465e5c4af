"""Plain fp64 CPU oracle of the HySparse2 hybrid sparse attention step.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check in
``__graft_entry__.py`` and the CPU-baseline leg of ``bench.py`` may import it.
It shares no code with the CUDA path: it reads the bf16 bit patterns the input
generator wrote, widens them exactly to float64 and evaluates the definitions
below with NumPy, one (batch, kv head, query) at a time.  Nothing here is
blocked, fused or reordered beyond what the definitions state; a NumPy matmul,
``exp``/``log`` and a lexicographic sort are the only library primitives used.

What the step computes, and where it comes from
-----------------------------------------------
HySparse2 puts hybrid sparse attention in the cross-decoder: occasional
full-attention layers, each followed by sparse layers ("HySparse2 Cuts the
Prefill Path for Tool-Using Agents", section "One Cache Plan, Two Sharing
Layers").  Each sparse layer reuses the KV cache of the full-attention layer
before it *and* that layer's selection of tokens (KV Reuse); selection is per
token, not per block, and the most recent tokens are always included, so the
local window and the selected distant tokens share one cache ("HySparse2 od
Xiaomi zkracuje zpracování dlouhého kontextu", section "Proč není nutné znovu
zpracovat celý dlouhý vstup", third paragraph; "DAIR.AI周报：HySparse2长上下文优化与
SIFT代码Agent自改进", bullets "Two levels of KV sharing" and "Prefill exits early").

The pages leave the selection score, its tie rule and the window's relation to
the top-k pool open.  This library fixes them, and the oracle follows:

1. full attention (standard definition): for query head hq of kv head
   h = floor(hq / G) and key j <= pos_t, l_j = d^-1/2 * <q_hq,t , k_h,j>,
   LSE = log sum_j exp(l_j), O_full = sum_j exp(l_j - LSE) v_h,j;
2. selection score of key j for (b, h, t): the max over the G query heads of
   kv head h of the log-softmax probability, s_j = max_g (l_{hG+g,j} - LSE_{hG+g}),
   for j in the pool [0, pos_t - W];
3. selection: the min(k, |pool|) pool keys of largest score, ties to the lower
   index, plus the forced window [max(0, pos_t - W + 1), pos_t] (never part of
   the pool);
4. sparse attention (KV Reuse): the full-attention definition with Q_sparse,
   restricted to the selected keys, the same index set for all G query heads of
   kv head h.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np


# ----------------------------------------------------------------------------- helpers

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def softmax_scale(d: int) -> float:
    """Attention scale d^-1/2 (standard scaled dot-product attention)."""
    return 1.0 / math.sqrt(d)


def kv_head_of(hq: int, G: int) -> int:
    """GQA grouping: query head hq reads kv head floor(hq / G) (consecutive groups)."""
    return hq // G


def window_keys(pos: int, W: int) -> np.ndarray:
    """Forced window: the W most recent keys up to and including the query position."""
    lo = max(0, pos - W + 1)
    return np.arange(lo, pos + 1, dtype=np.int64)


def pool_size(pos: int, W: int) -> int:
    """Number of keys in the top-k pool [0, pos - W] (the window is excluded)."""
    return max(0, pos - W + 1)


def attend(q: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, scale: float):
    """Softmax attention of query rows ``q`` [R, d] over key rows ``Kh`` [n, d].

    Returns (O [R, d], LSE [R], logits [R, n]); LSE is shifted by the row max
    before exponentiating, which is exact in real arithmetic.
    """
    logits = scale * (q @ Kh.T)
    m = logits.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
    p = np.exp(logits - lse[:, None])
    return p @ Vh, lse, logits


def rank_pool(s: np.ndarray) -> np.ndarray:
    """Pool positions ordered best first: by score descending, then index ascending."""
    j = np.arange(s.shape[0], dtype=np.int64)
    return np.lexsort((j, -s))


def topk_pool(s: np.ndarray, k: int) -> np.ndarray:
    """The min(k, |pool|) best pool keys (ties to the lower index), sorted by index."""
    return np.sort(rank_pool(s)[:min(k, s.shape[0])])


# ----------------------------------------------------------------------------- the step

@dataclass
class RowResult:
    """Everything the oracle knows about one (b, kv head, query) row."""

    b: int
    h: int
    t: int
    pos: int
    k: int
    W: int
    heads: np.ndarray         # the G query heads of kv head h
    lse_full: np.ndarray      # [G] natural-log LSE of the G query heads
    o_full: np.ndarray        # [G, d]
    scores: np.ndarray        # [|pool|] selection scores of keys 0 .. pos-W
    selected: np.ndarray      # sorted int64 key indices: top-k of the pool + window
    o_sparse: np.ndarray      # [G, d]
    lse_sparse: np.ndarray    # [G]

    @property
    def n_top(self) -> int:
        """How many selected keys come from the pool: min(k, |pool|)."""
        return min(self.k, self.scores.shape[0])

    @property
    def kth_score(self) -> float:
        """Score of the worst selected pool key (nan if nothing came from the pool)."""
        if self.n_top <= 0:
            return float("nan")
        return float(np.sort(self.scores)[::-1][self.n_top - 1])


def full_attention_row(Qf: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, pos: int, scale: float):
    """Full attention of the G query rows of one (b, kv head, t) over keys 0..pos."""
    return attend(Qf, Kh[:pos + 1], Vh[:pos + 1], scale)


def selection_scores_row(logits: np.ndarray, lse: np.ndarray, pos: int, W: int) -> np.ndarray:
    """s_j = max over the G heads of (l_j - LSE) for j in the pool [0, pos - W]."""
    P = pool_size(pos, W)
    if P == 0:
        return np.zeros((0,), dtype=np.float64)
    return (logits[:, :P] - lse[:, None]).max(axis=0)


def select_row(scores: np.ndarray, pos: int, k: int, W: int) -> np.ndarray:
    """Top-k of the pool (ties to lower index) plus the forced window, sorted."""
    top = topk_pool(scores, k)
    return np.union1d(top, window_keys(pos, W))


def sparse_attention_row(Qs: np.ndarray, Kh: np.ndarray, Vh: np.ndarray,
                         selected: np.ndarray, scale: float):
    """Sparse attention of the G query rows over the selected keys only (KV Reuse).

    An empty selection (k = 0 and W = 0) is an empty sum: O = 0 and LSE = -inf.
    """
    if selected.shape[0] == 0:
        return np.zeros((Qs.shape[0], Kh.shape[1])), np.full((Qs.shape[0],), -np.inf)
    O, lse, _ = attend(Qs, Kh[selected], Vh[selected], scale)
    return O, lse


def step_rows(inp, rows: Optional[Iterable[Tuple[int, int, int]]] = None,
              selected_override: Optional[Dict[Tuple[int, int, int], np.ndarray]] = None
              ) -> Dict[Tuple[int, int, int], RowResult]:
    """Run the whole step for the requested (b, kv head, t) rows (default: all).

    ``selected_override`` replaces the oracle's own selection for a row when
    evaluating sparse attention (used to score a different but valid index set).
    """
    B, Hq, T, d = inp.Qf.shape
    Hkv, N = inp.K.shape[1], inp.K.shape[2]
    G = Hq // Hkv
    scale = softmax_scale(d)
    if rows is None:
        rows = [(b, h, t) for b in range(B) for h in range(Hkv) for t in range(T)]
    rows = list(rows)
    by_head: Dict[Tuple[int, int], List[int]] = {}
    for b, h, t in rows:
        by_head.setdefault((b, h), []).append(t)
    out: Dict[Tuple[int, int, int], RowResult] = {}
    for (b, h), ts in by_head.items():
        Kh = bf16_to_f64(inp.K[b, h])
        Vh = bf16_to_f64(inp.V[b, h])
        heads = [hq for hq in range(Hq) if kv_head_of(hq, G) == h]
        for t in ts:
            pos = int(inp.pos[b, t])
            qf = bf16_to_f64(inp.Qf[b, heads, t])
            qs = bf16_to_f64(inp.Qs[b, heads, t])
            o_full, lse, logits = full_attention_row(qf, Kh, Vh, pos, scale)
            scores = selection_scores_row(logits, lse, pos, inp.W)
            selected = select_row(scores, pos, inp.k, inp.W)
            use = selected
            if selected_override is not None and (b, h, t) in selected_override:
                use = np.asarray(selected_override[(b, h, t)], dtype=np.int64)
            o_sp, lse_sp = sparse_attention_row(qs, Kh, Vh, use, scale)
            out[(b, h, t)] = RowResult(
                b=b, h=h, t=t, pos=pos, k=inp.k, W=inp.W, heads=np.asarray(heads),
                lse_full=lse, o_full=o_full, scores=scores, selected=selected,
                o_sparse=o_sp, lse_sparse=lse_sp)
    return out


@dataclass
class StepResult:
    """Dense outputs of the step, laid out like the library's outputs."""

    O_full: np.ndarray        # [B, Hq, T, d] float64
    LSE_full: np.ndarray      # [B, Hq, T]
    O_sparse: np.ndarray      # [B, Hq, T, d]
    LSE_sparse: np.ndarray    # [B, Hq, T]
    selected: Dict[Tuple[int, int, int], np.ndarray]
    scores: Dict[Tuple[int, int, int], np.ndarray]


def step(inp) -> StepResult:
    """The whole step over every row, as dense arrays (small inputs only)."""
    B, Hq, T, d = inp.Qf.shape
    rows = step_rows(inp)
    O_full = np.zeros((B, Hq, T, d))
    LSE_full = np.zeros((B, Hq, T))
    O_sp = np.zeros((B, Hq, T, d))
    LSE_sp = np.zeros((B, Hq, T))
    sel, sc = {}, {}
    for (b, h, t), r in rows.items():
        hs = r.heads
        O_full[b, hs, t] = r.o_full
        LSE_full[b, hs, t] = r.lse_full
        O_sp[b, hs, t] = r.o_sparse
        LSE_sp[b, hs, t] = r.lse_sparse
        sel[(b, h, t)] = r.selected
        sc[(b, h, t)] = r.scores
    return StepResult(O_full, LSE_full, O_sp, LSE_sp, sel, sc)
