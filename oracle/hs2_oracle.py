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

The shared cache may be stored in other ways than contiguous bf16 (the pages
give no storage format; the 2.69 GB cache figure comes without its precision:
"HySparse2 od Xiaomi zkracuje zpracování dlouhého kontextu", section "Co říkají
výsledky — a co z nich neplyne").  The oracle reads every stored form back to
exact float64 values first (section "KV cache as stored" below) and then applies
the same four definitions:

* FP8 E4M3 codes with one fp32 scale per (b, kv head) for K and one for V: the
  value of a code is its exact E4M3 value times the scale;
* a paged pool: token j of batch row b lives in page page_table[b][j // page_size]
  at slot j % page_size;
* a run of decode steps: each step first writes the new token's K/V at position
  pos + 1 (rounded to E4M3 for an fp8 cache) and then computes the step for a
  query at that position.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
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


# ----------------------------------------------------------------------------- KV cache as stored

def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Exact value of FP8 E4M3 codes: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal, (m / 8) * 2^-6; otherwise (1 + m / 8) * 2^(e - 7).  The
    codes S.1111.111 are NaN; the format has no infinities (largest finite value 448)."""
    c = np.asarray(codes).astype(np.int64)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return np.where(c & 0x80, -mag, mag)


def quantize_e4m3(x_f32: np.ndarray, scale: float) -> np.ndarray:
    """E4M3 code of the float32 quotient x / scale: round to nearest, ties to even, magnitudes
    beyond 448 saturate to 448 (codes 0x7E / 0xFE), NaN gives 0x7F.

    The quotient is one IEEE float32 division (the precision the rounding decision is taken
    in); the rounding itself is done exactly in float64 on that quotient."""
    v = (np.asarray(x_f32, np.float32) / np.float32(scale)).astype(np.float64)
    sign = np.where(np.signbit(v), 0x80, 0).astype(np.int64)
    a = np.abs(v)
    code = np.zeros(a.shape, np.int64)
    sub = a < 2.0 ** -6
    # subnormal range: multiples of 2^-9 (a count of 8 is the smallest normal, code 0x08)
    code = np.where(sub, np.rint(np.where(sub, a, 0.0) / 2.0 ** -9).astype(np.int64), code)
    # normal range: a = f * 2^ex with f in [0.5, 1) -> exponent ex - 1, 3 mantissa bits
    with np.errstate(divide="ignore", invalid="ignore"):
        _, ex = np.frexp(np.where(sub | ~np.isfinite(a), 1.0, a))
    e = ex.astype(np.int64) - 1
    q = np.rint(np.where(sub | ~np.isfinite(a), 8.0, a / np.exp2(e - 3.0))).astype(np.int64)  # in [8, 16]
    carry = q == 16
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 8, q)
    normal = ((e + 7) << 3) | (q - 8)
    normal = np.where((e > 8) | ((e == 8) & (q > 14)) | np.isinf(a), 0x7E, normal)
    code = np.where(sub, code, normal)
    code = code | sign
    code = np.where(np.isnan(v), 0x7F, code)
    return code.astype(np.uint8)


def cache_token_slot(c, b: int, j: int) -> Tuple[object, int]:
    """Where token j of batch row b is stored: (index into the first axis, token slot)."""
    if c.page_size:
        return int(c.page_table[b, j // c.page_size]), j % c.page_size
    return b, j


def cache_rows_f64(inp, b: int, h: int) -> Tuple[np.ndarray, np.ndarray]:
    """Keys and values of (b, kv head h) as exact float64 [N, d], read from the cache as stored."""
    c = getattr(inp, "cache", None)
    if c is None:
        return bf16_to_f64(inp.K[b, h]), bf16_to_f64(inp.V[b, h])
    if c.page_size:
        rows = [cache_token_slot(c, b, j) for j in range(c.N)]
        Kc = np.stack([c.K[p, h, slot] for p, slot in rows])
        Vc = np.stack([c.V[p, h, slot] for p, slot in rows])
    else:
        Kc, Vc = c.K[b, h], c.V[b, h]
    if c.dtype == "bf16":
        return bf16_to_f64(Kc), bf16_to_f64(Vc)
    if c.dtype == "fp8_e4m3":
        return e4m3_to_f64(Kc) * float(c.k_scale[b, h]), e4m3_to_f64(Vc) * float(c.v_scale[b, h])
    raise ValueError(f"unknown cache dtype {c.dtype}")


def append_token(c, b: int, j: int, k_bits: np.ndarray, v_bits: np.ndarray) -> None:
    """Write one new token (bf16 K and V rows [Hkv, d]) into the cache at position j, in place:
    bf16 caches store the bits as they are, fp8 caches the E4M3 codes of value / scale."""
    p, slot = cache_token_slot(c, b, j)
    for h in range(c.Hkv):
        if c.dtype == "bf16":
            c.K[p, h, slot] = k_bits[h]
            c.V[p, h, slot] = v_bits[h]
        else:
            c.K[p, h, slot] = quantize_e4m3(bf16_to_f64(k_bits[h]).astype(np.float32), c.k_scale[b, h])
            c.V[p, h, slot] = quantize_e4m3(bf16_to_f64(v_bits[h]).astype(np.float32), c.v_scale[b, h])


def decode_loop(steps, cache):
    """A run of decode steps (``DecodeSteps``) over ``cache`` (a ``KVCache``, copied first).

    Step s appends token s of every batch row at position pos + 1 and computes the hybrid step
    for a query at that position.  Returns (per-step {(b, h, 0): RowResult}, final cache)."""
    c = cache.copy()
    pos = steps.start.pos[:, -1].astype(np.int64).copy()
    results = []
    for s in range(steps.Qf.shape[0]):
        pos += 1
        for b in range(pos.shape[0]):
            append_token(c, b, int(pos[b]), steps.K_new[s, b], steps.V_new[s, b])
        inp = replace(steps.start, Qf=steps.Qf[s], Qs=steps.Qs[s], pos=pos[:, None].astype(np.int32), cache=c)
        results.append(step_rows(inp))
    return results, c


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
    Hkv = inp.dims["Hkv"]
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
        Kh, Vh = cache_rows_f64(inp, b, h)
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
