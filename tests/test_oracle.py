"""The fp64 oracle against its pins, and the pins against planted oracle mistakes."""
import numpy as np
import pytest

import oracle.hs2_oracle as O
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_needles_rank_high():
    """Sanity, not a pin: keys planted with a +3 logit boost are selected far above chance."""
    from long_context_sparse_hs2_b200.inputs import WORKLOADS, generate

    inp = generate(WORKLOADS["tiny"])
    r = O.step_rows(inp)[(0, 0, 0)]
    needles = set(inp.needle_pos[0, 0].tolist()) - set(range(r.pos - inp.W + 1, r.pos + 1))
    hit = len(needles & set(r.selected.tolist())) / len(needles)
    base = inp.k / r.scores.shape[0]
    assert hit >= 0.4 and hit >= 10 * base


# Each mutant plants one plausible mistake in the oracle (on the CPU, by patching one
# helper); at least one pin must catch it.
def _m_scale(d):
    return 1.0 / d


def _m_gqa(hq, G):
    return hq % G


def _m_window(pos, W):
    return np.arange(max(0, pos - W), pos + 1, dtype=np.int64)


def _m_pool(pos, W):
    return max(0, pos - W + 2)


def _m_tie_high(s):
    j = np.arange(s.shape[0], dtype=np.int64)
    return np.lexsort((-j, -s))


def _m_lse_no_shift(q, Kh, Vh, scale):
    logits = scale * (q @ Kh.T)
    m = logits.max(axis=1, keepdims=True)
    lse = np.log(np.exp(logits - m).sum(axis=1))
    p = np.exp(logits - lse[:, None])
    return p @ Vh, lse, logits


def _m_score_min(logits, lse, pos, W):
    Pn = O.pool_size(pos, W)
    return (logits[:, :Pn] - lse[:, None]).min(axis=0)


def _m_score_raw(logits, lse, pos, W):
    Pn = O.pool_size(pos, W)
    return logits[:, :Pn].max(axis=0)


def _m_score_head0_lse(logits, lse, pos, W):
    Pn = O.pool_size(pos, W)
    return (logits[:, :Pn] - lse[0]).max(axis=0)


def _m_no_window(scores, pos, k, W):
    return O.topk_pool(scores, k)


def _m_topk_plus_one(s, k):
    return np.sort(O.rank_pool(s)[:min(k + 1, s.shape[0])])


def _m_causal_off_by_one(Qf, Kh, Vh, pos, scale):
    n = max(pos, 1)
    return O.attend(Qf, Kh[:n], Vh[:n], scale)


def _m_sparse_unrestricted(Qs, Kh, Vh, selected, scale):
    n = int(selected.max()) + 1
    out, lse, _ = O.attend(Qs, Kh[:n], Vh[:n], scale)
    return out, lse


def _m_transposed_v(q, Kh, Vh, scale):
    logits = scale * (q @ Kh.T)
    m = logits.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
    p = np.exp(logits - lse[:, None])
    return p @ Vh[::-1], lse, logits


def _m_e4m3_bias8(codes):
    return O.e4m3_to_f64(codes) / 2.0


def _m_e4m3_subnormal_as_normal(codes):
    c = np.asarray(codes).astype(np.int64)
    v = O.e4m3_to_f64(codes)
    e, m = (c >> 3) & 0xF, (c & 7).astype(np.float64)
    alt = (1.0 + m / 8.0) * 2.0 ** -7
    return np.where(e == 0, np.where(c & 0x80, -alt, alt), v)


_quantize = O.quantize_e4m3
_cache_rows = O.cache_rows_f64
_slot = O.cache_token_slot


def _m_round_half_away(x, scale):
    # the oracle's rounding with every np.rint replaced by floor(v + 1/2): ties away from zero
    real_rint = np.rint
    try:
        np.rint = lambda v: np.floor(np.asarray(v) + 0.5)
        return _quantize(x, scale)
    finally:
        np.rint = real_rint


def _m_no_saturation(x, scale):
    c = _quantize(x, scale)
    v = np.asarray(x, np.float32) / np.float32(scale)
    return np.where(np.abs(v) > 448, 0x7F, c).astype(np.uint8)


def _m_swapped_scales(inp, b, h):
    c = getattr(inp, "cache", None)
    if c is None or c.dtype != "fp8_e4m3":
        return _cache_rows(inp, b, h)
    from dataclasses import replace as _r
    return _cache_rows(_r(inp, cache=_r(c, k_scale=c.v_scale, v_scale=c.k_scale)), b, h)


def _m_slot_off_by_one(c, b, j):
    if c.page_size:
        return int(c.page_table[b, j // c.page_size]), (j + 1) % c.page_size
    return _slot(c, b, j)


def _m_append_unscaled(c, b, j, k_bits, v_bits):
    p, slot = O.cache_token_slot(c, b, j)
    for h in range(c.Hkv):
        if c.dtype == "bf16":
            c.K[p, h, slot], c.V[p, h, slot] = k_bits[h], v_bits[h]
        else:
            c.K[p, h, slot] = _quantize(O.bf16_to_f64(k_bits[h]).astype(np.float32), 1.0)
            c.V[p, h, slot] = _quantize(O.bf16_to_f64(v_bits[h]).astype(np.float32), 1.0)


def _m_decode_append_at_old_position(steps, cache):
    from dataclasses import replace as _r
    c = cache.copy()
    pos = steps.start.pos[:, -1].astype(np.int64).copy()
    results = []
    for s in range(steps.Qf.shape[0]):
        for b in range(pos.shape[0]):
            O.append_token(c, b, int(pos[b]), steps.K_new[s, b], steps.V_new[s, b])
        pos += 1
        inp = _r(steps.start, Qf=steps.Qf[s], Qs=steps.Qs[s], pos=pos[:, None].astype(np.int32), cache=c)
        results.append(O.step_rows(inp))
    return results, c


MUTANTS = [
    ("softmax_scale", _m_scale),
    ("kv_head_of", _m_gqa),
    ("window_keys", _m_window),
    ("pool_size", _m_pool),
    ("rank_pool", _m_tie_high),
    ("attend", _m_lse_no_shift),
    ("attend", _m_transposed_v),
    ("selection_scores_row", _m_score_min),
    ("selection_scores_row", _m_score_raw),
    ("selection_scores_row", _m_score_head0_lse),
    ("select_row", _m_no_window),
    ("topk_pool", _m_topk_plus_one),
    ("full_attention_row", _m_causal_off_by_one),
    ("sparse_attention_row", _m_sparse_unrestricted),
    ("e4m3_to_f64", _m_e4m3_bias8),
    ("e4m3_to_f64", _m_e4m3_subnormal_as_normal),
    ("quantize_e4m3", _m_round_half_away),
    ("quantize_e4m3", _m_no_saturation),
    ("cache_rows_f64", _m_swapped_scales),
    ("cache_token_slot", _m_slot_off_by_one),
    ("append_token", _m_append_unscaled),
    ("decode_loop", _m_decode_append_at_old_position),
]


@pytest.mark.parametrize("name,mutant", MUTANTS, ids=[f"{n}:{m.__name__}" for n, m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, name, mutant):
    monkeypatch.setattr(O, name, mutant)
    tripped = []
    for pin in P.ALL_PINS:
        try:
            pin()
        except Exception:  # an assertion or a crash both count as caught
            tripped.append(pin.__name__)
    assert tripped, f"no pin caught the mutant {mutant.__name__} of {name}"
