"""Pins of the oracle's stored-cache readers: FP8 E4M3 codes with per-head scales, the paged
pool, and the decode loop that appends one token per step.

Each ``pin_*`` ties the oracle to something outside its own code:

* the E4M3 value of all 256 codes against PyTorch's float8_e4m3fn conversion, plus closed
  forms (smallest subnormal 2^-9, smallest normal 2^-6, 1.0, largest finite 448);
* the E4M3 rounding of float32 values (subnormals, exact ties, both signs) against PyTorch's
  round-to-nearest-even conversion, and the saturation rule by its definition;
* a step on an fp8 cache whose values, code x scale, are exactly representable in bf16 must
  equal the step on that bf16 cache (K and V have different power-of-two scales, so applying a
  scale to the wrong tensor shows);
* a paged cache built by scattering a contiguous cache over a shuffled page pool (junk in the
  unused slots) must read back token for token and give the same step;
* a run of decode steps must leave the appended tokens at positions pos+1, pos+2, ..., leave
  the older tokens untouched, and each step must equal a fresh step, at that step's position,
  on the final cache (later tokens are invisible to an earlier query: causality).
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import torch

from long_context_sparse_hs2_b200.inputs import (KVCache, bf16_bits_to_f32, bf16_cache, f32_to_bf16_bits,
                                                  fp8_e4m3_cache, make_decode_steps, make_inputs, paged_cache)
import oracle.hs2_oracle as O


def _torch_e4m3_values(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_e4m3_codes(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_e4m3_decode_table():
    codes = np.arange(256, dtype=np.uint8)
    got = O.e4m3_to_f64(codes)
    np.testing.assert_array_equal(got, _torch_e4m3_values(codes))
    closed = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
              0x7E: 448.0, 0xFE: -448.0, 0x80: -0.0, 0xB8: -1.0}
    for c, v in closed.items():
        assert O.e4m3_to_f64(np.array([c], np.uint8))[0] == v, hex(c)
    assert np.isnan(O.e4m3_to_f64(np.array([0x7F, 0xFF], np.uint8))).all()


def pin_e4m3_rounding():
    rng = np.random.default_rng(12)
    finite = _torch_e4m3_values(np.arange(256, dtype=np.uint8))
    finite = np.unique(finite[np.isfinite(finite)])
    mids = (finite[1:] + finite[:-1]) / 2  # exact ties between neighbouring codes (float32-exact)
    x = np.concatenate([
        rng.standard_normal(20000) * 40, rng.standard_normal(5000) * 0.01,  # normals, subnormals
        mids, -mids, finite, np.array([0.0, -0.0, 2.0 ** -10, 3 * 2.0 ** -11, 447.9, -447.9])]).astype(np.float32)
    np.testing.assert_array_equal(O.quantize_e4m3(x, 1.0), _torch_e4m3_codes(x))
    # a non-unit scale: the code is taken from the float32 quotient
    s = np.float32(0.0371)
    xs = x[:5000][np.abs(x[:5000] / s) <= 448]
    np.testing.assert_array_equal(O.quantize_e4m3(xs, s), _torch_e4m3_codes(xs / s))
    # saturation (by definition: finite magnitudes beyond 448 become 448) and NaN
    big = np.array([449.0, 463.9, 464.0, 1e30, np.inf, -500.0, -np.inf], np.float32)
    np.testing.assert_array_equal(O.quantize_e4m3(big, 1.0), [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE])
    assert O.quantize_e4m3(np.array([np.nan], np.float32), 1.0)[0] == 0x7F


def _exact_fp8_case(seed, paged=0):
    """An fp8 cache with power-of-two scales (2^-3 for K, 2^2 for V) and the bf16 inputs that
    hold exactly the same values."""
    inp = make_inputs(2, 4, 2, 64, 48, 3, 6, 5, seed=seed, pos=np.array([[20, 33, 47], [5, 40, 47]], np.int32))
    rng = np.random.default_rng(seed)
    B, Hkv, N, d = inp.K.shape
    codes = [rng.integers(0, 256, size=(B, Hkv, N, d)).astype(np.uint8) for _ in range(2)]
    for c in codes:  # no NaN codes
        c[(c & 0x7F) == 0x7F] = 0x3C
    ks = np.full((B, Hkv), 2.0 ** -3, np.float32)
    vs = np.full((B, Hkv), 2.0 ** 2, np.float32)
    cache = KVCache("fp8_e4m3", codes[0], codes[1], N=N, k_scale=ks, v_scale=vs)
    vals = [O.e4m3_to_f64(codes[0]) * 2.0 ** -3, O.e4m3_to_f64(codes[1]) * 2.0 ** 2]
    bits = [f32_to_bf16_bits(v.astype(np.float32)) for v in vals]
    for v, bb in zip(vals, bits):
        assert np.array_equal(O.bf16_to_f64(bb), v)  # E4M3 x 2^e is exact in bf16
    as_bf16 = replace(inp, K=bits[0], V=bits[1])
    if paged:
        cache = paged_cache(cache, paged, seed=seed)
    return replace(inp, cache=cache), as_bf16


def _same_steps(a, b):
    ra, rb = O.step_rows(a), O.step_rows(b)
    assert ra.keys() == rb.keys()
    for key in ra:
        x, y = ra[key], rb[key]
        for f in ("lse_full", "o_full", "scores", "selected", "o_sparse", "lse_sparse"):
            np.testing.assert_array_equal(getattr(x, f), getattr(y, f), err_msg=f"{key} {f}")


def pin_fp8_cache_reads_scaled_values():
    for seed in (1, 2):
        fp8, bf16 = _exact_fp8_case(seed)
        _same_steps(fp8, bf16)


def pin_paged_cache_reads_the_same_tokens():
    for seed, ps in ((3, 8), (4, 16), (5, 64)):
        inp = make_inputs(2, 4, 2, 64, 45, 2, 6, 5, seed=seed, pos=np.array([[30, 44], [9, 44]], np.int32))
        pc = paged_cache(bf16_cache(inp), ps, seed=seed)
        paged = replace(inp, cache=pc)
        for b in range(2):
            for h in range(2):
                k, v = O.cache_rows_f64(paged, b, h)
                np.testing.assert_array_equal(k, O.bf16_to_f64(inp.K[b, h]))
                np.testing.assert_array_equal(v, O.bf16_to_f64(inp.V[b, h]))
                for j in (0, min(ps - 1, 44), 44):  # token j by an explicit page lookup
                    page = pc.page_table[b, j // ps]
                    np.testing.assert_array_equal(O.bf16_to_f64(pc.K[page, h, j % ps]), k[j])
        _same_steps(paged, inp)
        fp8, bf16 = _exact_fp8_case(seed, paged=ps)
        _same_steps(fp8, bf16)


def _decode_case(dtype, paged, seed):
    start = make_inputs(2, 4, 2, 64, 60, 1, 5, 4, seed=seed, pos=np.array([[40], [17]], np.int32))
    steps = make_decode_steps(start, 4, seed=seed + 1, drift=0.2)
    if dtype == "fp8_e4m3":
        cache = fp8_e4m3_cache(start.K, start.V)
        # power-of-two scales and new tokens exactly representable as code x scale, so that the
        # codes they must be stored as are known exactly
        cache.k_scale[...] = 2.0 ** -5
        cache.v_scale[...] = 2.0 ** -4
        rng = np.random.default_rng(seed)
        for arr, sc in ((steps.K_new, cache.k_scale), (steps.V_new, cache.v_scale)):
            codes = rng.integers(0, 0x7E, size=arr.shape).astype(np.uint8)
            vals = O.e4m3_to_f64(codes) * sc[None, :, :, None]
            arr[...] = f32_to_bf16_bits(vals.astype(np.float32))
            assert np.array_equal(O.bf16_to_f64(arr), vals)
    else:
        cache = bf16_cache(start)
    if paged:
        cache = paged_cache(cache, paged, seed=seed)
    return start, steps, cache


def pin_decode_loop_appends_and_stays_causal():
    for dtype, paged in (("bf16", 0), ("fp8_e4m3", 0), ("bf16", 16), ("fp8_e4m3", 8)):
        start, steps, cache = _decode_case(dtype, paged, seed=7)
        results, final = O.decode_loop(steps, cache)
        p0 = start.pos[:, 0]
        S = steps.Qf.shape[0]
        fin = replace(start, cache=final)
        before = replace(start, cache=cache)
        for b in range(2):
            for h in range(2):
                k1, v1 = O.cache_rows_f64(fin, b, h)
                k0, v0 = O.cache_rows_f64(before, b, h)
                last = int(p0[b])
                np.testing.assert_array_equal(k1[:last + 1], k0[:last + 1])  # older tokens untouched
                np.testing.assert_array_equal(v1[:last + 1], v0[:last + 1])
                for s in range(S):  # token s sits at p0 + 1 + s, with the value it was given
                    np.testing.assert_array_equal(k1[last + 1 + s], O.bf16_to_f64(steps.K_new[s, b, h]))
                    np.testing.assert_array_equal(v1[last + 1 + s], O.bf16_to_f64(steps.V_new[s, b, h]))
                np.testing.assert_array_equal(k1[last + 1 + S:], k0[last + 1 + S:])
        for s in range(S):
            fresh = O.step_rows(replace(start, Qf=steps.Qf[s], Qs=steps.Qs[s], cache=final,
                                        pos=(p0 + 1 + s)[:, None].astype(np.int32)))
            for key, r in results[s].items():
                f = fresh[key]
                assert r.pos == int(p0[key[0]]) + 1 + s
                for fld in ("lse_full", "o_full", "selected", "o_sparse", "lse_sparse"):
                    np.testing.assert_array_equal(getattr(r, fld), getattr(f, fld), err_msg=f"step {s} {key} {fld}")


CACHE_PINS = [
    pin_e4m3_decode_table,
    pin_e4m3_rounding,
    pin_fp8_cache_reads_scaled_values,
    pin_paged_cache_reads_the_same_tokens,
    pin_decode_loop_appends_and_stays_causal,
]
