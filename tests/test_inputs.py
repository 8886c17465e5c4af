"""The seeded input generator: bf16 rounding, determinism and the recipe's structure."""
import numpy as np
import torch

from long_context_sparse_hs2_b200.inputs import (WORKLOADS, bf16_bits_to_f32, f32_to_bf16_bits,
                                                  generate, make_inputs)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10 ** rng.uniform(-3, 3, 100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(f32_to_bf16_bits(x), want)
    np.testing.assert_array_equal(bf16_bits_to_f32(want), torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_deterministic_and_shapes():
    a = generate(WORKLOADS["tiny"])
    b = generate(WORKLOADS["tiny"])
    for f in ("Qf", "Qs", "K", "V", "pos", "needle_pos"):
        np.testing.assert_array_equal(getattr(a, f), getattr(b, f))
    w = WORKLOADS["tiny"]
    assert a.Qf.shape == (w.B, w.Hq, w.T, w.d) and a.K.shape == (w.B, w.Hkv, w.N, w.d)
    assert a.pos.tolist() == [[w.N - 1]]
    assert a.needle_pos.shape == (1, 1, 16) and len(set(a.needle_pos[0, 0].tolist())) == 16


def test_needles_raise_their_heads_logit():
    inp = make_inputs(1, 4, 1, 64, 512, 1, 8, 8, seed=3, needles=8)
    q = bf16_bits_to_f32(inp.Qf[0, :, 0]).astype(np.float64)
    K = bf16_bits_to_f32(inp.K[0, 0]).astype(np.float64)
    base = make_inputs(1, 4, 1, 64, 512, 1, 8, 8, seed=3, needles=0)
    K0 = bf16_bits_to_f32(base.K[0, 0]).astype(np.float64)
    for n, j in enumerate(inp.needle_pos[0, 0]):
        g = n % 4
        boost = (q[g] @ (K[j] - K0[j])) / np.linalg.norm(q[g])
        assert abs(boost - 3.0) < 0.1


def test_prefill_positions_are_the_last_T():
    inp = make_inputs(1, 2, 1, 64, 64, 8, 4, 4, seed=0)
    assert inp.pos.tolist() == [list(range(56, 64))]
