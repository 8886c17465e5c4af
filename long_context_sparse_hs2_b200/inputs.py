"""Seeded synthetic inputs for the HySparse2 hybrid sparse attention step.

This module draws the tensors one step consumes -- Q_full, Q_sparse, K, V and the
causal query positions -- and nothing else.  It holds none of the method's
arithmetic (no logits, softmax, scores or selection), so the CUDA path and the
fp64 oracle can both start from the same bytes without sharing any of the
computation they are compared on.

Recipe (stated once here, repeated in the design notes):

* draws use ``numpy.random.Generator(PCG64(seed))`` in float32, in the order
  Q_full, Q_sparse, K, V (each standard normal), then the AR(1) drift noise (only
  for workloads that have drift), then the needle positions;
* every tensor is rounded once to bfloat16 with round-to-nearest-even and kept as
  raw bf16 bit patterns (``uint16``), layout ``[B, H, T|N, d]`` row-major;
* AR(1) drift: per (b, kv head, dim) a mean ``m_n = rho*m_{n-1} + sigma*eps_n``,
  ``m_{-1} = 0``, added to K in float32 before rounding;
* needles: per (b, kv head), ``needles`` distinct positions drawn uniformly from
  ``[0, N)``; needle ``n`` adds ``3 * q_hat`` to its key row before rounding, where
  ``q_hat`` is the unit vector of the (already rounded) Q_full row of query head
  ``h*G + (n mod G)`` at the last query ``T-1``.  This raises that head's logit for
  the needle by about 3 (``|q| ~ sqrt(d)``);
* query positions are the last ``T`` positions of the cache:
  ``pos[b, t] = N - T + t``.

The named workloads are the five shapes the long-context decode and chunked
prefill benchmarks use (the 1M-token decode appears twice, at T=1 and T=16), plus
a reduced chunked-prefill shape for profiler captures.
The pages run no public benchmark for this step; these needle-in-noise inputs
stand in for long-context retrieval traffic.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np


@dataclass(frozen=True)
class Workload:
    """Shape and recipe of one synthetic workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    T: int
    k: int
    W: int
    seed: int
    needles: int = 0                              # per (b, kv head)
    drift: Optional[Tuple[float, float]] = None   # (rho, sigma) of the AR(1) mean drift on K

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, d=64, N=2048, T=1, k=64, W=64,
                     seed=0, needles=16),
    "batched": Workload("batched", B=8, Hq=32, Hkv=4, d=128, N=32768, T=1, k=2048, W=128,
                        seed=1, needles=64),
    "long": Workload("long", B=1, Hq=64, Hkv=8, d=128, N=131072, T=1, k=4096, W=512,
                     seed=2, needles=128, drift=(0.999, 0.05)),
    "prefill": Workload("prefill", B=1, Hq=32, Hkv=4, d=128, N=131072, T=4096, k=2048, W=128,
                        seed=3, needles=256),
    "1m_t1": Workload("1m_t1", B=1, Hq=32, Hkv=4, d=128, N=1048576, T=1, k=8192, W=1024,
                      seed=4, needles=512),
    "1m_t16": Workload("1m_t16", B=1, Hq=32, Hkv=4, d=128, N=1048576, T=16, k=8192, W=1024,
                       seed=4, needles=512),
    # the chunked-prefill shape at a quarter of the context and of the chunk: small enough for
    # multi-pass profiler captures of the prefill kernels (K/V 64 MiB, score keys 512 MiB)
    "prefill_32k": Workload("prefill_32k", B=1, Hq=32, Hkv=4, d=128, N=32768, T=1024, k=2048, W=128,
                            seed=3, needles=64),
}


# ----------------------------------------------------------------------------- bf16 bits

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); return the bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    flat_in = x.reshape(-1).view(np.uint32)
    flat_out = out.reshape(-1)
    step = 1 << 24
    for s in range(0, flat_in.size, step):
        u = flat_in[s:s + step].astype(np.uint32)
        lsb = (u >> np.uint32(16)) & np.uint32(1)
        u = u + np.uint32(0x7FFF) + lsb
        flat_out[s:s + step] = (u >> np.uint32(16)).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------- inputs

@dataclass
class Inputs:
    """One step's inputs as bf16 bit patterns plus the integer arguments."""

    Qf: np.ndarray          # uint16 [B, Hq, T, d]
    Qs: np.ndarray          # uint16 [B, Hq, T, d]
    K: np.ndarray           # uint16 [B, Hkv, N, d]
    V: np.ndarray           # uint16 [B, Hkv, N, d]
    pos: np.ndarray         # int32  [B, T]
    k: int
    W: int
    needle_pos: np.ndarray = field(default_factory=lambda: np.zeros((0,), np.int64))

    @property
    def dims(self):
        B, Hq, T, d = self.Qf.shape
        Hkv, N = self.K.shape[1], self.K.shape[2]
        return dict(B=B, Hq=Hq, Hkv=Hkv, T=T, N=N, d=d, k=self.k, W=self.W)


def _ar1_drift(rng: np.random.Generator, shape, rho: float, sigma: float) -> np.ndarray:
    """AR(1) walk along axis 2 of ``shape`` = (B, H, N, d): m_n = rho*m_{n-1} + sigma*eps_n."""
    from scipy.signal import lfilter

    eps = rng.standard_normal(shape, dtype=np.float32)
    m = lfilter([sigma], [1.0, -rho], eps.astype(np.float64), axis=2)
    return m.astype(np.float32)


def make_inputs(B: int, Hq: int, Hkv: int, d: int, N: int, T: int, k: int, W: int,
                seed: int, needles: int = 0,
                drift: Optional[Tuple[float, float]] = None,
                pos: Optional[np.ndarray] = None,
                q_scale: float = 1.0, k_scale: float = 1.0) -> Inputs:
    """Draw one step's inputs with the recipe in the module docstring.

    ``pos`` overrides the default ``N - T + t`` positions (shape ``[B, T]``).
    ``q_scale`` / ``k_scale`` multiply Q and K before rounding, to sharpen or
    flatten the softmax in edge-case tests.
    """
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    rng = np.random.Generator(np.random.PCG64(seed))
    qf = rng.standard_normal((B, Hq, T, d), dtype=np.float32)
    qs = rng.standard_normal((B, Hq, T, d), dtype=np.float32)
    kk = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    vv = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    if q_scale != 1.0:
        qf *= np.float32(q_scale)
        qs *= np.float32(q_scale)
    if k_scale != 1.0:
        kk *= np.float32(k_scale)
    if drift is not None:
        kk += _ar1_drift(rng, kk.shape, drift[0], drift[1])
    Qf = f32_to_bf16_bits(qf)
    Qs = f32_to_bf16_bits(qs)
    del qf, qs
    needle_pos = np.zeros((B, Hkv, needles), dtype=np.int64)
    if needles:
        qf_r = bf16_bits_to_f32(Qf)
        for b in range(B):
            for h in range(Hkv):
                p = rng.choice(N, size=needles, replace=False)
                needle_pos[b, h] = p
                for n, j in enumerate(p):
                    q = qf_r[b, h * G + (n % G), T - 1].astype(np.float64)
                    nrm = np.linalg.norm(q)
                    if nrm > 0:
                        kk[b, h, j] += (3.0 * q / nrm).astype(np.float32)
        del qf_r
    K = f32_to_bf16_bits(kk)
    del kk
    V = f32_to_bf16_bits(vv)
    del vv
    if pos is None:
        pos = np.broadcast_to(np.arange(N - T, N, dtype=np.int32), (B, T)).copy()
    else:
        pos = np.ascontiguousarray(pos, dtype=np.int32).reshape(B, T)
    return Inputs(Qf=Qf, Qs=Qs, K=K, V=V, pos=pos, k=int(k), W=int(W), needle_pos=needle_pos)


def generate(w: Workload, **overrides) -> Inputs:
    """Inputs of a named workload (``overrides`` replace fields, e.g. a smaller N)."""
    if overrides:
        w = replace(w, **overrides)
    return make_inputs(w.B, w.Hq, w.Hkv, w.d, w.N, w.T, w.k, w.W, w.seed,
                       needles=w.needles, drift=w.drift)
