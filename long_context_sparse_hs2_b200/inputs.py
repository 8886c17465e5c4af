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
class KVCache:
    """The shared KV cache as it is stored, when it is not plain contiguous bf16.

    dtype "bf16": K/V hold bfloat16 bit patterns (uint16).  dtype "fp8_e4m3": K/V hold FP8
    E4M3 codes (uint8) and a token's value is code * scale, with one fp32 scale per
    (b, kv head) for K and one for V.  Contiguous layout: K/V are [B, Hkv, N, d].  Paged
    layout (page_size > 0): K/V are a pool [num_pages, Hkv, page_size, d] and token j of
    batch row b sits in page page_table[b, j // page_size] at slot j % page_size.
    """

    dtype: str
    K: np.ndarray
    V: np.ndarray
    N: int
    k_scale: Optional[np.ndarray] = None    # float32 [B, Hkv] (fp8 only)
    v_scale: Optional[np.ndarray] = None
    page_size: int = 0
    page_table: Optional[np.ndarray] = None  # int32 [B, max_pages] (paged only)

    @property
    def Hkv(self) -> int:
        return self.K.shape[1]

    def copy(self) -> "KVCache":
        c = lambda a: None if a is None else a.copy()  # noqa: E731
        return replace(self, K=self.K.copy(), V=self.V.copy(), k_scale=c(self.k_scale), v_scale=c(self.v_scale),
                       page_table=c(self.page_table))


@dataclass
class Inputs:
    """One step's inputs as bf16 bit patterns plus the integer arguments.

    ``cache`` replaces K/V when the cache is stored in another format or layout (then K and V
    keep the bf16 draw it was made from, for reference only)."""

    Qf: np.ndarray          # uint16 [B, Hq, T, d]
    Qs: np.ndarray          # uint16 [B, Hq, T, d]
    K: np.ndarray           # uint16 [B, Hkv, N, d]
    V: np.ndarray           # uint16 [B, Hkv, N, d]
    pos: np.ndarray         # int32  [B, T]
    k: int
    W: int
    needle_pos: np.ndarray = field(default_factory=lambda: np.zeros((0,), np.int64))
    cache: Optional[KVCache] = None

    @property
    def dims(self):
        B, Hq, T, d = self.Qf.shape
        if self.cache is not None:
            Hkv, N = self.cache.Hkv, self.cache.N
        else:
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


# ----------------------------------------------------------------------------- cache formats

FP8_E4M3_MAX = 448.0


def fp8_e4m3_cache(K_bits: np.ndarray, V_bits: np.ndarray) -> KVCache:
    """FP8 E4M3 image of a bf16 cache [B, Hkv, N, d] with one amax scale per (b, kv head).

    scale = max|x| / 448 in float32, code = the float32 quotient x / scale rounded to E4M3
    (nearest, ties to even; PyTorch's float8_e4m3fn conversion).  This is how the synthetic
    fp8 workloads are stored; it is data preparation, done once per workload."""
    import torch

    B, Hkv = K_bits.shape[:2]
    out = []
    for bits in (K_bits, V_bits):
        codes = np.empty(bits.shape, np.uint8)
        scale = np.empty((B, Hkv), np.float32)
        for b in range(B):
            for h in range(Hkv):
                x = bf16_bits_to_f32(bits[b, h])
                amax = np.float32(np.abs(x).max())
                sc = np.float32(amax / np.float32(FP8_E4M3_MAX)) if amax > 0 else np.float32(1.0)
                q = np.clip(x / sc, -FP8_E4M3_MAX, FP8_E4M3_MAX).astype(np.float32)
                codes[b, h] = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                scale[b, h] = sc
        out.append((codes, scale))
    (K8, ks), (V8, vs) = out
    return KVCache("fp8_e4m3", K8, V8, N=K_bits.shape[2], k_scale=ks, v_scale=vs)


def bf16_cache(inp: Inputs) -> KVCache:
    """The inputs' own contiguous bf16 cache as a KVCache."""
    return KVCache("bf16", inp.K, inp.V, N=inp.K.shape[2])


def paged_cache(c: KVCache, page_size: int, seed: int, spare_pages: int = 3) -> KVCache:
    """The same cache in a paged pool [num_pages, Hkv, page_size, d] with a shuffled page table.

    Every batch row owns ceil(N / page_size) pages; the pool also holds ``spare_pages`` pages no
    row uses, and the physical order of all pages is a seeded random permutation.  Slots past N
    in a row's last page and the spare pages are filled with junk (all bytes 0x7F: NaN in both
    bf16 and E4M3), so a read of anything but the mapped tokens shows in the results."""
    if c.page_size:
        raise ValueError("already paged")
    B, Hkv, N, d = c.K.shape
    per = -(-N // page_size)
    num = B * per + spare_pages
    rng = np.random.Generator(np.random.PCG64(seed))
    perm = rng.permutation(num).astype(np.int32)
    table = perm[:B * per].reshape(B, per).copy()
    pools = []
    for x in (c.K, c.V):
        pool = np.full((num, Hkv, page_size, d), 0x7F, dtype=x.dtype)
        if x.dtype == np.uint16:
            pool[...] = 0x7F7F
        for b in range(B):
            for i in range(per):
                j0, j1 = i * page_size, min(N, (i + 1) * page_size)
                pool[table[b, i], :, :j1 - j0] = x[b, :, j0:j1]
        pools.append(pool)
    return replace(c, K=pools[0], V=pools[1], page_size=page_size, page_table=table)


@dataclass
class DecodeSteps:
    """Inputs of a run of consecutive decode steps: each step appends one token per batch row
    to the cache and then runs the hybrid step for that token as the query (T = 1).

    ``start`` is the cache before the first step (``start.pos[b, 0]`` = the newest token already
    cached); step s brings Q_full/Q_sparse [B, Hq, 1, d] and the new token's K/V [B, Hkv, d]."""

    start: Inputs
    Qf: np.ndarray      # uint16 [S, B, Hq, 1, d]
    Qs: np.ndarray      # uint16 [S, B, Hq, 1, d]
    K_new: np.ndarray   # uint16 [S, B, Hkv, d]
    V_new: np.ndarray   # uint16 [S, B, Hkv, d]


def make_decode_steps(start: Inputs, steps: int, seed: int, drift: float = 0.0) -> DecodeSteps:
    """Draw ``steps`` decode steps after ``start``: new tokens' K/V ~ N(0,1); each query is the
    previous query plus ``drift``-scaled N(0,1) noise (0: independent N(0,1) queries), the
    first one continuing from the start's last query."""
    rng = np.random.Generator(np.random.PCG64(seed))
    B, Hq, T, d = start.Qf.shape
    Hkv = start.dims["Hkv"]
    qf, qs = bf16_bits_to_f32(start.Qf[:, :, -1:]), bf16_bits_to_f32(start.Qs[:, :, -1:])
    Qf, Qs = [], []
    for _ in range(steps):
        nf = rng.standard_normal(qf.shape, dtype=np.float32)
        ns = rng.standard_normal(qs.shape, dtype=np.float32)
        if drift > 0:
            qf = (qf + np.float32(drift) * nf) / np.float32(np.sqrt(1 + drift * drift))
            qs = (qs + np.float32(drift) * ns) / np.float32(np.sqrt(1 + drift * drift))
        else:
            qf, qs = nf, ns
        Qf.append(f32_to_bf16_bits(qf))
        Qs.append(f32_to_bf16_bits(qs))
    K_new = f32_to_bf16_bits(rng.standard_normal((steps, B, Hkv, d), dtype=np.float32))
    V_new = f32_to_bf16_bits(rng.standard_normal((steps, B, Hkv, d), dtype=np.float32))
    return DecodeSteps(start=start, Qf=np.stack(Qf), Qs=np.stack(Qs), K_new=K_new, V_new=V_new)
