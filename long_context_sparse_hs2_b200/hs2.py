"""Thin Python binding of ``libhs2.so`` (the C ABI declared in ``include/hs2.h``).

Argument marshalling only: it checks tensor dtypes, shapes, devices and contiguity,
allocates outputs and the workspace with PyTorch (device memory is PyTorch's job
here), and passes raw pointers and the current CUDA stream to the library.  Every
step of the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and a missing library is an error.

Names mirror the C entry points: ``full_attn``, ``select``, ``sparse_attn``,
``step``, ``workspace_size``, ``read_device_status``, ``status_string``, and for a cache
described by a ``KVCache`` (bf16 or FP8 E4M3, contiguous or paged) ``full_attn_kv``,
``select_kv``, ``sparse_attn_kv``, ``step_kv``, ``workspace_size_kv``, ``kv_append`` and
``decode_step``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

HS2_OK, HS2_ERR_INVALID_ARG, HS2_ERR_UNSUPPORTED, HS2_ERR_WORKSPACE, HS2_ERR_CUDA, HS2_ERR_DEVICE = range(6)
DEV_BAD_POS, DEV_BAD_INDEX, DEV_NONFINITE, DEV_TIMEOUT, DEV_CAND_OVERFLOW = 0x1, 0x2, 0x4, 0x8, 0x10

DEV_BAD_PAGE = 0x20
KV_BF16, KV_FP8_E4M3 = 0, 1

ENTRY_POINTS = ("hs2_workspace_size", "hs2_full_attn", "hs2_select", "hs2_sparse_attn", "hs2_step",
                "hs2_read_device_status", "hs2_status_string", "hs2_trace_enable", "hs2_trace_collect",
                "hs2_launch_count", "hs2_version", "hs2_sparse_attn_static", "hs2_workspace_size_kv",
                "hs2_full_attn_kv", "hs2_select_kv", "hs2_sparse_attn_kv", "hs2_step_kv", "hs2_kv_append",
                "hs2_decode_step", "hs2_selftest_wait_bound")
STATIC_SCRATCH_BYTES = 4 << 20  # HS2_STATIC_SCRATCH_BYTES


class Dims(ctypes.Structure):
    """``hs2_dims``: problem shape (the attention scale is fixed to d^-1/2)."""

    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "T", "N", "d", "k", "W")]

    def as_tuple(self):
        return tuple(getattr(self, n) for n, _ in self._fields_)


class KvCacheDesc(ctypes.Structure):
    """``hs2_kv_cache``: storage format and layout of the shared KV cache."""

    _fields_ = [("dtype", ctypes.c_int32), ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("K", ctypes.c_void_p), ("V", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p)]


class HS2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libhs2.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m long_context_sparse_hs2_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32p, f32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
    dp = ctypes.POINTER(Dims)
    L.hs2_workspace_size.argtypes = [dp]
    L.hs2_workspace_size.restype = sz
    L.hs2_full_attn.argtypes = [dp, vp, vp, vp, i32p, vp, f32p, vp, sz, vp]
    L.hs2_select.argtypes = [dp, vp, vp, f32p, i32p, i32p, i32p, vp, sz, vp]
    L.hs2_sparse_attn.argtypes = [dp, vp, vp, vp, i32p, i32p, i32p, vp, f32p, vp, sz, vp]
    L.hs2_step.argtypes = [dp, vp, vp, vp, vp, i32p, vp, vp, f32p, f32p, i32p, i32p, vp, sz, vp]
    L.hs2_sparse_attn_static.argtypes = [dp, vp, vp, vp, i32p, i32p, i32p, vp, f32p, vp]
    L.hs2_sparse_attn_static.restype = ctypes.c_int
    cp = ctypes.POINTER(KvCacheDesc)
    L.hs2_workspace_size_kv.argtypes = [dp, cp]
    L.hs2_workspace_size_kv.restype = sz
    L.hs2_full_attn_kv.argtypes = [dp, vp, cp, i32p, vp, f32p, vp, sz, vp]
    L.hs2_select_kv.argtypes = [dp, vp, cp, f32p, i32p, i32p, i32p, vp, sz, vp]
    L.hs2_sparse_attn_kv.argtypes = [dp, vp, cp, i32p, i32p, i32p, vp, f32p, vp, sz, vp]
    L.hs2_step_kv.argtypes = [dp, vp, vp, cp, i32p, vp, vp, f32p, f32p, i32p, i32p, vp, sz, vp]
    L.hs2_kv_append.argtypes = [dp, cp, vp, vp, i32p, vp, sz, vp]
    L.hs2_decode_step.argtypes = [dp, cp, vp, vp, vp, vp, i32p, vp, vp, f32p, f32p, i32p, i32p, vp, sz, vp]
    for f in ("hs2_full_attn_kv", "hs2_select_kv", "hs2_sparse_attn_kv", "hs2_step_kv", "hs2_kv_append",
              "hs2_decode_step"):
        getattr(L, f).restype = ctypes.c_int
    L.hs2_selftest_wait_bound.argtypes = [vp, sz, ctypes.c_uint64, vp]
    L.hs2_selftest_wait_bound.restype = ctypes.c_int
    L.hs2_read_device_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    L.hs2_status_string.argtypes = [ctypes.c_int]
    L.hs2_status_string.restype = ctypes.c_char_p
    L.hs2_version.restype = ctypes.c_uint32
    L.hs2_trace_enable.argtypes = [ctypes.c_int]
    L.hs2_trace_enable.restype = ctypes.c_int
    L.hs2_trace_collect.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_int64), ctypes.c_int]
    L.hs2_trace_collect.restype = ctypes.c_int
    L.hs2_launch_count.restype = ctypes.c_uint64
    for f in ("hs2_full_attn", "hs2_select", "hs2_sparse_attn", "hs2_step", "hs2_read_device_status"):
        getattr(L, f).restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().hs2_status_string(int(status)).decode()


def make_dims(B, Hq, Hkv, T, N, d, k, W) -> Dims:
    return Dims(int(B), int(Hq), int(Hkv), int(T), int(N), int(d), int(k), int(W))


def workspace_size(dims: Dims) -> int:
    """Bytes of workspace the entry points need for ``dims`` (0 if unsupported)."""
    return int(lib().hs2_workspace_size(ctypes.byref(dims)))


def alloc_workspace(dims: Dims, device) -> torch.Tensor:
    n = workspace_size(dims)
    if n == 0:
        raise HS2Error(HS2_ERR_UNSUPPORTED, "workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream, device) -> Optional[int]:
    """Raw handle of ``stream`` (default: the current stream of ``device``).  A torch stream must
    belong to ``device``: the library launches on whatever device is current, so a stream of
    another GPU would run the kernels there."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if hasattr(stream, "cuda_stream"):
        if getattr(stream, "device", device) != device:
            raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
        return stream.cuda_stream
    return int(stream)


def device_of(where: str, **tensors) -> torch.device:
    """The one CUDA device every given tensor lives on (``None`` entries are skipped).

    The kernels run on the current device and dereference every pointer there, so tensors on
    two GPUs would read the wrong memory or fault: this raises before anything is launched."""
    devs = {name: t.device for name, t in tensors.items() if t is not None}
    if len(set(devs.values())) != 1:
        listing = ", ".join(f"{n} on {d}" for n, d in devs.items())
        raise ValueError(f"{where}: every tensor must be on one CUDA device ({listing})")
    return next(iter(devs.values()))


def _need(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def dims_of(Q: torch.Tensor, K: torch.Tensor, k: int, W: int) -> Dims:
    B, Hq, T, d = Q.shape
    Hkv, N = K.shape[1], K.shape[2]
    return make_dims(B, Hq, Hkv, T, N, d, k, W)


def _ws(dims: Dims, ws: Optional[torch.Tensor], device) -> torch.Tensor:
    if ws is None:
        return alloc_workspace(dims, device)
    return ws


def _check(status: int, where: str):
    if status != HS2_OK:
        raise HS2Error(status, where)


def full_attn(Q_full, K, V, pos, *, k: int = 0, W: int = 0, O_full=None, LSE_full=None, ws=None, stream=None):
    """Full-attention layer: returns (O_full bf16 [B,Hq,T,d], LSE_full fp32 [B,Hq,T])."""
    dm = dims_of(Q_full, K, k, W)
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_full, "Q_full", torch.bfloat16, (B, Hq, T, d))
    _need(K, "K", torch.bfloat16, (B, Hkv, N, d))
    _need(V, "V", torch.bfloat16, (B, Hkv, N, d))
    _need(pos, "pos", torch.int32, (B, T))
    dev = device_of("full_attn", Q_full=Q_full, K=K, V=V, pos=pos, O_full=O_full, LSE_full=LSE_full, ws=ws)
    with torch.cuda.device(dev):
        O_full = torch.empty_like(Q_full) if O_full is None else O_full
        LSE_full = torch.empty((B, Hq, T), dtype=torch.float32, device=dev) if LSE_full is None else LSE_full
        ws = _ws(dm, ws, dev)
        _check(lib().hs2_full_attn(ctypes.byref(dm), _p(Q_full), _p(K), _p(V), _p(pos), _p(O_full), _p(LSE_full),
                                   _p(ws), ws.numel(), _stream(stream, dev)), "hs2_full_attn")
    return O_full, LSE_full


def select(Q_full, K, LSE_full, pos, *, k: int, W: int, idx=None, cnt=None, ws=None, stream=None):
    """Token-level top-k + forced window: returns (idx int32 [B,Hkv,T,k+W], cnt int32 [B,Hkv,T])."""
    dm = dims_of(Q_full, K, k, W)
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_full, "Q_full", torch.bfloat16, (B, Hq, T, d))
    _need(K, "K", torch.bfloat16, (B, Hkv, N, d))
    _need(LSE_full, "LSE_full", torch.float32, (B, Hq, T))
    _need(pos, "pos", torch.int32, (B, T))
    dev = device_of("select", Q_full=Q_full, K=K, LSE_full=LSE_full, pos=pos, idx=idx, cnt=cnt, ws=ws)
    with torch.cuda.device(dev):
        idx = torch.empty((B, Hkv, T, k + W), dtype=torch.int32, device=dev) if idx is None else idx
        cnt = torch.empty((B, Hkv, T), dtype=torch.int32, device=dev) if cnt is None else cnt
        ws = _ws(dm, ws, dev)
        _check(lib().hs2_select(ctypes.byref(dm), _p(Q_full), _p(K), _p(LSE_full), _p(pos), _p(idx), _p(cnt),
                                _p(ws), ws.numel(), _stream(stream, dev)), "hs2_select")
    return idx, cnt


def _sparse_checks(where, Q_sparse, K, V, pos, idx, cnt, k, W, O_sparse, LSE_sparse, ws=None):
    dm = dims_of(Q_sparse, K, k, W)
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_sparse, "Q_sparse", torch.bfloat16, (B, Hq, T, d))
    _need(K, "K", torch.bfloat16, (B, Hkv, N, d))
    _need(V, "V", torch.bfloat16, (B, Hkv, N, d))
    _need(pos, "pos", torch.int32, (B, T))
    _need(idx, "idx", torch.int32, (B, Hkv, T, k + W))
    _need(cnt, "cnt", torch.int32, (B, Hkv, T))
    dev = device_of(where, Q_sparse=Q_sparse, K=K, V=V, pos=pos, idx=idx, cnt=cnt, O_sparse=O_sparse,
                    LSE_sparse=LSE_sparse, ws=ws)
    return dm, dev


def sparse_attn(Q_sparse, K, V, pos, idx, cnt, *, k: int, W: int, O_sparse=None, LSE_sparse=None, ws=None,
                stream=None):
    """Sparse layer with KV Reuse over idx/cnt: returns (O_sparse bf16, LSE_sparse fp32)."""
    dm, dev = _sparse_checks("sparse_attn", Q_sparse, K, V, pos, idx, cnt, k, W, O_sparse, LSE_sparse, ws)
    B, Hq, _, T = dm.B, dm.Hq, dm.Hkv, dm.T
    with torch.cuda.device(dev):
        O_sparse = torch.empty_like(Q_sparse) if O_sparse is None else O_sparse
        LSE_sparse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev) if LSE_sparse is None else LSE_sparse
        ws = _ws(dm, ws, dev)
        _check(lib().hs2_sparse_attn(ctypes.byref(dm), _p(Q_sparse), _p(K), _p(V), _p(pos), _p(idx), _p(cnt),
                                     _p(O_sparse), _p(LSE_sparse), _p(ws), ws.numel(), _stream(stream, dev)),
               "hs2_sparse_attn")
    return O_sparse, LSE_sparse


def sparse_attn_static(Q_sparse, K, V, pos, idx, cnt, *, k: int, W: int, O_sparse=None, LSE_sparse=None,
                       stream=None):
    """hs2_sparse_attn_static: the sparse layer with its scratch in the library's fixed device
    array (no workspace).  The outputs are allocated here only if the caller passes none."""
    dm, dev = _sparse_checks("sparse_attn_static", Q_sparse, K, V, pos, idx, cnt, k, W, O_sparse, LSE_sparse)
    B, Hq, T = dm.B, dm.Hq, dm.T
    with torch.cuda.device(dev):
        O_sparse = torch.empty_like(Q_sparse) if O_sparse is None else O_sparse
        LSE_sparse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev) if LSE_sparse is None else LSE_sparse
        _check(lib().hs2_sparse_attn_static(ctypes.byref(dm), _p(Q_sparse), _p(K), _p(V), _p(pos), _p(idx),
                                            _p(cnt), _p(O_sparse), _p(LSE_sparse), _stream(stream, dev)),
               "hs2_sparse_attn_static")
    return O_sparse, LSE_sparse


@dataclass
class StepOutputs:
    O_full: torch.Tensor
    O_sparse: torch.Tensor
    LSE_full: torch.Tensor
    LSE_sparse: torch.Tensor
    idx: torch.Tensor
    cnt: torch.Tensor

    def as_dict(self) -> Dict[str, torch.Tensor]:
        return dict(O_full=self.O_full, O_sparse=self.O_sparse, LSE_full=self.LSE_full,
                    LSE_sparse=self.LSE_sparse, idx=self.idx, cnt=self.cnt)


def alloc_step_outputs(dims: Dims, device) -> StepOutputs:
    B, Hq, Hkv, T, N, d, k, W = dims.as_tuple()
    return StepOutputs(
        O_full=torch.empty((B, Hq, T, d), dtype=torch.bfloat16, device=device),
        O_sparse=torch.empty((B, Hq, T, d), dtype=torch.bfloat16, device=device),
        LSE_full=torch.empty((B, Hq, T), dtype=torch.float32, device=device),
        LSE_sparse=torch.empty((B, Hq, T), dtype=torch.float32, device=device),
        idx=torch.empty((B, Hkv, T, k + W), dtype=torch.int32, device=device),
        cnt=torch.empty((B, Hkv, T), dtype=torch.int32, device=device))


def step(Q_full, Q_sparse, K, V, pos, *, k: int, W: int, out: Optional[StepOutputs] = None, ws=None,
         stream=None) -> StepOutputs:
    """The whole hybrid step (full attention -> selection -> sparse attention) on one stream."""
    dm = dims_of(Q_full, K, k, W)
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_full, "Q_full", torch.bfloat16, (B, Hq, T, d))
    _need(Q_sparse, "Q_sparse", torch.bfloat16, (B, Hq, T, d))
    _need(K, "K", torch.bfloat16, (B, Hkv, N, d))
    _need(V, "V", torch.bfloat16, (B, Hkv, N, d))
    _need(pos, "pos", torch.int32, (B, T))
    outs = out.as_dict() if out is not None else {}
    dev = device_of("step", Q_full=Q_full, Q_sparse=Q_sparse, K=K, V=V, pos=pos, ws=ws, **outs)
    with torch.cuda.device(dev):
        out = alloc_step_outputs(dm, dev) if out is None else out
        ws = _ws(dm, ws, dev)
        _check(lib().hs2_step(ctypes.byref(dm), _p(Q_full), _p(Q_sparse), _p(K), _p(V), _p(pos), _p(out.O_full),
                              _p(out.O_sparse), _p(out.LSE_full), _p(out.LSE_sparse), _p(out.idx), _p(out.cnt),
                              _p(ws), ws.numel(), _stream(stream, dev)), "hs2_step")
    return out


# ----------------------------------------------------------------------------- cache descriptors

@dataclass
class KVCache:
    """The shared KV cache as stored (``hs2_kv_cache``).

    dtype "bf16": K/V are bfloat16 tensors.  dtype "fp8_e4m3": K/V hold E4M3 codes (uint8 or
    torch.float8_e4m3fn) and k_scale/v_scale (float32 [B, Hkv]) turn them into values.
    page_size = 0: K/V are [B, Hkv, N, d].  page_size > 0: K/V are pools
    [num_pages, Hkv, page_size, d] and page_table (int32 [B, max_pages]) maps token j of row b
    to page page_table[b, j // page_size].  N is the number of token positions per row."""

    K: torch.Tensor
    V: torch.Tensor
    N: int
    dtype: str = "bf16"
    k_scale: Optional[torch.Tensor] = None
    v_scale: Optional[torch.Tensor] = None
    page_size: int = 0
    page_table: Optional[torch.Tensor] = None

    @property
    def Hkv(self) -> int:
        return int(self.K.shape[1])

    def tensors(self) -> Dict[str, torch.Tensor]:
        out = dict(K=self.K, V=self.V, k_scale=self.k_scale, v_scale=self.v_scale, page_table=self.page_table)
        return {k: v for k, v in out.items() if v is not None}

    def check(self, B: int, d: int) -> None:
        if self.dtype not in ("bf16", "fp8_e4m3"):
            raise ValueError(f"unknown cache dtype {self.dtype}")
        fp8 = self.dtype == "fp8_e4m3"
        allowed = (torch.uint8, torch.float8_e4m3fn) if fp8 else (torch.bfloat16,)
        Hkv = self.Hkv
        if self.page_size:
            npg = int(self.K.shape[0])
            shape = (npg, Hkv, self.page_size, d)
            if self.page_table is None:
                raise ValueError("a paged cache needs page_table")
            _need(self.page_table, "page_table", torch.int32, (B, int(self.page_table.shape[1])))
        else:
            shape = (B, Hkv, self.N, d)
        for name in ("K", "V"):
            t = getattr(self, name)
            if t.dtype not in allowed:
                raise TypeError(f"{name} must be one of {allowed} for a {self.dtype} cache, got {t.dtype}")
            _need(t, name, t.dtype, shape)
        if fp8:
            for name in ("k_scale", "v_scale"):
                t = getattr(self, name)
                if t is None:
                    raise ValueError(f"an fp8 cache needs {name}")
                _need(t, name, torch.float32, (B, Hkv))

    def desc(self) -> KvCacheDesc:
        return KvCacheDesc(dtype=KV_FP8_E4M3 if self.dtype == "fp8_e4m3" else KV_BF16,
                           page_size=int(self.page_size),
                           num_pages=int(self.K.shape[0]) if self.page_size else 0,
                           max_pages=int(self.page_table.shape[1]) if self.page_size else 0,
                           K=_p(self.K), V=_p(self.V), page_table=_p(self.page_table), k_scale=_p(self.k_scale),
                           v_scale=_p(self.v_scale))


def dims_kv(Q: torch.Tensor, cache: KVCache, k: int, W: int) -> Dims:
    B, Hq, T, d = Q.shape
    return make_dims(B, Hq, cache.Hkv, T, cache.N, d, k, W)


def workspace_size_kv(dims: Dims, cache: KVCache) -> int:
    """Bytes of workspace the cache-descriptor entry points need (0 if unsupported)."""
    desc = cache.desc()
    return int(lib().hs2_workspace_size_kv(ctypes.byref(dims), ctypes.byref(desc)))


def alloc_workspace_kv(dims: Dims, cache: KVCache, device) -> torch.Tensor:
    n = workspace_size_kv(dims, cache)
    if n == 0:
        raise HS2Error(HS2_ERR_UNSUPPORTED, "workspace_size_kv")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _kv_call(where, Q, cache, k, W, ws, extra):
    """Shape/device checks shared by the cache-descriptor calls; returns (dims, desc, device)."""
    dm = dims_kv(Q, cache, k, W)
    cache.check(dm.B, dm.d)
    dev = device_of(where, Q=Q, ws=ws, **cache.tensors(), **{n: t for n, t in extra.items() if t is not None})
    return dm, cache.desc(), dev


def full_attn_kv(Q_full, cache: KVCache, pos, *, k: int = 0, W: int = 0, O_full=None, LSE_full=None, ws=None,
                 stream=None):
    """hs2_full_attn_kv: the full-attention layer over a cache descriptor."""
    dm, desc, dev = _kv_call("full_attn_kv", Q_full, cache, k, W, ws, dict(pos=pos, O_full=O_full, LSE_full=LSE_full))
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_full, "Q_full", torch.bfloat16, (B, Hq, T, d))
    _need(pos, "pos", torch.int32, (B, T))
    with torch.cuda.device(dev):
        O_full = torch.empty_like(Q_full) if O_full is None else O_full
        LSE_full = torch.empty((B, Hq, T), dtype=torch.float32, device=dev) if LSE_full is None else LSE_full
        ws = alloc_workspace_kv(dm, cache, dev) if ws is None else ws
        _check(lib().hs2_full_attn_kv(ctypes.byref(dm), _p(Q_full), ctypes.byref(desc), _p(pos), _p(O_full),
                                      _p(LSE_full), _p(ws), ws.numel(), _stream(stream, dev)), "hs2_full_attn_kv")
    return O_full, LSE_full


def select_kv(Q_full, cache: KVCache, LSE_full, pos, *, k: int, W: int, idx=None, cnt=None, ws=None, stream=None):
    """hs2_select_kv: top-k + window over a cache descriptor."""
    dm, desc, dev = _kv_call("select_kv", Q_full, cache, k, W, ws, dict(LSE_full=LSE_full, pos=pos, idx=idx, cnt=cnt))
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_full, "Q_full", torch.bfloat16, (B, Hq, T, d))
    _need(LSE_full, "LSE_full", torch.float32, (B, Hq, T))
    _need(pos, "pos", torch.int32, (B, T))
    with torch.cuda.device(dev):
        idx = torch.empty((B, Hkv, T, k + W), dtype=torch.int32, device=dev) if idx is None else idx
        cnt = torch.empty((B, Hkv, T), dtype=torch.int32, device=dev) if cnt is None else cnt
        ws = alloc_workspace_kv(dm, cache, dev) if ws is None else ws
        _check(lib().hs2_select_kv(ctypes.byref(dm), _p(Q_full), ctypes.byref(desc), _p(LSE_full), _p(pos), _p(idx),
                                   _p(cnt), _p(ws), ws.numel(), _stream(stream, dev)), "hs2_select_kv")
    return idx, cnt


def sparse_attn_kv(Q_sparse, cache: KVCache, pos, idx, cnt, *, k: int, W: int, O_sparse=None, LSE_sparse=None,
                   ws=None, stream=None):
    """hs2_sparse_attn_kv: the sparse layer (KV Reuse over idx/cnt) over a cache descriptor."""
    dm, desc, dev = _kv_call("sparse_attn_kv", Q_sparse, cache, k, W, ws,
                             dict(pos=pos, idx=idx, cnt=cnt, O_sparse=O_sparse, LSE_sparse=LSE_sparse))
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_sparse, "Q_sparse", torch.bfloat16, (B, Hq, T, d))
    _need(pos, "pos", torch.int32, (B, T))
    _need(idx, "idx", torch.int32, (B, Hkv, T, k + W))
    _need(cnt, "cnt", torch.int32, (B, Hkv, T))
    with torch.cuda.device(dev):
        O_sparse = torch.empty_like(Q_sparse) if O_sparse is None else O_sparse
        LSE_sparse = torch.empty((B, Hq, T), dtype=torch.float32, device=dev) if LSE_sparse is None else LSE_sparse
        ws = alloc_workspace_kv(dm, cache, dev) if ws is None else ws
        _check(lib().hs2_sparse_attn_kv(ctypes.byref(dm), _p(Q_sparse), ctypes.byref(desc), _p(pos), _p(idx),
                                        _p(cnt), _p(O_sparse), _p(LSE_sparse), _p(ws), ws.numel(),
                                        _stream(stream, dev)), "hs2_sparse_attn_kv")
    return O_sparse, LSE_sparse


def step_kv(Q_full, Q_sparse, cache: KVCache, pos, *, k: int, W: int, out: Optional["StepOutputs"] = None, ws=None,
            stream=None) -> "StepOutputs":
    """hs2_step_kv: the whole hybrid step over a cache descriptor."""
    outs = out.as_dict() if out is not None else {}
    dm, desc, dev = _kv_call("step_kv", Q_full, cache, k, W, ws, dict(Q_sparse=Q_sparse, pos=pos, **outs))
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    _need(Q_full, "Q_full", torch.bfloat16, (B, Hq, T, d))
    _need(Q_sparse, "Q_sparse", torch.bfloat16, (B, Hq, T, d))
    _need(pos, "pos", torch.int32, (B, T))
    with torch.cuda.device(dev):
        out = alloc_step_outputs(dm, dev) if out is None else out
        ws = alloc_workspace_kv(dm, cache, dev) if ws is None else ws
        _check(lib().hs2_step_kv(ctypes.byref(dm), _p(Q_full), _p(Q_sparse), ctypes.byref(desc), _p(pos),
                                 _p(out.O_full), _p(out.O_sparse), _p(out.LSE_full), _p(out.LSE_sparse), _p(out.idx),
                                 _p(out.cnt), _p(ws), ws.numel(), _stream(stream, dev)), "hs2_step_kv")
    return out


def kv_append(cache: KVCache, K_new, V_new, pos, *, ws=None, stream=None) -> torch.Tensor:
    """hs2_kv_append: K_new/V_new (bf16 [B, Hkv, T, d]) become tokens pos[b, t] of the cache.
    Returns the status workspace (read it with read_device_status)."""
    B, Hkv, T, d = K_new.shape
    cache.check(B, d)
    _need(K_new, "K_new", torch.bfloat16, (B, cache.Hkv, T, d))
    _need(V_new, "V_new", torch.bfloat16, (B, cache.Hkv, T, d))
    _need(pos, "pos", torch.int32, (B, T))
    dev = device_of("kv_append", K_new=K_new, V_new=V_new, pos=pos, ws=ws, **cache.tensors())
    dm = make_dims(B, cache.Hkv, cache.Hkv, T, cache.N, d, 0, 0)
    desc = cache.desc()
    with torch.cuda.device(dev):
        ws = torch.empty(256, dtype=torch.uint8, device=dev) if ws is None else ws
        _check(lib().hs2_kv_append(ctypes.byref(dm), ctypes.byref(desc), _p(K_new), _p(V_new), _p(pos), _p(ws),
                                   ws.numel(), _stream(stream, dev)), "hs2_kv_append")
    return ws


def decode_step(Q_full, Q_sparse, cache: KVCache, K_new, V_new, pos, *, k: int, W: int,
                out: Optional["StepOutputs"] = None, ws=None, stream=None) -> "StepOutputs":
    """hs2_decode_step: append the new token at pos[b] + 1 (device-side pos advances) and run the
    step for it.  Q_full/Q_sparse [B, Hq, 1, d], K_new/V_new [B, Hkv, 1, d] bf16, pos int32 [B]."""
    outs = out.as_dict() if out is not None else {}
    dm, desc, dev = _kv_call("decode_step", Q_full, cache, k, W, ws,
                             dict(Q_sparse=Q_sparse, K_new=K_new, V_new=V_new, pos=pos, **outs))
    B, Hq, Hkv, T, N, d, _, _ = dm.as_tuple()
    if T != 1:
        raise ValueError("decode_step takes one query per batch row (T = 1)")
    _need(Q_full, "Q_full", torch.bfloat16, (B, Hq, 1, d))
    _need(Q_sparse, "Q_sparse", torch.bfloat16, (B, Hq, 1, d))
    _need(K_new, "K_new", torch.bfloat16, (B, Hkv, 1, d))
    _need(V_new, "V_new", torch.bfloat16, (B, Hkv, 1, d))
    _need(pos, "pos", torch.int32, (B,))
    with torch.cuda.device(dev):
        out = alloc_step_outputs(dm, dev) if out is None else out
        ws = alloc_workspace_kv(dm, cache, dev) if ws is None else ws
        _check(lib().hs2_decode_step(ctypes.byref(dm), ctypes.byref(desc), _p(Q_full), _p(Q_sparse), _p(K_new),
                                     _p(V_new), _p(pos), _p(out.O_full), _p(out.O_sparse), _p(out.LSE_full),
                                     _p(out.LSE_sparse), _p(out.idx), _p(out.cnt), _p(ws), ws.numel(),
                                     _stream(stream, dev)), "hs2_decode_step")
    return out


def selftest_wait_bound(ws: torch.Tensor, limit_ns: int, stream=None) -> None:
    """hs2_selftest_wait_bound: run a bounded device wait that runs out (sets DEV_TIMEOUT in ws)."""
    with torch.cuda.device(ws.device):
        _check(lib().hs2_selftest_wait_bound(_p(ws), ws.numel(), int(limit_ns), _stream(stream, ws.device)),
               "hs2_selftest_wait_bound")


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    """Device status bits of the last call that used ``ws`` (synchronises the stream)."""
    bits = ctypes.c_uint32(0)
    with torch.cuda.device(ws.device):
        st = lib().hs2_read_device_status(_p(ws), _stream(stream, ws.device), ctypes.byref(bits))
    if st not in (HS2_OK, HS2_ERR_DEVICE):
        raise HS2Error(st, "hs2_read_device_status")
    return int(bits.value)


def trace_enable(enable: bool = True) -> None:
    """Start (or stop) per-kernel CUDA-event timing inside the library; clears the record."""
    _check(lib().hs2_trace_enable(1 if enable else 0), "hs2_trace_enable")


def trace_collect(max_entries: int = 64) -> Dict[str, tuple]:
    """{kernel name: (total ms, launches)} since the last collect (waits for the events)."""
    names = (ctypes.c_char_p * max_entries)()
    ms = (ctypes.c_double * max_entries)()
    cnt = (ctypes.c_int64 * max_entries)()
    n = lib().hs2_trace_collect(names, ms, cnt, max_entries)
    if n == -1:
        raise HS2Error(HS2_ERR_CUDA, "hs2_trace_collect")
    if n < 0:
        raise RuntimeError("trace event pool exhausted: collect more often")
    return {names[i].decode(): (ms[i], int(cnt[i])) for i in range(n)}


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(lib().hs2_launch_count())


def version() -> str:
    v = int(lib().hs2_version())
    return f"{v >> 16}.{v & 0xFFFF}"
