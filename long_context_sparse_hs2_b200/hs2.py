"""Thin Python binding of ``libhs2.so`` (the C ABI declared in ``include/hs2.h``).

Argument marshalling only: it checks tensor dtypes, shapes, devices and contiguity,
allocates outputs and the workspace with PyTorch (device memory is PyTorch's job
here), and passes raw pointers and the current CUDA stream to the library.  Every
step of the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and a missing library is an error.

Names mirror the C entry points: ``full_attn``, ``select``, ``sparse_attn``,
``step``, ``workspace_size``, ``read_device_status``, ``status_string``.
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

ENTRY_POINTS = ("hs2_workspace_size", "hs2_full_attn", "hs2_select", "hs2_sparse_attn", "hs2_step",
                "hs2_read_device_status", "hs2_status_string", "hs2_trace_enable", "hs2_trace_collect",
                "hs2_launch_count", "hs2_version", "hs2_sparse_attn_static")
STATIC_SCRATCH_BYTES = 4 << 20  # HS2_STATIC_SCRATCH_BYTES


class Dims(ctypes.Structure):
    """``hs2_dims``: problem shape (the attention scale is fixed to d^-1/2)."""

    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "T", "N", "d", "k", "W")]

    def as_tuple(self):
        return tuple(getattr(self, n) for n, _ in self._fields_)


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
