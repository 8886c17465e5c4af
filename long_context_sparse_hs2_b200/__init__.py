"""HySparse2 hybrid sparse attention step on NVIDIA B200 (sm_100a).

The compute path lives in ``libhs2.so`` (hand-written CUDA behind a C ABI,
declared in ``include/hs2.h``); ``long_context_sparse_hs2_b200.hs2`` is the thin
ctypes binding.  The binding is imported lazily so that the input generator
(``long_context_sparse_hs2_b200.inputs``) can be used without loading CUDA.
"""

__all__ = ["hs2", "inputs"]


def __getattr__(name):
    if name in ("hs2", "inputs"):
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
