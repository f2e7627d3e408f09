"""TwoTower layer-aligned block attention on B200 (sm_100a).

The compute lives in ``libtt_block_attn.so`` (CUDA kernels behind a C ABI,
declared in ``include/tt_block_attn.h``).  ``two_tower_block_b200.ops`` is the
thin ctypes binding with the same names; it loads the library on first use
and raises if it is missing.  There is no CPU fallback.
"""
import importlib

__all__ = ["ops", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
