"""libkvq: rotate-then-quantize int4 KV-cache codec for NVIDIA B200 (sm_100a).

The compute path is the C-ABI shared library ``libkvq.so`` built from
``csrc/`` (see ``build.py``).  ``kvq`` is a thin ctypes binding over it; it is
imported lazily so that ``workloads`` can be used without the library.
"""

SRFT = 0
SRHT = 1

__all__ = ["SRFT", "SRHT", "kvq", "workloads"]


def __getattr__(name):
    if name in ("kvq", "workloads"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
