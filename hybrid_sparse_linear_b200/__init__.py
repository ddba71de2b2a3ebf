"""SALA hybrid attention forward for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libsala.so`` (hand-written CUDA kernels, declared in
``include/sala.h``); ``hybrid_sparse_linear_b200.sala`` is the thin ctypes binding over it and
``hybrid_sparse_linear_b200.synth`` draws the seeded synthetic inputs.  Importing the package
itself loads nothing; importing ``.sala`` loads the library and raises if it is missing.
"""
__all__ = ["sala", "synth"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
