"""Thin ctypes binding over libpagedattn.so (filled in with the C ABI)."""
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")
_lib = None


def load_library():
    global _lib
    if _lib is None:
        import ctypes
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library {LIB_PATH} is not built; run __graft_entry__.build()")
        _lib = ctypes.CDLL(LIB_PATH)
    return _lib
