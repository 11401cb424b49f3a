"""Head-wise sparse decode attention for B200 (sm_100a).

The CUDA library (lib/libsparsedecode.so, C ABI in include/sparse_decode.h)
does all the work; `sparse_decode` is its thin ctypes binding and `decode`
wires a full decode step.  Both are imported on first use so that the build
script can run before the library exists.
"""

import importlib

__all__ = ["sparse_decode", "decode"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
