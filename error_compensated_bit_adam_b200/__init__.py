"""B200-native compression-phase step of 1-bit Adam.

libonebit (csrc/, C ABI in include/onebit.h) runs the method in hand-written
sm_100a CUDA kernels; this package is its Python binding:

* ``_binding``  -- one function per C entry point, same names (ctypes);
* ``optimizer`` -- ``OneBitAdam``, a context with torch-owned device memory;
* ``workloads`` -- seeded synthetic inputs (no method arithmetic);
* ``build``     -- nvcc build of libonebit.so for sm_100a.

The library is loaded on first use; if it is not built, that use raises.
"""
from ._binding import *  # noqa: F401,F403
from ._binding import OnebitError, lib  # noqa: F401


def __getattr__(name):
    if name == "OneBitAdam":
        from .optimizer import OneBitAdam
        return OneBitAdam
    raise AttributeError(name)
