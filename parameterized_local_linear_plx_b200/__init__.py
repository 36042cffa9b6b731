"""parameterized_local_linear_plx_b200: the Parallax attention forward pass
(causal prefill and split-KV decode) as hand-written sm_100a CUDA kernels
behind a small C ABI (``libplx.so``).

``from parameterized_local_linear_plx_b200 import plx`` loads the compiled
library and exposes ``plx.fwd`` and ``plx.decode``; it raises if the library
has not been built. ``inputs`` (seeded synthetic tensors) needs no library.
"""

__all__ = ["plx", "inputs"]


def __getattr__(name):
    if name == "plx":
        from . import plx as _plx
        return _plx
    if name == "inputs":
        from . import inputs as _inputs
        return _inputs
    raise AttributeError(name)
