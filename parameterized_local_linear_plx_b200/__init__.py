"""parameterized_local_linear_plx_b200: the Parallax attention forward pass
(causal prefill and split-KV decode) as hand-written sm_100a CUDA kernels
behind a small C ABI (``libplx.so``, declared in include/plx.h).

``from parameterized_local_linear_plx_b200 import plx`` loads the compiled
library and exposes ``plx.plx_fwd`` and ``plx.plx_decode``; that import raises
if the library has not been built.  ``inputs`` (seeded synthetic tensors) and
``build`` need no library.
"""
