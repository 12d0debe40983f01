"""CPU oracle for the NVFP4 W4A4 linear.  TEST INFRASTRUCTURE, NOT PRODUCT CODE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference arm may import this package.  It shares no code with the CUDA library
(``nvfp4_w4a4_quantized_02_b200``) and never imports it.
"""
from .nvfp4_oracle import *  # noqa: F401,F403
from . import layout  # noqa: F401
