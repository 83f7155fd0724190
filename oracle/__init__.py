"""FP64 CPU oracle of the CGTP convolution -- test infrastructure only.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline /
reference legs may import this package.  It shares no code with the CUDA
product path.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import build, lib, set_fault  # noqa: F401
