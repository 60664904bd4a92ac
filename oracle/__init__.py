"""CPU oracle for the QLoRA NF4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import anything from here.  The product path (the CUDA library and its
Python binding) never does, and shares no code with it.
"""
from .oracle import *  # noqa: F401,F403
