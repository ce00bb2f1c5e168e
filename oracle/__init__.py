"""CPU oracle for the ConvRot W8A8 INT8 linear.

Test infrastructure only: tests/, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the product package never does.
"""
from .oracle import *  # noqa: F401,F403
