"""B200-native ConvRot W8A8 INT8 linear.

The compute path lives in the C-ABI library ``libconvrot.so`` (hand-written
sm_100a CUDA); :mod:`.convrot` is a thin ctypes binding over it and
:mod:`.workloads` draws the seeded synthetic inputs.  Importing this package
loads nothing; the binding loads the library on first use and raises if it is
missing.
"""

__all__ = ["convrot", "workloads"]
