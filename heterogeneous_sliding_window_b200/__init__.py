"""heterogeneous_sliding_window_b200: MoA heterogeneous sliding-window attention on B200.

The compute lives in ``libmoa.so`` (C ABI, ``include/moa.h``); :mod:`.moa` is
its ctypes binding and :mod:`.inputs` the seeded synthetic-input generators.
Build the library with ``python -m heterogeneous_sliding_window_b200.build``.
"""

from . import moa  # noqa: F401  (loads libmoa.so lazily, on first call)

__all__ = ["moa"]
