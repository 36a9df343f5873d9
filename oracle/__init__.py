"""CPU oracle of the mHC decode boundary.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow float64 restatement
of what the boundary computes. It exists to check the CUDA library and to be
timed as a CPU baseline. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` (``cpu_baseline`` and ``--impl reference``) may import
it. The product (``mhc_residual_stream_b200`` and its CUDA library) never
imports, links or calls anything here, and this package imports nothing from
the product: the two share no code.

Parity status of each function is stated in its docstring. Functions whose
result rests on a convention that no independent value can fix carry the words
"parity unpinned" for that convention.
"""

from .mhc import *  # noqa: F401,F403
