"""B200-native mHC decode boundary.

The compute path is the CUDA library ``libmhc.so`` (built from ``csrc/``);
``mhc_residual_stream_b200.mhc`` is its thin ctypes binding. Importing the
package itself loads nothing, so that the seeded input generator
(``synthetic``) is usable on machines without the library.
"""

__all__ = ["synthetic"]
