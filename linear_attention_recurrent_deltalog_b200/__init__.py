"""DeltaLog decoding for delta-rule linear attention on B200 (sm_100a).

The compute path is the C-ABI library ``libdeltalog.so`` (CUDA kernels for
sm_100a) reached through :mod:`.deltalog`; :mod:`.workloads` draws the seeded
synthetic inputs.  Importing the package loads nothing native: the library is
loaded (and a missing build reported) when :mod:`.deltalog` is imported.
"""

__version__ = "0.1.0"
