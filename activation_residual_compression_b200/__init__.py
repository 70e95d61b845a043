"""B200 residual compression with error feedback (CompactFusion-style).

The product is ``libcf.so`` (C ABI in ``include/cf.h``, sm_100a kernels in
``csrc/``); this package is its thin Python binding (``_cf``), plus the seeded
synthetic activation streams used by the tests and the benchmark
(``inputs``).  The binding loads the library on its first call and raises
ImportError if it has not been built: there is no CPU fallback.
"""
from . import _cf  # noqa: F401
from ._cf import *  # noqa: F401,F403

__all__ = [n for n in dir(_cf) if n.startswith(("cf_", "CF_"))] + ["MODE_NAMES", "CFError"]
