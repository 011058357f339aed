"""librswa: B200-native (sm_100a) R-SWA decode hot path behind a C ABI.

The CUDA library ``librswa.so`` (built from ``csrc/``) exports the ``rswa_*``
calls declared in ``include/rswa.h``; ``ring_sliding_window_b200.rswa`` is the
thin ctypes binding with the same names.  ``synth`` holds the seeded input
generators.  Importing this package does not load the CUDA library; the first
access to a binding name (``rswa_*``, ``RSWA_*``, ``State``) does, and fails
loudly if it is missing.
"""
import importlib


def __getattr__(name):
    if name.startswith(("rswa_", "RSWA_", "Rswa")) or name in ("State", "Config", "lib"):
        mod = importlib.import_module(".rswa", __name__)
        return getattr(mod, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
