"""B200-native Gram Newton-Schulz (Muon) update.

The work runs in hand-written sm_100a CUDA kernels behind the C ABI in
``include/dmu.h`` (``libdmu.so``); ``gram_newton_schulz_b200.dmu`` is the
ctypes binding (argument marshalling only).  Importing this package does
not load the shared library; ``dmu.load()`` does, and fails loudly when it
is missing.
"""

__version__ = "0.1.0"
