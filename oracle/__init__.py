"""Plain fp64 CPU oracle for the Muon / Gram Newton-Schulz update.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA path
(``gram_newton_schulz_b200``) and imports nothing from it.

Every function is written from the method as the DMuon, Dion3 and DeMuon
pages state it (see the per-function citations in ``gram_ns.py``), in
float64, with ``numpy.matmul`` as the only library primitive.

Pins (``tests/test_oracle_pins.py``): SVD polar factor, spectral closed
form, Gram-form == rectangular form, transpose / scale / orthogonal
invariance, the quintic singular-value band, and exact rational special
cases.  ``demuon.py`` (one DeMuon iteration over N agents) is pinned in
``tests/test_demuon_oracle.py``: the single-agent reduction to Muon, the
gradient-tracking mean invariant, one-step consensus on the complete
graph, a hand-computed scalar case, and the ring's closed-form mixing rate.
No function here is "parity unpinned".
"""

from .gram_ns import (  # noqa: F401
    QUINTIC,
    K_STEPS,
    momentum,
    frobenius_normalize,
    ns_rectangular,
    ns_gram,
    gram_trace,
    orthogonalize,
    update_scale,
    muon_step,
    bf16_bits_to_f64,
)
