"""Plain fp64 CPU oracle for the TurboQuant hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import anything from this package.  The
product path (the C-ABI library and its Python binding) never imports it, and
this package imports nothing from the product: the two share no code, no
tables and no constant generators.  The one module both sides' tests use is
the seeded input generator ``kv_cache_vector_15_b200.inputs``, which holds none
of the method's arithmetic.

Everything here is written for a reader to check by eye against the pages:

* ``params``      -- the seeded Rademacher diagonal D, the seeded Gaussian
                     projection S and the Lloyd-Max codebook for the rotated
                     coordinate law;
* ``turboquant``  -- rotation, quantize (write half), packing, the logit
                     estimator, dequantization and top-k (read half).

Parity status per function is stated in each docstring; the pins live in
``tests/test_oracle_*.py``.  Nothing here is "parity unpinned" except the
exact values of D and S, which depend on the chosen generator and are
pinned only by their published generator definitions (SplitMix64, Box-Muller)
and by their statistics.
"""

from . import params, turboquant  # noqa: F401
