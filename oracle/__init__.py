"""FP64 CPU oracle for Flint's sink-aware attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg, never by the CUDA library. It shares no code
with the library; only the seeded input generators in ``flint_inputs`` serve
both sides.

* ``flint_oracle`` - vectorised FP64 NumPy definition (forward, analytic
  backward, sampled rows for large inputs).
* ``brute`` - pure-Python scalar-loop forward for tiny inputs.
"""
