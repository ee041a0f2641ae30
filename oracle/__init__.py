"""The oracle: plain, slow CPU implementations of the emulated MMA arithmetic.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference leg of ``bench.py`` may import or run anything
in this package.  The product library (``bit_exact_tensor_b200``) never
imports it, and it shares no code with the CUDA kernels.

* ``mma_model``  -- the authority: arbitrary-precision Python integers, one
  output element at a time, parametric in format and model so tiny formats
  can be checked exhaustively.
* ``mmaemu_ref.c`` / ``cref`` -- the same rules restated in plain C with
  64-bit integers, threaded over independent output elements, for
  full-size workloads and the timed CPU baseline.

Parity of the oracle itself is pinned by ``tests/test_oracle_*.py`` against
facts that do not come from the oracle: the worked example and the behaviour
the pages print, closed-form probe values, exact-rational agreement,
exhaustive tiny-format enumeration and algebraic invariants.
"""
