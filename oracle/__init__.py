"""fp64 CPU oracle for block-sparse causal attention (test infrastructure).

This package is test infrastructure only.  It is a plain, slow, obviously
correct restatement of what the block-sparse causal attention forward
computes, written from the pages' statement of the method.  Only the test
suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import it; the CUDA product path never does, and the two
share no code (the seeded input generator they both consume lives in its own
module and contains none of the method's arithmetic).

Modules:
  layouts   -- kept-block sets for each pattern family, the SplitMix64
               generator, CSR and transposed (CSC) assembly, pair counts and
               reachability depth.
  attention -- the masked-softmax definition (dense, tiny n), the same
               definition restricted to its support (large n), and a pure
               Python brute force for tiny inputs.
  decode    -- one selected-page decode step through a page table.
  backward  -- the gradients of the masked softmax, written out.
  bsbr      -- BSBR's chunk states, meta weights and retrieval term.

Every function is pinned by a ``-m "not gpu"`` test against something other
than itself (printed page values, closed forms, library routines, invariants,
brute force): ``tests/test_oracle_layouts.py``,
``tests/test_oracle_attention.py``, ``tests/test_oracle_decode.py``,
``tests/test_oracle_backward.py`` and ``tests/test_oracle_bsbr.py``.
"""
from . import layouts, attention  # noqa: F401
