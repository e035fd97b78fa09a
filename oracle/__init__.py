"""CPU oracle for the forward pass of shared-QK LSH attention (Reformer).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may use it.  It shares no code,
header, table or helper with the CUDA library in ``lsh_attention_hash_b200``.

Every function is plain float64 NumPy that follows the method step by step, in
the order the pages describe it.  See ``lsh_oracle`` for the functions and the
passages each one follows.  Every function here is pinned by ``-m "not gpu"``
tests in ``tests/test_oracle_pins.py`` (worked example, closed forms,
invariants and brute-force enumeration); none is "parity unpinned".
"""

from .lsh_oracle import (  # noqa: F401
    TIE_REL,
    oracle_hash,
    oracle_sort,
    oracle_attend,
    oracle_attend_slots,
    oracle_combine,
    oracle_lsh_attention,
    oracle_attend_backward,
)
