"""CPU oracle for mixed-format paged decode attention (FP8 anchor pages + packed TQ3 pages).

TEST INFRASTRUCTURE ONLY.  A plain, slow float64 numpy restatement of what the method
computes, used to check the CUDA library.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the library never
does, and the oracle imports nothing from the library.

Modules:
  formats    -- E4M3 codec, FP8 page write with rescale-on-grow, TQ3 quantise/pack, slot bytes
  pool       -- allocator, block tables, anchor policy, demotion, sequence copy
  attention  -- float64 attention over the dequantised cache, partial states, merge

Every function is pinned by ``tests/test_oracle_*.py`` against values the pages or the
mathematics fix (closed forms, library conversions, exact rationals, invariants, brute force).
"""
from . import attention, formats, pool  # noqa: F401
