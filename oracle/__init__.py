"""CPU oracle for mask-aware attention forward: plain, slow, obviously correct.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, header,
table or helper with the CUDA library; the two meet only on the seeded inputs
produced by ``workloads``.

Everything here computes in float64 (bf16 inputs are upcast exactly) with NumPy.
Each function cites the passage of the source pages it restates, by page title
and section.

Modules
-------
masks      dense boolean mask builders for every mask form (block ids, causal,
           sliding window, varlen packing, BSR, predicate algebra)
attention  masked softmax attention with log-sum-exp
plan       the tile plan a dense mask defines (classes, packed bits, CSR, order)

Parity status: every function is pinned by a ``-m "not gpu"`` test against
brute force, closed forms, a library routine or a printed example; none is
"parity unpinned".
"""

from . import masks, attention, plan  # noqa: F401
