"""ORACLE — test infrastructure, not product code.

A plain, slow CPU restatement of block-sparse attention with cumulant-order block
selection (COBS), written from the method's description: the NSA three-branch
attention (compressed tokens, selected blocks, sliding window, mixed by per-head
gates) whose selected-block branch ranks key blocks by the first two cumulants
of the log attention mass.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import, call, link or execute anything in this package. It shares no code
with the CUDA library and imports nothing from it.

* ``cobs_oracle``     float64 restatement of every step (numpy; library matmul and
                      sort are the only primitives used).
* ``canonical_fp32.c`` the float32 selector arithmetic in a fixed order, in which the
                      integer selection decision is taken (C, ``fmaf``).

Parity status: every function is pinned by ``tests/test_oracle_*.py`` except the
way per-head scores of one GQA group are combined into one group score (their sum),
which the pages leave open: that reading is "parity unpinned".
"""
