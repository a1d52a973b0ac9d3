"""CPU oracle for fused hybrid-batch (prefill + decode) attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg use it.  It shares no code with the
CUDA path (``prefill_decode_b200/``); the two meet only in the seeded input
generator ``synth``, which holds no attention arithmetic.

Contents
  attention.py  plain float64 attention: causal chunked prefill, paged decode,
                split-KV partials and their log-sum-exp merge, and a
                pure-Python brute-force version for tiny inputs.
  plan_ref.py   the scheduling plan rule (work items, split-KV partition,
                prefill:decode ticket ratio), restated in plain Python.

Parity status
  attention.*   pinned by brute force, closed forms and invariants
                (tests/test_oracle.py, tests/golden/).
  plan_ref.*    parity unpinned by the sources: they fix no split or ratio
                formula, so the rule is the library's own; it is pinned only by
                invariants (every (row, key) covered once, caps respected,
                degenerate batches) and by bit-exact agreement with the C
                planner, which is a separate implementation of the same rule.
"""
from .attention import (  # noqa: F401
    gather_tokens,
    attend_decode,
    attend_prefill,
    attend_prefill_batched,
    attend_rows,
    attend_partial,
    lse_merge,
    attend_brute_decode,
    attend_brute_prefill,
)
from .plan_ref import plan_ref, plan_ref_batched, PlanRef  # noqa: F401
