"""CPU oracle for one DSpark-style speculative round (fp64, numpy).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import, call or execute
anything under ``oracle/``. The product path (the CUDA library and its Python
binding) never does, and this package imports nothing from the product.

Parity pins: every function here is checked in ``tests/`` against something
other than itself (published Philox known answers and an independent Philox
implementation, hand-computed distributions, brute-force enumeration,
closed forms and invariants of rejection sampling). ``prefix_cut``'s
early-stopping rule is pinned only as a definition (hand-worked examples):
parity unpinned against the rule of the DSpark paper itself, whose appendix
is not among the pages.
"""
from .philox import philox4x32_10, uniform  # noqa: F401
from . import dspark  # noqa: F401
