"""CPU oracle for the attention core: TEST INFRASTRUCTURE, not part of the product.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import, call or run anything in this package. The CUDA library and its Python binding
never import it, and the two share no code: only the seeded input generators in
``workloads.py`` (which hold none of the method's arithmetic) serve both sides.

Modules
  attention  the plain definition in fp64: RoPE, ALiBi slopes, masked softmax attention
             (prefill), one decode step over a cache, and the projection block.
  online     the tiled online-softmax recurrences (a second, independent route to the
             same numbers, used only to pin ``attention``).
  brute      scalar Python loops on tiny shapes (a third route, used only as a pin).

Every function is pinned by tests under ``tests/`` marked ``not gpu``: printed values of
the worked example, closed forms, invariants the pages state, and agreement between the
three independent routes. No function here is "parity unpinned".
"""
from . import attention, online, brute  # noqa: F401
