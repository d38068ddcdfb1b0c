"""CPU oracle for the MOSS-Image DiT denoising step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.  The product library never does, and it shares no code with it.

Pinned parts and how: see ``tests/test_oracle_pins.py``.  Parity unpinned: the block's
internal structure against the trained MOSS-Image checkpoint (no code or weights of the
real model exist to compare with); the readings it rests on are listed in
``moss_oracle``'s header.
"""
from . import moss_oracle  # noqa: F401
