"""CPU oracle for the low-bit MoE hot path -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously correct numpy (float64) restatement
of what the path computes. It exists to check the CUDA library, never to stand
in for it: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` may import or run anything here.
The product path (``quantized_rl_fine_b200``) never imports this package and
shares no code with it; the two meet only through the seeded input bytes made
by ``quantized_rl_fine_b200.synth``.

Every function cites the passage of the source pages it follows. Where the
pages are silent the docstring says which plain reading was taken.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test against
something other than itself (hand-worked tables, closed forms, brute force,
finite differences, the pages' storage arithmetic); no function is "parity
unpinned".
"""

from .moe_oracle import *  # noqa: F401,F403
