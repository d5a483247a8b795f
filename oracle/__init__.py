"""CPU oracle for activation-sparse decoding -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 numpy definitions of what the activation-sparse GEMV/FFN
path computes. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference legs of ``bench.py`` may import this package; the product
package ``sparse_input_gemv_b200`` never imports it and shares no code with it
(only the seeded input generators in ``sparse_input_gemv_b200.synth`` feed
both sides).

Every function is pinned by ``tests/test_oracle_pins.py`` against values the
source pages print, closed forms, invariants or brute force.
"""
from .sfx_oracle import *  # noqa: F401,F403
