"""Activation-sparse GEMV / FFN for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libsfx.so`` (include/sfx.h), built
in-tree by ``sparse_input_gemv_b200.build``; ``binding`` exposes its entry
points to Python with the same names. ``synth`` draws the seeded synthetic
inputs. Importing this package loads nothing; the library is loaded on the
first call and its absence raises.
"""

__all__ = ["binding", "synth", "build"]
