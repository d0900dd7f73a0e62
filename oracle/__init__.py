"""fp64 CPU oracle of the gated delta-rule recurrence (KDA / Complex-KDA).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the CUDA library or its
Python binding.  Every function is pinned by ``tests/pins.py`` against closed
forms and invariants of the method (run by ``tests/test_oracle_pins.py``).
"""
from .oracle import (SOURCE, Oracle, build, ckda_bwd, ckda_fwd, ckda_fwd_explicit,
                     ckda_fwd_product, compile_c, decode_step, default, gates, transition)

__all__ = ["SOURCE", "Oracle", "build", "ckda_bwd", "ckda_fwd", "ckda_fwd_explicit",
           "ckda_fwd_product", "compile_c", "decode_step", "default", "gates", "transition"]
