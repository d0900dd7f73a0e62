"""B200-native (sm_100a) gated delta-rule recurrence: KDA and Complex-KDA.

``ops`` binds the C ABI of ``libckda.so`` (``include/ckda.h``): the chunkwise
forward (``chunk_fwd``) and the one-token decode step (``decode_step``).
``synth`` draws the seeded synthetic workloads.  ``build`` compiles the
library with nvcc for sm_100a.
"""
__version__ = "0.1.0"
