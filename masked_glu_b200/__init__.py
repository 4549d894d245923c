"""masked_glu_b200: a B200-native (sm_100a) Masked Gated Linear Unit forward.

The compute lives in ``libmglu.so`` (hand-written CUDA behind a C ABI, see
``include/mglu.h``); :mod:`masked_glu_b200.mglu` is the thin ctypes binding
with the same names.  :mod:`masked_glu_b200.inputs` draws seeded synthetic
inputs and holds no part of the method.
"""
