"""CPU oracle for the Masked Gated Linear Unit forward -- test infrastructure.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / ``--impl reference`` leg may import this package.  The
product library never loads it, and it never loads the product library.

* :mod:`oracle.core`  -- ctypes binding to ``mglu_oracle.c`` (float64,
  OpenMP over output columns, explicit bit-by-bit mask unpacking).
* :mod:`oracle.brute` -- pure-Python loops over logical (d x h) tensors, used
  to cross-check the C oracle at tiny sizes.
* :mod:`oracle.train` -- numpy float64 training path: mask binarisation
  from logits and the straight-through backward (dx, dW, mask-logit
  gradients), plus the down-projection backward.
* :mod:`oracle.routed` -- per-token mask weights and top-k mask routing.

The method: "Masked Gated Linear Unit" (atlas.scime.ai summary page of the
MGLU paper), "Approach" and "Key results" and the "Measured effects" rows on
summing masks and on GELU / ReLU gating.
"""
from .core import (  # noqa: F401
    ACT_GELU,
    ACT_RELU,
    ACT_SWISH,
    GATE_DENSE,
    activation,
    build,
    down,
    down_elems,
    forward,
    forward_elems,
    gate_value,
    pack_masks,
    packed_bytes,
    unpack_masks, max_threads, set_threads)
