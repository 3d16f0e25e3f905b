"""B200 (sm_100a) hot path of a BASE layer: affinity scores, balanced
auction / greedy routing, expert-major permutation, expert FFNs with the
eq. 1 gated residual, combine, and the backward -- each a CUDA kernel behind
the C ABI of include/base.h.  ``binding`` exposes that ABI one-to-one;
``buffers`` allocates the caller-owned device buffers with torch."""
from .binding import *  # noqa: F401,F403
from . import binding, buffers, synth  # noqa: F401
