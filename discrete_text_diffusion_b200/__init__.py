"""B200 (sm_100a) denoising-step library for block-autoregressive multinomial
text diffusion with a top-k MoE.  The compute path is libdg.so (hand-written
CUDA behind the C ABI in include/dg.h); ``dg`` is its thin ctypes binding and
``synth`` the seeded synthetic-input recipes shared with the tests."""
from . import synth  # noqa: F401
from .dg import *  # noqa: F401,F403
