"""Canvas-step library for block-wise discrete-diffusion decoding on B200 (sm_100a).

The computation lives in ``libdg.so`` (C ABI, include/dg.h); :mod:`.binding` marshals torch
tensors to it.  Build the library with ``python -m block_discrete_diffusion_dg_b200.build``.
"""
from . import binding  # noqa: F401
from .binding import DgError  # noqa: F401

__all__ = ["binding", "DgError"]
