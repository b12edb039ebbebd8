"""Exact ring attention on one B200: C-ABI library (libringattn.so) + thin binding.

The library (built in-tree by ``python -m sequence_exact_attention_ring_b200.build``)
holds every kernel; this package only marshals arguments. Importing the package
does not load the library; the first call does, and raises if it is missing.
"""
from . import binding  # noqa: F401
from . import ring  # noqa: F401
from .api import (  # noqa: F401
    HostRunner, merge, ring_attention, ring_attention_backward, ring_attention_decode, ring_attention_ring_step,
    ring_attention_step, ring_backward_prep, ring_backward_step, status, workspace_bytes)
from .binding import RingAttnError  # noqa: F401

__all__ = ["binding", "ring", "ring_attention", "ring_attention_step", "ring_attention_ring_step", "merge", "status",
           "workspace_bytes", "HostRunner", "RingAttnError", "ring_attention_backward", "ring_attention_decode",
           "ring_backward_prep", "ring_backward_step"]
