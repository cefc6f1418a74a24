"""Orthrus dual-view block decoding on B200 (sm_100a).

The hot path lives in ``liborthrus.so`` (hand-written CUDA behind a C ABI,
declared in ``include/orthrus.h``). ``diffusion_draft_ar_b200.orthrus`` is the
thin ctypes binding with the same call names; importing it loads the library
and fails loudly when it has not been built.

``diffusion_draft_ar_b200.workloads`` holds the seeded synthetic inputs.
"""

__all__ = ["orthrus", "workloads"]
