"""Kimi Delta Attention (KDA) on NVIDIA B200: a C-ABI CUDA library (sm_100a)
with a thin Python binding.

The compute entry points (``kda_chunk_fwd``, ``kda_decode_step``,
``kda_decode_tokens``) live in
``gated_delta_rule_132_b200.kda`` and load the in-tree ``libkda_b200.so`` on
first use; ``inputs`` holds the seeded synthetic-input generators.
"""
import importlib

from . import inputs  # noqa: F401  (no CUDA needed)

_EXPORTS = ("kda_chunk_fwd", "kda_chunk_fwd_prepare", "kda_chunk_fwd_carry",
            "kda_decode_step", "kda_decode_tokens", "kda_gdn_chunk_fwd", "kda_chunk_bwd",
            "kda_chunk_fwd_workspace_size",
            "ChunkFwdCall", "lib", "KdaError")


def __getattr__(name):
    if name in _EXPORTS:
        return getattr(importlib.import_module(".kda", __name__), name)
    raise AttributeError(name)
