"""Kimi Delta Attention (KDA) on NVIDIA B200: a C-ABI CUDA library (sm_100a)
with a thin Python binding.

The compute entry points (``chunk_fwd``, ``decode_step``) live in
``gated_delta_rule_132_b200.kda`` and load the in-tree ``libkda_b200.so`` on
first use; ``inputs`` holds the seeded synthetic-input generators.
"""
from . import inputs  # noqa: F401  (no CUDA needed)


def __getattr__(name):
    if name in ("chunk_fwd", "decode_step", "chunk_fwd_workspace_size", "lib", "kda",
                "KdaError"):
        from . import kda
        return kda if name == "kda" else getattr(kda, name)
    raise AttributeError(name)
