"""kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot
allocate device memory (for example a plugin whose host application owns all
device memory). It must give the same results as kda_chunk_fwd, using the
library's fixed scratch array instead of a caller-provided workspace.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from common import to_cuda
from gated_delta_rule_132_b200 import inputs as I
from gated_delta_rule_132_b200 import kda

KDA_OK, KDA_ERR_WORKSPACE = 0, 4
SCRATCH_BYTES = 32 * 1024 * 1024  # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h


def _entry():
    f = kda.lib().kda_chunk_fwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.restype = i
    f.argtypes = [vp, vp, vp, i, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp, vp,
                  i, vp]
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(x, o, S_final, algo=0):
    B, T, H, d = x["q"].shape
    n_seqs = 0 if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1
    dt = 1 if x["q"].dtype == torch.bfloat16 else 0
    return _entry()(_p(x["q"]), _p(x["k"]), _p(x["v"]), dt, _p(x["log_alpha"]), _p(x["beta"]),
                    _p(x["S0"]), _p(x["cu_seqlens"]), n_seqs, B, T, H, d, x["v"].shape[-1],
                    x["scale"], _p(o), _p(S_final), algo,
                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
def test_noalloc_matches_chunk_fwd_on_two_calls_in_a_row():
    """Two calls in a row with different problems (a batched tensor-core
    prefill, then a packed variable-length one) each match kda_chunk_fwd."""
    problems = [
        I.make_prefill(2, 300, 4, 128, torch.bfloat16, -1.0, 0.05, seed=61),
        I.make_prefill(1, 0, 3, 128, torch.bfloat16, -2.0, 0.05, seed=62,
                       lengths=[65, 1, 190, 0, 64]),
    ]
    for x in problems:
        g = to_cuda(x)
        o_ref, S_ref = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                                         g["S0"], g["cu_seqlens"], g["scale"])
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        assert _call_noalloc(g, o, S) == KDA_OK
        torch.cuda.synchronize()
        # the same kernels on the same inputs: bit-identical results
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_noalloc_rejects_problems_beyond_the_scratch_size():
    """A problem whose workspace exceeds the fixed scratch array is rejected on
    the host (placeholder pointers, never dereferenced; no CUDA call is made)."""
    need = kda.lib().kda_chunk_fwd_workspace_size(1, 1 << 20, 32, 128, 128, 0, 1)
    assert need > SCRATCH_BYTES
    f = ctypes.c_void_p(0x10000)
    st = _entry()(f, f, f, 1, f, f, None, None, 0, 1, 1 << 20, 32, 128, 128, 0.1, f, None, 0,
                  None)
    assert st == KDA_ERR_WORKSPACE


@pytest.mark.parametrize("dt,d,status", [(7, 128, 2), (1, 96, 2), (1, 0, 1)])
def test_noalloc_rejects_bad_arguments_on_the_host(dt, d, status):
    """An unsupported dtype or head size, or a non-positive size, is rejected on
    the host with the status kda_chunk_fwd_ex gives, before any CUDA call
    (placeholder pointers, never dereferenced)."""
    f = ctypes.c_void_p(0x10000)
    st = _entry()(f, f, f, dt, f, f, None, None, 0, 1, 64, 2, d, d, 0.1, f, None, 0, None)
    assert st == status
