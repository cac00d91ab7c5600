"""The time-split prefill on the tensor-core path against the fp64 oracle.

A long sequence with few heads leaves most SMs idle during the sequential
chunk walk; kda_chunk_fwd_timesplit runs that walk in two parallel passes over
time segments (zero-start states and transitions, a combine, then the true
entry states). Results must equal the token-by-token recurrence within the
bf16 tolerance for any segment count, including segments left empty.
"""
import numpy as np
import pytest
import torch

import oracle
from common import TOL, rel_l2, to_cuda, unit_errors_o, unit_errors_S
from gated_delta_rule_132_b200 import inputs as I
from gated_delta_rule_132_b200 import kda

pytestmark = pytest.mark.gpu
BF16 = TOL[torch.bfloat16]


def _oracle(x, heads=None):
    sel = slice(None) if heads is None else heads
    S0 = None if x["S0"] is None else x["S0"][:, sel].cpu()
    return oracle.forward(x["q"][:, :, sel].cpu(), x["k"][:, :, sel].cpu(),
                          x["v"][:, :, sel].cpu(), x["log_alpha"][:, :, sel].cpu(),
                          x["beta"][:, :, sel].cpu(), S0,
                          None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu(),
                          scale=x["scale"])


def _split(g, segments, output_final_state=True):
    return kda.kda_chunk_fwd_timesplit(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                                       g["S0"], g["cu_seqlens"], g["scale"], segments=segments,
                                       output_final_state=output_final_state)


@pytest.mark.parametrize("segments", [1, 2, 3, 5, 14, 20])
def test_segments_against_the_oracle(segments):
    """B=2, H=2, 837 tokens (14 chunks, a ragged tail): every segment count,
    including more segments than chunks (empty segments)."""
    x = I.make_prefill(2, 837, 2, 128, torch.bfloat16, gate_shift=-1.0, s0_std=0.05, seed=81)
    o, Sf = _split(to_cuda(x), segments)
    o_ref, S_ref = _oracle(x)
    assert rel_l2(o, o_ref) <= BF16 and rel_l2(Sf, S_ref) <= BF16
    assert unit_errors_o(o, o_ref).max() <= BF16 and unit_errors_S(Sf, S_ref).max() <= BF16


@pytest.mark.parametrize("segments", [3, 7])
def test_varlen_with_empty_and_ragged_sequences(segments):
    lengths = [1, 640, 0, 1000, 65, 2048]
    x = I.make_prefill(1, 0, 2, 128, torch.bfloat16, gate_shift=-2.0, s0_std=0.05, seed=82,
                       lengths=lengths)
    o, Sf = _split(to_cuda(x), segments)
    o_ref, S_ref = _oracle(x)
    assert unit_errors_o(o, o_ref, x["cu_seqlens"]).max() <= BF16
    assert unit_errors_S(Sf, S_ref).max() <= BF16
    assert torch.equal(Sf[2].cpu(), x["S0"][2])  # the empty sequence keeps its S0


@pytest.mark.parametrize("gate_shift", [-6.0, 3.0])
def test_slow_and_strong_decay(gate_shift):
    """Nearly no decay (the transition stays close to the delta rule's own
    contraction over many chunks) and strong decay (the exact fixup chunks)."""
    x = I.make_prefill(1, 64 * 24 + 17, 2, 128, torch.bfloat16, gate_shift=gate_shift,
                       s0_std=0.05, seed=83)
    o, Sf = _split(to_cuda(x), 4)
    o_ref, S_ref = _oracle(x)
    assert rel_l2(o, o_ref) <= BF16 and rel_l2(Sf, S_ref) <= BF16


def test_zero_state_and_no_final_state():
    x = I.make_prefill(1, 64 * 10, 3, 128, torch.bfloat16, gate_shift=-1.0, s0_std=0.0, seed=84)
    o, Sf = _split(to_cuda(x), 3, output_final_state=False)
    assert Sf is None
    o_ref, _ = _oracle(x)
    assert rel_l2(o, o_ref) <= BF16


def test_split_matches_the_unsplit_path_and_is_deterministic():
    g = to_cuda(I.make_prefill(1, 64 * 40, 4, 128, torch.bfloat16, -2.0, 0.05, seed=85))
    o1, S1 = _split(g, 1)
    o2, S2 = _split(g, 6)
    o3, S3 = _split(g, 6)
    assert torch.equal(o2, o3) and torch.equal(S2, S3)
    assert rel_l2(o2, o1.double().cpu().numpy()) <= 1e-2
    assert rel_l2(S2, S1.double().cpu().numpy()) <= 1e-2


def test_automatic_choice():
    """AUTO splits only when few chains would leave SMs idle: H = 4 at 64k
    tokens splits (the workspace holds the segment states), H = 32 does not."""
    L = kda.lib()
    few = L.kda_chunk_fwd_workspace_size_ex(1, 1 << 16, 4, 128, 128, 0, 1, 0)
    few_seq = L.kda_chunk_fwd_workspace_size_ex(1, 1 << 16, 4, 128, 128, 0, 1, 3)
    many = L.kda_chunk_fwd_workspace_size_ex(1, 1 << 16, 32, 128, 128, 0, 1, 0)
    many_seq = L.kda_chunk_fwd_workspace_size_ex(1, 1 << 16, 32, 128, 128, 0, 1, 3)
    assert few > few_seq and many == many_seq


@pytest.mark.slow
@pytest.mark.parametrize("H", [4, 32])
def test_one_million_tokens_single_sequence(H):
    """B=1, T=2^20 (the pages' 1M-token setting), d=128, bf16, slow decay:
    H=4 takes the time split, H=32 the plain sequential walk (AUTO). All heads
    run on the GPU; the oracle checks 2 of them end to end."""
    T = 1 << 20
    x = I.make_prefill(1, T, H, 128, torch.bfloat16, gate_shift=-3.0, s0_std=0.0, seed=86,
                       device="cuda")
    o, Sf = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None,
                              scale=x["scale"])
    torch.cuda.synchronize()
    heads = [0, H - 1]
    o_ref, S_ref = _oracle(x, heads)
    o_h, S_h = o[:, :, heads].cpu(), Sf[:, heads].cpu()
    del x, o, Sf
    torch.cuda.empty_cache()
    assert unit_errors_o(o_h, o_ref).max() <= BF16
    assert unit_errors_S(S_h, S_ref).max() <= BF16
    assert np.isfinite(o_h.float().numpy()).all()
