"""kda_chunk_fwd on the GPU against the fp64 oracle, on both prefill paths."""
import numpy as np
import pytest
import torch

import oracle
from common import REGRESSION_GUARD, TOL, rel_l2, to_cuda, unit_errors_o, unit_errors_S
from gated_delta_rule_132_b200 import inputs as I
from gated_delta_rule_132_b200 import kda

pytestmark = pytest.mark.gpu

# (algo, dtype, d) combinations each path implements.
PATHS = [("simt", torch.float32, 32), ("simt", torch.float32, 64),
         ("simt", torch.float32, 128), ("simt", torch.bfloat16, 64),
         ("simt", torch.bfloat16, 128), ("tcgen05", torch.bfloat16, 128)]


def _has_tc():
    """True when the library accepts KDA_ALGO_TCGEN05 for bf16, d=128 (checked on
    the host with placeholder pointers: the call is rejected for its zero-size
    workspace before anything could be launched)."""
    import ctypes
    f = ctypes.c_void_p(0x10000)
    st = kda.lib().kda_chunk_fwd_ex(f, f, f, 1, f, f, None, None, 0, 1, 64, 1, 128, 128, 0.1,
                                    f, None, f, 0, 2, None)
    return st == 4  # KDA_ERR_WORKSPACE: the tcgen05 path exists for this problem


def run_both(x, algo="auto", heads=None, output_final_state=True):
    """GPU result and oracle result on the same inputs (optionally only some heads
    go through the oracle)."""
    g = to_cuda(x)
    o, Sf = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["S0"],
                              g["cu_seqlens"], x["scale"], output_final_state, algo=algo)
    torch.cuda.synchronize()
    sel = slice(None) if heads is None else heads
    ref_in = {k: (x[k][:, :, sel] if x[k] is not None and k != "S0" and k != "cu_seqlens"
                  else x[k]) for k in ("q", "k", "v", "log_alpha", "beta", "S0", "cu_seqlens")}
    if x["S0"] is not None:
        ref_in["S0"] = x["S0"][:, sel]
    o_ref, S_ref = oracle.forward(ref_in["q"], ref_in["k"], ref_in["v"], ref_in["log_alpha"],
                                  ref_in["beta"], ref_in["S0"], ref_in["cu_seqlens"],
                                  scale=x["scale"])
    o_gpu = o[:, :, sel]
    S_gpu = None if Sf is None else Sf[:, sel]
    return o_gpu, S_gpu, o_ref, S_ref


def _skip_unless(algo):
    if algo == "tcgen05" and not _has_tc():
        pytest.skip("tcgen05 path not built")


def test_tiny_fp32_config():
    """B=1, H=2, T=64, d=32, fp32: rel-L2 <= 1e-4 on o and S_final."""
    x = I.make_preset(I.TINY)
    o, Sf, o_ref, S_ref = run_both(x)
    assert rel_l2(o, o_ref) <= 1e-4
    assert rel_l2(Sf, S_ref) <= 1e-4


@pytest.mark.parametrize("algo,dtype,d", PATHS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_lengths_and_tails(algo, dtype, d, T):
    _skip_unless(algo)
    x = I.make_prefill(2, T, 3, d, dtype, gate_shift=-1.0, s0_std=0.05, seed=T * 7 + d)
    o, Sf, o_ref, S_ref = run_both(x, algo=algo)
    assert rel_l2(o, o_ref) <= TOL[dtype]
    assert rel_l2(Sf, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("algo,dtype,d", PATHS)
def test_varlen_with_empty_and_ragged_sequences(algo, dtype, d):
    _skip_unless(algo)
    lengths = [1, 64, 0, 65, 127, 3, 190, 0, 64]
    x = I.make_prefill(1, 0, 2, d, dtype, gate_shift=-1.0, s0_std=0.05, seed=31 + d,
                       lengths=lengths)
    o, Sf, o_ref, S_ref = run_both(x, algo=algo)
    assert rel_l2(o, o_ref) <= TOL[dtype]
    assert rel_l2(Sf, S_ref) <= TOL[dtype]
    # zero-length sequences return their S0 exactly
    assert torch.equal(Sf[2].cpu(), x["S0"][2]) and torch.equal(Sf[7].cpu(), x["S0"][7])


@pytest.mark.parametrize("algo,dtype,d", PATHS)
def test_zero_state_and_no_final_state(algo, dtype, d):
    _skip_unless(algo)
    x = I.make_prefill(1, 150, 2, d, dtype, gate_shift=0.0, s0_std=0.0, seed=5)
    o, Sf, o_ref, S_ref = run_both(x, algo=algo, output_final_state=False)
    assert Sf is None
    assert rel_l2(o, o_ref) <= TOL[dtype]


@pytest.mark.parametrize("algo", ["simt", "tcgen05"])
def test_empty_time_axis_copies_state(algo):
    _skip_unless(algo)
    x = I.make_prefill(3, 0, 2, 128, torch.bfloat16, s0_std=0.05, seed=9)
    g = to_cuda(x)
    o, Sf = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], g["S0"],
                              algo=algo)
    assert o.numel() == 0 and torch.equal(Sf, g["S0"])
    o, Sf = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], None,
                              algo=algo)
    assert torch.count_nonzero(Sf) == 0


@pytest.mark.parametrize("algo", ["simt", "tcgen05"])
def test_split_prefill_equals_single_call(algo):
    """forward(T) == forward(T1) then forward(T - T1) from its S_final (the state
    is the whole checkpoint of a sequence)."""
    _skip_unless(algo)
    x = to_cuda(I.make_prefill(2, 300, 4, 128, torch.bfloat16, -1.0, 0.05, seed=12))
    args = lambda s, e: (x["q"][:, s:e].contiguous(), x["k"][:, s:e].contiguous(),
                         x["v"][:, s:e].contiguous(), x["log_alpha"][:, s:e].contiguous(),
                         x["beta"][:, s:e].contiguous())
    o, Sf = kda.kda_chunk_fwd(*args(0, 300), x["S0"], algo=algo)
    oa, Sa = kda.kda_chunk_fwd(*args(0, 100), x["S0"], algo=algo)
    ob, Sb = kda.kda_chunk_fwd(*args(100, 300), Sa, algo=algo)
    assert rel_l2(torch.cat([oa, ob], 1), o.double().cpu().numpy()) <= 1e-2
    assert rel_l2(Sb, Sf.double().cpu().numpy()) <= 1e-2


@pytest.mark.parametrize("algo", ["simt", "tcgen05"])
def test_deterministic_and_in_place_state(algo):
    _skip_unless(algo)
    x = to_cuda(I.make_prefill(2, 260, 4, 128, torch.bfloat16, -1.0, 0.05, seed=13))
    a = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"])
    o1, S1 = kda.kda_chunk_fwd(*a, x["S0"], algo=algo)
    o2, S2 = kda.kda_chunk_fwd(*a, x["S0"], algo=algo)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    S = x["S0"].clone()
    o3, S3 = kda.kda_chunk_fwd(*a, S, S_final=S, algo=algo)  # S0 aliases S_final
    assert torch.equal(o3, o1) and torch.equal(S, S1)


def check_full_size(o, Sf, o_ref, S_ref, cu_seqlens=None):
    """Every (sequence, head) unit within the bf16 tolerance on its own (a fault
    in one unit is not diluted by the others), the whole tensors within it too,
    and the global errors within the regression guard (about twice the errors
    measured for the tensor-core path; not a tolerance)."""
    eo = unit_errors_o(o, o_ref, cu_seqlens)
    eS = unit_errors_S(Sf, S_ref)
    assert eo.max() <= TOL[torch.bfloat16], f"worst (sequence, head) of o: {eo.max():.3e}"
    assert eS.max() <= TOL[torch.bfloat16], f"worst (sequence, head) of S: {eS.max():.3e}"
    go, gS = rel_l2(o, o_ref), rel_l2(Sf, S_ref)
    assert go <= TOL[torch.bfloat16] and gS <= TOL[torch.bfloat16]
    assert go <= REGRESSION_GUARD["o"], f"o error {go:.3e} regressed"
    assert gS <= REGRESSION_GUARD["S"], f"S_final error {gS:.3e} regressed"


def test_chunked_config_full_size():
    """B=4, H=16, T=4096, d=128, bf16, S0 ~ N(0, 0.01): every output checked,
    each of the 64 (sequence, head) units on its own."""
    x = I.make_preset(I.CHUNKED)
    o, Sf, o_ref, S_ref = run_both(x)
    check_full_size(o, Sf, o_ref, S_ref)


@pytest.mark.slow
def test_long_context_config_sampled_heads():
    """B=1, H=32, T=131072, d=128, bf16, slow decay: the GPU runs all 32 heads;
    the oracle checks 8 of them end to end (heads are independent), each on its
    own."""
    x = I.make_preset(I.LONG)
    heads = [0, 4, 9, 13, 18, 21, 26, 31]
    o, Sf, o_ref, S_ref = run_both(x, heads=heads)
    check_full_size(o, Sf, o_ref, S_ref)


@pytest.mark.slow
def test_varlen_config_sampled_heads():
    """8 packed sequences of seeded lengths in [1024, 65536], H=32, d=128, bf16,
    per-sequence S0: the oracle checks every sequence on 3 heads, each
    (sequence, head) on its own."""
    x = I.make_preset(I.VARLEN)
    heads = [2, 17, 30]
    o, Sf, o_ref, S_ref = run_both(x, heads=heads)
    check_full_size(o, Sf, o_ref, S_ref, cu_seqlens=x["cu_seqlens"])


@pytest.mark.parametrize("algo", ["simt", "tcgen05"])
def test_prepare_then_carry_equals_one_call(algo):
    _skip_unless(algo)
    x = to_cuda(I.make_prefill(1, 0, 3, 128, torch.bfloat16, -1.0, 0.05, seed=14,
                               lengths=[70, 1, 200]))
    a = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], x["cu_seqlens"])
    o1, S1 = kda.kda_chunk_fwd(*a, algo=algo)
    call = kda.kda_chunk_fwd_prepare(*a, algo=algo)
    o2, S2 = kda.kda_chunk_fwd_carry(call)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("algo", ["simt", "tcgen05"])
@pytest.mark.parametrize("gate_shift", [1.0, 3.0])
def test_strong_decay_gates(algo, gate_shift):
    """Fast-forgetting gates: log_alpha = -softplus(N(0,1) + shift). With shift 1 a
    chunk decays by ~80 nats (the tensor-core prep switches to direct
    exponentials); with shift 3 half a chunk decays by ~100 nats (the chunk is
    recomputed by the exact fixup). Results must match the oracle either way."""
    _skip_unless(algo)
    x = I.make_prefill(2, 300, 3, 128, torch.bfloat16, gate_shift=gate_shift, s0_std=0.05,
                       seed=41)
    o, Sf, o_ref, S_ref = run_both(x, algo=algo)
    assert rel_l2(o, o_ref) <= 2e-2
    assert rel_l2(Sf, S_ref) <= 2e-2


@pytest.mark.parametrize("gate_shift", [-3.0, 0.0, 3.0])
def test_tcgen05_matches_simt(gate_shift):
    """The two GPU paths agree with each other on the same inputs."""
    if not _has_tc():
        pytest.skip("tcgen05 path not built")
    x = to_cuda(I.make_prefill(2, 333, 4, 128, torch.bfloat16, gate_shift, 0.05, seed=42))
    a = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    o1, S1 = kda.kda_chunk_fwd(*a, algo="simt")
    o2, S2 = kda.kda_chunk_fwd(*a, algo="tcgen05")
    assert rel_l2(o2, o1.double().cpu().numpy()) <= 2e-2
    assert rel_l2(S2, S1.double().cpu().numpy()) <= 2e-2
