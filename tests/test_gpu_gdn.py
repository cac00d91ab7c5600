"""The GDN entry points (one gate per token and head) on the GPU against the
fp64 oracle, which receives the gate broadcast over the channels: the rule with
Diag(alpha_t) = alpha_t I."""
import pytest
import torch

import oracle
from common import TOL, rel_l2
from gated_delta_rule_132_b200 import inputs as I
from gated_delta_rule_132_b200 import kda

pytestmark = pytest.mark.gpu

PATHS = [("simt", torch.float32, 32), ("simt", torch.float32, 128),
         ("simt", torch.bfloat16, 128), ("tcgen05", torch.bfloat16, 128)]


def gdn(x):
    """The per-head gate: channel 0 of the generated per-channel gate (same
    distribution), and its broadcast over the channels for the oracle."""
    la = x["log_alpha"][..., 0].contiguous()
    return la, la[..., None].expand_as(x["log_alpha"]).contiguous()


def run_gdn(x, algo="auto"):
    la, la_full = gdn(x)
    dev = lambda t: None if t is None else t.cuda()
    o, Sf = kda.kda_gdn_chunk_fwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), la.cuda(),
                                  dev(x["beta"]), dev(x["S0"]), dev(x["cu_seqlens"]),
                                  x["scale"], algo=algo)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], la_full, x["beta"], x["S0"],
                                  x["cu_seqlens"], scale=x["scale"])
    return o, Sf, o_ref, S_ref


@pytest.mark.parametrize("algo,dtype,d", PATHS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_gdn_prefill_lengths(algo, dtype, d, T):
    x = I.make_prefill(2, T, 3, d, dtype, gate_shift=-1.0, s0_std=0.05, seed=600 + T + d)
    o, Sf, o_ref, S_ref = run_gdn(x, algo)
    assert rel_l2(o, o_ref) <= TOL[dtype]
    assert rel_l2(Sf, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("algo", ["simt", "tcgen05"])
def test_gdn_prefill_varlen(algo):
    x = I.make_prefill(1, 0, 4, 128, torch.bfloat16, gate_shift=-2.0, s0_std=0.01, seed=61,
                       lengths=[1, 64, 100, 0, 333, 65])
    o, Sf, o_ref, S_ref = run_gdn(x, algo)
    assert rel_l2(o, o_ref) <= TOL[torch.bfloat16]
    assert rel_l2(Sf, S_ref) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("shift", [1.0, 4.0])
def test_gdn_strong_decay(shift):
    """Gates far below zero (e^{g} underflows inside a chunk): every factor the
    scalar-gate prep forms is e^{<= 0}, so nothing overflows."""
    x = I.make_prefill(1, 300, 2, 128, torch.bfloat16, gate_shift=shift, s0_std=0.05, seed=62)
    x["log_alpha"] = x["log_alpha"] * 8.0
    o, Sf, o_ref, S_ref = run_gdn(x, "tcgen05")
    assert torch.isfinite(o).all() and torch.isfinite(Sf).all()
    assert rel_l2(o, o_ref) <= TOL[torch.bfloat16]
    assert rel_l2(Sf, S_ref) <= TOL[torch.bfloat16]


def test_gdn_equals_kda_with_broadcast_gate():
    """The GDN path and the per-channel path given the broadcast gate compute
    the same function (both within the bf16 tolerance of each other)."""
    x = I.make_prefill(2, 500, 4, 128, torch.bfloat16, gate_shift=-2.0, s0_std=0.02, seed=63)
    la, la_full = gdn(x)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    o1, S1 = kda.kda_gdn_chunk_fwd(g["q"], g["k"], g["v"], la.cuda(), g["beta"], g["S0"],
                                   scale=x["scale"])
    o2, S2 = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], la_full.cuda(), g["beta"], g["S0"],
                               scale=x["scale"])
    assert rel_l2(o1, o2.float().cpu()) <= 1e-2
    assert rel_l2(S1, S2.cpu()) <= 1e-2


def test_gdn_prepare_then_carry():
    x = I.make_prefill(1, 1000, 4, 128, torch.bfloat16, gate_shift=-2.0, s0_std=0.01, seed=64)
    la, la_full = gdn(x)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    call = kda.ChunkFwdCall(g["q"], g["k"], g["v"], la.cuda(), g["beta"], g["S0"], None,
                            x["scale"], gate="head")
    call.prepare()
    o, Sf = call.carry()
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], la_full, x["beta"], x["S0"],
                                  scale=x["scale"])
    assert rel_l2(o, o_ref) <= TOL[torch.bfloat16]
    assert rel_l2(Sf, S_ref) <= TOL[torch.bfloat16]


def test_gdn_long_sampled_heads():
    """The long-context shape (B=1, H=32, T=131072) with per-head gates; 2 heads
    go through the oracle (heads are independent, so the subset is exact)."""
    P = I.LONG
    x = I.make_prefill(P.B, P.T, P.H, P.d, P.dtype, P.gate_shift, P.s0_std, P.seed)
    la, la_full = gdn(x)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    o, Sf = kda.kda_gdn_chunk_fwd(g["q"], g["k"], g["v"], la.cuda(), g["beta"], g["S0"],
                                  scale=x["scale"])
    heads = [3, 29]
    sub = lambda t: t[:, :, heads].contiguous()
    o_ref, S_ref = oracle.forward(sub(x["q"]), sub(x["k"]), sub(x["v"]), sub(la_full),
                                  sub(x["beta"]), None, scale=x["scale"])
    assert rel_l2(o[:, :, heads], o_ref) <= TOL[P.dtype]
    assert rel_l2(Sf[:, heads], S_ref) <= TOL[P.dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gdn_decode_tokens(dtype):
    N, T, H, d = 3, 9, 2, 128
    x = I.make_prefill(N, T, H, d, dtype, gate_shift=-2.0, seed=65)
    la, la_full = gdn(x)
    S = I.make_decode_state(N, H, d, 0.05, seed=66)
    S_gpu = S.cuda()
    o = kda.kda_decode_tokens(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), la.cuda(),
                              x["beta"].cuda(), S_gpu, scale=x["scale"], gate="head")
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], la_full, x["beta"], S0=S,
                                  scale=x["scale"])
    assert rel_l2(o, o_ref) <= TOL[dtype]
    assert rel_l2(S_gpu, S_ref) <= TOL[torch.float32]
