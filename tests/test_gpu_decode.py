"""kda_decode_step on the GPU against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from common import TOL, rel_l2
from gated_delta_rule_132_b200 import inputs as I
from gated_delta_rule_132_b200 import kda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_small_chain(d, dtype):
    N, H = 5, 3
    S = I.make_decode_state(N, H, d, 0.05, seed=100 + d)
    S_gpu = S.cuda()
    S_ref = S.double().numpy()
    for step in range(4):
        tok = I.make_decode_token(N, H, d, dtype, -2.0, seed=200 + step)
        o = kda.kda_decode_step(**{k: v.cuda() for k, v in tok.items()}, S=S_gpu)
        o_ref, S_ref = oracle.decode_step(**tok, S=S_ref)
        assert rel_l2(o, o_ref) <= TOL[dtype]
        assert rel_l2(S_gpu, S_ref) <= TOL[torch.float32]


def test_decode_full_batch_256x32_first_steps_and_long_chain_subset():
    """The decode workload at full size: 256 sequences x 32 heads x 128 x 128
    state (537 MB). All 10 first steps are checked on the whole batch; then the
    chain runs to 1000 steps and a seeded subset of 16 sequences is checked at
    every step (units are independent, so the subset is exact)."""
    P = I.DECODE
    S = I.make_decode_state(P.N, P.H, P.d, P.s_std, P.seed)
    S_gpu = S.cuda()
    subset = torch.randperm(P.N, generator=torch.Generator().manual_seed(7))[:16].sort().values
    S_ref_full = S.double().numpy()
    S_ref = None
    worst_o = 0.0
    for step in range(P.steps):
        tok = I.make_decode_token(P.N, P.H, P.d, P.dtype, P.gate_shift,
                                  seed=P.step_seed0 + step)
        o = kda.kda_decode_step(**{k: v.cuda(non_blocking=True) for k, v in tok.items()},
                                S=S_gpu)
        if step < 10:
            o_ref, S_ref_full = oracle.decode_step(**tok, S=S_ref_full)
            assert rel_l2(o, o_ref) <= TOL[P.dtype], step
            if step == 9:
                assert rel_l2(S_gpu, S_ref_full) <= 1e-4
                S_ref = S_ref_full[subset.numpy()]
        else:
            sub = {k: v[subset] for k, v in tok.items()}
            o_ref, S_ref = oracle.decode_step(**sub, S=S_ref)
            worst_o = max(worst_o, rel_l2(o[subset.cuda()], o_ref))
    assert worst_o <= TOL[P.dtype]
    assert rel_l2(S_gpu[subset.cuda()], S_ref) <= 1e-4


def test_decode_is_deterministic():
    N, H, d = 7, 4, 128
    S = I.make_decode_state(N, H, d, 0.05, seed=3).cuda()
    tok = {k: v.cuda() for k, v in I.make_decode_token(N, H, d, seed=4).items()}
    S1, S2 = S.clone(), S.clone()
    o1 = kda.kda_decode_step(**tok, S=S1)
    o2 = kda.kda_decode_step(**tok, S=S2)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


# ----------------------------------------------------------------- multi-token decode
def _tokens_problem(N, T, H, d, dtype, seed):
    x = I.make_prefill(N, T, H, d, dtype, gate_shift=-2.0, seed=seed)
    S = I.make_decode_state(N, H, d, 0.05, seed=seed + 1)
    return x, S


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 2, 7, 33])
def test_decode_tokens_vs_oracle(T, dtype, d):
    """T tokens in one call against the fp64 token-by-token forward started from S."""
    N, H = 3, 2
    x, S = _tokens_problem(N, T, H, d, dtype, seed=300 + T + d)
    S_gpu = S.cuda()
    o = kda.kda_decode_tokens(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(),
                              x["log_alpha"].cuda(), x["beta"].cuda(), S_gpu, scale=x["scale"])
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S0=S,
                                  scale=x["scale"])
    assert o.shape == (N, T, H, d)
    assert rel_l2(o, o_ref) <= TOL[dtype]
    assert rel_l2(S_gpu, S_ref) <= TOL[torch.float32]


def test_decode_tokens_equals_chained_steps():
    """One T-token call and T single-step calls apply the same rule to the same
    fp32 state; only the order of the fp32 sums over the key rows differs (warp
    shuffles against shared-memory row groups), so they agree to rounding."""
    N, T, H, d = 4, 5, 3, 128
    x, S = _tokens_problem(N, T, H, d, torch.bfloat16, seed=41)
    g = {k: v.cuda() for k, v in x.items() if isinstance(v, torch.Tensor)}
    S1, S2 = S.cuda(), S.cuda()
    o1 = kda.kda_decode_tokens(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S1,
                               scale=x["scale"])
    for t in range(T):
        o2 = kda.kda_decode_step(g["q"][:, t].contiguous(), g["k"][:, t].contiguous(),
                                 g["v"][:, t].contiguous(), g["log_alpha"][:, t].contiguous(),
                                 g["beta"][:, t].contiguous(), S2, scale=x["scale"])
        assert rel_l2(o1[:, t], o2.double().cpu().numpy()) <= 4e-3, t  # a bf16 rounding step
    assert rel_l2(S1, S2.double().cpu().numpy()) <= 1e-5


def test_decode_tokens_matches_prefill_continuation():
    """Continuing from a state with T tokens equals the chunked prefill with
    S0 = that state (both within the bf16 tolerance of the oracle)."""
    N, T, H, d = 2, 24, 4, 128
    x, S = _tokens_problem(N, T, H, d, torch.bfloat16, seed=52)
    g = {k: v.cuda() for k, v in x.items() if isinstance(v, torch.Tensor)}
    S_dec = S.cuda()
    o_dec = kda.kda_decode_tokens(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S_dec,
                                  scale=x["scale"])
    o_pre, S_pre = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"],
                                     S0=S.cuda(), scale=x["scale"])
    assert rel_l2(o_dec, o_pre.float().cpu()) <= TOL[torch.bfloat16]
    assert rel_l2(S_dec, S_pre.cpu()) <= 1e-2


def test_decode_tokens_zero_tokens_leaves_state():
    N, H, d = 2, 2, 64
    S = I.make_decode_state(N, H, d, 0.05, seed=9).cuda()
    S0 = S.clone()
    e = torch.empty((N, 0, H, d), device="cuda")
    o = kda.kda_decode_tokens(e, e, e, e, torch.empty((N, 0, H), device="cuda"), S)
    assert o.shape == (N, 0, H, d) and torch.equal(S, S0)


def test_decode_tokens_full_batch_sampled():
    """Decode workload shape (256 sequences x 32 heads, d=128) with 8 tokens per
    call; a seeded subset of 16 sequences is checked against the oracle (units
    are independent, so the subset is exact)."""
    P = I.DECODE
    T = 8
    x = I.make_prefill(P.N, T, P.H, P.d, P.dtype, gate_shift=P.gate_shift, seed=77)
    S = I.make_decode_state(P.N, P.H, P.d, P.s_std, P.seed)
    subset = torch.randperm(P.N, generator=torch.Generator().manual_seed(8))[:16].sort().values
    S_gpu = S.cuda()
    o = kda.kda_decode_tokens(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(),
                              x["log_alpha"].cuda(), x["beta"].cuda(), S_gpu, scale=x["scale"])
    sub = {k: x[k][subset] for k in ("q", "k", "v", "log_alpha", "beta")}
    o_ref, S_ref = oracle.forward(**sub, S0=S[subset], scale=x["scale"])
    assert rel_l2(o[subset.cuda()], o_ref) <= TOL[P.dtype]
    assert rel_l2(S_gpu[subset.cuda()], S_ref) <= 1e-4
