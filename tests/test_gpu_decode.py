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
