"""kda_chunk_bwd / kda_gdn_chunk_bwd / kda_chunk_bwd_ex on the GPU against the
fp64 oracle's backward (itself pinned by central differences of the forward):
every gradient of <dO, o> + <dS_final, S_final>, element by element, on the
same inputs, for both backward algorithms (the token walk and the
chunk-parallel form)."""
import numpy as np
import pytest
import torch

import oracle
from common import rel_l2
from gated_delta_rule_132_b200 import inputs as I
from gated_delta_rule_132_b200 import kda

pytestmark = pytest.mark.gpu

TOL = 1e-4  # fp32 arithmetic on both gate forms; the oracle sees the same input values
KEYS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def _problem(B, T, H, d, dtype, seed, lengths=None, s0=True):
    x = I.make_prefill(B, T, H, d, dtype, gate_shift=-1.0, s0_std=0.1 if s0 else 0.0,
                       seed=seed, lengths=lengths)
    g = torch.Generator().manual_seed(seed + 1)
    N = B if lengths is None else len(lengths)
    dO = torch.randn(x["v"].shape, generator=g).to(dtype)
    dSf = torch.randn((N, H, d, d), generator=g) if s0 else None
    return x, dO, dSf


ALGOS = ["token", "chunked"]


def _check(x, dO, dSf, gate="channel", algo="auto"):
    la = x["log_alpha"] if gate == "channel" else x["log_alpha"][..., 0].contiguous()
    la_full = la if gate == "channel" else la[..., None].expand_as(x["log_alpha"]).contiguous()
    dev = lambda t: None if t is None else t.cuda()
    got = kda.kda_chunk_bwd(dev(x["q"]), dev(x["k"]), dev(x["v"]), la.cuda(), dev(x["beta"]),
                            dO.cuda(), dev(x["S0"]), dev(x["cu_seqlens"]), x["scale"],
                            dev(dSf), gate=gate, algo=algo)
    torch.cuda.synchronize()
    ref = oracle.backward(x["q"], x["k"], x["v"], la_full, x["beta"], dO, x["S0"], dSf,
                          x["cu_seqlens"], scale=x["scale"])
    if gate == "head":
        ref["dlog_alpha"] = ref["dlog_alpha"].sum(axis=-1)
    errs = {key: rel_l2(got[key], ref[key]) for key in KEYS}
    assert all(np.isfinite(e) and e <= TOL for e in errs.values()), errs


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype,d", [(torch.float32, 32), (torch.float32, 64),
                                     (torch.float32, 128), (torch.bfloat16, 128)])
def test_backward_crossing_checkpoints(dtype, d, algo):
    """70 tokens per sequence: two full 32-token replay blocks and a ragged one
    (one full 64-token chunk and a ragged one)."""
    _check(*_problem(2, 70, 2, d, dtype, seed=700 + d), algo=algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_backward_varlen_with_empty_sequence(algo):
    _check(*_problem(1, 0, 2, 64, torch.float32, seed=710, lengths=[5, 0, 65, 130]), algo=algo)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("gate_dtype", [torch.float32, torch.bfloat16])
def test_backward_one_gate_per_head(gate_dtype, algo):
    _check(*_problem(2, 100, 2, 128 if gate_dtype == torch.bfloat16 else 32, gate_dtype,
                     seed=720), gate="head", algo=algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_backward_without_states(algo):
    """S0 and dS_final absent (zero); the initial-state gradient still comes back."""
    x, dO, dSf = _problem(1, 90, 3, 64, torch.float32, seed=730, s0=False)
    _check(x, dO, dSf, algo=algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_backward_long_bf16(algo):
    """300 tokens (five checkpoint blocks, five chunks), 4 heads, d = 128, bf16 inputs."""
    _check(*_problem(1, 300, 4, 128, torch.bfloat16, seed=740), algo=algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_backward_block_edges(algo):
    """Lengths around the 32-token replay block and the 64-token chunk."""
    _check(*_problem(1, 0, 2, 64, torch.float32, seed=750, lengths=[1, 31, 32, 33, 64, 65]),
           algo=algo)


def test_backward_chunked_strong_decay():
    """Gates far outside any factorised range: the chunked form takes only
    exponentials of non-positive numbers."""
    x = I.make_prefill(1, 200, 2, 64, torch.float32, gate_shift=3.0, s0_std=0.1, seed=770)
    g = torch.Generator().manual_seed(771)
    dO = torch.randn(x["v"].shape, generator=g)
    dSf = torch.randn((1, 2, 64, 64), generator=g)
    _check(x, dO, dSf, algo="chunked")


def test_backward_algorithms_agree():
    """The two algorithms on the same bf16 problem agree to fp32 rounding."""
    x, dO, dSf = _problem(2, 200, 3, 128, torch.bfloat16, seed=780)
    dev = lambda t: None if t is None else t.cuda()
    args = (dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["beta"]),
            dO.cuda(), dev(x["S0"]), None, x["scale"], dev(dSf))
    a = kda.kda_chunk_bwd(*args, algo="token")
    b = kda.kda_chunk_bwd(*args, algo="chunked")
    for key in KEYS:
        assert rel_l2(b[key], a[key].double().cpu().numpy()) <= 2e-5, key


def test_backward_leaves_tokens_outside_sequences_unwritten():
    """cu_seqlens ending before B*T: the trailing tokens keep what the caller put there;
    the covered ones match the oracle (they do not depend on later sequences)."""
    x, dO, dSf = _problem(1, 0, 2, 128, torch.float32, seed=760, lengths=[40, 30, 10])
    ref = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dO, x["S0"], dSf,
                          x["cu_seqlens"], scale=x["scale"])
    cu = x["cu_seqlens"][:3].cuda()
    B, T, H, d = x["q"].shape
    sentinel = 12345.0
    out = {key: torch.full(ref[key].shape, sentinel, device="cuda") for key in KEYS}
    out["dS0"] = torch.full((2, H, d, d), sentinel, device="cuda")
    dev = {key: x[key].cuda() for key in ("q", "k", "v", "log_alpha", "beta", "S0")}
    dS0_in = dev["S0"][:2].contiguous()
    dSf2 = dSf[:2].contiguous().cuda()
    dOc = dO.cuda()
    need = int(kda.lib().kda_chunk_bwd_workspace_size(B, T, H, d, d, 2, kda._dt(dev["q"])))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = kda.lib().kda_chunk_bwd(
        kda._p(dev["q"]), kda._p(dev["k"]), kda._p(dev["v"]), kda._dt(dev["q"]),
        kda._p(dev["log_alpha"]), kda._p(dev["beta"]), kda._p(dS0_in), kda._p(cu), 2, B, T, H,
        d, d, float(x["scale"]), kda._p(dOc), kda._p(dSf2), kda._p(out["dq"]),
        kda._p(out["dk"]), kda._p(out["dv"]), kda._p(out["dlog_alpha"]), kda._p(out["dbeta"]),
        kda._p(out["dS0"]), kda._p(ws), need, kda._stream(None))
    assert st == 0
    torch.cuda.synchronize()
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        got = out[key].cpu()
        assert torch.all(got[:, 70:] == sentinel), key
        assert rel_l2(got[:, :70], ref[key][:, :70]) <= TOL, key
    assert rel_l2(out["dS0"].cpu(), ref["dS0"][:2]) <= TOL


def test_backward_chunked_leaves_tokens_outside_sequences_unwritten():
    """As above, through kda_chunk_bwd_ex with the chunk-parallel algorithm."""
    x, dO, dSf = _problem(1, 0, 2, 64, torch.float32, seed=761, lengths=[40, 30, 10])
    ref = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dO, x["S0"], dSf,
                          x["cu_seqlens"], scale=x["scale"])
    cu = x["cu_seqlens"][:3].cuda()
    B, T, H, d = x["q"].shape
    sentinel = 12345.0
    out = {key: torch.full(ref[key].shape, sentinel, device="cuda") for key in KEYS}
    out["dS0"] = torch.full((2, H, d, d), sentinel, device="cuda")
    dev = {key: x[key].cuda() for key in ("q", "k", "v", "log_alpha", "beta", "S0")}
    S0 = dev["S0"][:2].contiguous()
    dSf2 = dSf[:2].contiguous().cuda()
    dOc = dO.cuda()
    L = kda.lib()
    need = int(L.kda_chunk_bwd_workspace_size_ex(B, T, H, d, d, 2, kda._dt(dev["q"]), 2))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = L.kda_chunk_bwd_ex(
        kda._p(dev["q"]), kda._p(dev["k"]), kda._p(dev["v"]), kda._dt(dev["q"]),
        kda._p(dev["log_alpha"]), kda._p(dev["beta"]), kda._p(S0), kda._p(cu), 2, B, T, H,
        d, d, float(x["scale"]), kda._p(dOc), kda._p(dSf2), kda._p(out["dq"]),
        kda._p(out["dk"]), kda._p(out["dv"]), kda._p(out["dlog_alpha"]), kda._p(out["dbeta"]),
        kda._p(out["dS0"]), kda._p(ws), need, 1, 2, kda._stream(None))
    assert st == 0
    torch.cuda.synchronize()
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        got = out[key].cpu()
        assert torch.all(got[:, 70:] == sentinel), key
        assert rel_l2(got[:, :70], ref[key][:, :70]) <= TOL, key
    assert rel_l2(out["dS0"].cpu(), ref["dS0"][:2]) <= TOL


@pytest.mark.slow
@pytest.mark.parametrize("algo", ALGOS)
def test_backward_bench_shape_sampled_heads(algo):
    """The benchmark's backward shape and launch configuration (B=1, H=32, T=8192,
    d=128, bf16 inputs, slow decay; token walk: 128 CTAs, 256 replay blocks per
    CTA; chunked: 128 chunks x 32 heads per chunk-parallel kernel). The GPU
    computes all 32 heads. The oracle checks 8 of them, since heads are independent."""
    P = I.LONG
    x = I.make_prefill(1, 8192, P.H, P.d, P.dtype, P.gate_shift, 0.0, P.seed + 1000)
    g = torch.Generator().manual_seed(P.seed + 7)
    dO = torch.randn(x["v"].shape, generator=g).to(P.dtype)
    got = kda.kda_chunk_bwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["log_alpha"].cuda(),
                            x["beta"].cuda(), dO.cuda(), scale=x["scale"], algo=algo)
    torch.cuda.synchronize()
    heads = [0, 4, 9, 13, 18, 22, 27, 31]
    sel = lambda t: t[:, :, heads].contiguous()
    ref = oracle.backward(sel(x["q"]), sel(x["k"]), sel(x["v"]), sel(x["log_alpha"]),
                          sel(x["beta"]), sel(dO), scale=x["scale"])
    errs = {key: rel_l2(got[key][:, :, heads], ref[key]) for key in KEYS if key != "dS0"}
    errs["dS0"] = rel_l2(got["dS0"][:, heads], ref["dS0"])
    assert all(np.isfinite(e) and e <= TOL for e in errs.values()), errs
