"""The chunk-parallel backward's kernel bodies (csrc/kda_cbwd_body.cuh) compiled
for the host and run with one fiber per CUDA thread (tests/cuda_host), against
the fp64 oracle's backward. This checks the bodies' arithmetic, indexing and
barrier placement on the CPU. The per-chunk records they read are formed here
in numpy from their definition (the backward's prep writes the same matrices on the
GPU)."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import pins

HERE = os.path.dirname(os.path.abspath(__file__))
C = 64


@pytest.fixture(scope="module")
def host_lib(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ is not available")
    so = str(tmp_path_factory.mktemp("cbwd") / "cbwd_host.so")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run([gxx, "-O2", "-std=c++17", "-fPIC", "-shared", "-I", cuda_inc, "-o", so,
                    os.path.join(HERE, "cuda_host", "cbwd_host.cpp")], check=True)
    return ctypes.CDLL(so)


def _records(q, k, v, la, beta):
    """Per chunk: W, Ut, Qt, Kh (C x D), Pm (C x C), gamma (D), the tail padded
    with identity tokens (k = q = v = 0, beta = 0, log_alpha = 0)."""
    T, D = q.shape
    out = []
    for a in range(0, T, C):
        L = min(C, T - a)
        pad = lambda x: np.concatenate([x[a:a + L], np.zeros((C - L,) + x.shape[1:])])
        qc, kc, vc, lc, bc = pad(q), pad(k), pad(v), pad(la), pad(beta)
        g = np.cumsum(lc, 0)
        low = np.tril(np.ones((C, C)))
        E = np.exp(np.minimum(g[:, None] - g[None], 0.0)) * low[:, :, None]
        kk = np.einsum("rc,sc,rsc->rs", kc, kc, E) * np.tril(np.ones((C, C)), -1)
        Pm = np.einsum("rc,sc,rsc->rs", qc, kc, E)
        Ti = np.linalg.inv(np.eye(C) + bc[:, None] * kk)
        W = Ti @ (bc[:, None] * kc * np.exp(g))
        Ut = Ti @ (bc[:, None] * vc)
        out.append(np.concatenate([W.ravel(), Ut.ravel(), (qc * np.exp(g)).ravel(),
                                   (kc * np.exp(g[-1] - g)).ravel(), Pm.ravel(), np.exp(g[-1])]))
    return out


def _run(lib, lengths, H, D, gpc=True, s0=True, dsf=True, decay=1.0, seed=0, scale=0.3,
         own_prep=False, bf16=False):
    T, N = sum(lengths), len(lengths)
    q, k, v, la, b, _ = pins._rand(seed, B=1, T=T, H=H, dk=D, dv=D, unit_k=True)
    la = la * decay
    if bf16:  # both sides read the same bf16-rounded q, k, v and dO
        import torch
        rnd = lambda a: torch.from_numpy(a).to(torch.bfloat16).double().numpy()
        q, k, v = rnd(q), rnd(k), rnd(v)
    if not gpc:
        la = np.repeat(la[..., :1], D, axis=-1)
    r = np.random.default_rng(seed + 1)
    S0 = r.normal(size=(N, H, D, D)) * 0.3 if s0 else None
    dO = r.normal(size=v.shape)
    if bf16:
        dO = rnd(dO)
    dSf = r.normal(size=(N, H, D, D)) if dsf else None
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    ref = oracle.backward(q, k, v, la, b, dO, S0, dSf, cu, scale=scale)
    seq_start = cu.astype(np.int32)
    chunk_off = np.concatenate([[0], np.cumsum([(n + C - 1) // C for n in lengths])]).astype(np.int32)
    order = np.array(sorted(range(N), key=lambda n: (-lengths[n], n)), dtype=np.int32)
    n_alloc = int(chunk_off[-1]) + 1  # one chunk index past the end: must be skipped
    rec = np.zeros((n_alloc, H, 4 * C * D + C * C + D), np.float32)
    for n in range(N):
        for h in range(H):
            a, e = cu[n], cu[n + 1]
            for lc, x in enumerate(_records(q[0, a:e, h], k[0, a:e, h], v[0, a:e, h],
                                             la[0, a:e, h], b[0, a:e, h]) if e > a else []):
                rec[chunk_off[n] + lc, h] = x
    f32 = lambda x: None if x is None else np.ascontiguousarray(x, dtype=np.float32)
    big = lambda *s: np.zeros(s, np.float32)
    Sst, dSst = big(n_alloc, H, D, D), big(n_alloc, H, D, D)
    Ust, dUst = big(n_alloc, H, C, D), big(n_alloc, H, C, D)
    scr = big(n_alloc, H, 3 * C * D + C * C + D)
    nan = lambda s: np.full(s, np.nan, np.float32)
    rec_own = np.full(rec.shape, np.nan, np.float32)
    g = dict(dq=nan(q.shape), dk=nan(q.shape), dv=nan(v.shape),
             dlog_alpha=nan(la.shape if gpc else la.shape[:3]), dbeta=nan(b.shape),
             dS0=nan((N, H, D, D)))
    if bf16:
        import torch
        raw = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).view(torch.int16).numpy()
        tok = [raw(q), raw(k), raw(v), raw(dO)]
    else:
        tok = [f32(q), f32(k), f32(v), f32(dO)]
    args = tok + [f32(la if gpc else la[..., 0]), f32(b), f32(S0), f32(dSf)]
    ptr = lambda x: None if x is None else x.ctypes.data_as(ctypes.c_void_p)
    st = lib.cbwd_host_run(
        ctypes.c_int(D), ctypes.c_int(int(bf16)), *map(ptr, args), ctypes.c_int(N), ctypes.c_int(H), ctypes.c_int(int(gpc)),
        ctypes.c_float(scale), ptr(seq_start), ptr(chunk_off), ptr(order), ptr(rec), ptr(Sst),
        ptr(dSst), ptr(Ust), ptr(dUst), ptr(scr), ptr(g["dq"]), ptr(g["dk"]), ptr(g["dv"]),
        ptr(g["dlog_alpha"]), ptr(g["dbeta"]), ptr(g["dS0"]), ctypes.c_int(n_alloc),
        ptr(rec_own) if own_prep else None)
    assert st == 0
    if not gpc:
        ref["dlog_alpha"] = ref["dlog_alpha"].sum(-1)
    errs = {key: float(np.linalg.norm(g[key] - ref[key]) / np.linalg.norm(ref[key])) for key in g}
    assert all(np.isfinite(e) and e <= 2e-5 for e in errs.values()), errs
    if own_prep:  # the kernel's records equal the definition's on every live chunk
        live = np.zeros(n_alloc, bool)
        live[:chunk_off[-1]] = True
        np.testing.assert_allclose(rec_own[live], rec[live], rtol=0, atol=2e-4 * max(1.0, np.abs(rec).max()))


@pytest.mark.parametrize("kw", [
    dict(lengths=[70], H=1, D=32),
    dict(lengths=[150, 1, 64, 0, 65], H=2, D=32, seed=3),
    dict(lengths=[130], H=1, D=64, decay=4.0, seed=4),
    dict(lengths=[100], H=2, D=32, gpc=False, seed=5),
    dict(lengths=[90], H=1, D=32, s0=False, dsf=False, seed=6),
    dict(lengths=[70, 3], H=1, D=128, seed=9),
    dict(lengths=[130, 7], H=2, D=128, seed=10, bf16=True),
], ids=["one-seq", "varlen-empty", "strong-decay-d64", "head-gate", "no-states", "d128",
        "bf16-d128"])
@pytest.mark.parametrize("own_prep", [False, True], ids=["given-records", "own-prep"])
def test_chunked_backward_bodies_on_host(host_lib, kw, own_prep):
    _run(host_lib, **kw, own_prep=own_prep)
