"""Pins for the fp64 oracle: facts about the KDA recurrence that hold
independently of the oracle's own code.

Each ``pin_*`` function takes an oracle binding (``oracle.OracleLib``) and
returns the largest deviation it finds (0 for a perfect match); ``TOL`` gives
the bound each must meet. Every check is written from the mathematics of the
update rule in "Kimi Linear：让长上下文大模型真正实用的线性注意力架构", section
三 5️⃣ (S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T),
the per-channel gate of section 三 1️⃣ and the read-out o_t = scale S_t^T q_t —
not by re-calling or retyping the oracle's loop. The same functions run
against deliberately broken builds of the oracle to show that each planted
mistake trips at least one of them.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

TOL = {
    "p1_bruteforce": 1e-12,
    "p1_bruteforce_rect": 1e-12,
    "p2_deltanet": 1e-12,
    "p3_gdn_scalar_gate": 1e-12,
    "p4_pure_decay": 1e-12,
    "p5_exact_write": 1e-12,
    "p6_orthonormal_keys": 1e-12,
    "p7_online_gradient_step": 1e-6,
    "p8a_value_columns_independent": 1e-12,
    "p8b_decode_chain_equals_prefill": 1e-12,
    "p8c_split_prefill": 1e-12,
    "p8d_varlen_equals_separate": 1e-12,
    "p9_non_expansion": 1e-12,
    "golden_hand_example": 1e-12,
}


def _rand(seed, B=2, T=12, H=2, dk=6, dv=6, s0=True, unit_k=False):
    r = np.random.default_rng(seed)
    q = r.normal(size=(B, T, H, dk))
    k = r.normal(size=(B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.normal(size=(B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-r.normal(size=(B, T, H))))
    log_alpha = -np.log1p(np.exp(r.normal(size=(B, T, H, dk))))
    S0 = r.normal(size=(B, H, dk, dv)) if s0 else None
    return q, k, v, log_alpha, beta, S0


def _dense_reference(q, k, v, log_alpha, beta, S0, scale):
    """Brute force: form the dk x dk transition M_t = (I - beta k k^T) Diag(alpha)
    as a dense matrix and apply it with a matrix product."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    Sf = np.zeros((B, H, dk, dv))
    I = np.eye(dk)
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for t in range(T):
                kt = k[b, t, h][:, None]
                M = (I - beta[b, t, h] * (kt @ kt.T)) @ np.diag(np.exp(log_alpha[b, t, h]))
                S = M @ S + beta[b, t, h] * (kt @ v[b, t, h][None, :])
                o[b, t, h] = scale * (S.T @ q[b, t, h])
            Sf[b, h] = S
    return o, Sf


def _maxdiff(*pairs):
    return max(float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) for a, b in pairs)


def pin_p1_bruteforce(orc):
    q, k, v, la, b, S0 = _rand(11)
    scale = 0.37
    o, Sf = orc.forward(q, k, v, la, b, S0, scale=scale)
    ro, rS = _dense_reference(q, k, v, la, b, S0, scale)
    return _maxdiff((o, ro), (Sf, rS))


def pin_p1_bruteforce_rect(orc):
    """Same as P1 with dk != dv, so a swapped row/column index cannot pass."""
    q, k, v, la, b, S0 = _rand(12, B=1, T=9, H=3, dk=5, dv=3)
    scale = 5 ** -0.5
    o, Sf = orc.forward(q, k, v, la, b, S0, scale=scale)
    ro, rS = _dense_reference(q, k, v, la, b, S0, scale)
    return _maxdiff((o, ro), (Sf, rS))


def pin_p2_deltanet(orc):
    """alpha == 1 (log_alpha == 0) is the DeltaNet update
    S_t = S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T."""
    q, k, v, la, b, S0 = _rand(21)
    la = np.zeros_like(la)
    scale = 0.5
    o, Sf = orc.forward(q, k, v, la, b, S0, scale=scale)
    B, T, H, _ = q.shape
    err = 0.0
    for bb in range(B):
        for h in range(H):
            S = S0[bb, h].copy()
            for t in range(T):
                kt, vt = k[bb, t, h], v[bb, t, h]
                S = S + b[bb, t, h] * np.outer(kt, vt - S.T @ kt)
                err = max(err, _maxdiff((o[bb, t, h], scale * S.T @ q[bb, t, h])))
            err = max(err, _maxdiff((Sf[bb, h], S)))
    return err


def pin_p3_gdn_scalar_gate(orc):
    """alpha_t constant across channels (a_t * 1) is per-head scalar gating:
    S_t = a_t (S_{t-1} - beta_t k_t k_t^T S_{t-1}) + beta_t k_t v_t^T."""
    q, k, v, la, b, S0 = _rand(31)
    la = np.repeat(la[..., :1], la.shape[-1], axis=-1)
    scale = 0.25
    o, Sf = orc.forward(q, k, v, la, b, S0, scale=scale)
    B, T, H, _ = q.shape
    err = 0.0
    for bb in range(B):
        for h in range(H):
            S = S0[bb, h].copy()
            for t in range(T):
                a = math.exp(la[bb, t, h, 0])
                kt = k[bb, t, h]
                S = a * (S - b[bb, t, h] * np.outer(kt, kt @ S)) \
                    + b[bb, t, h] * np.outer(kt, v[bb, t, h])
                err = max(err, _maxdiff((o[bb, t, h], scale * S.T @ q[bb, t, h])))
            err = max(err, _maxdiff((Sf[bb, h], S)))
    return err


def pin_p4_pure_decay(orc):
    """beta == 0: S_t = Diag(exp(sum_{s<=t} log_alpha_s)) S_0 in closed form."""
    q, k, v, la, b, S0 = _rand(41)
    b = np.zeros_like(b)
    scale = 0.8
    o, Sf = orc.forward(q, k, v, la, b, S0, scale=scale)
    G = np.cumsum(la, axis=1)                           # [B,T,H,dk]
    St = np.exp(G)[..., None] * S0[:, None]             # [B,T,H,dk,dv]
    ro = scale * np.einsum("bthij,bthi->bthj", St, q)
    return _maxdiff((o, ro), (Sf, St[:, -1]))


def pin_p5_exact_write(orc):
    """|k_t| = 1 and beta_t = 1: the update writes v_t exactly at key k_t,
    k_t^T S_t = v_t^T. Reading out with q_t = k_t therefore returns scale*v_t."""
    q, k, v, la, b, S0 = _rand(51, unit_k=True)
    b = np.ones_like(b)
    scale = 0.3
    o, Sf = orc.forward(k, k, v, la, b, S0, scale=scale)
    last = np.einsum("bhi,bhij->bhj", k[:, -1], Sf)
    return _maxdiff((o, scale * v), (last, v[:, -1]))


def pin_p6_orthonormal_keys(orc):
    """S0 = 0 and k_t = e_t (T <= dk): row s of the state is written once, at
    t = s, with beta_s v_s and then only decays, so
    o_t = scale * sum_{s<=t} q_t[s] exp(sum_{r=s+1..t} log_alpha_r[s]) beta_s v_s."""
    B, T, H, dk, dv = 2, 7, 2, 8, 5
    q, _, v, la, b, _ = _rand(61, B=B, T=T, H=H, dk=dk, dv=dv, s0=False)
    k = np.zeros((B, T, H, dk))
    for t in range(T):
        k[:, t, :, t] = 1.0
    scale = 0.6
    o, Sf = orc.forward(q, k, v, la, b, None, scale=scale)
    ro = np.zeros_like(o)
    rS = np.zeros_like(Sf)
    for bb in range(B):
        for h in range(H):
            for t in range(T):
                for s in range(t + 1):
                    w = math.exp(la[bb, s + 1:t + 1, h, s].sum()) * b[bb, s, h]
                    ro[bb, t, h] += scale * q[bb, t, h, s] * w * v[bb, s, h]
            for s in range(T):
                rS[bb, h, s] = math.exp(la[bb, s + 1:, h, s].sum()) * b[bb, s, h] * v[bb, s, h]
    return _maxdiff((o, ro), (Sf, rS))


def pin_p7_online_gradient_step(orc):
    """The delta rule is one gradient step on L(S) = 1/2 |S^T k - v|^2 taken
    from the decayed state S' = Diag(alpha) S_{t-1}, with step size beta:
    S_t = S' - beta * grad L(S'). The gradient is taken by central finite
    differences (exact up to rounding for a quadratic)."""
    r = np.random.default_rng(71)
    dk, dv = 4, 3
    err = 0.0
    for _ in range(3):
        Sp = r.normal(size=(dk, dv))
        k = r.normal(size=dk)
        v = r.normal(size=dv)
        q = r.normal(size=dk)
        la = -np.log1p(np.exp(r.normal(size=dk)))
        beta = float(1 / (1 + math.exp(-r.normal())))
        o, Sf = orc.forward(q[None, None, None], k[None, None, None], v[None, None, None],
                            la[None, None, None], np.array([[[beta]]]), Sp[None, None],
                            scale=1.0)
        Sdec = np.exp(la)[:, None] * Sp

        def L(S):
            e = S.T @ k - v
            return 0.5 * float(e @ e)

        g = np.zeros_like(Sdec)
        hstep = 1e-4
        for i in range(dk):
            for j in range(dv):
                Ep = Sdec.copy(); Ep[i, j] += hstep
                Em = Sdec.copy(); Em[i, j] -= hstep
                g[i, j] = (L(Ep) - L(Em)) / (2 * hstep)
        St = Sdec - beta * g
        err = max(err, _maxdiff((Sf[0, 0], St), (o[0, 0, 0], St.T @ q)))
    return err


def pin_p8a_value_columns_independent(orc):
    """The columns of S (value channels) never mix: slicing v and S0 by
    columns gives the column slice of the full result."""
    q, k, v, la, b, S0 = _rand(81, dk=6, dv=8)
    o, Sf = orc.forward(q, k, v, la, b, S0)
    cols = [1, 4, 7]
    o2, Sf2 = orc.forward(q, k, v[..., cols], la, b, S0[..., cols])
    return _maxdiff((o[..., cols], o2), (Sf[..., cols], Sf2))


def pin_p8b_decode_chain_equals_prefill(orc):
    """T single-token decode steps reproduce the T-token forward."""
    q, k, v, la, b, S0 = _rand(82, B=3, T=10)
    o, Sf = orc.forward(q, k, v, la, b, S0)
    S = S0.copy()
    err = 0.0
    for t in range(q.shape[1]):
        ot, S = orc.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], b[:, t], S)
        err = max(err, _maxdiff((ot, o[:, t])))
    return max(err, _maxdiff((S, Sf)))


def pin_p8c_split_prefill(orc):
    """forward(T) == forward(T1) followed by forward(T - T1) from its S_final."""
    q, k, v, la, b, S0 = _rand(83, T=13)
    o, Sf = orc.forward(q, k, v, la, b, S0)
    T1 = 5
    oa, Sa = orc.forward(q[:, :T1], k[:, :T1], v[:, :T1], la[:, :T1], b[:, :T1], S0)
    ob, Sb = orc.forward(q[:, T1:], k[:, T1:], v[:, T1:], la[:, T1:], b[:, T1:], Sa)
    return _maxdiff((np.concatenate([oa, ob], axis=1), o), (Sb, Sf))


def pin_p8d_varlen_equals_separate(orc):
    """Packing sequences along time with cu_seqlens equals separate calls."""
    lens = [3, 1, 7, 5]
    T = sum(lens)
    q, k, v, la, b, _ = _rand(84, B=1, T=T)
    r = np.random.default_rng(85)
    S0 = r.normal(size=(len(lens), q.shape[2], q.shape[3], v.shape[3]))
    cu = np.cumsum([0] + lens)
    o, Sf = orc.forward(q, k, v, la, b, S0, cu_seqlens=cu)
    err = 0.0
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        on, Sn = orc.forward(q[:, s:e], k[:, s:e], v[:, s:e], la[:, s:e], b[:, s:e],
                             S0[n:n + 1])
        err = max(err, _maxdiff((o[:, s:e], on), (Sf[n:n + 1], Sn)))
    return err


def pin_p9_non_expansion(orc):
    """With |k_t| = 1, beta_t in [0,1] and alpha_t in (0,1]:
    |I - beta k k^T|_2 <= 1 and |Diag(alpha)|_2 <= 1, so
    |S_t|_F <= |S_{t-1}|_F + beta_t |v_t|. Returns the largest violation."""
    q, k, v, la, b, S0 = _rand(91, T=16, unit_k=True)
    S = S0.copy()
    worst = 0.0
    for t in range(q.shape[1]):
        _, Sn = orc.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], b[:, t], S)
        lhs = np.linalg.norm(Sn, axis=(-2, -1))
        rhs = np.linalg.norm(S, axis=(-2, -1)) + b[:, t] * np.linalg.norm(v[:, t], axis=-1)
        worst = max(worst, float(np.max(lhs - rhs)))
        S = Sn
    return max(worst, 0.0)


def load_hand_example(path=os.path.join(GOLDEN, "kda_hand_d2_T3.txt")):
    vals = {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *rest = line.split()
            vals[key] = [Fraction(x) for x in rest]
    return vals


def hand_example_exact(vals):
    """Re-derive the hand example in exact rational arithmetic."""
    S = [[vals["S0"][0], vals["S0"][1]], [vals["S0"][2], vals["S0"][3]]]
    scale = vals["scale"][0]
    outs = []
    for t in (1, 2, 3):
        k, v, q = vals[f"k{t}"], vals[f"v{t}"], vals[f"q{t}"]
        beta, alpha = vals[f"beta{t}"][0], vals[f"alpha{t}"]
        Sd = [[alpha[i] * S[i][j] for j in range(2)] for i in range(2)]
        kS = [sum(k[i] * Sd[i][j] for i in range(2)) for j in range(2)]
        u = [beta * (v[j] - kS[j]) for j in range(2)]
        S = [[Sd[i][j] + k[i] * u[j] for j in range(2)] for i in range(2)]
        outs.append([scale * sum(S[i][j] * q[i] for i in range(2)) for j in range(2)])
    return outs, S


def pin_golden_hand_example(orc):
    vals = load_hand_example()
    f = lambda key: np.array([float(x) for x in vals[key]])
    q = np.stack([f(f"q{t}") for t in (1, 2, 3)])[None, :, None]
    k = np.stack([f(f"k{t}") for t in (1, 2, 3)])[None, :, None]
    v = np.stack([f(f"v{t}") for t in (1, 2, 3)])[None, :, None]
    la = np.log(np.stack([f(f"alpha{t}") for t in (1, 2, 3)]))[None, :, None]
    b = np.array([float(vals[f"beta{t}"][0]) for t in (1, 2, 3)])[None, :, None]
    S0 = f("S0").reshape(1, 1, 2, 2)
    o, Sf = orc.forward(q, k, v, la, b, S0, scale=float(vals["scale"][0]))
    ro = np.stack([f(f"o{t}") for t in (1, 2, 3)])
    return _maxdiff((o[0, :, 0], ro), (Sf[0, 0], f("S_final").reshape(2, 2)))


ALL = {
    "p1_bruteforce": pin_p1_bruteforce,
    "p1_bruteforce_rect": pin_p1_bruteforce_rect,
    "p2_deltanet": pin_p2_deltanet,
    "p3_gdn_scalar_gate": pin_p3_gdn_scalar_gate,
    "p4_pure_decay": pin_p4_pure_decay,
    "p5_exact_write": pin_p5_exact_write,
    "p6_orthonormal_keys": pin_p6_orthonormal_keys,
    "p7_online_gradient_step": pin_p7_online_gradient_step,
    "p8a_value_columns_independent": pin_p8a_value_columns_independent,
    "p8b_decode_chain_equals_prefill": pin_p8b_decode_chain_equals_prefill,
    "p8c_split_prefill": pin_p8c_split_prefill,
    "p8d_varlen_equals_separate": pin_p8d_varlen_equals_separate,
    "p9_non_expansion": pin_p9_non_expansion,
    "golden_hand_example": pin_golden_hand_example,
}


def failing_pins(orc):
    """Names of the pins that ``orc`` violates (an exception counts as a
    violation)."""
    bad = []
    for name, fn in ALL.items():
        try:
            e = fn(orc)
            ok = np.isfinite(e) and e <= TOL[name]
        except Exception:  # noqa: BLE001 - a crash or rejection is a failure
            ok = False
        if not ok:
            bad.append(name)
    return bad


# ---------------------------------------------------------------------------
# Backward pins. L = <dO, o> + <dS_final, S_final>; the oracle's backward must
# give dL/d(every input). Checked against central differences of the (pinned)
# forward and against a closed form where the rule makes one exact.
BACKWARD_TOL = {
    "b1_central_differences": 1e-7,
    "b2_varlen_central_differences": 1e-7,
    "b3_pure_decay_closed_form": 1e-12,
    "b4_chunk_parallel_form": 1e-10,
}

_GRAD_OF = (("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_alpha", "dlog_alpha"),
            ("beta", "dbeta"), ("S0", "dS0"))


def _fd_gap(orc, x, dO, dSf, cu=None, h=1e-6):
    """Largest gap between the backward and central differences of
    L(x) = <dO, o> + <dSf, S_final>, over every element of every input,
    relative to max(1, |finite difference|) per input."""
    def loss(z):
        o, sf = orc.forward(z["q"], z["k"], z["v"], z["log_alpha"], z["beta"], z["S0"], cu)
        return float((o * dO).sum() + (sf * dSf).sum())

    g = orc.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], dO, x["S0"], dSf, cu)
    worst = 0.0
    for name, key in _GRAD_OF:
        a = x[name]
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            old = a[idx]
            a[idx] = old + h
            lp = loss(x)
            a[idx] = old - h
            lm = loss(x)
            a[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        worst = max(worst, float(np.abs(fd - g[key]).max() / max(1.0, np.abs(fd).max())))
    return worst


def pin_b1_central_differences(orc):
    """Every input's gradient against central differences, on a problem whose
    sequences (70 tokens) cross the backward's 64-token replay blocks."""
    q, k, v, la, b, S0 = _rand(101, B=2, T=70, H=1, dk=3, dv=2, unit_k=True)
    r = np.random.default_rng(102)
    S0 = S0 * 0.3
    x = dict(q=q, k=k, v=v, log_alpha=la, beta=b, S0=S0)
    return _fd_gap(orc, x, r.normal(size=v.shape), r.normal(size=S0.shape))


def pin_b2_varlen_central_differences(orc):
    """The same with packed sequences of 5, 0 and 7 tokens, one state each."""
    q, k, v, la, b, _ = _rand(103, B=1, T=12, H=2, dk=3, dv=2, s0=False, unit_k=True)
    r = np.random.default_rng(104)
    S0 = r.normal(size=(3, 2, 3, 2)) * 0.3
    x = dict(q=q, k=k, v=v, log_alpha=la, beta=b, S0=S0)
    cu = np.array([0, 5, 5, 12], dtype=np.int64)
    return _fd_gap(orc, x, r.normal(size=v.shape), r.normal(size=S0.shape), cu)


def pin_b3_pure_decay_closed_form(orc):
    """beta = 0 leaves only the decay: S_t = Diag(e^{g_t}) S0 with g_t the
    cumulative log_alpha, so o_t = scale S0^T Diag(e^{g_t}) q_t and
        dq_t   = scale Diag(e^{g_t}) S0 dO_t,
        dS0    = sum_t scale Diag(e^{g_t}) q_t dO_t^T + Diag(e^{g_T}) dS_final,
        dlog_alpha_s[i] = sum_{t>=s} scale q_t[i] e^{g_t[i]} (S0 dO_t)_i
                          + e^{g_T[i]} sum_j S0_ij dS_final_ij,
        dk = dv = 0."""
    q, k, v, la, _, S0 = _rand(105, B=1, T=9, H=1, dk=4, dv=3)
    b = np.zeros((1, 9, 1))
    r = np.random.default_rng(106)
    dO, dSf = r.normal(size=v.shape), r.normal(size=S0.shape)
    scale = 0.5
    g = orc.backward(q, k, v, la, b, dO, S0, dSf, scale=scale)
    G = np.cumsum(la[0, :, 0], axis=0)  # [T, dk]
    s0 = S0[0, 0]
    dq = np.stack([scale * np.exp(G[t]) * (s0 @ dO[0, t, 0]) for t in range(9)])
    dS0 = sum(scale * np.outer(np.exp(G[t]) * q[0, t, 0], dO[0, t, 0]) for t in range(9))
    dS0 = dS0 + np.exp(G[-1])[:, None] * dSf[0, 0]
    per_t = np.stack([scale * q[0, t, 0] * np.exp(G[t]) * (s0 @ dO[0, t, 0]) for t in range(9)])
    dla = np.cumsum(per_t[::-1], axis=0)[::-1] + np.exp(G[-1]) * (s0 * dSf[0, 0]).sum(axis=1)
    return _maxdiff((g["dq"][0, :, 0], dq), (g["dS0"][0, 0], dS0),
                    (g["dlog_alpha"][0, :, 0], dla), (g["dk"], 0 * k), (g["dv"], 0 * v))


def _chunked_backward(q, k, v, la, beta, S0, dO, dSf, scale, C):
    """Gradients of one (sequence, head) through the chunk-parallel form of the
    rule, an independent derivation. In a chunk with entry state S and inclusive
    cumulative log-decay g (per channel), with E_rs = e^{g_r - g_s} (r >= s):
        A_rs = beta_r k_r.(E_rs k_s) (s < r),  Pm_rs = q_r.(E_rs k_s) (s <= r),
        T = (I + A)^{-1},  W = T Diag(beta) (e^g k),  U = T Diag(beta) V - W S,
        O = scale (e^g q) S + scale Pm U,  S_end = Diag(e^{g_C}) S + (e^{g_C - g} k)^T U.
    Reverse-mode through these block products, written so that every
    exponential is an E_rs <= 1. Only e^{g_r - g_s} with r >= s appears, so
    strong decay cannot overflow."""
    T_, dk = q.shape
    n_ch = (T_ + C - 1) // C
    S = S0.copy()
    saved = []
    for c in range(n_ch):
        a, e = c * C, min(T_, (c + 1) * C)
        n = e - a
        g = np.cumsum(la[a:e], axis=0)
        low = np.tril(np.ones((n, n)))
        E = np.exp(np.minimum(g[:, None, :] - g[None, :, :], 0.0)) * low[:, :, None]
        kk = np.einsum("rc,sc,rsc->rs", k[a:e], k[a:e], E) * np.tril(np.ones((n, n)), -1)
        Pm = np.einsum("rc,sc,rsc->rs", q[a:e], k[a:e], E)
        Tm = np.linalg.inv(np.eye(n) + beta[a:e, None] * kk)
        bv = beta[a:e, None] * v[a:e]
        bk = beta[a:e, None] * k[a:e] * np.exp(g)
        W = Tm @ bk
        U = Tm @ bv - W @ S
        saved.append((a, e, g, E, kk, Pm, Tm, bv, bk, W, U, S.copy()))
        S = np.exp(g[-1])[:, None] * S + (k[a:e] * np.exp(g[-1] - g)).T @ U
    G = dSf.copy()
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dlog_alpha=np.zeros_like(la), dbeta=np.zeros_like(beta))
    for a, e, g, E, kk, Pm, Tm, bv, bk, W, U, S in reversed(saved):
        qc, kc, vc, bc, do = q[a:e], k[a:e], v[a:e], beta[a:e], dO[a:e]
        eg, egC = np.exp(g), np.exp(g[-1])
        kh = kc * np.exp(g[-1] - g)
        dU = scale * Pm.T @ do + kh @ G
        dPm = np.tril(scale * do @ U.T)
        dW = -dU @ S.T
        xv, xk = Tm.T @ dU, Tm.T @ dW
        dA = np.tril(-Tm.T @ (dU @ bv.T + dW @ bk.T) @ Tm.T, -1)
        bdA = bc[:, None] * dA
        X = np.einsum("rs,sc,rsc->rc", dPm, kc, E)
        Y = np.einsum("rs,rc,rsc->sc", dPm, qc, E)
        Z = np.einsum("rs,sc,rsc->rc", bdA, kc, E)
        R = np.einsum("rs,rc,rsc->sc", bdA, kc, E)
        Kt = np.exp(g[-1] - g) * (U @ G.T)
        dq = scale * eg * (do @ S.T) + X
        dk_ = bc[:, None] * eg * xk + Z + Y + R + Kt
        dg = qc * dq + kc * (dk_ - 2.0 * (Y + R + Kt))
        dg[-1] += np.sum(kc * Kt, axis=0) + egC * np.sum(G * S, axis=1)
        out["dq"][a:e], out["dk"][a:e], out["dv"][a:e] = dq, dk_, bc[:, None] * xv
        out["dbeta"][a:e] = (np.sum(xv * vc, 1) + np.sum(xk * kc * eg, 1) + np.sum(dA * kk, 1))
        out["dlog_alpha"][a:e] = np.cumsum(dg[::-1], axis=0)[::-1]
        G = scale * (qc * eg).T @ do + egC[:, None] * G - W.T @ dU
    out["dS0"] = G
    return out


def pin_b4_chunk_parallel_form(orc):
    """The backward equals the reverse of the chunk-parallel form (chunks of 16
    over 150 tokens, so that the oracle's own 64-token replay blocks are crossed
    too; dk != dv, two heads, with and without strong decay), relative to the
    largest gradient of each kind."""
    worst = 0.0
    for seed, shift in ((107, 0.0), (108, 3.0)):
        q, k, v, la, b, S0 = _rand(seed, B=1, T=150, H=2, dk=5, dv=4, unit_k=True)
        la = la * (1.0 + shift)  # at shift 3 the log-decay inside one chunk reaches about -68
        r = np.random.default_rng(seed + 50)
        dO, dSf = r.normal(size=v.shape), r.normal(size=S0.shape)
        scale = 0.45
        g = orc.backward(q, k, v, la, b, dO, S0, dSf, scale=scale)
        for h in range(2):
            ref = _chunked_backward(q[0, :, h], k[0, :, h], v[0, :, h], la[0, :, h], b[0, :, h],
                                    S0[0, h], dO[0, :, h], dSf[0, h], scale, 16)
            for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
                x, y = g[key][0, :, h], ref[key]
                worst = max(worst, float(np.abs(x - y).max() / max(1e-30, np.abs(y).max())))
            x, y = g["dS0"][0, h], ref["dS0"]
            worst = max(worst, float(np.abs(x - y).max() / max(1e-30, np.abs(y).max())))
    return worst


BACKWARD_ALL = {
    "b1_central_differences": pin_b1_central_differences,
    "b2_varlen_central_differences": pin_b2_varlen_central_differences,
    "b3_pure_decay_closed_form": pin_b3_pure_decay_closed_form,
    "b4_chunk_parallel_form": pin_b4_chunk_parallel_form,
}


def failing_backward_pins(orc):
    """Names of the backward pins that ``orc`` violates (an exception counts)."""
    bad = []
    for name, fn in BACKWARD_ALL.items():
        try:
            e = fn(orc)
            ok = np.isfinite(e) and e <= BACKWARD_TOL[name]
        except Exception:  # noqa: BLE001 - a crash or rejection is a failure
            ok = False
        if not ok:
            bad.append(name)
    return bad
