"""Python handle on the fp64 CPU oracle for the Kimi Delta Attention recurrence.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers. The CUDA library never imports this
module and this module never imports the CUDA library.

The arithmetic lives in ``kda_oracle.c`` (the token-by-token update rule of
"Kimi Linear：让长上下文大模型真正实用的线性注意力架构", section 三 5️⃣, with the
read-out o_t = scale * S_t^T q_t on the post-update state). This file only
builds that C file with gcc, widens every input to float64 and passes pointers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libkda_oracle.so`` (plain gcc, no
    fast-math, no FMA contraction) unless an up-to-date build exists."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class OracleLib:
    """ctypes binding of one build of ``kda_oracle.c`` (the default build, or a
    variant built elsewhere, which the test suite uses to check that its pins
    catch planted mistakes)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.kda_oracle_forward.restype = ctypes.c_int
        lib.kda_oracle_forward.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, _dp, _dp, ctypes.c_int]
        lib.kda_oracle_decode_step.restype = ctypes.c_int
        lib.kda_oracle_decode_step.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, _dp, ctypes.c_int]
        lib.kda_oracle_backward.restype = ctypes.c_int
        lib.kda_oracle_backward.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int]
        lib.kda_oracle_num_threads.restype = ctypes.c_int
        lib.kda_oracle_num_threads.argtypes = [ctypes.c_int]
        self.lib = lib
        self.path = path

    def num_threads(self, requested: int = 0) -> int:
        """Threads used for ``n_threads=requested`` (0 = all online cores)."""
        return self.lib.kda_oracle_num_threads(int(requested))

    def forward(self, q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, scale=None,
                n_threads: int = 0, return_final: bool = True):
        """fp64 token-by-token forward.

        Shapes: q, k, log_alpha [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H];
        S0 [N,H,dk,dv] or None (zero state); cu_seqlens [N+1] or None (then N = B).
        Returns (o [B,T,H,dv], S_final [N,H,dk,dv]) as float64 arrays
        (S_final is None when ``return_final`` is False).
        """
        q, k, v, la, b = map(_f64, (q, k, v, log_alpha, beta))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        if k.shape != q.shape or la.shape != q.shape or v.shape[:3] != (B, T, H) \
                or b.shape != (B, T, H):
            raise ValueError("shape mismatch")
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(np.asarray(
                cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                dtype=np.int64))
            N = cu.shape[0] - 1
            if B != 1:
                raise ValueError("cu_seqlens needs B == 1")
        else:
            cu, N = None, B
        s0 = _f64(S0)
        if s0 is not None and s0.shape != (N, H, dk, dv):
            raise ValueError("S0 shape mismatch")
        if scale is None:
            scale = dk ** -0.5
        o = np.zeros((B, T, H, dv), dtype=np.float64)
        sf = np.zeros((N, H, dk, dv), dtype=np.float64) if return_final else None
        rc = self.lib.kda_oracle_forward(
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
            None if cu is None else cu.ctypes.data_as(_i64p), int(N),
            int(B), int(T), int(H), int(dk), int(dv), float(scale),
            _ptr(o), _ptr(sf), int(n_threads))
        if rc != 0:
            raise ValueError(f"kda_oracle_forward rejected its arguments (rc={rc})")
        return o, sf

    def backward(self, q, k, v, log_alpha, beta, dO, S0=None, dS_final=None,
                 cu_seqlens=None, scale=None, n_threads: int = 0):
        """fp64 reverse-mode derivatives of L = <dO, o> + <dS_final, S_final>.

        Inputs as :meth:`forward`, plus dO [B,T,H,dv] and dS_final [N,H,dk,dv] (or
        None for zero). Returns a dict of float64 arrays with the inputs' shapes:
        dq, dk, dv, dlog_alpha, dbeta and dS0 (the gradient of the initial state,
        also when S0 is None, i.e. zero).
        """
        q, k, v, la, b, do = map(_f64, (q, k, v, log_alpha, beta, dO))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        if k.shape != q.shape or la.shape != q.shape or v.shape[:3] != (B, T, H) \
                or b.shape != (B, T, H) or do.shape != v.shape:
            raise ValueError("shape mismatch")
        if cu_seqlens is not None:
            cu = np.ascontiguousarray(np.asarray(
                cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                dtype=np.int64))
            N = cu.shape[0] - 1
            if B != 1:
                raise ValueError("cu_seqlens needs B == 1")
        else:
            cu, N = None, B
        s0, dsf = _f64(S0), _f64(dS_final)
        for t, name in ((s0, "S0"), (dsf, "dS_final")):
            if t is not None and t.shape != (N, H, dk, dv):
                raise ValueError(f"{name} shape mismatch")
        if scale is None:
            scale = dk ** -0.5
        out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
               "dlog_alpha": np.zeros_like(la), "dbeta": np.zeros_like(b),
               "dS0": np.zeros((N, H, dk, dv), dtype=np.float64)}
        rc = self.lib.kda_oracle_backward(
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0),
            None if cu is None else cu.ctypes.data_as(_i64p), int(N),
            int(B), int(T), int(H), int(dk), int(dv), float(scale), _ptr(do), _ptr(dsf),
            _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_alpha"]),
            _ptr(out["dbeta"]), _ptr(out["dS0"]), int(n_threads))
        if rc != 0:
            raise ValueError(f"kda_oracle_backward rejected its arguments (rc={rc})")
        return out

    def decode_step(self, q, k, v, log_alpha, beta, S, scale=None, n_threads: int = 0):
        """One recurrent step for N sequences. q, k, log_alpha [N,H,dk]; v [N,H,dv];
        beta [N,H]; S [N,H,dk,dv]. Returns (o [N,H,dv], S_new) as float64 arrays;
        the input S is not modified."""
        q, k, v, la, b = map(_f64, (q, k, v, log_alpha, beta))
        S = _f64(S).copy()
        N, H, dk = q.shape
        dv = v.shape[-1]
        if scale is None:
            scale = dk ** -0.5
        o = np.zeros((N, H, dv), dtype=np.float64)
        rc = self.lib.kda_oracle_decode_step(
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(S),
            int(N), int(H), int(dk), int(dv), float(scale), _ptr(o), int(n_threads))
        if rc != 0:
            raise ValueError(f"kda_oracle_decode_step rejected its arguments (rc={rc})")
        return o, S


def default() -> OracleLib:
    """The oracle built from ``kda_oracle.c`` in this directory."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = OracleLib(build())
    return _lib


def _f64(x):
    """Widen to a contiguous float64 numpy array. Accepts numpy arrays and torch
    CPU tensors (bf16 included: bf16 -> fp32 -> fp64 is exact)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor
        x = x.detach()
        if x.device.type != "cpu":
            raise ValueError("the oracle takes host data only")
        x = x.float().numpy() if x.dtype.is_floating_point else x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def num_threads(requested: int = 0) -> int:
    """Threads the default oracle uses for ``n_threads=requested``."""
    return default().num_threads(requested)


def forward(*args, **kwargs):
    """:meth:`OracleLib.forward` of the default build."""
    return default().forward(*args, **kwargs)


def decode_step(*args, **kwargs):
    """:meth:`OracleLib.decode_step` of the default build."""
    return default().decode_step(*args, **kwargs)


def backward(*args, **kwargs):
    """:meth:`OracleLib.backward` of the default build."""
    return default().backward(*args, **kwargs)
