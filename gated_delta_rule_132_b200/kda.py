"""Thin ctypes binding of the KDA C ABI (include/kda.h) for torch CUDA tensors.

Argument marshalling only: these functions check dtypes/shapes, allocate the
outputs and the workspace with torch (device memory is torch's job here), and
pass raw pointers plus ``torch.cuda.current_stream()`` to the C entry points of
the same names. Every step of the computation runs in the library's kernels;
there is no fallback of any kind. If the library is missing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda_b200.so")

KDA_DTYPE_F32, KDA_DTYPE_BF16 = 0, 1
ALGOS = {"auto": 0, "simt": 1, "tcgen05": 2, "tcgen05_sequential": 3}
STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
          3: "KDA_ERR_ALIGNMENT", 4: "KDA_ERR_WORKSPACE", 5: "KDA_ERR_CUDA",
          6: "KDA_ERR_DEVICE_STATUS"}

_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_f = ctypes.c_float


class KdaError(RuntimeError):
    """A KDA C entry point returned a non-OK status."""

    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().kda_status_string(status).decode()
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({msg})")


def lib() -> ctypes.CDLL:
    """The loaded ``libkda_b200.so``; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m gated_delta_rule_132_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        L.kda_status_string.restype = ctypes.c_char_p
        L.kda_status_string.argtypes = [_i]
        L.kda_version.restype = _i
        L.kda_version.argtypes = []
        L.kda_launch_count.restype = ctypes.c_ulonglong
        L.kda_launch_count.argtypes = []
        L.kda_chunk_fwd_status.restype = _i
        L.kda_chunk_fwd_status.argtypes = [_vp, _sz, ctypes.POINTER(_i), _vp]
        L.kda_debug_set_wait_limit.restype = _i
        L.kda_debug_set_wait_limit.argtypes = [ctypes.c_uint, _i]
        L.kda_chunk_fwd_workspace_size.restype = _sz
        L.kda_chunk_fwd_workspace_size.argtypes = [_i] * 7
        L.kda_chunk_fwd_workspace_size_ex.restype = _sz
        L.kda_chunk_fwd_workspace_size_ex.argtypes = [_i] * 8
        L.kda_chunk_fwd_timesplit_workspace_size.restype = _sz
        L.kda_chunk_fwd_timesplit_workspace_size.argtypes = [_i] * 8
        common = [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f,
                  _vp, _vp, _vp, _sz]
        L.kda_chunk_fwd.restype = _i
        L.kda_chunk_fwd.argtypes = common + [_vp]
        for fn in ("kda_chunk_fwd_ex", "kda_chunk_fwd_prepare", "kda_chunk_fwd_carry",
                   "kda_gdn_chunk_fwd", "kda_gdn_chunk_fwd_prepare", "kda_chunk_fwd_timesplit"):
            getattr(L, fn).restype = _i
            getattr(L, fn).argtypes = common + [_i, _vp]
        L.kda_decode_step.restype = _i
        L.kda_decode_step.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _f,
                                      _vp, _vp]
        L.kda_chunk_bwd_workspace_size.restype = _sz
        L.kda_chunk_bwd_workspace_size.argtypes = [_i] * 7
        L.kda_chunk_bwd_workspace_size_ex.restype = _sz
        L.kda_chunk_bwd_workspace_size_ex.argtypes = [_i] * 8
        for fn in ("kda_chunk_bwd", "kda_gdn_chunk_bwd"):
            getattr(L, fn).restype = _i
            getattr(L, fn).argtypes = ([_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                        _i, _i, _f] + [_vp] * 9 + [_sz, _vp])
        L.kda_chunk_bwd_ex.restype = _i
        L.kda_chunk_bwd_ex.argtypes = ([_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                        _i, _i, _f] + [_vp] * 9 + [_sz, _i, _i, _vp])
        for fn in ("kda_decode_tokens", "kda_gdn_decode_tokens"):
            getattr(L, fn).restype = _i
            getattr(L, fn).argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                       _f, _vp, _vp]
        _lib = L
    return _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError(f"q/k/v must be bf16 or fp32, got {t.dtype}")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def kda_chunk_fwd_workspace_size(B, T, H, dk, dv, n_seqs=0, dtype=torch.bfloat16,
                                 algo="auto") -> int:
    """Bytes of workspace :func:`kda_chunk_fwd` needs with ``algo``
    (C: ``kda_chunk_fwd_workspace_size_ex``)."""
    d = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_F32
    return int(lib().kda_chunk_fwd_workspace_size_ex(B, T, H, dk, dv, n_seqs, d, ALGOS[algo]))


class ChunkFwdCall:
    """One prefill problem marshalled for the C ABI: the checked tensors, the
    outputs, the workspace and the ctypes argument list. Calling ``run``,
    ``prepare`` or ``carry`` enqueues ``kda_chunk_fwd_ex`` or one of its two
    phases on ``stream`` (default: the current torch stream). With
    ``gate="head"`` log_alpha is [B,T,H] (one gate per head, the GDN entry
    points ``kda_gdn_chunk_fwd`` and ``kda_gdn_chunk_fwd_prepare``)."""

    def __init__(self, q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, scale=None,
                 output_final_state=True, workspace=None, o=None, S_final=None,
                 algo="auto", gate="channel"):
        if gate not in ("channel", "head"):
            raise ValueError(f"gate must be 'channel' or 'head', not {gate!r}")
        self.gate = gate
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        dtype = q.dtype
        _dt(q)
        for t, name in ((q, "q"), (k, "k")):
            _need(t, name, dtype, (B, T, H, dk))
        _need(v, "v", dtype, (B, T, H, dv))
        _need(log_alpha, "log_alpha", torch.float32,
              (B, T, H, dk) if gate == "channel" else (B, T, H))
        _need(beta, "beta", torch.float32, (B, T, H))
        if cu_seqlens is not None:
            _need(cu_seqlens, "cu_seqlens", torch.int32)
            N = cu_seqlens.shape[0] - 1
        else:
            N = B
        if S0 is not None:
            _need(S0, "S0", torch.float32, (N, H, dk, dv))
        if scale is None:
            scale = dk ** -0.5
        if o is None:
            o = torch.empty((B, T, H, dv), dtype=dtype, device=q.device)
        else:
            _need(o, "o", dtype, (B, T, H, dv))
        if output_final_state and S_final is None:
            S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
        elif S_final is not None:
            _need(S_final, "S_final", torch.float32, (N, H, dk, dv))
        n_seqs = N if cu_seqlens is not None else 0
        need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, n_seqs, dtype, algo)
        if workspace is None:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        self.tensors = (q, k, v, log_alpha, beta, S0, cu_seqlens, workspace)
        self.o, self.S_final, self.workspace = o, S_final, workspace
        self.args = [_p(q), _p(k), _p(v), _dt(q), _p(log_alpha), _p(beta), _p(S0),
                     _p(cu_seqlens), int(n_seqs), B, T, H, dk, dv, float(scale), _p(o),
                     _p(S_final), _p(workspace), workspace.numel() * workspace.element_size(),
                     ALGOS[algo]]

    def _call(self, fn, stream):
        st = getattr(lib(), fn)(*self.args, _stream(stream))
        if st != 0:
            raise KdaError(fn, st)
        return self.o, self.S_final

    def run(self, stream=None):
        return self._call("kda_chunk_fwd_ex" if self.gate == "channel" else "kda_gdn_chunk_fwd",
                          stream)

    def prepare(self, stream=None):
        return self._call("kda_chunk_fwd_prepare" if self.gate == "channel"
                          else "kda_gdn_chunk_fwd_prepare", stream)

    def carry(self, stream=None):
        return self._call("kda_chunk_fwd_carry", stream)


def kda_launch_count() -> int:
    """Kernels the library has launched in this process (C: ``kda_launch_count``)."""
    return int(lib().kda_launch_count())


def kda_chunk_fwd_status(workspace: torch.Tensor, stream=None):
    """Device status word of the last prefill that used ``workspace`` (C:
    ``kda_chunk_fwd_status``; waits for the stream). Returns ``(status, code)``:
    status 0 (KDA_OK) with code 0, or 6 (KDA_ERR_DEVICE_STATUS) with the code of
    the first bounded wait that ran out."""
    code = _i(0)
    st = lib().kda_chunk_fwd_status(_p(workspace), workspace.numel() * workspace.element_size(),
                                    ctypes.byref(code), _stream(stream))
    if st not in (0, 6):
        raise KdaError("kda_chunk_fwd_status", st)
    return st, code.value


def kda_debug_set_wait_limit(polls: int = 0, starve_carry: bool = False) -> None:
    """Debugging aid (C: ``kda_debug_set_wait_limit``): poll limit of the
    tensor-core kernels' bounded waits (0: default) and whether the sequential
    kernel's copy producer issues nothing."""
    lib().kda_debug_set_wait_limit(int(polls), 1 if starve_carry else 0)


def kda_chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, scale=None,
                  output_final_state=True, workspace=None, o=None, S_final=None,
                  algo="auto", stream=None):
    """Chunked KDA prefill (C: ``kda_chunk_fwd`` / ``kda_chunk_fwd_ex``).

    q, k [B,T,H,dk] and v [B,T,H,dv] in bf16 or fp32; log_alpha [B,T,H,dk] fp32;
    beta [B,T,H] fp32; S0 [N,H,dk,dv] fp32 or None; cu_seqlens int32 [N+1] or None
    (then N = B). Returns (o [B,T,H,dv] in q's dtype, S_final [N,H,dk,dv] fp32 or None).
    """
    return ChunkFwdCall(q, k, v, log_alpha, beta, S0, cu_seqlens, scale, output_final_state,
                        workspace, o, S_final, algo).run(stream)


def kda_chunk_fwd_timesplit(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, scale=None,
                            segments=0, output_final_state=True, workspace=None, o=None,
                            S_final=None, stream=None):
    """Tensor-core prefill with the sequential phase split into ``segments``
    time segments per sequence (C: ``kda_chunk_fwd_timesplit``; 0 = automatic,
    1 = no split). bf16, dk = dv = 128. Arguments and results as
    :func:`kda_chunk_fwd`."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    n_seqs = cu_seqlens.shape[0] - 1 if cu_seqlens is not None else 0
    need = int(lib().kda_chunk_fwd_timesplit_workspace_size(B, T, H, dk, dv, n_seqs, _dt(q),
                                                            int(segments)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    call = ChunkFwdCall(q, k, v, log_alpha, beta, S0, cu_seqlens, scale, output_final_state,
                        workspace, o, S_final, "tcgen05")
    args = call.args[:-1]  # the algo is replaced by the segment count
    st = lib().kda_chunk_fwd_timesplit(*args, int(segments), _stream(stream))
    if st != 0:
        raise KdaError("kda_chunk_fwd_timesplit", st)
    return call.o, call.S_final


def kda_chunk_fwd_prepare(*args, stream=None, **kwargs) -> ChunkFwdCall:
    """The chunk-parallel phase (C: ``kda_chunk_fwd_prepare``). Takes the
    arguments of :func:`kda_chunk_fwd` and returns the marshalled call, whose
    ``carry()`` runs the sequential phase on the same workspace."""
    call = ChunkFwdCall(*args, **kwargs)
    call.prepare(stream)
    return call


def kda_chunk_fwd_carry(call: ChunkFwdCall, stream=None):
    """The sequential phase (C: ``kda_chunk_fwd_carry``) of a prepared call."""
    return call.carry(stream)


def kda_gdn_chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, scale=None,
                      output_final_state=True, workspace=None, o=None, S_final=None,
                      algo="auto", stream=None):
    """Chunked prefill with one gate per token and head (C: ``kda_gdn_chunk_fwd``).

    As :func:`kda_chunk_fwd`, except log_alpha is [B,T,H] fp32.
    """
    return ChunkFwdCall(q, k, v, log_alpha, beta, S0, cu_seqlens, scale, output_final_state,
                        workspace, o, S_final, algo, gate="head").run(stream)


BWD_ALGOS = {"auto": 0, "token": 1, "chunked": 2}


def kda_chunk_bwd(q, k, v, log_alpha, beta, dO, S0=None, cu_seqlens=None, scale=None,
                  dS_final=None, want_dS0=True, workspace=None, gate="channel", stream=None,
                  algo="auto"):
    """Backward of the prefill (C: ``kda_chunk_bwd_ex``): the gradients of
    <dO, o> + <dS_final, S_final>.

    Arguments as :func:`kda_chunk_fwd` (``gate="head"``: log_alpha [B,T,H]), plus
    dO [B,T,H,dv] in q's dtype and dS_final [N,H,dk,dv] fp32 or None. ``algo`` is
    "auto", "token" (token-by-token walk) or "chunked" (chunk-parallel). Returns a
    dict of fp32 tensors dq, dk, dv, dlog_alpha, dbeta and dS0 (None unless want_dS0).
    """
    if gate not in ("channel", "head"):
        raise ValueError(f"gate must be 'channel' or 'head', not {gate!r}")
    if algo not in BWD_ALGOS:
        raise ValueError(f"algo must be one of {sorted(BWD_ALGOS)}, not {algo!r}")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dtype = q.dtype
    _dt(q)
    for t, name in ((q, "q"), (k, "k")):
        _need(t, name, dtype, (B, T, H, dk))
    _need(v, "v", dtype, (B, T, H, dv))
    _need(dO, "dO", dtype, (B, T, H, dv))
    la_shape = (B, T, H, dk) if gate == "channel" else (B, T, H)
    _need(log_alpha, "log_alpha", torch.float32, la_shape)
    _need(beta, "beta", torch.float32, (B, T, H))
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32)
        N = cu_seqlens.shape[0] - 1
    else:
        N = B
    for t, name in ((S0, "S0"), (dS_final, "dS_final")):
        if t is not None:
            _need(t, name, torch.float32, (N, H, dk, dv))
    if scale is None:
        scale = dk ** -0.5
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"dq": torch.empty((B, T, H, dk), **f32), "dk": torch.empty((B, T, H, dk), **f32),
         "dv": torch.empty((B, T, H, dv), **f32), "dlog_alpha": torch.empty(la_shape, **f32),
         "dbeta": torch.empty((B, T, H), **f32),
         "dS0": torch.empty((N, H, dk, dv), **f32) if want_dS0 else None}
    n_seqs = N if cu_seqlens is not None else 0
    need = int(lib().kda_chunk_bwd_workspace_size_ex(B, T, H, dk, dv, n_seqs, _dt(q),
                                                     BWD_ALGOS[algo]))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().kda_chunk_bwd_ex(
        _p(q), _p(k), _p(v), _dt(q), _p(log_alpha), _p(beta), _p(S0), _p(cu_seqlens),
        int(n_seqs), B, T, H, dk, dv, float(scale), _p(dO), _p(dS_final), _p(g["dq"]),
        _p(g["dk"]), _p(g["dv"]), _p(g["dlog_alpha"]), _p(g["dbeta"]), _p(g["dS0"]),
        _p(workspace), workspace.numel() * workspace.element_size(),
        1 if gate == "channel" else 0, BWD_ALGOS[algo], _stream(stream))
    if st != 0:
        raise KdaError("kda_chunk_bwd_ex", st)
    return g


def kda_decode_step(q, k, v, log_alpha, beta, S, scale=None, o=None, stream=None):
    """One recurrent decode step (C: ``kda_decode_step``); updates S in place.

    q, k [N,H,dk]; v [N,H,dv] (bf16 or fp32); log_alpha [N,H,dk] fp32; beta [N,H]
    fp32; S [N,H,dk,dv] fp32. Returns o [N,H,dv] in q's dtype.
    """
    N, H, dk = q.shape
    dv = v.shape[-1]
    dtype = q.dtype
    _dt(q)
    _need(q, "q", dtype, (N, H, dk))
    _need(k, "k", dtype, (N, H, dk))
    _need(v, "v", dtype, (N, H, dv))
    _need(log_alpha, "log_alpha", torch.float32, (N, H, dk))
    _need(beta, "beta", torch.float32, (N, H))
    _need(S, "S", torch.float32, (N, H, dk, dv))
    if scale is None:
        scale = dk ** -0.5
    if o is None:
        o = torch.empty((N, H, dv), dtype=dtype, device=q.device)
    else:
        _need(o, "o", dtype, (N, H, dv))
    st = lib().kda_decode_step(_p(q), _p(k), _p(v), _dt(q), _p(log_alpha), _p(beta), _p(S),
                               N, H, dk, dv, float(scale), _p(o), _stream(stream))
    if st != 0:
        raise KdaError("kda_decode_step", st)
    return o


def kda_decode_tokens(q, k, v, log_alpha, beta, S, scale=None, o=None, stream=None,
                      gate="channel"):
    """T recurrent decode steps in one call (C: ``kda_decode_tokens``); updates S in place.

    q, k [N,T,H,dk]; v [N,T,H,dv] (bf16 or fp32); log_alpha [N,T,H,dk] fp32
    ([N,T,H] with ``gate="head"``, C: ``kda_gdn_decode_tokens``); beta [N,T,H]
    fp32; S [N,H,dk,dv] fp32. Returns o [N,T,H,dv] in q's dtype.
    """
    N, T, H, dk = q.shape
    dv = v.shape[-1]
    dtype = q.dtype
    _dt(q)
    _need(q, "q", dtype, (N, T, H, dk))
    _need(k, "k", dtype, (N, T, H, dk))
    _need(v, "v", dtype, (N, T, H, dv))
    if gate not in ("channel", "head"):
        raise ValueError(f"gate must be 'channel' or 'head', not {gate!r}")
    _need(log_alpha, "log_alpha", torch.float32,
          (N, T, H, dk) if gate == "channel" else (N, T, H))
    _need(beta, "beta", torch.float32, (N, T, H))
    _need(S, "S", torch.float32, (N, H, dk, dv))
    if scale is None:
        scale = dk ** -0.5
    if o is None:
        o = torch.empty((N, T, H, dv), dtype=dtype, device=q.device)
    else:
        _need(o, "o", dtype, (N, T, H, dv))
    fn = "kda_decode_tokens" if gate == "channel" else "kda_gdn_decode_tokens"
    st = getattr(lib(), fn)(_p(q), _p(k), _p(v), _dt(q), _p(log_alpha), _p(beta), _p(S),
                            N, T, H, dk, dv, float(scale), _p(o), _stream(stream))
    if st != 0:
        raise KdaError(fn, st)
    return o
