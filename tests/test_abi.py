"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_132_b200 import build, kda
    build.build()
    return kda.lib()


def declared_functions():
    src = open(HEADER, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("kda_chunk_fwd", "kda_decode_step", "kda_decode_tokens",
                     "kda_chunk_fwd_workspace_size", "kda_status_string"):
        assert required in names


@pytest.mark.parametrize("name", declared_functions())
def test_symbol_exported(L, name):
    assert hasattr(L, name), f"{name} declared in include/kda.h but not exported"


def test_status_strings(L):
    for s in range(7):
        assert L.kda_status_string(s)
    assert L.kda_version() >= 100


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def _chunk(L, **kw):
    a = dict(q=_fake(), k=_fake(), v=_fake(), dt=1, la=_fake(), beta=_fake(), S0=None,
             cu=None, n_seqs=0, B=1, T=64, H=2, dk=128, dv=128, scale=0.1, o=_fake(),
             Sf=None, ws=_fake(), ws_bytes=1 << 40, algo=0, stream=None)
    a.update(kw)
    return L.kda_chunk_fwd_ex(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"], a["S0"],
                              a["cu"], a["n_seqs"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                              a["scale"], a["o"], a["Sf"], a["ws"], a["ws_bytes"], a["algo"],
                              a["stream"])


# Every case below must be rejected on the host: the fake device pointers are
# never dereferenced and no CUDA call is made.
@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(beta=None), 1), (dict(o=None), 1),
    (dict(B=0), 1), (dict(T=-1), 1), (dict(H=0), 1),
    (dict(dk=96, dv=96), 2), (dict(dk=128, dv=64), 2), (dict(dt=7), 2),
    (dict(q=_fake(0x10004)), 3), (dict(la=_fake(0x10008)), 3), (dict(Sf=_fake(0x10001)), 3),
    (dict(ws=None), 4), (dict(ws_bytes=16), 4),
    (dict(cu=_fake(), n_seqs=0), 1), (dict(cu=_fake(), n_seqs=2, B=2), 1),
    (dict(algo=9), 1), (dict(scale=float("nan")), 1),
    (dict(dk=64, dv=64, algo=2), 2), (dict(dt=0, algo=2), 2),
])
def test_chunk_fwd_rejects(L, kw, status):
    assert _chunk(L, **kw) == status


def test_workspace_size(L):
    a = L.kda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 0, 1)
    b = L.kda_chunk_fwd_workspace_size(4, 4097, 16, 128, 128, 0, 1)
    assert 0 < a < b
    assert L.kda_chunk_fwd_workspace_size(1, 1000, 4, 64, 64, 3, 0) > 0
    assert L.kda_chunk_fwd_workspace_size(1, 100, 4, 96, 96, 0, 0) == 0
    assert L.kda_chunk_fwd_workspace_size(0, 100, 4, 64, 64, 0, 0) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(N=0), 1), (dict(S=None), 1), (dict(dk=48, dv=48), 2), (dict(dt=3), 2),
    (dict(S=_fake(0x10008)), 3), (dict(o=_fake(0x10002)), 3), (dict(scale=float("inf")), 1),
])
def test_decode_rejects(L, kw, status):
    a = dict(q=_fake(), k=_fake(), v=_fake(), dt=1, la=_fake(), beta=_fake(), S=_fake(),
             N=4, H=2, dk=128, dv=128, scale=0.1, o=_fake(), stream=None)
    a.update(kw)
    assert L.kda_decode_step(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"], a["S"],
                             a["N"], a["H"], a["dk"], a["dv"], a["scale"], a["o"],
                             a["stream"]) == status


@pytest.mark.parametrize("kw,status", [
    (dict(N=0), 1), (dict(T=-1), 1), (dict(S=None), 1), (dict(q=None), 1), (dict(o=None), 1),
    (dict(dk=48, dv=48), 2), (dict(dt=3), 2), (dict(N=1 << 20, T=1 << 12), 2),
    (dict(S=_fake(0x10008)), 3), (dict(v=_fake(0x10002)), 3), (dict(scale=float("nan")), 1),
    # no token: nothing is read, written or launched, and only S must be given
    (dict(T=0, q=None, k=None, v=None, la=None, beta=None, o=None), 0),
])
def test_decode_tokens_rejects(L, kw, status):
    a = dict(q=_fake(), k=_fake(), v=_fake(), dt=1, la=_fake(), beta=_fake(), S=_fake(),
             N=4, T=3, H=2, dk=128, dv=128, scale=0.1, o=_fake(), stream=None)
    a.update(kw)
    assert L.kda_decode_tokens(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"], a["S"],
                               a["N"], a["T"], a["H"], a["dk"], a["dv"], a["scale"], a["o"],
                               a["stream"]) == status


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(la=None), 1), (dict(B=0), 1), (dict(dk=96, dv=96), 2),
    (dict(la=_fake(0x10004)), 3), (dict(ws_bytes=16), 4), (dict(algo=9), 1),
    (dict(dt=0, algo=2), 2),
])
@pytest.mark.parametrize("fn", ["kda_gdn_chunk_fwd", "kda_gdn_chunk_fwd_prepare"])
def test_gdn_chunk_fwd_rejects(L, fn, kw, status):
    """The one-gate-per-head prefill checks its arguments like kda_chunk_fwd_ex."""
    a = dict(q=_fake(), k=_fake(), v=_fake(), dt=1, la=_fake(), beta=_fake(), S0=None,
             cu=None, n_seqs=0, B=1, T=64, H=2, dk=128, dv=128, scale=0.1, o=_fake(),
             Sf=None, ws=_fake(), ws_bytes=1 << 40, algo=0, stream=None)
    a.update(kw)
    assert getattr(L, fn)(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"], a["S0"],
                          a["cu"], a["n_seqs"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                          a["scale"], a["o"], a["Sf"], a["ws"], a["ws_bytes"], a["algo"],
                          a["stream"]) == status


@pytest.mark.parametrize("kw,status", [
    (dict(N=0), 1), (dict(la=None), 1), (dict(S=None), 1), (dict(dk=48, dv=48), 2),
    (dict(S=_fake(0x10008)), 3), (dict(T=0, q=None, la=None), 0),
])
def test_gdn_decode_tokens_rejects(L, kw, status):
    a = dict(q=_fake(), k=_fake(), v=_fake(), dt=1, la=_fake(), beta=_fake(), S=_fake(),
             N=4, T=3, H=2, dk=128, dv=128, scale=0.1, o=_fake(), stream=None)
    a.update(kw)
    assert L.kda_gdn_decode_tokens(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"],
                                   a["S"], a["N"], a["T"], a["H"], a["dk"], a["dv"],
                                   a["scale"], a["o"], a["stream"]) == status


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(dO=None), 1), (dict(gq=None), 1), (dict(gbeta=None), 1),
    (dict(B=0), 1), (dict(dk=96, dv=96), 2), (dict(dt=5), 2), (dict(gla=_fake(0x10004)), 3),
    (dict(dO=_fake(0x10002)), 3), (dict(ws=None), 4), (dict(ws_bytes=64), 4),
    (dict(scale=float("nan")), 1),
])
@pytest.mark.parametrize("fn", ["kda_chunk_bwd", "kda_gdn_chunk_bwd"])
def test_chunk_bwd_rejects(L, fn, kw, status):
    a = dict(q=_fake(), k=_fake(), v=_fake(), dt=1, la=_fake(), beta=_fake(), S0=None,
             cu=None, n_seqs=0, B=1, T=64, H=2, dk=128, dv=128, scale=0.1, dO=_fake(),
             dSf=None, gq=_fake(), gk=_fake(), gv=_fake(), gla=_fake(), gbeta=_fake(),
             gS0=None, ws=_fake(), ws_bytes=1 << 40, stream=None)
    a.update(kw)
    assert getattr(L, fn)(a["q"], a["k"], a["v"], a["dt"], a["la"], a["beta"], a["S0"],
                          a["cu"], a["n_seqs"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                          a["scale"], a["dO"], a["dSf"], a["gq"], a["gk"], a["gv"],
                          a["gla"], a["gbeta"], a["gS0"], a["ws"], a["ws_bytes"],
                          a["stream"]) == status


@pytest.mark.parametrize("algo,status", [(3, 1), (-1, 1)])
def test_chunk_bwd_ex_rejects_unknown_algorithm(L, algo, status):
    assert L.kda_chunk_bwd_ex(_fake(), _fake(), _fake(), 1, _fake(), _fake(), None, None, 0, 1,
                              64, 2, 128, 128, 0.1, _fake(), None, _fake(), _fake(), _fake(),
                              _fake(), _fake(), None, _fake(), 1 << 40, 1, algo, None) == status


def test_chunk_bwd_ex_rejects_like_the_plain_call(L):
    """Bad sizes, dtype, alignment and workspace fail on the host for both algorithms."""
    for algo in (0, 1, 2):
        base = [_fake(), _fake(), _fake(), 1, _fake(), _fake(), None, None, 0, 1, 64, 2, 128,
                128, 0.1, _fake(), None, _fake(), _fake(), _fake(), _fake(), _fake(), None,
                _fake(), 1 << 40, 1, algo, None]
        bad_dtype = list(base); bad_dtype[3] = 5
        bad_head = list(base); bad_head[12] = bad_head[13] = 96
        small_ws = list(base); small_ws[24] = 64
        misaligned = list(base); misaligned[15] = _fake(0x10002)
        assert L.kda_chunk_bwd_ex(*bad_dtype) == 2
        assert L.kda_chunk_bwd_ex(*bad_head) == 2
        assert L.kda_chunk_bwd_ex(*small_ws) == 4
        assert L.kda_chunk_bwd_ex(*misaligned) == 3


def test_chunk_bwd_workspace_size_ex(L):
    token = L.kda_chunk_bwd_workspace_size_ex(1, 8192, 32, 128, 128, 0, 1, 1)
    chunked = L.kda_chunk_bwd_workspace_size_ex(1, 8192, 32, 128, 128, 0, 1, 2)
    # AUTO is the chunk-parallel form, also for the plain size query
    assert chunked == L.kda_chunk_bwd_workspace_size(1, 8192, 32, 128, 128, 0, 1)
    assert chunked == L.kda_chunk_bwd_workspace_size_ex(1, 8192, 32, 128, 128, 0, 1, 0)
    assert token > chunked
    # chunked: about 7.1 KB per token and head at d = 128
    assert 6.5e3 * 8192 * 32 < chunked < 7.5e3 * 8192 * 32
    assert L.kda_chunk_bwd_workspace_size_ex(1, 8192, 32, 128, 128, 0, 1, 3) == 0


def test_chunk_bwd_workspace_size(L):
    a = L.kda_chunk_bwd_workspace_size(1, 4096, 8, 128, 128, 0, 1)
    b = L.kda_chunk_bwd_workspace_size(1, 4097, 8, 128, 128, 0, 1)
    assert 0 < a < b
    assert L.kda_chunk_bwd_workspace_size(1, 100, 4, 96, 96, 0, 0) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from gated_delta_rule_132_b200 import kda
    monkeypatch.setattr(kda, "_lib", None)
    monkeypatch.setattr(kda, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        kda.lib()


def test_workspace_size_per_algorithm(L):
    """The tcgen05 path needs less workspace than the SIMT path; asking for a
    path a problem does not support gives 0."""
    L.kda_chunk_fwd_workspace_size_ex.restype = ctypes.c_size_t
    tc = L.kda_chunk_fwd_workspace_size_ex(1, 4096, 8, 128, 128, 0, 1, 2)
    simt = L.kda_chunk_fwd_workspace_size_ex(1, 4096, 8, 128, 128, 0, 1, 1)
    auto = L.kda_chunk_fwd_workspace_size_ex(1, 4096, 8, 128, 128, 0, 1, 0)
    assert 0 < tc < simt and auto == tc
    assert L.kda_chunk_fwd_workspace_size(1, 4096, 8, 128, 128, 0, 1) == tc
    assert L.kda_chunk_fwd_workspace_size_ex(1, 4096, 8, 64, 64, 0, 1, 2) == 0
    assert L.kda_chunk_fwd_workspace_size_ex(1, 4096, 8, 128, 128, 0, 1, 7) == 0


def test_status_query_rejects_bad_arguments(L):
    """kda_chunk_fwd_status checks its arguments on the host (no CUDA call)."""
    code = ctypes.c_int(0)
    assert L.kda_chunk_fwd_status(None, 1024, ctypes.byref(code), None) == 1
    assert L.kda_chunk_fwd_status(_fake(), 1024, None, None) == 1
    assert L.kda_chunk_fwd_status(_fake(0x10004), 1024, ctypes.byref(code), None) == 3
    assert L.kda_chunk_fwd_status(_fake(), 255, ctypes.byref(code), None) == 4


def test_launch_count_and_debug_knobs(L):
    """The launch counter starts at a number and rejected calls launch nothing;
    the debug knobs accept any value and are reset."""
    L.kda_launch_count.restype = ctypes.c_ulonglong
    before = L.kda_launch_count()
    assert _chunk(L, q=None) == 1
    assert L.kda_launch_count() == before
    assert L.kda_debug_set_wait_limit(1000, 1) == 0
    assert L.kda_debug_set_wait_limit(0, 0) == 0


def _split_call(L, segments, **kw):
    f = _fake()
    a = dict(dt=1, dk=128, ws=f, ws_bytes=1 << 40)
    a.update(kw)
    return L.kda_chunk_fwd_timesplit(f, f, f, a["dt"], f, f, None, None, 0, 1, 4096, 4,
                                     a["dk"], a["dk"], 0.1, f, None, a["ws"], a["ws_bytes"],
                                     segments, None)


@pytest.mark.parametrize("segments,kw,status", [
    (-1, {}, 1), (65, {}, 1),                 # segment count outside 0..64
    (3, dict(dt=0), 2), (3, dict(dk=64), 2),  # not a tensor-core problem
    (3, dict(ws_bytes=1024), 4),              # workspace too small
])
def test_timesplit_rejects(L, segments, kw, status):
    assert _split_call(L, segments, **kw) == status


def test_timesplit_workspace_grows_with_segments(L):
    f = L.kda_chunk_fwd_timesplit_workspace_size
    one, four = f(1, 4096, 4, 128, 128, 0, 1, 1), f(1, 4096, 4, 128, 128, 0, 1, 4)
    assert one > 0 and four - one == 3 * 4 * 1 * 4 * 128 * 128 * 4
    assert f(1, 4096, 4, 128, 128, 0, 1, 65) == 0 and f(1, 4096, 4, 64, 64, 0, 1, 2) == 0
    # the sequential algorithm never reserves segment states
    assert L.kda_chunk_fwd_workspace_size_ex(1, 4096, 4, 128, 128, 0, 1, 3) == one
