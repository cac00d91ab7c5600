"""The fp64 oracle against facts the update rule fixes (CPU only)."""
import numpy as np
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("name", sorted(pins.ALL))
def test_pin(orc, name):
    err = pins.ALL[name](orc)
    assert np.isfinite(err) and err <= pins.TOL[name], f"{name}: {err}"


def test_hand_example_fixture_is_exact():
    """The stored hand-derived values equal an exact rational re-derivation."""
    vals = pins.load_hand_example()
    outs, S = pins.hand_example_exact(vals)
    for t, o in enumerate(outs, start=1):
        assert o == vals[f"o{t}"]
    assert [x for row in S for x in row] == vals["S_final"]
    # the exact-write property holds in the fixture's last step (beta=1, |k|=1)
    k3 = vals["k3"]
    assert sum(x * x for x in k3) == 1 and vals["beta3"][0] == 1
    kS = [sum(k3[i] * S[i][j] for i in range(2)) for j in range(2)]
    assert kS == vals["v3"]


def test_oracle_threads_do_not_change_results(orc):
    q, k, v, la, b, S0 = pins._rand(5, B=3, T=9, H=4)
    o1, s1 = orc.forward(q, k, v, la, b, S0, n_threads=1)
    o8, s8 = orc.forward(q, k, v, la, b, S0, n_threads=8)
    assert np.array_equal(o1, o8) and np.array_equal(s1, s8)


def test_oracle_rejects_bad_cu_seqlens(orc):
    q, k, v, la, b, _ = pins._rand(6, B=1, T=8)
    with pytest.raises(ValueError):
        orc.forward(q, k, v, la, b, cu_seqlens=np.array([0, 5, 3, 8]))
    with pytest.raises(ValueError):
        orc.forward(q, k, v, la, b, cu_seqlens=np.array([0, 5, 7]))


def test_empty_sequence_keeps_state(orc):
    """A zero-length sequence in a packed batch returns its S0 unchanged."""
    q, k, v, la, b, _ = pins._rand(7, B=1, T=6)
    S0 = np.random.default_rng(8).normal(size=(3, q.shape[2], q.shape[3], v.shape[3]))
    o, Sf = orc.forward(q, k, v, la, b, S0, cu_seqlens=np.array([0, 4, 4, 6]))
    assert np.array_equal(Sf[1], S0[1])
