"""The fp64 oracle against what the pages and the mathematics fix (no GPU)."""
import numpy as np
import pytest

import oracle
from tests import pins


def fwd_c(q, k, v, la, beta, s0):
    s0 = None if s0 is None else np.asarray(s0)[None]
    out, fs = oracle.forward(q, k, v, la, beta, s0, num_threads=2)
    return out, fs[0]


def fwd_np(q, k, v, la, beta, s0):
    return oracle.forward_np(q, k, v, la, beta, s0)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("impl", [fwd_c, fwd_np], ids=["c", "numpy"])
def test_pin(pin, impl):
    pin(impl)


def test_c_matches_numpy_twin_varlen():
    r = np.random.default_rng(3)
    lens = [0, 5, 1, 9, 0, 3]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T, H, dk, dv = int(cu[-1]), 3, 6, 5
    q, k, v, la, beta, _ = pins.random_case(4, T=T, H=H, dk=dk, dv=dv)
    s0 = r.standard_normal((len(lens), H, dk, dv))
    out, fs = oracle.forward(q, k, v, la, beta, s0, cu)
    for n, L in enumerate(lens):
        a, b = cu[n], cu[n + 1]
        o2, s2 = oracle.forward_np(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b], s0[n])
        np.testing.assert_allclose(out[a:b], o2, atol=1e-12, rtol=0)
        np.testing.assert_allclose(fs[n], s2, atol=1e-12, rtol=0)
    # empty sequences pass their initial state through unchanged
    assert np.array_equal(fs[0], s0[0]) and np.array_equal(fs[4], s0[4])


def test_thread_count_does_not_change_results():
    q, k, v, la, beta, s0 = pins.random_case(5, T=40, H=4, dk=8, dv=8)
    a = oracle.forward(q, k, v, la, beta, s0[None], num_threads=1)
    b = oracle.forward(q, k, v, la, beta, s0[None], num_threads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_bad_arguments_rejected():
    q, k, v, la, beta, _ = pins.random_case(6, T=4, H=1)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, la, beta, None, np.array([0, 3], dtype=np.int64))
    with pytest.raises(RuntimeError):
        oracle.forward(q, k, v, la, beta, None, np.array([0, 3, 2, 4], dtype=np.int64))


def test_window_bound_holds():
    """Truncating the history to a window changes the end state by at most the bound."""
    r = np.random.default_rng(8)
    T, H, dk, dv = 600, 1, 8, 4
    q = r.standard_normal((T, H, dk))
    k = pins._unit(r.standard_normal((T, H, dk)))
    v = r.standard_normal((T, H, dv))
    la = -np.log1p(np.exp(r.standard_normal((T, H, dk)))) / 4.0
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((T, H))))
    _, full = oracle.forward(q, k, v, la, beta)
    t0 = 450
    _, win = oracle.forward(q[t0:], k[t0:], v[t0:], la[t0:], beta[t0:])
    ld, nb = oracle.window_bound(k, v, la, beta, 0, 0, t0, T)
    diff = float(np.max(np.abs(full - win)))
    bound = float(np.exp(ld) * nb)
    assert diff <= bound * (1 + 1e-9) + 1e-12, (diff, bound)
    # and the bound is not vacuous here
    assert bound < 1e-2


# ---- the prologue functions, pinned to closed forms and identities ---------------------------
@pytest.mark.parametrize("pin", pins.PROLOGUE_PINS, ids=lambda f: f.__name__)
def test_prologue_pin(pin):
    pin(oracle)


def test_prologue_flags_are_independent():
    rng = np.random.default_rng(5)
    q, k, g = (rng.standard_normal((4, 2, 32)) for _ in range(3))
    b = rng.standard_normal((4, 2))
    for flags in range(8):
        q2, k2, la, beta = oracle.prologue(q, k, g, b, flags, gate_scale=1 / 16)
        assert np.array_equal(q2, oracle.l2_normalise(q) if flags & 1 else q)
        assert np.array_equal(k2, oracle.l2_normalise(k) if flags & 1 else k)
        assert np.array_equal(la, -oracle.softplus(g) / 16 if flags & 2 else g)
        assert np.array_equal(beta, oracle.sigmoid(b) if flags & 4 else b)
    _, _, la, _ = oracle.prologue(q, k, np.zeros_like(g), b, 2, gate_scale=1 / 16)
    assert np.all(np.abs(la + np.log(2.0) / 16) < 1e-16)  # g = 0: alpha = 2^(-1/16)
