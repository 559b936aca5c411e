"""Plausible mistakes planted in a CPU copy of the oracle must each fail a pin.

This shows the pins in tests/pins.py are strong enough to catch a dropped
term, a wrong sign, a wrong order of steps or a transposed operand. Mistakes
are planted only here, in a numpy copy on the CPU.
"""
import numpy as np
import pytest

from tests import pins


def make_mutant(kind):
    def fwd(q, k, v, la, beta, s0):
        T, H, dk = q.shape
        dv = v.shape[-1]
        S = np.zeros((H, dk, dv)) if s0 is None else np.array(s0, dtype=np.float64, copy=True)
        out = np.zeros((T, H, dv))
        for t in range(T):
            for h in range(H):
                a = np.exp(la[t, h])
                if kind == "decay_exp_sign":
                    a = np.exp(-la[t, h])
                if kind == "decay_value_channels":
                    # gate applied along value channels (needs dk == dv to run)
                    S[h] *= np.resize(a, dv)[None, :]
                elif kind not in ("no_decay", "decay_after_write"):
                    S[h] *= a[:, None]
                if kind == "read_before_write":
                    out[t, h] = S[h].T @ q[t, h]
                pred = S[h].T @ k[t, h]
                if kind == "recall_transposed" and dk == dv:
                    pred = S[h] @ k[t, h]
                err = v[t, h] - pred
                if kind == "err_sign":
                    err = pred - v[t, h]
                if kind == "no_recall":
                    err = v[t, h]
                b = beta[t, h]
                if kind == "beta_squared":
                    b = b * b
                S[h] += b * np.outer(k[t, h], err)
                if kind == "decay_after_write":
                    S[h] *= a[:, None]
                if kind != "read_before_write":
                    out[t, h] = S[h].T @ (k[t, h] if kind == "read_with_key" else q[t, h])
        return out, S
    return fwd


MUTANTS = ["decay_exp_sign", "decay_value_channels", "no_decay", "decay_after_write",
           "read_before_write", "recall_transposed", "err_sign", "no_recall", "beta_squared",
           "read_with_key"]


def test_unmutated_copy_passes():
    fwd = make_mutant("none")
    for pin in pins.ALL_PINS:
        pin(fwd)


@pytest.mark.parametrize("kind", MUTANTS)
def test_mutant_fails_some_pin(kind):
    fwd = make_mutant(kind)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(fwd)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {kind} passed every pin"
