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



class _PrologueMutant:
    """A numpy copy of the oracle's prologue functions with one planted mistake."""
    L2NORM_EPS = 1e-6

    def __init__(self, kind):
        self.kind = kind

    def softplus(self, x):
        x = np.asarray(x, dtype=np.float64)
        with np.errstate(over="ignore"):
            if self.kind == "softplus_naive":
                return np.log1p(np.exp(x))                          # overflows for large x
            if self.kind == "softplus_sign":
                return np.maximum(-x, 0.0) + np.log1p(np.exp(-np.abs(x)))
            if self.kind == "softplus_log_not_log1p":
                return np.maximum(x, 0.0) + np.log(np.exp(-np.abs(x)))
            if self.kind == "softplus_dropped_tail":
                return np.maximum(x, 0.0)
            return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))

    def sigmoid(self, x):
        x = np.asarray(x, dtype=np.float64)
        e = np.exp(-np.abs(x))
        if self.kind == "sigmoid_sign":
            return np.where(x >= 0, e / (1.0 + e), 1.0 / (1.0 + e))
        if self.kind == "sigmoid_tanh":
            return 0.5 * (1.0 + np.tanh(x))                        # tanh(x), not tanh(x / 2)
        return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))

    def l2_normalise(self, x):
        x = np.asarray(x, dtype=np.float64)
        ss = np.sum(x * x, axis=-1, keepdims=True)
        if self.kind == "l2_no_sqrt":
            return x / (ss + self.L2NORM_EPS)
        if self.kind == "l2_wrong_axis":
            return x / np.sqrt(np.sum(x * x, axis=0, keepdims=True) + self.L2NORM_EPS)
        if self.kind == "l2_l1_norm":
            return x / (np.sum(np.abs(x), axis=-1, keepdims=True) + self.L2NORM_EPS)
        return x / np.sqrt(ss + self.L2NORM_EPS)


PROLOGUE_MUTANTS = ["softplus_naive", "softplus_sign", "softplus_log_not_log1p",
                    "softplus_dropped_tail", "sigmoid_sign", "sigmoid_tanh", "l2_no_sqrt",
                    "l2_wrong_axis", "l2_l1_norm"]


def test_unmutated_prologue_copy_passes():
    for pin in pins.PROLOGUE_PINS:
        pin(_PrologueMutant("none"))


@pytest.mark.parametrize("kind", PROLOGUE_MUTANTS)
def test_prologue_mutant_fails_some_pin(kind):
    f = _PrologueMutant(kind)
    failed = []
    for pin in pins.PROLOGUE_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(f)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"mutant {kind} passed every prologue pin"
