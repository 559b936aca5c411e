"""Pins for a KDA recurrence implementation, independent of the implementation.

Each ``pin_*`` takes ``fwd(q, k, v, log_alpha, beta, s0) -> (out, final_state)`` for
ONE sequence (q, k, log_alpha [T, H, d_k]; v [T, H, d_v]; beta [T, H];
s0 [H, d_k, d_v] or None) and raises AssertionError when the implementation
disagrees with something the pages or the mathematics fix:

* hand-derived examples (tests/golden) of the delta rule ("How the delta rule
  actually works", shivam2003.com Kimi K3 article) with channel-wise decay;
* the no-op case alpha = 1, beta = 0;
* exact recall: beta = 1 and a unit key make S^T k = v right after the write,
  whatever alpha and the prior state are; with orthonormal keys and no decay
  every written pair is recalled exactly;
* pure decay: beta = 0 reduces to S_T = Diag(exp(sum_t log_alpha_t)) S_0;
* brute force: the state equals the explicit product of the per-token
  transition matrices (I - beta k k^T) Diag(alpha) plus the written terms;
* structure: linearity in (S_0, v), equivariance under permuting value
  channels, and prefix/suffix resume (the prefill-cache property of the
  "Serving infrastructure" section of the same article).

tests/test_oracle_pins.py applies them to the C oracle and its numpy twin, and
tests/test_oracle_mutants.py checks that each planted mistake fails one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_case(seed, T=7, H=2, dk=4, dv=3, unit_keys=True, s0=True):
    r = _rng(seed)
    q = r.standard_normal((T, H, dk))
    k = r.standard_normal((T, H, dk))
    if unit_keys:
        k = _unit(k)
    v = r.standard_normal((T, H, dv))
    la = -r.uniform(0.0, 0.7, size=(T, H, dk))
    beta = r.uniform(0.0, 1.0, size=(T, H))
    S0 = r.standard_normal((H, dk, dv)) if s0 else None
    return q, k, v, la, beta, S0


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3g}"


def pin_golden(fwd):
    with open(os.path.join(GOLDEN, "delta_rule_hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        T = len(c["beta"])
        dk, dv = c["dk"], c["dv"]
        q = np.array(c["q"], dtype=np.float64).reshape(T, 1, dk)
        k = np.array(c["k"], dtype=np.float64).reshape(T, 1, dk)
        v = np.array(c["v"], dtype=np.float64).reshape(T, 1, dv)
        la = np.log(np.array(c["alpha"], dtype=np.float64)).reshape(T, 1, dk)
        beta = np.array(c["beta"], dtype=np.float64).reshape(T, 1)
        s0 = np.array(c["initial_state"], dtype=np.float64).reshape(1, dk, dv)
        out, S = fwd(q, k, v, la, beta, s0)
        _close(out, np.array(c["out"]).reshape(T, 1, dv), 1e-12, c["name"] + " out")
        _close(S, np.array(c["final_state"]).reshape(1, dk, dv), 1e-12, c["name"] + " state")


def pin_noop(fwd, seed=11):
    q, k, v, la, beta, S0 = random_case(seed)
    la[:] = 0.0
    beta[:] = 0.0
    out, S = fwd(q, k, v, la, beta, S0)
    assert np.array_equal(S, S0), "alpha=1, beta=0 must leave the state bit-exactly unchanged"
    _close(out, np.einsum("hcj,thc->thj", S0, q), TOL, "noop out = S0^T q")


def pin_exact_recall(fwd, seed=12):
    """beta = 1 with unit keys: the just-written value is recalled exactly (any alpha, S0)."""
    q, k, v, la, beta, S0 = random_case(seed, T=9, dk=5, dv=4)
    beta[:] = 1.0
    out, _ = fwd(k.copy(), k, v, la, beta, S0)  # read with q_t = k_t
    _close(out, v, TOL, "S_t^T k_t = v_t")


def pin_orthonormal_recall(fwd, seed=13, d=6, dv=5):
    """alpha = 1, beta = 1, orthonormal keys, S0 = 0: S_T^T k_i = v_i for every i."""
    r = _rng(seed)
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    k = Qm.T.reshape(d, 1, d)  # token i gets the i-th orthonormal row
    v = r.standard_normal((d, 1, dv))
    q = r.standard_normal((d, 1, d))
    la = np.zeros((d, 1, d))
    beta = np.ones((d, 1))
    _, S = fwd(q, k, v, la, beta, None)
    rec = np.einsum("cj,ic->ij", S[0], k[:, 0, :])
    _close(rec, v[:, 0, :], TOL, "orthonormal recall")


def pin_pure_decay(fwd, seed=14):
    """beta = 0: closed form S_t = Diag(exp(sum_{s<=t} log_alpha_s)) S0, out_t = S_t^T q_t."""
    q, k, v, la, beta, S0 = random_case(seed, T=8, dk=5, dv=3)
    beta[:] = 0.0
    out, S = fwd(q, k, v, la, beta, S0)
    cum = np.cumsum(la, axis=0)  # [T, H, dk]
    St = np.exp(cum)[..., None] * S0[None]  # [T, H, dk, dv]
    _close(S, St[-1], TOL, "decay closed form (state)")
    _close(out, np.einsum("thcj,thc->thj", St, q), TOL, "decay closed form (out)")


def brute_force(q, k, v, la, beta, S0):
    """Explicit transition matrices: S_t = A_t S_{t-1} + beta_t k_t v_t^T, A_t = (I - beta k k^T) Diag(alpha)."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((T, H, dv))
    S = np.zeros((H, dk, dv)) if S0 is None else S0.copy()
    for h in range(H):
        P = np.eye(dk)  # product A_t ... A_1
        acc = np.zeros((dk, dv))  # sum_s (A_t ... A_{s+1}) beta_s k_s v_s^T
        for t in range(T):
            A = (np.eye(dk) - beta[t, h] * np.outer(k[t, h], k[t, h])) @ np.diag(np.exp(la[t, h]))
            P = A @ P
            acc = A @ acc + beta[t, h] * np.outer(k[t, h], v[t, h])
            St = P @ S[h] + acc
            out[t, h] = St.T @ q[t, h]
        S[h] = P @ S[h] + acc
    return out, S


def pin_brute_force(fwd, seeds=(21, 22, 23)):
    for s in seeds:
        case = random_case(s, T=8, H=2, dk=4, dv=4, unit_keys=(s % 2 == 0))
        out, S = fwd(*case)
        bo, bS = brute_force(*case)
        _close(out, bo, 1e-11, f"brute force out (seed {s})")
        _close(S, bS, 1e-11, f"brute force state (seed {s})")


def pin_linearity(fwd, seed=31):
    q, k, v, la, beta, S0 = random_case(seed)
    _, _, v2, _, _, S02 = random_case(seed + 1)
    a, b = 0.75, -1.5
    o1, s1 = fwd(q, k, v, la, beta, S0)
    o2, s2 = fwd(q, k, v2, la, beta, S02)
    o3, s3 = fwd(q, k, a * v + b * v2, la, beta, a * S0 + b * S02)
    _close(o3, a * o1 + b * o2, 1e-11, "linear in (S0, v): out")
    _close(s3, a * s1 + b * s2, 1e-11, "linear in (S0, v): state")


def pin_value_permutation(fwd, seed=41):
    q, k, v, la, beta, S0 = random_case(seed, dv=5)
    perm = _rng(seed).permutation(5)
    o1, s1 = fwd(q, k, v, la, beta, S0)
    o2, s2 = fwd(q, k, v[..., perm], la, beta, S0[..., perm])
    _close(o2, o1[..., perm], 1e-12, "permute value channels: out")
    _close(s2, s1[..., perm], 1e-12, "permute value channels: state")


def pin_resume(fwd, seed=51, split=5):
    """Prefix then suffix from the saved state equals the whole sequence."""
    q, k, v, la, beta, S0 = random_case(seed, T=11)
    o, s = fwd(q, k, v, la, beta, S0)
    oa, sa = fwd(q[:split], k[:split], v[:split], la[:split], beta[:split], S0)
    ob, sb = fwd(q[split:], k[split:], v[split:], la[split:], beta[split:], sa)
    _close(np.concatenate([oa, ob]), o, 1e-12, "resume: out")
    _close(sb, s, 1e-12, "resume: state")


def pin_key_channel_decay(fwd, seed=61):
    """The gate decays key-channel rows: with a single decaying channel c and keys
    orthogonal to it, only row c of the state shrinks."""
    r = _rng(seed)
    dk, dv = 4, 3
    S0 = r.standard_normal((1, dk, dv))
    T = 3
    k = np.zeros((T, 1, dk))
    k[:, 0, 1] = 1.0  # keys along channel 1
    v = r.standard_normal((T, 1, dv))
    q = r.standard_normal((T, 1, dk))
    la = np.zeros((T, 1, dk))
    la[:, 0, 3] = math.log(0.5)  # only channel 3 forgets
    beta = np.full((T, 1), 0.5)
    _, S = fwd(q, k, v, la, beta, S0)
    _close(S[0, 3], S0[0, 3] * 0.125, 1e-12, "row 3 decays by 1/8")
    _close(S[0, 0], S0[0, 0], 1e-12, "row 0 untouched")
    _close(S[0, 2], S0[0, 2], 1e-12, "row 2 untouched")


ALL_PINS = [pin_golden, pin_noop, pin_exact_recall, pin_orthonormal_recall, pin_pure_decay,
            pin_brute_force, pin_linearity, pin_value_permutation, pin_resume,
            pin_key_channel_decay]


# ---- the prologue functions (q/k L2 normalisation, gate -softplus, beta sigmoid) -------------
# Each pin takes an object with softplus(x), sigmoid(x), l2_normalise(x) and L2NORM_EPS, and
# checks it against closed forms and identities that owe nothing to its code.
def pin_softplus(f):
    assert abs(float(f.softplus(0.0)) - math.log(2.0)) < 1e-15          # log(1 + 1)
    assert abs(float(f.softplus(math.log(3.0))) - math.log(4.0)) < 1e-15  # log(1 + 3)
    x = np.linspace(-40.0, 40.0, 801)
    y = f.softplus(x)
    # softplus(x) - softplus(-x) = log((1 + e^x) / (1 + e^-x)) = x
    assert np.max(np.abs(y - f.softplus(-x) - x)) < 1e-12
    assert np.all(y > 0) and np.all(np.diff(y) > 0)
    assert float(f.softplus(800.0)) == 800.0 and float(f.softplus(-800.0)) == 0.0  # no overflow


def pin_sigmoid(f):
    assert float(f.sigmoid(0.0)) == 0.5
    assert abs(float(f.sigmoid(math.log(3.0))) - 0.75) < 1e-15           # 3 / (1 + 3)
    x = np.linspace(-40.0, 40.0, 801)
    assert np.max(np.abs(f.sigmoid(x) + f.sigmoid(-x) - 1.0)) < 1e-15
    assert float(f.sigmoid(800.0)) == 1.0 and float(f.sigmoid(-800.0)) == 0.0


def pin_softplus_slope_is_sigmoid(f, h=1e-5):
    x = np.linspace(-40.0, 40.0, 801)
    d = (f.softplus(x + h) - f.softplus(x - h)) / (2 * h)
    assert np.max(np.abs(d - f.sigmoid(x))) < 1e-8


def pin_l2_normalise(f):
    y = f.l2_normalise(np.array([[3.0, 4.0], [0.0, 0.0]]))
    assert np.max(np.abs(y[0] - np.array([0.6, 0.8]))) < 1e-7   # eps / 25 relative
    assert np.all(y[1] == 0.0)
    x = _rng(3).standard_normal((7, 5, 128))
    z = f.l2_normalise(x)
    n = np.linalg.norm(x, axis=-1)
    want = n / np.sqrt(n * n + f.L2NORM_EPS)
    assert np.max(np.abs(np.linalg.norm(z, axis=-1) - want)) < 1e-12
    # parallel to the input: z . x = |x|^2 / sqrt(|x|^2 + eps)
    assert np.max(np.abs(np.sum(z * x, -1) - n * want)) < 1e-10


PROLOGUE_PINS = [pin_softplus, pin_sigmoid, pin_softplus_slope_is_sigmoid, pin_l2_normalise]
