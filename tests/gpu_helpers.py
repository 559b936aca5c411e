"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on the same bits."""
import numpy as np
import torch

import oracle
from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W

# Tolerances on max-abs error relative to max|v| (fp32 inputs / bf16 inputs with fp32 state).
TOL = {"f32": 1e-4, "bf16": 2e-2}


def f64(t):
    return W.to_f64_numpy(t)


def assert_close(gpu, ref, tol, scale, what):
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    err = float(np.max(np.abs(g - ref))) if g.size else 0.0
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:g} * {scale:.3g}"
    return err


def oracle_forward(inp, heads=None, seqs=None):
    """fp64 oracle on the exact input values; optionally a subset of heads / sequences."""
    cu = inp["cu_seqlens"].numpy().astype(np.int64)
    hs = slice(None) if heads is None else list(heads)
    q, k, v, la, b = (f64(inp[n][:, hs]) for n in ("q", "k", "v", "log_alpha", "beta"))
    s0 = inp.get("initial_state")
    s0 = None if s0 is None else f64(s0[:, hs])
    if seqs is None:
        return oracle.forward(q, k, v, la, b, s0, cu)
    outs, states = {}, {}
    for n in seqs:
        a, e = int(cu[n]), int(cu[n + 1])
        o, s = oracle.forward(q[a:e], k[a:e], v[a:e], la[a:e], b[a:e],
                              None if s0 is None else s0[n:n + 1])
        outs[n], states[n] = o, s[0]
    return outs, states


def gpu_prefill(inp, algo="auto"):
    return K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                     inp.get("initial_state"), inp["cu_seqlens"], inp["cu_seqlens_dev"], algo=algo)


def vmax(inp):
    return max(float(inp["v"].abs().max().item()), 1e-30)
