"""fp64 CPU oracle of the KDA recurrence (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never imports or calls it, and it imports nothing from the
product package.

``forward`` runs the token-by-token fp64 recurrence in C (``kda_oracle.c``,
OpenMP over (sequence, head)); ``forward_np`` is a numpy restatement of the
same steps for tiny inputs. See ``kda_oracle.c`` for the definition and the
passages of the pages each step follows.
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


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libkda_oracle.so`` (gcc, OpenMP, generic x86-64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            lib.kda_oracle_forward.restype = ctypes.c_int
            lib.kda_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
                                               ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_int32, dp, dp, ctypes.c_int32]
            lib.kda_oracle_window_bound.restype = ctypes.c_int
            lib.kda_oracle_window_bound.argtypes = [dp, dp, dp, dp, ctypes.c_int32, ctypes.c_int32,
                                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                                    ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                                    dp, dp]
            lib.kda_oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.float64)
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"shape {a.shape} != {tuple(shape)}")
    return a


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(_load().kda_oracle_num_threads())


def forward(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, num_threads: int = 0):
    """Packed-varlen recurrence in fp64.

    q, k, log_alpha: [T, H, d_k]; v: [T, H, d_v]; beta: [T, H];
    initial_state: [N, H, d_k, d_v] or None (zeros); cu_seqlens: [N+1] (default: one sequence).
    Returns (out [T, H, d_v], final_state [N, H, d_k, d_v]) as float64 arrays.
    """
    q = _f64(q)
    T, H, dk = q.shape
    dv = np.shape(v)[-1]
    k = _f64(k, (T, H, dk))
    v = _f64(v, (T, H, dv))
    la = _f64(log_alpha, (T, H, dk))
    beta = _f64(beta, (T, H))
    if cu_seqlens is None:
        cu_seqlens = np.array([0, T], dtype=np.int64)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != T:
        raise ValueError("cu_seqlens must start at 0 and end at T")
    s0 = _f64(initial_state, (N, H, dk, dv)) if initial_state is not None else None
    out = np.zeros((T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(s0),
                                    cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                    N, H, dk, dv, _ptr(out), _ptr(fs), int(num_threads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_forward failed with {rc}")
    return out, fs


def window_bound(k, v, log_alpha, beta, h, t_start, t0, t1, s0_norm=0.0):
    """(log_decay, norm_bound) of ``kda_oracle_window_bound`` for head ``h`` (arrays [T, H, d])."""
    k = _f64(k)
    T, H, dk = k.shape
    v = _f64(v)
    dv = v.shape[-1]
    la = _f64(log_alpha, (T, H, dk))
    beta = _f64(beta, (T, H))
    ld = ctypes.c_double()
    nb = ctypes.c_double()
    rc = _load().kda_oracle_window_bound(_ptr(k), _ptr(v), _ptr(la), _ptr(beta), H, dk, dv, int(h),
                                         int(t_start), int(t0), int(t1), float(s0_norm),
                                         ctypes.byref(ld), ctypes.byref(nb))
    if rc != 0:
        raise RuntimeError("kda_oracle_window_bound: bad arguments")
    return ld.value, nb.value


def forward_np(q, k, v, log_alpha, beta, initial_state=None):
    """One sequence, numpy fp64, tiny sizes: the same five steps as the C oracle.

    q, k, log_alpha: [T, H, d_k]; v: [T, H, d_v]; beta: [T, H]; initial_state [H, d_k, d_v].
    Returns (out [T, H, d_v], final_state [H, d_k, d_v]).
    """
    q, k, v, la, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta))
    T, H, dk = q.shape
    dv = v.shape[-1]
    S = (np.zeros((H, dk, dv)) if initial_state is None
         else np.array(initial_state, dtype=np.float64, copy=True))
    out = np.zeros((T, H, dv))
    for t in range(T):
        for h in range(H):
            S[h] *= np.exp(la[t, h])[:, None]                 # forget, per key channel
            pred = S[h].T @ k[t, h]                          # recall
            S[h] += beta[t, h] * np.outer(k[t, h], v[t, h] - pred)  # write the error only
            out[t, h] = S[h].T @ q[t, h]                     # read after the write
    return out, S


# ---- the KDA layer's elementwise prologue (what kda_prefill_prologue fuses) ----------------
# Sources: "Kimi Delta Attention: the load-bearing choice" (shivam2003.com Kimi K3 article):
# per-key-channel forgetting gates alpha in (0, 1] and a writing strength beta; the synthetic
# workloads draw q, k ~ N(0, 1) then L2-normalise them per token, log alpha = -softplus(g)/16 and
# beta = sigmoid(b) with g, b ~ N(0, 1). The epsilon inside the norm is this library's reading.
L2NORM_EPS = 1e-6
QK_L2NORM, GATE_SOFTPLUS, BETA_SIGMOID = 1, 2, 4


def l2_normalise(x):
    """Rows along the last axis divided by sqrt(sum of squares + L2NORM_EPS), fp64."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + L2NORM_EPS)


def softplus(x):
    """log(1 + e^x), fp64, without overflow: max(x, 0) + log(1 + e^-|x|)."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    """1 / (1 + e^-x), fp64, without overflow."""
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def prologue(q, k, log_alpha, beta, flags, gate_scale=1.0):
    """The activated (q, k, log_alpha, beta) from raw ones, per ``flags`` (fp64 arrays)."""
    q, k, la, b = (np.asarray(x, dtype=np.float64) for x in (q, k, log_alpha, beta))
    if flags & QK_L2NORM:
        q, k = l2_normalise(q), l2_normalise(k)
    if flags & GATE_SOFTPLUS:
        la = -gate_scale * softplus(la)
    if flags & BETA_SIGMOID:
        b = sigmoid(b)
    return q, k, la, b
