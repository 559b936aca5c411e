"""ctypes binding of libkda (argument marshalling only; every step runs in the CUDA library).

PyTorch provides device memory and the current CUDA stream. There is no CPU
fallback: if ``libkda.so`` is missing or fails to load, every call raises.

Layouts follow ``include/kda.h``: q, k, log_alpha [T, H, d_k]; v, out [T, H, d_v];
beta [T, H]; states [N, H, d_k, d_v] fp32; cu_seqlens [N + 1] int32. Dense
[B, T, ...] inputs are accepted and packed as B sequences of T tokens.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# KDA_LIB selects another build of the library (e.g. the bounds-checked libkda_debug.so).
LIB_PATH = os.environ.get("KDA_LIB") or os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARGUMENT, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_ERR_INTERNAL = range(6)
KDA_F32, KDA_BF16 = 0, 1

_lock = threading.Lock()
_lib = None

_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t

SIGNATURES = {
    "kda_prefill_workspace_size": (_sz, [_i32, _i64, _i32, _i32, _i32, _i32]),
    "kda_prefill": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32,
                           _i32, _vp, _vp, _vp, _sz, _vp]),
    "kda_prefill_recurrent": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32,
                                     _i32, _i32, _i32, _vp, _vp, _vp]),
    "kda_decode_step": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                               _vp, _sz, _vp]),
    "kda_status_string": (ctypes.c_char_p, [_i32]),
    "kda_last_error": (ctypes.c_char_p, []),
    "kda_read_device_status": (_i32, [_vp, _vp]),
    "kda_version": (_i32, []),
    "kda_last_launch_count": (_i32, []),
    "kda_selftest_bounded_wait": (_i32, [_vp, _sz, ctypes.c_uint64, _vp]),
    "kda_selftest_flag_wait": (_i32, [_vp, _sz, ctypes.c_uint64, _vp]),
    "kda_prefill_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                                   _i32, _i32, _vp, _vp, _vp]),
    "kda_prefill_noalloc_status": (_i32, [_vp]),
    "kda_prefill_cp": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32,
                              _i32, _vp, _vp, _i32, _vp, _sz, _vp]),
    "kda_prefill_cp_workspace_size": (_sz, [_i32, _vp, _i32, _i32, _i32, _i32, _i32]),
    "kda_prefill_slots": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _i32, _i64,
                                 _i32, _i32, _i32, _i32, _vp, _vp, _sz, _vp]),
    "kda_decode_step_slots": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _i32,
                                     _i32, _vp, _vp, _sz, _vp]),
    "kda_decode_verify": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _i32,
                                 _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "kda_decode_commit": (_i32, [_vp, _vp, _vp, _vp, _i64, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                 _i32, _vp, _sz, _vp]),
    "kda_prefill_prologue": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                                    _i32, _i32, _vp, _vp, _vp, _sz, ctypes.c_uint32, ctypes.c_float,
                                    _vp]),
    "kda_decode_commit_verify": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                        _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _sz,
                                        _vp]),
}


class KdaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(message)


def lib():
    """Load libkda.so (raises if it is missing: there is no fallback path)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} not built; run python -m gated_delta_rule_62_b200.build")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _check(status: int, what: str):
    if status != KDA_OK:
        L = lib()
        name = L.kda_status_string(status).decode()
        msg = L.kda_last_error().decode()
        raise KdaError(status, f"{what}: {name}: {msg}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return KDA_BF16
    if dt == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported input dtype {dt}; use bfloat16 or float32")


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


def workspace_size(num_seqs: int, total_tokens: int, H: int, dk: int, dv: int, dtype) -> int:
    return int(lib().kda_prefill_workspace_size(num_seqs, total_tokens, H, dk, dv,
                                                _dtype_code(dtype)))


def prefill(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, cu_seqlens_dev=None,
            out=None, final_state=None, workspace=None, output_final_state=True,
            algo: str = "auto", stream=None, prologue: int = 0, gate_scale: float = 1.0,
            segments: int = 2):
    """Chunked KDA prefill over packed sequences (``kda_prefill``).

    prologue: KDA_PROLOGUE_* flags (``kda_prefill_prologue``): q, k, log_alpha, beta hold the
    layer's raw projections and are activated inside the kernels (gate_scale for the gate).

    q, k, log_alpha: [T, H, d_k] (or [B, T, H, d_k]); v: [T, H, d_v]; beta [T, H].
    cu_seqlens: host int32 offsets [N + 1] (default: one sequence, or B equal ones
    for 4-D inputs); cu_seqlens_dev: the same on the device (copied if omitted).
    algo: "auto" (``kda_prefill``), "recurrent" (``kda_prefill_recurrent``) or "cp"
    (``kda_prefill_cp``: context parallelism, each sequence cut into up to ``segments`` segments).
    Returns (out, final_state or None).
    """
    dense = q.dim() == 4
    if dense:
        B, T = q.shape[:2]
        q, k, v = q.reshape(B * T, *q.shape[2:]), k.reshape(B * T, *k.shape[2:]), v.reshape(B * T, *v.shape[2:])
        log_alpha = log_alpha.reshape(B * T, *log_alpha.shape[2:])
        beta = beta.reshape(B * T, *beta.shape[2:])
        if cu_seqlens is None:
            cu_seqlens = torch.arange(0, (B + 1) * T, T, dtype=torch.int32)
    dtype = q.dtype
    _need(q, "q", ndim=3)
    Ttot, H, dk = q.shape
    dv = v.shape[-1]
    _need(k, "k", dtype, 3)
    _need(v, "v", dtype, 3)
    _need(log_alpha, "log_alpha", torch.float32, 3)
    _need(beta, "beta", torch.float32, 2)
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:2] != (Ttot, H) or beta.shape != (Ttot, H):
        raise ValueError("inconsistent shapes among q, k, v, log_alpha, beta")
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, Ttot], dtype=torch.int32)
    cu_host = torch.as_tensor(cu_seqlens, dtype=torch.int32).cpu().contiguous()
    N = cu_host.numel() - 1
    if cu_seqlens_dev is None:
        cu_seqlens_dev = cu_host.to(q.device, non_blocking=False)
    _need(cu_seqlens_dev, "cu_seqlens_dev", torch.int32, 1)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, 4)
        if tuple(initial_state.shape) != (N, H, dk, dv):
            raise ValueError(f"initial_state must be {(N, H, dk, dv)}")
    if out is None:
        out = torch.empty(Ttot, H, dv, dtype=dtype, device=q.device)
    _need(out, "out", dtype, 3)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, 4)
    L = lib()
    code = _dtype_code(dtype)
    common = [_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
              _ptr(cu_seqlens_dev), ctypes.c_void_p(cu_host.data_ptr()), N, Ttot, H, dk, dv, code,
              _ptr(out), _ptr(final_state)]
    if algo == "recurrent":
        if prologue:
            raise ValueError("the prologue runs through kda_prefill_prologue (algo='auto')")
        _check(L.kda_prefill_recurrent(*common, _stream(stream)), "kda_prefill_recurrent")
    elif algo == "cp":
        if prologue:
            raise ValueError("the prologue runs through kda_prefill_prologue (algo='auto')")
        cu_p = ctypes.c_void_p(cu_host.data_ptr())
        need = int(L.kda_prefill_cp_workspace_size(N, cu_p, H, dk, dv, code, int(segments)))
        if need == 0:
            raise ValueError("kda_prefill_cp_workspace_size rejected the arguments")
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8, 1)
        _check(L.kda_prefill_cp(*common, int(segments), _ptr(workspace), workspace.numel(), _stream(stream)),
               "kda_prefill_cp")
    elif algo == "auto":
        need = workspace_size(N, Ttot, H, dk, dv, dtype)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _need(workspace, "workspace", torch.uint8, 1)
        if prologue:
            _check(L.kda_prefill_prologue(*common, _ptr(workspace), workspace.numel(), int(prologue),
                                          float(gate_scale), _stream(stream)), "kda_prefill_prologue")
        else:
            _check(L.kda_prefill(*common, _ptr(workspace), workspace.numel(), _stream(stream)),
                   "kda_prefill")
    else:
        raise ValueError(f"unknown algo {algo!r}")
    if dense:
        out = out.reshape(B, T, H, dv)
    return out, final_state


def decode_step(q, k, v, log_alpha, beta, state, out=None, stream=None):
    """One decode token per sequence (``kda_decode_step``); ``state`` is updated in place.

    q, k, log_alpha: [N, H, d_k]; v: [N, H, d_v]; beta: [N, H]; state [N, H, d_k, d_v] fp32.
    Returns out [N, H, d_v].
    """
    dtype = q.dtype
    _need(q, "q", ndim=3)
    N, H, dk = q.shape
    dv = v.shape[-1]
    _need(k, "k", dtype, 3)
    _need(v, "v", dtype, 3)
    _need(log_alpha, "log_alpha", torch.float32, 3)
    _need(beta, "beta", torch.float32, 2)
    _need(state, "state", torch.float32, 4)
    if k.shape != q.shape or log_alpha.shape != q.shape or tuple(state.shape) != (N, H, dk, dv):
        raise ValueError("inconsistent shapes among q, k, log_alpha, state")
    if out is None:
        out = torch.empty(N, H, dv, dtype=dtype, device=q.device)
    _need(out, "out", dtype, 3)
    _check(lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                 _ptr(state), N, H, dk, dv, _dtype_code(dtype), _ptr(out), None, 0,
                                 _stream(stream)), "kda_decode_step")
    return out


def prefill_slots(q, k, v, log_alpha, beta, state_pool, init_slot, final_slot, cu_seqlens=None,
                  cu_seqlens_dev=None, out=None, workspace=None, stream=None):
    """Chunked prefill with the states in a pool of slots (``kda_prefill_slots``).

    q, k, log_alpha [T, H, d_k]; v [T, H, d_v]; beta [T, H]; state_pool [P, H, d_k, d_v] fp32
    (read and written); init_slot, final_slot: int32 device tensors [N] (-1: zeros / not stored).
    cu_seqlens: host int32 offsets [N + 1] (default: one sequence). Returns out.
    """
    dtype = q.dtype
    _need(q, "q", ndim=3)
    Ttot, H, dk = q.shape
    dv = v.shape[-1]
    _need(k, "k", dtype, 3)
    _need(v, "v", dtype, 3)
    _need(log_alpha, "log_alpha", torch.float32, 3)
    _need(beta, "beta", torch.float32, 2)
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:2] != (Ttot, H) or beta.shape != (Ttot, H):
        raise ValueError("inconsistent shapes among q, k, v, log_alpha, beta")
    _need(state_pool, "state_pool", torch.float32, 4)
    P = state_pool.shape[0]
    if tuple(state_pool.shape[1:]) != (H, dk, dv):
        raise ValueError(f"state_pool must be [P, {H}, {dk}, {dv}]")
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, Ttot], dtype=torch.int32)
    cu_host = torch.as_tensor(cu_seqlens, dtype=torch.int32).cpu().contiguous()
    N = cu_host.numel() - 1
    if cu_seqlens_dev is None:
        cu_seqlens_dev = cu_host.to(q.device, non_blocking=False)
    _need(cu_seqlens_dev, "cu_seqlens_dev", torch.int32, 1)
    for t, name in ((init_slot, "init_slot"), (final_slot, "final_slot")):
        _need(t, name, torch.int32, 1)
        if t.numel() != N:
            raise ValueError(f"{name} must have {N} entries")
    if out is None:
        out = torch.empty(Ttot, H, dv, dtype=dtype, device=q.device)
    _need(out, "out", dtype, 3)
    if workspace is None:
        workspace = torch.empty(workspace_size(N, Ttot, H, dk, dv, dtype), dtype=torch.uint8,
                                device=q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    _check(lib().kda_prefill_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                   _ptr(state_pool), P, _ptr(init_slot), _ptr(final_slot),
                                   _ptr(cu_seqlens_dev), ctypes.c_void_p(cu_host.data_ptr()), N,
                                   Ttot, H, dk, dv, _dtype_code(dtype), _ptr(out), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "kda_prefill_slots")
    return out


def decode_step_slots(q, k, v, log_alpha, beta, state_pool, slot, out=None, workspace=None,
                      stream=None):
    """One decode token per sequence on pooled states (``kda_decode_step_slots``).

    state_pool [P, H, d_k, d_v] fp32, updated in place at slot[n] (int32 device [N]; -1: a zero
    state that is not stored). Returns out [N, H, d_v].
    """
    dtype = q.dtype
    _need(q, "q", ndim=3)
    N, H, dk = q.shape
    dv = v.shape[-1]
    _need(k, "k", dtype, 3)
    _need(v, "v", dtype, 3)
    _need(log_alpha, "log_alpha", torch.float32, 3)
    _need(beta, "beta", torch.float32, 2)
    _need(state_pool, "state_pool", torch.float32, 4)
    _need(slot, "slot", torch.int32, 1)
    if k.shape != q.shape or log_alpha.shape != q.shape or tuple(state_pool.shape[1:]) != (H, dk, dv) \
            or slot.numel() != N:
        raise ValueError("inconsistent shapes among q, k, log_alpha, state_pool, slot")
    if out is None:
        out = torch.empty(N, H, dv, dtype=dtype, device=q.device)
    _need(out, "out", dtype, 3)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    _check(lib().kda_decode_step_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                       _ptr(state_pool), state_pool.shape[0], _ptr(slot), N, H, dk,
                                       dv, _dtype_code(dtype), _ptr(out), _ptr(workspace),
                                       workspace.numel(), _stream(stream)), "kda_decode_step_slots")
    return out


MAX_DRAFT_TOKENS = 16
PROLOGUE_QK_L2NORM, PROLOGUE_GATE_SOFTPLUS, PROLOGUE_BETA_SIGMOID = 1, 2, 4
PROLOGUE_ALL = 7


def _pool_args(state, slot, N, H, dk, dv):
    _need(state, "state", torch.float32, 4)
    if tuple(state.shape[1:]) != (H, dk, dv):
        raise ValueError(f"state shape {tuple(state.shape)} does not end in {(H, dk, dv)}")
    if slot is None:
        if state.shape[0] != N:
            raise ValueError(f"state holds {state.shape[0]} entries for {N} sequences")
        return state.shape[0], None
    _need(slot, "slot", torch.int32, 1)
    if slot.numel() != N:
        raise ValueError("slot must have one entry per sequence")
    return state.shape[0], slot


def decode_verify(q, k, v, log_alpha, beta, state, slot=None, out=None, u_cache=None,
                  workspace=None, stream=None):
    """Check T draft tokens per sequence in one pass (``kda_decode_verify``); states unchanged.

    q, k [N, T, H, d_k]; v [N, T, H, d_v]; log_alpha [N, T, H, d_k] fp32; beta [N, T, H] fp32;
    state [N, H, d_k, d_v] fp32, or a pool [P, ...] addressed by ``slot`` (int32 device [N]).
    Returns (out, u_cache), both [N, T, H, d_v] (out in the input dtype, u_cache fp32).
    """
    dtype = q.dtype
    _need(q, "q", ndim=4)
    N, T, H, dk = q.shape
    dv = v.shape[-1]
    _need(k, "k", dtype, 4)
    _need(v, "v", dtype, 4)
    _need(log_alpha, "log_alpha", torch.float32, 4)
    _need(beta, "beta", torch.float32, 3)
    if k.shape != q.shape or log_alpha.shape != q.shape or tuple(v.shape[:3]) != (N, T, H) \
            or tuple(beta.shape) != (N, T, H):
        raise ValueError("inconsistent shapes among q, k, v, log_alpha, beta")
    P, slot = _pool_args(state, slot, N, H, dk, dv)
    if out is None:
        out = torch.empty(N, T, H, dv, dtype=dtype, device=q.device)
    if u_cache is None:
        u_cache = torch.empty(N, T, H, dv, dtype=torch.float32, device=q.device)
    _need(out, "out", dtype, 4)
    _need(u_cache, "u_cache", torch.float32, 4)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    _check(lib().kda_decode_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                   _ptr(state), P, _ptr(slot), N, T, H, dk, dv, _dtype_code(dtype),
                                   _ptr(out), _ptr(u_cache), _ptr(workspace), workspace.numel(),
                                   _stream(stream)), "kda_decode_verify")
    return out, u_cache


def decode_commit(k, log_alpha, u_cache, state, accepted, slot=None, workspace=None, stream=None):
    """Advance each state by its accepted draft tokens (``kda_decode_commit``), in place.

    k, log_alpha, u_cache as given to / returned by :func:`decode_verify`; accepted int32 device
    [N], each in [0, T].
    """
    _need(k, "k", ndim=4)
    N, T, H, dk = k.shape
    dv = u_cache.shape[-1]
    _need(log_alpha, "log_alpha", torch.float32, 4)
    _need(u_cache, "u_cache", torch.float32, 4)
    _need(accepted, "accepted", torch.int32, 1)
    if log_alpha.shape != k.shape or tuple(u_cache.shape[:3]) != (N, T, H) or accepted.numel() != N:
        raise ValueError("inconsistent shapes among k, log_alpha, u_cache, accepted")
    P, slot = _pool_args(state, slot, N, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=k.device)
    _need(workspace, "workspace", torch.uint8, 1)
    _check(lib().kda_decode_commit(_ptr(k), _ptr(log_alpha), _ptr(u_cache), _ptr(state), P,
                                   _ptr(slot), _ptr(accepted), N, T, H, dk, dv,
                                   _dtype_code(k.dtype), _ptr(workspace), workspace.numel(),
                                   _stream(stream)), "kda_decode_commit")


def decode_commit_verify(prev_k, prev_log_alpha, prev_u, accepted, q, k, v, log_alpha, beta, state,
                         slot=None, out=None, u_cache=None, workspace=None, stream=None):
    """Commit the previous draft's accepted tokens and verify the next draft in one pass over the
    states (``kda_decode_commit_verify``). prev_* as the previous :func:`decode_verify` took and
    returned them ([N, T_prev, H, ...]); the rest as :func:`decode_verify`. Returns (out, u_cache),
    which must be new buffers (not prev_u)."""
    _need(prev_k, "prev_k", q.dtype, 4)
    _need(prev_log_alpha, "prev_log_alpha", torch.float32, 4)
    _need(prev_u, "prev_u", torch.float32, 4)
    _need(accepted, "accepted", torch.int32, 1)
    _need(q, "q", ndim=4)
    N, T, H, dk = q.shape
    dv = v.shape[-1]
    Tp = prev_k.shape[1]
    if prev_log_alpha.shape != prev_k.shape or tuple(prev_k.shape) != (N, Tp, H, dk) \
            or tuple(prev_u.shape) != (N, Tp, H, dv) or accepted.numel() != N:
        raise ValueError("inconsistent shapes among prev_k, prev_log_alpha, prev_u, accepted")
    _need(k, "k", q.dtype, 4)
    _need(v, "v", q.dtype, 4)
    _need(log_alpha, "log_alpha", torch.float32, 4)
    _need(beta, "beta", torch.float32, 3)
    if k.shape != q.shape or log_alpha.shape != q.shape or tuple(v.shape[:3]) != (N, T, H) \
            or tuple(beta.shape) != (N, T, H):
        raise ValueError("inconsistent shapes among q, k, v, log_alpha, beta")
    P, slot = _pool_args(state, slot, N, H, dk, dv)
    if out is None:
        out = torch.empty(N, T, H, dv, dtype=q.dtype, device=q.device)
    if u_cache is None:
        u_cache = torch.empty(N, T, H, dv, dtype=torch.float32, device=q.device)
    _need(out, "out", q.dtype, 4)
    _need(u_cache, "u_cache", torch.float32, 4)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    _check(lib().kda_decode_commit_verify(_ptr(prev_k), _ptr(prev_log_alpha), _ptr(prev_u),
                                          _ptr(accepted), Tp, _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(log_alpha), _ptr(beta), _ptr(state), P, _ptr(slot), N,
                                          T, H, dk, dv, _dtype_code(q.dtype), _ptr(out), _ptr(u_cache),
                                          _ptr(workspace), workspace.numel(), _stream(stream)),
           "kda_decode_commit_verify")
    return out, u_cache


def last_launch_count() -> int:
    """Kernels enqueued by this thread's last successful library call (``kda_last_launch_count``)."""
    return int(lib().kda_last_launch_count())


def selftest_bounded_wait(workspace, timeout_ns: int, stream=None):
    """Launch the bounded-wait probe (a wait nothing releases); see kda.h."""
    _check(lib().kda_selftest_bounded_wait(_ptr(workspace), workspace.numel(), int(timeout_ns),
                                           _stream(stream)), "kda_selftest_bounded_wait")


def selftest_flag_wait(workspace, timeout_ns: int, stream=None):
    """Launch the flag-wait probe (a global flag nothing releases); see kda.h."""
    _check(lib().kda_selftest_flag_wait(_ptr(workspace), workspace.numel(), int(timeout_ns),
                                        _stream(stream)), "kda_selftest_flag_wait")


def read_device_status(workspace, stream=None) -> int:
    """Status word of the last kda_prefill that used ``workspace`` (synchronises the stream)."""
    st = lib().kda_read_device_status(_ptr(workspace), _stream(stream))
    return int(st)
