"""Canary guard bands around every buffer the library writes, for the GPU tests.

compute-sanitizer is not available to these tests, so out-of-bounds writes are caught another
way: each output (and each state updated in place) the library is given lives inside one larger
allocation whose GUARD bytes before and after it are filled with a canary byte. After the call
the stream is synchronised and both bands must still hold the canary; a kernel that writes past
either end of a buffer fails the test that made the call.

Calls made while a CUDA graph is being captured go straight to the binding (a band check
synchronises the device, which a capture does not allow).

``install(K)`` replaces the binding's entry points (prefill, decode_step, prefill_slots,
decode_step_slots, decode_verify, decode_commit, decode_commit_verify) by guarded versions with
the same signatures: outputs the caller did not pass are allocated guarded, in-place states are
copied into guarded buffers, run there and copied back. ``checks()`` counts the bands checked.
"""
from __future__ import annotations

import functools
import inspect
import math

import torch

GUARD = 4096  # bytes each side (keeps the view 16-byte aligned)
CANARY = 0xA5
_count = {"bands": 0}


class _Bands:
    def __init__(self):
        self.items = []

    def empty(self, shape, dtype, device):
        n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        buf = torch.full((n + 2 * GUARD,), CANARY, dtype=torch.uint8, device=device)
        self.items.append((buf, n))
        return buf[GUARD:GUARD + n].view(dtype).view(*shape)

    def copy_of(self, t):
        g = self.empty(tuple(t.shape), t.dtype, t.device)
        g.copy_(t)
        return g

    def check(self, what):
        if not self.items:
            return
        torch.cuda.synchronize()
        for buf, n in self.items:
            lo, hi = buf[:GUARD], buf[GUARD + n:]
            bad_lo = int((lo != CANARY).sum())
            bad_hi = int((hi != CANARY).sum())
            assert bad_lo == 0 and bad_hi == 0, (
                f"{what}: {bad_lo} bytes before and {bad_hi} bytes after a {n}-byte output "
                f"were overwritten (out-of-bounds write)")
            _count["bands"] += 2


def checks() -> int:
    return _count["bands"]


def _seqs(a):
    cu = a.get("cu_seqlens")
    if cu is not None:
        return len(cu) - 1
    q = a["q"]
    return q.shape[0] if q.dim() == 4 else 1


def _guard_prefill(orig):
    sig = inspect.signature(orig)

    @functools.wraps(orig)
    def f(*args, **kwargs):
        if torch.cuda.is_current_stream_capturing():  # no synchronising check inside a CUDA graph
            return orig(*args, **kwargs)
        b = sig.bind(*args, **kwargs)
        a = b.arguments
        bands = _Bands()
        q, v = a["q"], a["v"]
        Ttot = q.shape[0] * q.shape[1] if q.dim() == 4 else q.shape[0]
        H, dk, dv = q.shape[-2], q.shape[-1], v.shape[-1]
        if a.get("out") is None:
            a["out"] = bands.empty((Ttot, H, dv), q.dtype, q.device)
        if a.get("final_state") is None and a.get("output_final_state", True):
            a["final_state"] = bands.empty((_seqs(a), H, dk, dv), torch.float32, q.device)
        r = orig(*b.args, **b.kwargs)
        bands.check("prefill")
        return r

    return f


def _guard_inplace(orig, name, outs, states):
    """outs: {arg: shape function of the bound arguments -> (shape, dtype)}; states: in-place args."""
    sig = inspect.signature(orig)

    @functools.wraps(orig)
    def f(*args, **kwargs):
        if torch.cuda.is_current_stream_capturing():  # no synchronising check inside a CUDA graph
            return orig(*args, **kwargs)
        b = sig.bind(*args, **kwargs)
        a = b.arguments
        bands = _Bands()
        for arg, shape_of in outs.items():
            if a.get(arg) is None:
                shape, dtype, dev = shape_of(a)
                a[arg] = bands.empty(shape, dtype, dev)
        originals = {}
        for arg in states:
            t = a.get(arg)
            if t is not None:
                originals[arg] = t
                a[arg] = bands.copy_of(t)
        r = orig(*b.args, **b.kwargs)
        bands.check(name)
        for arg, t in originals.items():
            t.copy_(a[arg])
        return r

    return f


def install(K):
    """Replace K's entry points by guarded versions (idempotent)."""
    if getattr(K, "_guards_installed", False):
        return
    K.prefill = _guard_prefill(K.prefill)
    K.decode_step = _guard_inplace(
        K.decode_step, "decode_step",
        {"out": lambda a: ((*a["q"].shape[:2], a["v"].shape[-1]), a["q"].dtype, a["q"].device)}, ["state"])
    K.prefill_slots = _guard_inplace(
        K.prefill_slots, "prefill_slots",
        {"out": lambda a: ((*a["q"].shape[:2], a["v"].shape[-1]), a["q"].dtype, a["q"].device)}, ["state_pool"])
    K.decode_step_slots = _guard_inplace(
        K.decode_step_slots, "decode_step_slots",
        {"out": lambda a: ((*a["q"].shape[:2], a["v"].shape[-1]), a["q"].dtype, a["q"].device)}, ["state_pool"])
    spec_out = {"out": lambda a: ((*a["q"].shape[:3], a["v"].shape[-1]), a["q"].dtype, a["q"].device),
                "u_cache": lambda a: ((*a["q"].shape[:3], a["v"].shape[-1]), torch.float32, a["q"].device)}
    K.decode_verify = _guard_inplace(K.decode_verify, "decode_verify", spec_out, ["state"])
    K.decode_commit = _guard_inplace(K.decode_commit, "decode_commit", {}, ["state"])
    K.decode_commit_verify = _guard_inplace(K.decode_commit_verify, "decode_commit_verify", spec_out, ["state"])
    K._guards_installed = True
