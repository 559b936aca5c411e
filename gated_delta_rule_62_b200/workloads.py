"""Seeded synthetic inputs for the KDA recurrence (shared by tests, bench and smoke).

This module holds only input recipes: shapes, seeds and value distributions.
It contains none of the recurrence's arithmetic, so both the CUDA path and the
CPU oracle can consume what it produces without sharing method code.

Recipe (the pages give no workload beyond "million-token context", decode at
constant per-token cost and prefix-cache resume; these synthetic shapes stand in
for them):

* q, k ~ N(0, 1), then L2-normalised over the key channels per token and head
  (in fp32), then cast to the input dtype;
* v ~ N(0, 1), cast to the input dtype;
* beta = sigmoid(N(0, 1)) in fp32, one per token and head (writing strength);
* log_alpha = -softplus(N(0, 1)) / 16 in fp32, one per token, head and key
  channel (channel-wise forgetting factor alpha = exp(log_alpha) in (0, 1]);
* initial state: zero, N(0, 0.02^2) per element, or the state left by a
  prefill (decode workload), always fp32 with layout [N, H, d_k, d_v].

Layouts (d contiguous): q, k, log_alpha [T_total, H, d_k]; v [T_total, H, d_v];
beta [T_total, H]; cu_seqlens [N + 1] int32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

# Tokens drawn per generator call; fixed so results do not depend on how many
# tokens a caller asks for at once.
_DRAW_BLOCK = 16384


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: sequence lengths, head geometry and dtypes."""

    name: str
    seed: int
    seqlens: tuple
    H: int
    dk: int
    dv: int
    dtype: str = "bf16"  # dtype of q, k, v and out: "bf16" or "f32"
    init_state: str = "zero"  # "zero" | "normal" (std 0.02) | "prefill"
    decode_steps: int = 0  # >0: a decode workload (one token per sequence per step)

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def describe(self) -> dict:
        d = {"workload": self.name, "num_seqs": self.num_seqs, "H": self.H,
             "d_k": self.dk, "d_v": self.dv, "dtype": self.dtype,
             "total_tokens": self.total_tokens, "init_state": self.init_state}
        if self.decode_steps:
            d["decode_steps"] = self.decode_steps
        return d


def varlen_lengths(n: int = 24, lo: int = 512, hi: int = 65536, seed: int = 5) -> tuple:
    """Log-uniform sequence lengths floor(exp(U[ln lo, ln hi])) from numpy's PCG64."""
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return tuple(int(x) for x in np.floor(np.exp(u)))


# The five workloads: a tiny fp32 single-chunk case, a 8K-token 32-head prefill,
# a 256-sequence decode, a million-token prefill and a 24-sequence varlen pack
# that resumes from random states.
TINY_F32 = Workload("tiny_prefill_T64_H2_d32_f32", 1001, (64,), 2, 32, 32, "f32")
PREFILL_8K = Workload("prefill_B1_T8192_H32_d128_bf16", 1002, (8192,), 32, 128, 128, "bf16")
DECODE_256 = Workload("decode_N256_H32_d128_bf16_1024steps", 1003, (512,) * 256, 32, 128, 128,
                      "bf16", init_state="prefill", decode_steps=1024)
PREFILL_1M = Workload("prefill_B1_T1048576_H16_d128_bf16", 1004, (1 << 20,), 16, 128, 128, "bf16")
VARLEN_24 = Workload("varlen_24seq_logU512-65536_H32_d128_bf16_resume", 1005,
                     varlen_lengths(), 32, 128, 128, "bf16", init_state="normal")

# Not a benchmark line: 64 of the decode workload's 512-token seeding prefills (2,048 chains, the
# fused kernel's regime), 1.8 GB on the device, for profiler captures that replay each launch.
PREFILL_64x512 = Workload("prefill_N64_T512_H32_d128_bf16", 1006, (512,) * 64, 32, 128, 128, "bf16")

WORKLOADS = {w.name: w for w in (TINY_F32, PREFILL_8K, DECODE_256, PREFILL_1M, VARLEN_24, PREFILL_64x512)}


def custom(seqlens, H, dk, dv, dtype="bf16", seed=7, init_state="zero", name=None) -> Workload:
    """A workload with explicit lengths (tests use these for edge shapes)."""
    seqlens = tuple(int(x) for x in seqlens)
    return Workload(name or f"custom_{len(seqlens)}seq_H{H}_dk{dk}_dv{dv}_{dtype}", seed,
                    seqlens, H, dk, dv, dtype, init_state)


def cu_seqlens_of(seqlens) -> np.ndarray:
    out = np.zeros(len(seqlens) + 1, dtype=np.int32)
    if len(seqlens):
        out[1:] = np.cumsum(np.asarray(seqlens, dtype=np.int64))
    if out[-1] > np.iinfo(np.int32).max:
        raise ValueError("total tokens exceed int32 cu_seqlens")
    return out


# log alpha = -softplus(g) * GATE_SCALE with g ~ N(0, 1) (the workloads' gate distribution)
GATE_SCALE = 1.0 / 16.0


def _l2n(x: torch.Tensor) -> torch.Tensor:
    # Input recipe, not method arithmetic: unit-norm keys/queries per token and head.
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-30)


def draw_tokens(gen: torch.Generator, ntok: int, H: int, dk: int, dv: int,
                dtype: torch.dtype, device, raw: bool = False) -> dict:
    """Draw ``ntok`` tokens of (q, k, v, beta, log_alpha) in blocks of _DRAW_BLOCK.

    ``raw``: the same draws before activation (q, k not normalised; ``log_alpha`` holds the
    N(0, 1) gates and ``beta`` the N(0, 1) logits), the inputs of the fused-prologue prefill."""
    q = torch.empty(ntok, H, dk, dtype=dtype, device=device)
    k = torch.empty(ntok, H, dk, dtype=dtype, device=device)
    v = torch.empty(ntok, H, dv, dtype=dtype, device=device)
    beta = torch.empty(ntok, H, dtype=torch.float32, device=device)
    la = torch.empty(ntok, H, dk, dtype=torch.float32, device=device)
    for s in range(0, ntok, _DRAW_BLOCK):
        n = min(_DRAW_BLOCK, ntok - s)
        f32 = dict(dtype=torch.float32, device=device, generator=gen)
        act = (lambda x: x) if raw else _l2n
        q[s:s + n] = act(torch.randn(n, H, dk, **f32)).to(dtype)
        k[s:s + n] = act(torch.randn(n, H, dk, **f32)).to(dtype)
        v[s:s + n] = torch.randn(n, H, dv, **f32).to(dtype)
        b = torch.randn(n, H, **f32)
        beta[s:s + n] = b if raw else torch.sigmoid(b)
        g = torch.randn(n, H, dk, **f32)
        la[s:s + n] = g if raw else -torch.nn.functional.softplus(g) * GATE_SCALE
    return {"q": q, "k": k, "v": v, "beta": beta, "log_alpha": la}


def make_inputs(wl: Workload, device="cpu", seed: Optional[int] = None, raw: bool = False) -> dict:
    """Prefill inputs of a workload: q, k, v, beta, log_alpha, initial_state, cu_seqlens.

    ``initial_state`` is None for a zero start. ``cu_seqlens`` is a CPU int32
    tensor; ``cu_seqlens_dev`` is the same on ``device``. For the decode
    workload these are the inputs of the 512-token prefill that seeds the state.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed if seed is None else seed)
    d = draw_tokens(gen, wl.total_tokens, wl.H, wl.dk, wl.dv, wl.torch_dtype, device, raw=raw)
    if wl.init_state == "normal":
        d["initial_state"] = 0.02 * torch.randn(wl.num_seqs, wl.H, wl.dk, wl.dv,
                                                dtype=torch.float32, device=device, generator=gen)
    else:
        d["initial_state"] = None
    cu = torch.from_numpy(cu_seqlens_of(wl.seqlens))
    d["cu_seqlens"] = cu
    d["cu_seqlens_dev"] = cu.to(device)
    d["_gen"] = gen
    return d


def make_decode_steps(wl: Workload, gen: torch.Generator, steps: int, device="cpu") -> dict:
    """Per-step decode inputs, stacked: q, k, log_alpha [steps, N, H, d_k]; v [steps, N, H, d_v];
    beta [steps, N, H]. Drawn after the seeding prefill's tokens from the same generator."""
    N = wl.num_seqs
    d = draw_tokens(gen, steps * N, wl.H, wl.dk, wl.dv, wl.torch_dtype, device)
    return {k_: t.reshape(steps, N, *t.shape[1:]) for k_, t in d.items()}


def to_f64_numpy(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """Exact upcast of a tensor's values (bf16/fp32 -> fp64) to a contiguous numpy array."""
    if t is None:
        return None
    return np.ascontiguousarray(t.detach().to("cpu", torch.float64).numpy())
