"""kda_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Callers such as an allocator or memory-pool callback, or a serving loop whose
device memory is fixed at start-up, cannot cudaMalloc a workspace when they run
a prefill. kda_prefill_noalloc takes no workspace and uses a fixed scratch array
inside the library instead. These tests call it through the C ABI and compare it
with kda_prefill (which takes a caller-allocated workspace) and with the fp64
oracle on two calls in a row, so the second call also shows that what the first
left in the shared scratch does not leak into its result; the status word the
calls leave in that scratch must read KDA_OK. This file is named so that pytest
collects it last.
"""
import ctypes

import numpy as np

import pytest
import torch

from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W
import oracle

MAX_SEQS = 16320  # (64 KiB - 256 B status word) / 4 B per scheduled sequence


def _noalloc(inp, out, fs, num_seqs=None):
    L = K.lib()
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    cu = inp["cu_seqlens"]
    N = cu.numel() - 1 if num_seqs is None else num_seqs
    T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    return L.kda_prefill_noalloc(p(inp["q"]), p(inp["k"]), p(inp["v"]), p(inp["log_alpha"]),
                                 p(inp["beta"]), p(inp.get("initial_state")),
                                 p(inp["cu_seqlens_dev"]), ctypes.c_void_p(cu.data_ptr()), N, T, H,
                                 dk, dv, K.KDA_BF16 if inp["q"].dtype == torch.bfloat16 else K.KDA_F32,
                                 p(out), p(fs), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_rejects_more_sequences_than_its_scratch_holds():
    """Host-side check only: nothing is enqueued (runs without a GPU)."""
    L = K.lib()
    N = MAX_SEQS + 1
    cu = (ctypes.c_int32 * (N + 1))(*range(N + 1))
    fake = ctypes.c_void_p(0x10000)
    rc = L.kda_prefill_noalloc(fake, fake, fake, fake, fake, None, fake, ctypes.cast(cu, ctypes.c_void_p),
                               N, N, 2, 128, 128, K.KDA_BF16, ctypes.c_void_p(0x20000), None, None)
    assert rc == K.KDA_ERR_INVALID_ARGUMENT
    assert b"scratch limit" in L.kda_last_error()


@pytest.mark.gpu
def test_noalloc_matches_prefill_on_two_calls_in_a_row():
    torch.cuda.set_device(0)
    oracle.build()
    problems = [((300, 0, 65, 128, 1), 31), ((200, 77, 9), 32)]  # different N, lengths, seeds
    for lens, seed in problems:
        wl = W.custom(lens, 4, 128, 128, "bf16", seed=seed, init_state="normal")
        inp = W.make_inputs(wl, "cuda")
        ref_out, ref_fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                    inp["initial_state"], inp["cu_seqlens"], inp["cu_seqlens_dev"])
        out = torch.full_like(ref_out, float("nan"))
        fs = torch.full_like(ref_fs, float("nan"))
        rc = _noalloc(inp, out, fs)
        assert rc == K.KDA_OK, K.lib().kda_last_error()
        torch.cuda.synchronize()
        tol = 2e-2 * float(inp["v"].abs().max())  # bf16 inputs with an fp32 state
        assert torch.isfinite(out).all() and torch.isfinite(fs).all()
        assert float((out.float() - ref_out.float()).abs().max()) <= tol, lens
        assert float((fs - ref_fs).abs().max()) <= tol, lens
        # and against the oracle directly, on the same input bits
        f64 = W.to_f64_numpy
        ro, rs = oracle.forward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["log_alpha"]),
                                f64(inp["beta"]), f64(inp["initial_state"]), inp["cu_seqlens"].numpy())
        assert float(np.abs(f64(out) - ro).max()) <= tol, lens
        assert float(np.abs(f64(fs) - rs).max()) <= tol, lens
        assert K.lib().kda_prefill_noalloc_status(
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == K.KDA_OK
