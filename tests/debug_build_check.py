"""Runs small prefills and decode steps on the bounds-checked build (KDA_LIB=.../libkda_debug.so).

Called by tests/test_gpu_debug_build.py in a subprocess, so the checked library is the only one
loaded in that process. Mode "clean": every kernel family on small ragged shapes must report
KDA_OK and match the oracle. Mode "shrunk" (KDA_DEBUG_SHRINK_OUT set): the output is declared
shorter than it is, and the writes past that point must be skipped and reported."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from gated_delta_rule_62_b200 import kda as K  # noqa: E402
from gated_delta_rule_62_b200 import workloads as W  # noqa: E402

f64 = W.to_f64_numpy


def check(out, fs, inp, tol, what):
    ro, rs = oracle.forward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["log_alpha"]),
                            f64(inp["beta"]), f64(inp.get("initial_state")), inp["cu_seqlens"].numpy())
    scale = float(inp["v"].abs().max())
    eo = float(np.abs(f64(out) - ro).max())
    es = float(np.abs(f64(fs) - rs).max())
    assert eo <= tol * scale and es <= tol * scale, (what, eo, es)


def run(wl, algo="auto", minimal_ws=False, segments=2):
    inp = W.make_inputs(wl, "cuda")
    N, T, H = wl.num_seqs, wl.total_tokens, wl.H
    if algo == "cp":
        import ctypes
        n = int(K.lib().kda_prefill_cp_workspace_size(N, ctypes.c_void_p(inp["cu_seqlens"].data_ptr()), H,
                                                      wl.dk, wl.dv, K.KDA_BF16, segments))
    elif minimal_ws:
        n = 256 + (4 * N + 255) // 256 * 256
    else:
        n = max(256, K.workspace_size(N, T, H, wl.dk, wl.dv, wl.torch_dtype))
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["initial_state"],
                        inp["cu_seqlens"], inp["cu_seqlens_dev"], workspace=None if algo == "recurrent" else ws,
                        algo=algo, segments=segments)
    st = K.read_device_status(ws) if algo != "recurrent" else K.KDA_OK
    return inp, out, fs, st, ws


def clean():
    oracle.build()
    few = W.custom((700, 0, 65, 130), 3, 128, 128, "bf16", seed=3, init_state="normal")
    cases = [("split", few, "auto", False), ("fused", few, "auto", True),
             ("recurrent f32", W.custom((90, 33), 2, 64, 64, "f32", seed=4, init_state="normal"), "recurrent", False),
             ("token-serial via kda_prefill", W.custom((50,), 2, 32, 32, "bf16", seed=6), "auto", False),
             ("context parallel", W.custom((1300, 200), 2, 128, 128, "bf16", seed=5, init_state="normal"), "cp", False)]
    for what, wl, algo, minimal in cases:
        inp, out, fs, st, _ = run(wl, algo, minimal)
        assert st == K.KDA_OK, (what, st, K.lib().kda_last_error())
        check(out, fs, inp, 1e-4 if wl.dtype == "f32" else 2e-2, what)
    # decode with a slot table (its workspace carries the status word)
    g = torch.Generator(device="cuda").manual_seed(9)
    d = W.make_decode_steps(W.custom((1,) * 3, 2, 128, 128), g, 1, "cuda")
    d = {n: t[0] for n, t in d.items()}
    pool = torch.randn(5, 2, 128, 128, device="cuda", generator=g)
    slots = torch.tensor([4, 0, 2], dtype=torch.int32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    ref_s = f64(pool[[4, 0, 2]])
    out = K.decode_step_slots(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, slots, workspace=ws)
    assert K.read_device_status(ws) == K.KDA_OK
    ro, rs = oracle.forward(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["log_alpha"]), f64(d["beta"]), ref_s,
                            np.arange(4))
    scale = float(d["v"].abs().max())
    assert float(np.abs(f64(out) - ro).max()) <= 2e-2 * scale
    assert float(np.abs(f64(pool[[4, 0, 2]]) - rs).max()) <= 2e-2 * scale
    print("clean ok")


def shrunk():
    """The output is declared to end after `keep` bytes: tokens past that point are not written."""
    keep = int(os.environ["KDA_DEBUG_SHRINK_OUT"])
    for what, minimal in (("split", False), ("fused", True)):
        wl = W.custom((300,), 2, 128, 128, "bf16", seed=8)
        inp = W.make_inputs(wl, "cuda")
        ws = torch.empty(256 + 256 if minimal else K.workspace_size(1, 300, 2, 128, 128, torch.bfloat16),
                         dtype=torch.uint8, device="cuda")
        out = torch.full((300, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None, inp["cu_seqlens"],
                  inp["cu_seqlens_dev"], out=out, workspace=ws)
        st = K.read_device_status(ws)
        msg = K.lib().kda_last_error().decode()
        assert st == K.KDA_ERR_INTERNAL, (what, st, msg)
        assert "outside its buffer" in msg, msg
        flat = out.view(-1)
        n_keep = keep // 2
        assert torch.isnan(flat[n_keep:].float()).all(), what      # past the declared end: untouched
        assert torch.isfinite(flat[:n_keep].float()).all(), what   # before it: written
        print(what, "shrunk ok:", msg)


if __name__ == "__main__":
    torch.cuda.set_device(0)
    {"clean": clean, "shrunk": shrunk}[sys.argv[1]]()
