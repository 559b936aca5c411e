"""Decode step on the GPU vs the fp64 oracle (a decode step is a one-token prefill)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W
from tests.gpu_helpers import TOL, assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_62_b200 import build
    build.build()
    oracle.build()


def _oracle_step(d, s):
    N = d["q"].shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    s = f64(s) if isinstance(s, torch.Tensor) else np.asarray(s, dtype=np.float64)
    return oracle.forward(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["log_alpha"]), f64(d["beta"]),
                          s, cu)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (32, 128), (128, 64), (64, 32)])
def test_decode_steps(dtype, dk, dv):
    wl = W.custom((1,) * 5, 3, dk, dv, dtype, seed=dk + 3 * dv)
    g = torch.Generator(device=DEV).manual_seed(17)
    state = torch.randn(5, 3, dk, dv, device=DEV, generator=g)
    steps = W.make_decode_steps(wl, g, 4, DEV)
    ref_s = f64(state)
    for t in range(4):
        d = {n: steps[n][t] for n in steps}
        out = K.decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state)
        ro, ref_s = _oracle_step(d, ref_s)
        scale = float(d["v"].abs().max())
        assert_close(out, ro, TOL[dtype], scale, f"decode out step {t}")
        assert_close(state, ref_s, TOL[dtype], scale, f"decode state step {t}")
        ref_s = f64(state)  # continue from the GPU state (no drift across steps)


def test_decode_equals_one_token_prefill():
    wl = W.custom((1,) * 7, 4, 128, 128, "bf16", seed=21, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    s = inp["initial_state"].clone()
    out_d = K.decode_step(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], s)
    out_p, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          inp["initial_state"], inp["cu_seqlens"], inp["cu_seqlens_dev"])
    # the decode kernel computes in fp32; the chunk kernel rounds MMA operands to bf16
    tol = 2e-2 * float(inp["v"].abs().max())
    assert float((out_d.float() - out_p.float()).abs().max()) <= tol
    assert float((s - fs).abs().max()) <= tol


def test_decode_256_sequences_from_prefill_state():
    """The 256-sequence, 32-head decode workload: state seeded by a 512-token GPU prefill, then
    decode steps checked against the oracle started from the GPU's seeded state."""
    wl = W.DECODE_256
    inp = W.make_inputs(wl, DEV)
    _, state = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                         inp["cu_seqlens"], inp["cu_seqlens_dev"])
    steps = W.make_decode_steps(wl, inp["_gen"], 3, DEV)
    ref_s = f64(state)
    for t in range(3):
        d = {n: steps[n][t] for n in steps}
        out = K.decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state)
        ro, ref_s = _oracle_step(d, ref_s)
        scale = float(d["v"].abs().max())
        assert_close(out, ro, TOL["bf16"], scale, f"decode256 out step {t}")
        assert_close(state, ref_s, TOL["bf16"], scale, f"decode256 state step {t}")


def test_decode_1024_steps_against_oracle_without_reseeding():
    """The full decode workload: 256 sequences x 32 heads seeded by the 512-token GPU prefill, then
    1,024 GPU decode steps. The oracle starts once from the GPU's seeded states and runs the same
    1,024 tokens per sequence on its own (no re-seeding between steps), so accumulated drift is
    compared. Oracle subset: 16 evenly spaced sequences x all 32 heads; every step's output and the
    final state are compared element by element at the bf16 tolerance."""
    wl = W.DECODE_256
    steps_n = wl.decode_steps
    inp = W.make_inputs(wl, DEV)
    _, state = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                         inp["cu_seqlens"], inp["cu_seqlens_dev"])
    sub = torch.arange(0, wl.num_seqs, wl.num_seqs // 16, device=DEV)
    assert sub.numel() == 16
    seeded = f64(state[sub])
    steps = W.make_decode_steps(wl, inp["_gen"], steps_n, DEV)
    outs = torch.empty(steps_n, sub.numel(), wl.H, wl.dv, dtype=steps["v"].dtype, device=DEV)
    for t in range(steps_n):
        out = K.decode_step(steps["q"][t], steps["k"][t], steps["v"][t], steps["log_alpha"][t],
                            steps["beta"][t], state)
        outs[t] = out[sub]
    torch.cuda.synchronize()
    # the subset's tokens packed sequence-major: row n * steps_n + t is step t of sequence sub[n]
    seq_major = {n: f64(steps[n][:, sub].transpose(0, 1).reshape(-1, *steps[n].shape[2:]))
                 for n in ("q", "k", "v", "log_alpha", "beta")}
    cu = np.arange(sub.numel() + 1, dtype=np.int64) * steps_n
    ro, rs = oracle.forward(seq_major["q"], seq_major["k"], seq_major["v"], seq_major["log_alpha"],
                            seq_major["beta"], seeded, cu)
    scale = float(steps["v"].abs().max())
    got = f64(outs.transpose(0, 1).reshape(-1, wl.H, wl.dv))
    assert_close(got, ro, TOL["bf16"], scale, "decode 1024 steps: every output")
    assert_close(state[sub], rs, TOL["bf16"], scale, "decode 1024 steps: final state")
    # drift stays far inside the tolerance: the last step alone, for the record
    last = got.reshape(sub.numel(), steps_n, wl.H, wl.dv)[:, -1]
    assert float(np.abs(last - ro.reshape(sub.numel(), steps_n, wl.H, wl.dv)[:, -1]).max()) <= TOL["bf16"] * scale


def test_back_to_back_steps_and_other_kernels_between():
    """Decode steps launched back to back (the programmatic launch lets a step's blocks become
    resident while the previous step drains), and with PyTorch kernels between them that rewrite
    the state and the next inputs: each step must see the writes of everything before it."""
    step = getattr(K.decode_step, "__wrapped__", K.decode_step)  # no guard copies between the calls
    wl = W.custom((1,) * 64, 8, 128, 128, "bf16", seed=91)
    g = torch.Generator(device=DEV).manual_seed(91)
    state = torch.randn(64, 8, 128, 128, device=DEV, generator=g) * 0.1
    steps = W.make_decode_steps(wl, g, 12, DEV)
    ref_s = f64(state)
    outs = torch.empty(12, 64, 8, 128, dtype=torch.bfloat16, device=DEV)
    ref_o = []
    for t in range(12):
        d = {n: steps[n][t] for n in steps}
        if t % 4 == 3:  # another kernel between two steps: halve the state, rescale v
            state.mul_(0.5)
            ref_s = ref_s * 0.5
            d["v"].mul_(2)
        step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state, out=outs[t])
        ro, ref_s = _oracle_step(d, ref_s)
        ref_o.append(ro)
    torch.cuda.synchronize()
    scale = float(torch.stack([steps["v"][t] for t in range(12)]).abs().max())
    assert_close(outs, np.stack(ref_o), TOL["bf16"], scale, "back-to-back decode outputs")
    assert_close(state, ref_s, TOL["bf16"], scale, "back-to-back decode state")
