"""Prefill with the layer's elementwise prologue fused (kda_prefill_prologue) vs the fp64 oracle
run on the activated inputs (oracle.prologue of the same raw values)."""
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


def _run(lens, H, d, dtype, flags, seed, init=False):
    """Raw inputs for the flagged parts, activated ones (as the workloads draw them) for the rest."""
    wl = W.custom(lens, H, d, d, dtype, seed=seed, init_state="normal" if init else "zero")
    raw = W.make_inputs(wl, DEV, raw=True)
    act = W.make_inputs(wl, DEV)  # the same draws, activated by the input recipe
    x = {"q": raw["q"] if flags & 1 else act["q"], "k": raw["k"] if flags & 1 else act["k"],
         "log_alpha": raw["log_alpha"] if flags & 2 else act["log_alpha"],
         "beta": raw["beta"] if flags & 4 else act["beta"], "v": act["v"]}
    out, fs = K.prefill(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], act["initial_state"],
                        act["cu_seqlens"], act["cu_seqlens_dev"], prologue=flags,
                        gate_scale=W.GATE_SCALE)
    torch.cuda.synchronize()
    q, k, la, b = oracle.prologue(f64(x["q"]), f64(x["k"]), f64(x["log_alpha"]), f64(x["beta"]),
                                  flags, W.GATE_SCALE)
    s0 = None if act["initial_state"] is None else f64(act["initial_state"])
    ref_o, ref_s = oracle.forward(q, k, f64(x["v"]), la, b, s0,
                                  act["cu_seqlens"].numpy().astype(np.int64))
    scale = max(float(act["v"].abs().max()), 1e-30)
    assert_close(out, ref_o, TOL[dtype], scale, f"out flags={flags}")
    assert_close(fs, ref_s, TOL[dtype], scale, f"final state flags={flags}")


# split-role kernel (bf16, few heads), fused chunk kernel (bf16, many heads), token-serial (fp32)
@pytest.mark.parametrize("lens,H,dtype,d", [((300, 0, 129), 2, "bf16", 128),
                                            ((200, 70), 40, "bf16", 128),
                                            ((90, 0, 33), 3, "f32", 64)])
def test_prologue_all_flags(lens, H, dtype, d):
    _run(lens, H, d, dtype, K.PROLOGUE_ALL, seed=sum(lens) + H, init=True)


@pytest.mark.parametrize("flags", [1, 2, 4])
@pytest.mark.parametrize("H,dtype,d", [(2, "bf16", 128), (40, "bf16", 128), (2, "f32", 32)])
def test_prologue_each_flag(flags, H, dtype, d):
    _run((150, 65), H, d, dtype, flags, seed=31 * flags + H)


def test_prologue_zero_flags_is_prefill():
    wl = W.custom((300, 65), 2, 128, 128, "bf16", seed=3)
    x = W.make_inputs(wl, DEV)
    ref = K.prefill(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, x["cu_seqlens"],
                    x["cu_seqlens_dev"])
    got = K.prefill(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, x["cu_seqlens"],
                    x["cu_seqlens_dev"], prologue=0)
    torch.cuda.synchronize()
    assert torch.equal(ref[0], got[0]) and torch.equal(ref[1], got[1])


def test_prologue_strong_raw_gates_take_the_exact_path():
    """Raw gates large enough that a chunk decays past the factored path's range."""
    wl = W.custom((200, 70), 2, 128, 128, "bf16", seed=17)
    raw = W.make_inputs(wl, DEV, raw=True)
    g = raw["log_alpha"] * 8.0 + 40.0  # softplus ~ 40 per token: log alpha ~ -2.5 with scale 1/16
    out, fs = K.prefill(raw["q"], raw["k"], raw["v"], g, raw["beta"], None, raw["cu_seqlens"],
                        raw["cu_seqlens_dev"], prologue=K.PROLOGUE_ALL, gate_scale=W.GATE_SCALE)
    torch.cuda.synchronize()
    q, k, la, b = oracle.prologue(f64(raw["q"]), f64(raw["k"]), f64(g), f64(raw["beta"]),
                                  K.PROLOGUE_ALL, W.GATE_SCALE)
    ref_o, ref_s = oracle.forward(q, k, f64(raw["v"]), la, b, None,
                                  raw["cu_seqlens"].numpy().astype(np.int64))
    scale = float(raw["v"].abs().max())
    assert_close(out, ref_o, TOL["bf16"], scale, "out")
    assert_close(fs, ref_s, TOL["bf16"], scale, "final state")


def test_prologue_8k_full_size():
    """The headline workload (8192 tokens x 32 heads, split-role kernel) on raw inputs."""
    wl = W.PREFILL_8K
    raw = W.make_inputs(wl, DEV, raw=True)
    out, fs = K.prefill(raw["q"], raw["k"], raw["v"], raw["log_alpha"], raw["beta"], None,
                        raw["cu_seqlens"], raw["cu_seqlens_dev"], prologue=K.PROLOGUE_ALL,
                        gate_scale=W.GATE_SCALE)
    torch.cuda.synchronize()
    q, k, la, b = oracle.prologue(f64(raw["q"]), f64(raw["k"]), f64(raw["log_alpha"]), f64(raw["beta"]),
                                  K.PROLOGUE_ALL, W.GATE_SCALE)
    ref_o, ref_s = oracle.forward(q, k, f64(raw["v"]), la, b, None,
                                  raw["cu_seqlens"].numpy().astype(np.int64))
    scale = float(raw["v"].abs().max())
    assert_close(out, ref_o, TOL["bf16"], scale, "out")
    assert_close(fs, ref_s, TOL["bf16"], scale, "final state")
