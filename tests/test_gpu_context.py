"""Context parallelism inside one GPU (kda_prefill_cp) against the fp64 oracle.

Long sequences are cut into segments whose chains run side by side; later segments run from a
zero state with their transition product and per-chunk correction tiles, a scan finds each
segment's true start state and a fix-up adds its contribution to the outputs. Every case is
compared element by element with the oracle (which has no segments) and with kda_prefill."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W
from tests.gpu_helpers import TOL, assert_close, f64, oracle_forward, vmax

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_62_b200 import build
    build.build()
    oracle.build()


def _cp(inp, segments, workspace=None):
    return K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp.get("initial_state"),
                     inp["cu_seqlens"], inp["cu_seqlens_dev"], algo="cp", segments=segments, workspace=workspace)


@pytest.mark.parametrize("lens,H,segments,init", [
    ((3000,), 4, 2, "zero"),
    ((3000,), 4, 5, "normal"),
    ((2500, 1, 0, 700, 129), 3, 3, "normal"),   # ragged: a one-token and an empty sequence
    ((64 * 7 + 5,), 2, 7, "normal"),            # one chunk per segment, ragged last chunk
    ((4096, 513), 8, 4, "zero"),
])
def test_context_parallel_matches_oracle(lens, H, segments, init):
    wl = W.custom(lens, H, 128, 128, "bf16", seed=sum(lens) % 997 + segments, init_state=init)
    inp = W.make_inputs(wl, DEV)
    out, fs = _cp(inp, segments)
    n_launch = K.last_launch_count()
    assert n_launch == 5, n_launch  # plan, split init, split kernel, scan, fix-up: the CP path ran
    ref_o, ref_s = oracle_forward(inp)
    scale = vmax(inp)
    assert_close(out, ref_o, TOL["bf16"], scale, "cp out")
    assert_close(fs, ref_s, TOL["bf16"], scale, "cp final state")
    # and kda_prefill on the same inputs agrees to the same bound
    out_p, fs_p = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["initial_state"], inp["cu_seqlens"], inp["cu_seqlens_dev"])
    assert float((out.float() - out_p.float()).abs().max()) <= 2 * TOL["bf16"] * scale
    assert float((fs - fs_p).abs().max()) <= 2 * TOL["bf16"] * scale


def test_context_parallel_reports_ok_and_resumes():
    """Status word OK; final_state aliasing initial_state (in-place resume) through the scan."""
    wl = W.custom((2000, 900), 4, 128, 128, "bf16", seed=5, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    N = 2
    need = int(K.lib().kda_prefill_cp_workspace_size(N, K.ctypes.c_void_p(inp["cu_seqlens"].data_ptr()),
                                                     4, 128, 128, K.KDA_BF16, 3))
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    ref_o, ref_s = oracle_forward(inp)
    state = inp["initial_state"].clone()
    out, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], state,
                        inp["cu_seqlens"], inp["cu_seqlens_dev"], final_state=state, algo="cp",
                        segments=3, workspace=ws)
    assert K.read_device_status(ws) == K.KDA_OK
    scale = vmax(inp)
    assert_close(out, ref_o, TOL["bf16"], scale, "cp in-place out")
    assert_close(state, ref_s, TOL["bf16"], scale, "cp in-place state")


def test_context_parallel_strong_decay_exact_path():
    """Gates strong enough for the chunk kernels' exact path, and a segment transition that is
    nearly zero: the scan and the fix-up must still agree with the oracle."""
    wl = W.custom((1500,), 2, 128, 128, "bf16", seed=11, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    la = inp["log_alpha"]
    la[::3] = -20.0
    ref_o, ref_s = oracle_forward(inp)
    out, fs = _cp(inp, 4)
    scale = vmax(inp)
    assert_close(out, ref_o, TOL["bf16"], scale, "cp strong decay out")
    assert_close(fs, ref_s, TOL["bf16"], scale, "cp strong decay state")


def test_context_parallel_no_decay_carries_start_state():
    """alpha = 1 and beta = 0: nothing decays and nothing is written, so every output is
    S_0^T q_t through all segments; the start state reaches the last segment only through the
    scan and the fix-up."""
    wl = W.custom((1200,), 2, 128, 128, "bf16", seed=13, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    inp["log_alpha"].zero_()
    inp["beta"].zero_()
    ref_o, ref_s = oracle_forward(inp)
    out, fs = _cp(inp, 6)
    scale = max(float(inp["initial_state"].abs().max()), 1e-30)
    assert_close(out, ref_o, TOL["bf16"], scale, "cp no-decay out")
    assert_close(fs, ref_s, TOL["bf16"], scale, "cp no-decay state")


def test_context_parallel_segments_one_is_plain_prefill():
    wl = W.custom((900,), 4, 128, 128, "bf16", seed=17)
    inp = W.make_inputs(wl, DEV)
    out1, fs1 = _cp(inp, 1)
    assert K.last_launch_count() == 2
    out_p, fs_p = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                            inp["cu_seqlens"], inp["cu_seqlens_dev"])
    assert torch.equal(out1, out_p) and torch.equal(fs1, fs_p)


def test_context_parallel_rejects_bad_segments():
    wl = W.custom((300,), 2, 128, 128, "bf16", seed=19)
    inp = W.make_inputs(wl, DEV)
    for bad in (0, 65):
        with pytest.raises((K.KdaError, ValueError)):
            _cp(inp, bad)


@pytest.mark.slow
def test_prefill_1m_context_parallel_windows_and_final_state():
    """The million-token, 16-head prefill with two segments: the first 16,384 outputs (first
    segment), the 16,384 outputs right after the segment boundary (zero-start outputs plus the
    fix-up's start-state term), and the final state (through the scan). The oracle runs each
    window from a zero state 16,384 tokens earlier; the contraction bound certifies the
    truncated history is far below the tolerance."""
    wl = W.PREFILL_1M
    inp = W.make_inputs(wl, DEV)
    out, fs = _cp(inp, 2)
    assert K.last_launch_count() == 5
    torch.cuda.synchronize()
    scale = vmax(inp)
    Wn = 16384
    T = wl.total_tokens
    heads = [0, 7, 15]
    names = ("q", "k", "v", "log_alpha", "beta")
    fo, _ = oracle.forward(*(f64(inp[n][:Wn, heads]) for n in names))
    assert_close(out[:Wn, heads], fo, TOL["bf16"], scale, "1M cp first window")
    chunks = T // 64
    boundary = 64 * (chunks // 2)  # where the second segment starts
    a, b = boundary - Wn, boundary + Wn
    wo, _ = oracle.forward(*(f64(inp[n][a:b, heads]) for n in names))
    lo, ls = oracle.forward(*(f64(inp[n][T - Wn:, heads]) for n in names))
    for i, h in enumerate(heads):
        arr = {n: f64(inp[n][:, [h]]) for n in ("k", "v", "log_alpha", "beta")}
        ld, nb = oracle.window_bound(arr["k"], arr["v"], arr["log_alpha"], arr["beta"], 0, 0, a, boundary)
        bound_w = float(np.exp(ld) * nb)
        ld, nb = oracle.window_bound(arr["k"], arr["v"], arr["log_alpha"], arr["beta"], 0, 0, T - Wn, T)
        bound_s = float(np.exp(ld) * nb)
        assert bound_w < 1e-6 * scale and bound_s < 1e-6 * scale, (bound_w, bound_s)
        assert_close(out[boundary:b, h], wo[Wn:, i], TOL["bf16"] + bound_w / scale, scale,
                     f"1M cp window after the segment boundary, head {h}")
        assert_close(fs[0, h], ls[0, i], TOL["bf16"] + bound_s / scale, scale, f"1M cp final state head {h}")
