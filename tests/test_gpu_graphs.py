"""The library's calls inside CUDA graphs: captured once, replayed, equal to eager calls bit for bit.

Nothing in the prefill, decode or speculative-decode paths allocates, synchronises or reads device
memory on the host, so each call can be captured; the decode kernel's programmatic launch becomes
a programmatic edge between consecutive steps in the graph. Every buffer is preallocated and the
graph replays on the same static tensors."""
import pytest
import torch

from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture (first-call set-up per kernel)
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_steps_replayed_from_a_graph():
    wl = W.custom((1,) * 16, 8, 128, 128, "bf16", seed=31)
    gen = torch.Generator(device=DEV).manual_seed(31)
    steps = W.make_decode_steps(wl, gen, 6, DEV)
    state0 = torch.randn(16, 8, 128, 128, device=DEV, generator=gen) * 0.1
    outs_e = torch.empty(6, 16, 8, 128, dtype=torch.bfloat16, device=DEV)
    state_e = state0.clone()
    for t in range(6):
        K.decode_step(steps["q"][t], steps["k"][t], steps["v"][t], steps["log_alpha"][t], steps["beta"][t],
                      state_e, out=outs_e[t])
    state_g = state0.clone()
    outs_g = torch.empty_like(outs_e)

    def six_steps():
        for t in range(6):
            K.decode_step(steps["q"][t], steps["k"][t], steps["v"][t], steps["log_alpha"][t],
                          steps["beta"][t], state_g, out=outs_g[t], stream=torch.cuda.current_stream())

    g = _capture(six_steps)
    for _ in range(2):  # each replay starts from the same state
        state_g.copy_(state0)
        outs_g.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(outs_g, outs_e) and torch.equal(state_g, state_e)


@pytest.mark.parametrize("lens,H,minimal", [((700, 65, 0, 130), 3, False),   # split-role kernel
                                             ((700, 65, 0, 130), 3, True),    # fused kernel
                                             ((64 * 3,) * 40, 8, False)])     # many heads: fused
def test_prefill_replayed_from_a_graph(lens, H, minimal):
    wl = W.custom(lens, H, 128, 128, "bf16", seed=sum(lens) % 101, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    N, T = wl.num_seqs, wl.total_tokens
    n = 256 + (4 * N + 255) // 256 * 256 if minimal else K.workspace_size(N, T, H, 128, 128, torch.bfloat16)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    out_e, fs_e = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["initial_state"],
                            inp["cu_seqlens"], inp["cu_seqlens_dev"], workspace=ws)
    out_g = torch.empty_like(out_e)
    fs_g = torch.empty_like(fs_e)

    def call():
        K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["initial_state"],
                  inp["cu_seqlens"], inp["cu_seqlens_dev"], out=out_g, final_state=fs_g, workspace=ws,
                  stream=torch.cuda.current_stream())

    g = _capture(call)
    out_g.zero_()
    fs_g.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert K.read_device_status(ws) == K.KDA_OK
    assert torch.equal(out_g, out_e) and torch.equal(fs_g, fs_e)


def test_speculative_step_replayed_from_a_graph():
    N, H, T = 8, 4, 3
    dr = W.make_inputs(W.custom((T,) * N, H, 128, 128, "bf16", seed=41), DEV)
    x = {n: dr[n].reshape(N, T, *dr[n].shape[1:]) for n in ("q", "k", "v", "log_alpha", "beta")}
    gen = torch.Generator(device=DEV).manual_seed(41)
    state0 = torch.randn(N, H, 128, 128, device=DEV, generator=gen) * 0.1
    acc = torch.tensor([3, 0, 1, 2, 3, 3, 1, 0], dtype=torch.int32, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    state_e = state0.clone()
    out_e, u_e = K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state_e, workspace=ws)
    K.decode_commit(x["k"], x["log_alpha"], u_e, state_e, acc, workspace=ws)
    state_g = state0.clone()
    out_g, u_g = torch.empty_like(out_e), torch.empty_like(u_e)

    def step():
        s = torch.cuda.current_stream()
        K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state_g, out=out_g, u_cache=u_g,
                        workspace=ws, stream=s)
        K.decode_commit(x["k"], x["log_alpha"], u_g, state_g, acc, workspace=ws, stream=s)

    g = _capture(step)
    state_g.copy_(state0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_e) and torch.equal(u_g, u_e) and torch.equal(state_g, state_e)
