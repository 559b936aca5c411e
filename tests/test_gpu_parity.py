"""CUDA path vs the fp64 oracle, element by element, on the same seeded inputs."""
import numpy as np
import pytest
import torch

from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W
from tests.gpu_helpers import TOL, assert_close, f64, gpu_prefill, oracle_forward, vmax

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_62_b200 import build
    build.build()
    import oracle
    oracle.build()


def _run_and_check(wl, algo="auto", heads=None, seqs=None, tol=None):
    inp = W.make_inputs(wl, DEV)
    out, fs = gpu_prefill(inp, algo)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle_forward(inp, heads, seqs)
    tol = TOL[wl.dtype] if tol is None else tol
    scale = vmax(inp)
    hs = slice(None) if heads is None else list(heads)
    if seqs is None:
        assert_close(out[:, hs], ref_o, tol, scale, f"{wl.name} out")
        assert_close(fs[:, hs], ref_s, tol, scale, f"{wl.name} final state")
    else:
        cu = inp["cu_seqlens"].numpy()
        for n in seqs:
            assert_close(out[cu[n]:cu[n + 1], hs], ref_o[n], tol, scale, f"{wl.name} out seq {n}")
            assert_close(fs[n, hs], ref_s[n], tol, scale, f"{wl.name} state seq {n}")
    return inp, out, fs


@pytest.mark.parametrize("algo", ["auto", "recurrent"])
def test_tiny_f32_single_chunk(algo):
    _run_and_check(W.TINY_F32, algo)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (32, 128), (128, 64), (64, 32)])
def test_head_sizes(dtype, dk, dv):
    wl = W.custom((70, 1, 130), 3, dk, dv, dtype, seed=dk * 7 + dv, init_state="normal")
    _run_and_check(wl)
    _run_and_check(wl, "recurrent")


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129, 300])
def test_ragged_lengths_bf16_d128(T):
    _run_and_check(W.custom((T,), 4, 128, 128, "bf16", seed=T, init_state="normal"))


def test_varlen_with_empty_sequences_and_resume_state():
    wl = W.custom((0, 77, 0, 1, 200, 64, 0, 333), 4, 128, 128, "bf16", seed=99, init_state="normal")
    inp, out, fs = _run_and_check(wl)
    # empty sequences pass the initial state through exactly
    for n in (0, 2, 6):
        assert torch.equal(fs[n], inp["initial_state"][n])


def test_no_final_state_and_no_initial_state():
    wl = W.custom((100, 50), 2, 128, 128, "bf16", seed=5)
    inp = W.make_inputs(wl, DEV)
    out, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                        inp["cu_seqlens"], inp["cu_seqlens_dev"], output_final_state=False)
    assert fs is None
    ref_o, _ = oracle_forward(inp)
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), "out without final state")


def test_final_state_may_alias_initial_state():
    wl = W.custom((90, 200), 2, 128, 128, "bf16", seed=6, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    ref_o, ref_s = oracle_forward(inp)
    s = inp["initial_state"].clone()
    out, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], s,
                        inp["cu_seqlens"], inp["cu_seqlens_dev"], final_state=s)
    assert fs.data_ptr() == s.data_ptr()
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), "aliased out")
    assert_close(s, ref_s, TOL["bf16"], vmax(inp), "aliased state")


def test_split_resume_equals_whole():
    """Prefix-cache resume: prefill(prefix) then prefill(suffix, from the saved state)."""
    wl = W.custom((333,), 4, 128, 128, "bf16", seed=8, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    out, fs = gpu_prefill(inp)
    m = 150
    part = lambda a, b: {n: inp[n][a:b] for n in ("q", "k", "v", "log_alpha", "beta")}
    p1 = part(0, m)
    o1, s1 = K.prefill(**p1, initial_state=inp["initial_state"])
    p2 = part(m, 333)
    o2, s2 = K.prefill(**p2, initial_state=s1)
    scale = vmax(inp)
    assert_close(torch.cat([o1, o2]), f64(out), TOL["bf16"], scale, "resume out")
    assert_close(s2, f64(fs), TOL["bf16"], scale, "resume state")


# (lens, H): 4 (sequence, head) pairs run two consumers per head in the split-role kernel, 33 one.
@pytest.mark.parametrize("lens,H", [((200, 70), 2), ((200, 70, 1), 11)])
@pytest.mark.parametrize("pattern", ["all_-20", "mix_0_-20", "one_channel_-30"])
def test_adversarial_decay(pattern, lens, H):
    wl = W.custom(lens, H, 128, 128, "bf16", seed=11, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    la = inp["log_alpha"]
    if pattern == "all_-20":
        la.fill_(-20.0)
    elif pattern == "mix_0_-20":
        g = torch.Generator(device=DEV).manual_seed(3)
        la.copy_(torch.where(torch.rand(la.shape, device=DEV, generator=g) < 0.5, 0.0, -20.0))
    else:
        la.fill_(0.0)
        la[..., 5] = -30.0
    out, fs = gpu_prefill(inp)
    ref_o, ref_s = oracle_forward(inp)
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), f"{pattern} out")
    assert_close(fs, ref_s, TOL["bf16"], vmax(inp), f"{pattern} state")


# 8192 tokens x 4 heads: 512 chunk items over the split kernel's producers, several per producer,
# so an exact-path item (which writes A over the previous item's, after waiting for it) follows
# factored and exact ones inside one producer's two-item pipeline.
@pytest.mark.parametrize("pattern", ["alternate_chunks", "mix_0_-20"])
def test_exact_path_items_in_one_producer(pattern):
    wl = W.custom((8192,), 4, 128, 128, "bf16", seed=17, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    la = inp["log_alpha"]
    if pattern == "alternate_chunks":  # even chunks decay by e^-1280 (exact path), odd ones not at all
        chunk = torch.arange(la.shape[0], device=DEV) // 64
        la.copy_(torch.where((chunk % 2 == 0)[:, None, None], torch.full_like(la, -20.0), torch.zeros_like(la)))
    else:
        g = torch.Generator(device=DEV).manual_seed(5)
        la.copy_(torch.where(torch.rand(la.shape, device=DEV, generator=g) < 0.5, 0.0, -20.0))
    out, fs = gpu_prefill(inp)
    ref_o, ref_s = oracle_forward(inp)
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), f"{pattern} out")
    assert_close(fs, ref_s, TOL["bf16"], vmax(inp), f"{pattern} state")


def test_noop_gates_keep_state():
    """alpha = 1, beta = 0 on the GPU: the state passes through unchanged."""
    wl = W.custom((130,), 2, 128, 128, "bf16", seed=12, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    inp["log_alpha"].zero_()
    inp["beta"].zero_()
    out, fs = gpu_prefill(inp)
    assert torch.allclose(fs, inp["initial_state"], atol=1e-6, rtol=0)


def test_prefill_8k_full_size():
    """The 8192-token, 32-head bf16 prefill, checked everywhere against the oracle."""
    _run_and_check(W.PREFILL_8K)


def test_varlen_24_sequences_resume_sampled_heads():
    """The 24-sequence log-uniform pack: every sequence, heads 0 and 31 checked by the oracle."""
    _run_and_check(W.VARLEN_24, heads=(0, 31))


@pytest.mark.slow
def test_prefill_1m_first_window_and_final_state():
    """Million-token prefill: outputs of the first 16,384 tokens, and the final state via a
    window whose truncated history is bounded by contraction."""
    import oracle
    wl = W.PREFILL_1M
    inp = W.make_inputs(wl, DEV)
    out, fs = gpu_prefill(inp)
    torch.cuda.synchronize()
    scale = vmax(inp)
    Wn = 16384
    heads = (0, 7, 15)
    first = {n: inp[n][:Wn] for n in ("q", "k", "v", "log_alpha", "beta")}
    fo, _ = oracle.forward(*(f64(first[n][:, list(heads)]) for n in ("q", "k", "v", "log_alpha", "beta")))
    assert_close(out[:Wn, list(heads)], fo, TOL["bf16"], scale, "1M first window")
    T = wl.total_tokens
    last = {n: inp[n][T - Wn:] for n in ("q", "k", "v", "log_alpha", "beta")}
    lo, ls = oracle.forward(*(f64(last[n][:, list(heads)]) for n in ("q", "k", "v", "log_alpha", "beta")))
    for i, h in enumerate(heads):
        cols = [h]
        arr = {n: f64(inp[n][:, cols]) for n in ("k", "v", "log_alpha", "beta")}
        ld, nb = oracle.window_bound(arr["k"], arr["v"], arr["log_alpha"], arr["beta"], 0, 0, T - Wn, T)
        bound = float(np.exp(ld) * nb)
        assert bound < 1e-6 * scale, bound
        assert_close(fs[0, h], ls[0, i], TOL["bf16"] + bound / scale, scale, f"1M final state head {h}")


# 37 chains: the most the split kernel takes on 148 SMs (4 blocks per chain); its consumers are
# then blocks 111..147 of the grid
LENS_37 = tuple((67 * i) % 331 for i in range(37))


@pytest.mark.parametrize("lens,H", [((8192,), 32), ((700, 0, 130, 64, 1), 6), ((1000,), 2),
                                     ((300, 0, 65, 129), 9), (LENS_37, 1)])
def test_split_role_and_fused_kernels_agree_with_oracle(lens, H):
    """Few-head problems run the split-role kernel when the workspace holds its ring; with only
    the minimum workspace they run the fused kernel. Both must match the oracle."""
    wl = W.custom(lens, H, 128, 128, "bf16", seed=len(lens) * 10 + H, init_state="normal")
    inp = W.make_inputs(wl, DEV)
    N = len(lens)
    full = torch.empty(K.workspace_size(N, wl.total_tokens, H, 128, 128, torch.bfloat16),
                       dtype=torch.uint8, device=DEV)
    minimal = torch.empty(256 + (4 * N + 255) // 256 * 256, dtype=torch.uint8, device=DEV)
    assert full.numel() > minimal.numel()
    heads = list(range(H)) if H <= 9 else [0, 13, 31]
    ref_o, ref_s = oracle_forward(inp, heads=heads)
    scale = vmax(inp)
    for ws in (full, minimal):
        out, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["initial_state"], inp["cu_seqlens"], inp["cu_seqlens_dev"], workspace=ws)
        assert K.read_device_status(ws) == K.KDA_OK
        assert_close(out[:, heads], ref_o, TOL["bf16"], scale, f"out ws={ws.numel()}")
        assert_close(fs[:, heads], ref_s, TOL["bf16"], scale, f"state ws={ws.numel()}")
