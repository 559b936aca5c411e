"""Speculative decode (verify T draft tokens in one pass, then commit the accepted prefix) vs the
fp64 oracle run on the same tokens, and vs T single decode steps bit for bit."""
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


def _draft(N, T, H, d, dtype, seed):
    """N sequences of T draft tokens each, as [N, T, H, ...] views of a packed prefill input."""
    inp = W.make_inputs(W.custom((T,) * N, H, d, d, dtype, seed=seed), DEV)
    x = {n: inp[n].reshape(N, T, *inp[n].shape[1:]) for n in ("q", "k", "v", "log_alpha", "beta")}
    return inp, x


def _states(P, H, d, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return 0.05 * torch.randn(P, H, d, d, device=DEV, generator=g)


def _oracle_prefix(x, s0, n, t):
    """Oracle outputs and final state of sequence n after its first t draft tokens."""
    if t == 0:
        return None, s0
    o, s = oracle.forward(*(f64(x[m][n, :t]) for m in ("q", "k", "v", "log_alpha", "beta")),
                          s0[None])
    return o, s[0]


@pytest.mark.parametrize("dtype,d,T", [("bf16", 128, 4), ("bf16", 128, 16), ("f32", 64, 3),
                                       ("bf16", 32, 1), ("f32", 128, 7)])
def test_verify_and_commit_match_oracle(dtype, d, T):
    N, H = 5, 3
    inp, x = _draft(N, T, H, d, dtype, seed=T * 10 + d)
    state = _states(N, H, d, seed=d + T)
    state0 = state.clone()
    out, u = K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state)
    torch.cuda.synchronize()
    assert torch.equal(state, state0), "verify must leave the states unchanged"
    s0 = f64(state0)
    cu = np.arange(N + 1, dtype=np.int64) * T
    ref_o, _ = oracle.forward(*(f64(inp[m]) for m in ("q", "k", "v", "log_alpha", "beta")), s0, cu)
    scale = max(float(inp["v"].abs().max()), 1e-30)
    assert_close(out.reshape(N * T, H, d), ref_o, TOL[dtype], scale, "verify out")

    # the corrections: S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T, so u_t = beta_t (v_t - (alpha_t * S_{t-1})^T k_t)
    for n in range(N):
        for t in range(T):
            _, s_prev = _oracle_prefix(x, s0[n], n, t)
            a = np.exp(f64(x["log_alpha"][n, t]))[:, :, None] * s_prev
            ref_u = f64(x["beta"][n, t])[:, None] * (f64(x["v"][n, t]) - np.einsum("hkv,hk->hv", a, f64(x["k"][n, t])))
            assert_close(u[n, t], ref_u, TOL[dtype], scale, f"u_cache seq {n} token {t}")

    accepted = [0, 1, T, T // 2, max(T - 1, 0)]
    acc = torch.tensor(accepted, dtype=torch.int32, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    K.decode_commit(x["k"], x["log_alpha"], u, state, acc, workspace=ws)
    assert K.read_device_status(ws) == K.KDA_OK
    for n, a in enumerate(accepted):
        if a == 0:
            assert torch.equal(state[n], state0[n])
            continue
        _, ref_s = _oracle_prefix(x, s0[n], n, a)
        assert_close(state[n], ref_s, TOL[dtype], scale, f"committed state seq {n} ({a} accepted)")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_verify_and_commit_equal_single_decode_steps_bitwise(dtype, d):
    N, T, H = 4, 6, 2
    _, x = _draft(N, T, H, d, dtype, seed=77 + d)
    state = _states(N, H, d, seed=3)
    ref = state.clone()
    outs, snaps = [], [ref.clone()]
    for t in range(T):
        outs.append(K.decode_step(*(x[m][:, t].contiguous() for m in ("q", "k", "v", "log_alpha", "beta")), ref))
        snaps.append(ref.clone())
    out, u = K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state)
    for t in range(T):
        assert torch.equal(out[:, t], outs[t]), f"token {t}"
    accepted = [3, 0, 6, 1]
    K.decode_commit(x["k"], x["log_alpha"], u, state,
                    torch.tensor(accepted, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    for n, a in enumerate(accepted):
        assert torch.equal(state[n], snaps[a][n]), f"seq {n}"


def test_speculative_on_state_slots():
    """Verify reads pooled states (two sequences share a slot, -1 is zeros); commit writes them."""
    N, T, H, d = 3, 5, 2, 128
    _, x = _draft(N, T, H, d, "bf16", seed=5)
    pool = _states(6, H, d, seed=8)
    pool0 = pool.clone()
    slot_r = torch.tensor([4, -1, 4], dtype=torch.int32, device=DEV)
    out, u = K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, slot=slot_r)
    torch.cuda.synchronize()
    assert torch.equal(pool, pool0)
    p0 = f64(pool0)
    s0 = [p0[4], np.zeros((H, d, d)), p0[4]]
    scale = float(x["v"].abs().max())
    for n in range(N):
        ref_o, _ = _oracle_prefix(x, s0[n], n, T)
        assert_close(out[n], ref_o, TOL["bf16"], scale, f"slot verify out seq {n}")
    # commit: sequence 0 in place (slot 4), sequence 1 not stored, sequence 2 has its own slot now
    slot_w = torch.tensor([4, -1, 1], dtype=torch.int32, device=DEV)
    pool[1] = pool[4]
    pool0 = pool.clone()
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    accepted = [2, 5, 5]
    K.decode_commit(x["k"], x["log_alpha"], u, pool, torch.tensor(accepted, dtype=torch.int32, device=DEV),
                    slot=slot_w, workspace=ws)
    assert K.read_device_status(ws) == K.KDA_OK
    for n, s in ((0, 4), (2, 1)):
        _, ref_s = _oracle_prefix(x, s0[n], n, accepted[n])
        assert_close(pool[s], ref_s, TOL["bf16"], scale, f"slot commit seq {n}")
    for s in (0, 2, 3, 5):
        assert torch.equal(pool[s], pool0[s]), s


def test_bad_accepted_count_and_slot_are_reported():
    N, T, H, d = 3, 4, 2, 64
    _, x = _draft(N, T, H, d, "f32", seed=9)
    state = _states(N, H, d, seed=1)
    out, u = K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state)
    state0 = state.clone()
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    K.decode_commit(x["k"], x["log_alpha"], u, state,
                    torch.tensor([T + 1, -1, 0], dtype=torch.int32, device=DEV), workspace=ws)
    assert K.read_device_status(ws) == K.KDA_ERR_INVALID_ARGUMENT
    assert torch.equal(state, state0)
    K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state,
                    slot=torch.tensor([0, 3, 1], dtype=torch.int32, device=DEV), workspace=ws)
    assert K.read_device_status(ws) == K.KDA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 32)])
def test_commit_verify_equals_commit_then_verify_bitwise(dtype, d):
    N, Tp, T, H = 4, 5, 3, 2
    _, x0 = _draft(N, Tp, H, d, dtype, seed=101 + d)
    _, x1 = _draft(N, T, H, d, dtype, seed=202 + d)
    state = _states(N, H, d, seed=12)
    _, u0 = K.decode_verify(x0["q"], x0["k"], x0["v"], x0["log_alpha"], x0["beta"], state)
    acc = torch.tensor([5, 0, 2, 4], dtype=torch.int32, device=DEV)
    two = state.clone()
    K.decode_commit(x0["k"], x0["log_alpha"], u0, two, acc)
    out_ref, u_ref = K.decode_verify(x1["q"], x1["k"], x1["v"], x1["log_alpha"], x1["beta"], two)
    out, u1 = K.decode_commit_verify(x0["k"], x0["log_alpha"], u0, acc, x1["q"], x1["k"], x1["v"],
                                     x1["log_alpha"], x1["beta"], state)
    torch.cuda.synchronize()
    assert torch.equal(out, out_ref) and torch.equal(u1, u_ref) and torch.equal(state, two)


@pytest.mark.parametrize("use_slots", [False, True])
def test_speculative_loop_matches_oracle_on_accepted_tokens(use_slots):
    """Three speculative steps (draft, accept a prefix, commit it while verifying the next draft)
    give the outputs and states of the oracle run on the accepted tokens only."""
    N, T, H, d, dtype = 3, 4, 2, 128, "bf16"
    drafts = [_draft(N, T, H, d, dtype, seed=300 + i)[1] for i in range(3)]
    accepted = [[4, 1, 0], [2, 4, 3], [0, 3, 4]]
    P = 5 if use_slots else N
    pool = _states(P, H, d, seed=4)
    slot = torch.tensor([3, 0, 4], dtype=torch.int32, device=DEV) if use_slots else None
    rows = [3, 0, 4] if use_slots else list(range(N))
    s_ref = [f64(pool[r]) for r in rows]
    hist = [{m: [] for m in ("q", "k", "v", "log_alpha", "beta")} for _ in range(N)]
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    x = drafts[0]
    out, u = K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, slot=slot,
                             workspace=ws)
    scale = max(float(dr["v"].abs().max()) for dr in drafts)
    for step in range(3):
        x = drafts[step]
        for n in range(N):  # the draft's outputs continue the accepted history
            ctx = {m: np.concatenate(hist[n][m] + [f64(x[m][n])]) if hist[n][m] else f64(x[m][n])
                   for m in hist[n]}
            o_ref, _ = oracle.forward(ctx["q"], ctx["k"], ctx["v"], ctx["log_alpha"], ctx["beta"],
                                      s_ref[n][None])
            assert_close(out[n], o_ref[-T:], TOL[dtype], scale, f"step {step} seq {n} out")
            for m in hist[n]:
                hist[n][m].append(f64(x[m][n, :accepted[step][n]]))
        acc = torch.tensor(accepted[step], dtype=torch.int32, device=DEV)
        if step < 2:
            nx = drafts[step + 1]
            out, u = K.decode_commit_verify(x["k"], x["log_alpha"], u, acc, nx["q"], nx["k"], nx["v"],
                                            nx["log_alpha"], nx["beta"], pool, slot=slot, workspace=ws)
        else:
            K.decode_commit(x["k"], x["log_alpha"], u, pool, acc, slot=slot, workspace=ws)
        assert K.read_device_status(ws) == K.KDA_OK
    for n in range(N):
        ctx = {m: np.concatenate(hist[n][m]) for m in hist[n]}
        if len(ctx["q"]) == 0:
            continue
        _, s_fin = oracle.forward(ctx["q"], ctx["k"], ctx["v"], ctx["log_alpha"], ctx["beta"],
                                  s_ref[n][None])
        assert_close(pool[rows[n]], s_fin[0], TOL[dtype], scale, f"final state seq {n}")


def test_speculative_decode_256_full_size():
    """The decode workload's 256 x 32 states (seeded by the GPU prefill), 4 draft tokens each:
    verify, then the fused commit (a mix of accepted counts) + verify of a second draft."""
    wl = W.DECODE_256
    inp = W.make_inputs(wl, DEV)
    _, state = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                         inp["cu_seqlens"], inp["cu_seqlens_dev"])
    N, H, T = wl.num_seqs, wl.H, 4
    g = torch.Generator(device=DEV).manual_seed(99)
    drafts = []
    for _ in range(2):
        st = W.make_decode_steps(wl, g, T, DEV)  # [T, N, ...] -> [N, T, ...]
        drafts.append({n: t.transpose(0, 1).contiguous() for n, t in st.items()})
    s0 = f64(state)
    x = drafts[0]
    out, u = K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state)
    accepted = torch.arange(N, dtype=torch.int32, device=DEV) % (T + 1)
    y = drafts[1]
    out2, _ = K.decode_commit_verify(x["k"], x["log_alpha"], u, accepted, y["q"], y["k"], y["v"],
                                     y["log_alpha"], y["beta"], state)
    torch.cuda.synchronize()
    scale = max(float(x["v"].abs().max()), float(y["v"].abs().max()))
    cu = np.arange(N + 1, dtype=np.int64) * T
    ref_o, _ = oracle.forward(*(f64(x[m]).reshape(N * T, *x[m].shape[2:]) for m in
                                ("q", "k", "v", "log_alpha", "beta")), s0, cu)
    assert_close(out.reshape(N * T, H, -1), ref_o, TOL["bf16"], scale, "verify out")
    acc = accepted.cpu().numpy()
    s1 = np.empty_like(s0)
    for n in range(N):  # the states after each sequence's accepted prefix
        if acc[n] == 0:
            s1[n] = s0[n]
        else:
            _, s = oracle.forward(*(f64(x[m][n, :acc[n]]) for m in ("q", "k", "v", "log_alpha", "beta")),
                                  s0[n][None])
            s1[n] = s[0]
    assert_close(state, s1, TOL["bf16"], scale, "committed states")
    ref_o2, _ = oracle.forward(*(f64(y[m]).reshape(N * T, *y[m].shape[2:]) for m in
                                 ("q", "k", "v", "log_alpha", "beta")), s1, cu)
    assert_close(out2.reshape(N * T, H, -1), ref_o2, TOL["bf16"], scale, "second verify out")
