"""Prefill and decode on a pool of state slots (the prefill cache's restore / store) vs the fp64
oracle run on the states gathered by slot: outputs element by element, and every slot of the
pool afterwards (written slots hold the oracle's final states, the others are untouched)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W
from tests.gpu_helpers import TOL, assert_close, f64, vmax

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_62_b200 import build
    build.build()
    oracle.build()


def _pool(P, H, dk, dv, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return 0.02 * torch.randn(P, H, dk, dv, device=DEV, generator=g)


def _expected(inp, pool0, init_slot, final_slot):
    """Oracle outputs and the pool after the call, from the states gathered by slot."""
    P, H, dk, dv = pool0.shape
    N = len(init_slot)
    p0 = f64(pool0)
    s0 = np.stack([p0[s] if s >= 0 else np.zeros((H, dk, dv)) for s in init_slot])
    cu = inp["cu_seqlens"].numpy().astype(np.int64)
    o, sT = oracle.forward(*(f64(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")), s0, cu)
    pool = p0.copy()
    for n in range(N):
        if final_slot[n] >= 0:
            pool[final_slot[n]] = sT[n]
    return o, pool


# (lens, H, dtype, d): the split-role kernel (bf16, d = 128, few heads), the fused kernel
# (bf16, d = 128, many heads) and the token-serial kernel (fp32).
CASES = [((200, 0, 70), 2, "bf16", 128), ((100, 0, 70), 48, "bf16", 128), ((90, 0, 33), 3, "f32", 64)]


@pytest.mark.parametrize("lens,H,dtype,d", CASES)
def test_prefill_slots_gather_and_scatter(lens, H, dtype, d):
    wl = W.custom(lens, H, d, d, dtype, seed=sum(lens) + H)
    inp = W.make_inputs(wl, DEV)
    pool = _pool(7, H, d, d, seed=H)
    pool0 = pool.clone()
    init_slot, final_slot = [4, 2, -1], [1, 2, 5]  # seq 1 (empty) resumes in place
    out = K.prefill_slots(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], pool,
                          torch.tensor(init_slot, dtype=torch.int32, device=DEV),
                          torch.tensor(final_slot, dtype=torch.int32, device=DEV),
                          inp["cu_seqlens"], inp["cu_seqlens_dev"])
    torch.cuda.synchronize()
    ref_o, ref_pool = _expected(inp, pool0, init_slot, final_slot)
    scale = vmax(inp)
    assert_close(out, ref_o, TOL[dtype], scale, "slots out")
    assert_close(pool, ref_pool, TOL[dtype], scale, "slots pool")
    for s in (0, 3, 4, 6):  # never written: bit-identical
        assert torch.equal(pool[s], pool0[s]), s


def test_prefill_slots_shared_source_and_in_place():
    """Two requests resume from the same cached slot; a third resumes in place."""
    wl = W.custom((130, 64, 200), 2, 128, 128, "bf16", seed=21)
    inp = W.make_inputs(wl, DEV)
    pool = _pool(4, 2, 128, 128, seed=5)
    pool0 = pool.clone()
    init_slot, final_slot = [0, 0, 3], [1, 2, 3]
    out = K.prefill_slots(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], pool,
                          torch.tensor(init_slot, dtype=torch.int32, device=DEV),
                          torch.tensor(final_slot, dtype=torch.int32, device=DEV),
                          inp["cu_seqlens"], inp["cu_seqlens_dev"])
    torch.cuda.synchronize()
    ref_o, ref_pool = _expected(inp, pool0, init_slot, final_slot)
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), "out")
    assert_close(pool, ref_pool, TOL["bf16"], vmax(inp), "pool")


def test_prefill_slots_equals_prefill_with_gathered_states():
    """The slot path and kda_prefill on the gathered states give identical bits."""
    wl = W.custom((300, 65), 2, 128, 128, "bf16", seed=31)
    inp = W.make_inputs(wl, DEV)
    pool = _pool(3, 2, 128, 128, seed=9)
    s0 = pool[[2, 0]].contiguous()
    out_ref, fs_ref = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], s0,
                                inp["cu_seqlens"], inp["cu_seqlens_dev"])
    out = K.prefill_slots(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], pool,
                          torch.tensor([2, 0], dtype=torch.int32, device=DEV),
                          torch.tensor([1, 2], dtype=torch.int32, device=DEV),
                          inp["cu_seqlens"], inp["cu_seqlens_dev"])
    torch.cuda.synchronize()
    assert torch.equal(out, out_ref)
    assert torch.equal(pool[1], fs_ref[0]) and torch.equal(pool[2], fs_ref[1])


def test_prefill_slots_out_of_range_slot_is_reported():
    wl = W.custom((100, 80), 2, 128, 128, "bf16", seed=41)
    inp = W.make_inputs(wl, DEV)
    pool = _pool(3, 2, 128, 128, seed=2)
    pool0 = pool.clone()
    ws = torch.empty(K.workspace_size(2, wl.total_tokens, 2, 128, 128, torch.bfloat16),
                     dtype=torch.uint8, device=DEV)
    init_slot, final_slot = [0, 7], [1, -1]  # slot 7 does not exist: read as zeros, reported
    out = K.prefill_slots(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], pool,
                          torch.tensor(init_slot, dtype=torch.int32, device=DEV),
                          torch.tensor(final_slot, dtype=torch.int32, device=DEV),
                          inp["cu_seqlens"], inp["cu_seqlens_dev"], workspace=ws)
    assert K.read_device_status(ws) == K.KDA_ERR_INVALID_ARGUMENT
    ref_o, ref_pool = _expected(inp, pool0, [0, -1], final_slot)
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), "out")
    assert_close(pool, ref_pool, TOL["bf16"], vmax(inp), "pool")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_decode_step_slots(dtype, d):
    wl = W.custom((1,) * 4, 3, d, d, dtype, seed=d)
    g = torch.Generator(device=DEV).manual_seed(23)
    steps = W.make_decode_steps(wl, g, 3, DEV)
    pool = _pool(6, 3, d, d, seed=d + 1)
    slot = [4, -1, 0, 2]
    slot_t = torch.tensor(slot, dtype=torch.int32, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    ref_pool = f64(pool)
    for t in range(3):
        x = {n: steps[n][t] for n in steps}
        out = K.decode_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, slot_t,
                                  workspace=ws)
        torch.cuda.synchronize()
        assert K.read_device_status(ws) == K.KDA_OK
        s0 = np.stack([ref_pool[s] if s >= 0 else np.zeros((3, d, d)) for s in slot])
        cu = np.arange(5, dtype=np.int64)
        ref_o, ref_s = oracle.forward(*(f64(x[n]) for n in ("q", "k", "v", "log_alpha", "beta")), s0, cu)
        for n, s in enumerate(slot):
            if s >= 0:
                ref_pool[s] = ref_s[n]
        scale = max(float(x["v"].abs().max()), 1e-30)
        assert_close(out, ref_o, TOL[dtype], scale, f"decode slots out step {t}")
        assert_close(pool, ref_pool, TOL[dtype], scale, f"decode slots pool step {t}")
    bad = torch.tensor([4, 9, 0, 2], dtype=torch.int32, device=DEV)
    K.decode_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, bad, workspace=ws)
    assert K.read_device_status(ws) == K.KDA_ERR_INVALID_ARGUMENT
