"""kda_last_launch_count reports the kernels each entry point enqueued (the bench's gpu_launches)."""
import pytest
import torch

from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from gated_delta_rule_62_b200 import build
    build.build()


@pytest.mark.parametrize("lens,H,dtype,want", [((200,), 2, "bf16", 2),      # split: init + split kernel
                                               ((100, 70), 48, "bf16", 2),  # fused: plan + chunk kernel
                                               ((50,), 2, "f32", 1)])       # token-serial kernel
def test_prefill_launch_count(lens, H, dtype, want):
    x = W.make_inputs(W.custom(lens, H, 128 if dtype == "bf16" else 64, 128 if dtype == "bf16" else 64,
                               dtype, seed=1), DEV)
    K.prefill(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, x["cu_seqlens"], x["cu_seqlens_dev"])
    torch.cuda.synchronize()
    assert K.last_launch_count() == want


def test_decode_and_speculative_launch_count():
    wl = W.custom((1,) * 4, 2, 64, 64, "f32", seed=2)
    g = torch.Generator(device=DEV).manual_seed(3)
    d = {n: t[0] for n, t in W.make_decode_steps(wl, g, 1, DEV).items()}
    state = torch.zeros(4, 2, 64, 64, device=DEV)
    K.decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state)
    assert K.last_launch_count() == 1
    x = {n: t[None].transpose(0, 1).contiguous() for n, t in d.items()}  # [N, 1, ...]
    K.decode_verify(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state)
    assert K.last_launch_count() == 1
    torch.cuda.synchronize()
