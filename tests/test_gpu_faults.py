"""Failure detection without a GPU fault: a stuck on-device wait ends by itself."""
import time

import pytest
import torch

from gated_delta_rule_62_b200 import kda as K
from gated_delta_rule_62_b200 import workloads as W
from tests.gpu_helpers import TOL, assert_close, gpu_prefill, oracle_forward, vmax

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    t = time.time()
    K.selftest_bounded_wait(ws, 50_000_000)  # 50 ms
    assert K.read_device_status(ws) == K.KDA_ERR_TIMEOUT
    assert time.time() - t < 5.0
    # the context is still usable: a prefill right after is correct and reports OK
    wl = W.custom((100,), 2, 128, 128, "bf16", seed=77)
    inp = W.make_inputs(wl, "cuda")
    work = torch.empty(K.workspace_size(1, 100, 2, 128, 128, torch.bfloat16), dtype=torch.uint8,
                       device="cuda")
    out, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                        inp["cu_seqlens"], inp["cu_seqlens_dev"], workspace=work)
    assert K.read_device_status(work) == K.KDA_OK
    ref_o, _ = oracle_forward(inp)
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), "prefill after timeout probe")


def test_selftest_rejects_bad_arguments():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KdaError):
        K.selftest_bounded_wait(ws, 0)


def test_flag_wait_reports_timeout_and_context_survives():
    """The split-role kernel's other wait: a spin on a global flag released by another thread
    block. A flag nothing releases ends the wait by itself with KDA_ERR_TIMEOUT, the context
    stays usable, and a split-kernel prefill right after matches the oracle."""
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    t = time.time()
    K.selftest_flag_wait(ws, 50_000_000)  # 50 ms
    assert K.read_device_status(ws) == K.KDA_ERR_TIMEOUT
    assert time.time() - t < 5.0
    wl = W.custom((700,), 4, 128, 128, "bf16", seed=78)  # few heads: the split-role kernel
    inp = W.make_inputs(wl, "cuda")
    work = torch.empty(K.workspace_size(1, 700, 4, 128, 128, torch.bfloat16), dtype=torch.uint8,
                       device="cuda")
    out, fs = K.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None,
                        inp["cu_seqlens"], inp["cu_seqlens_dev"], workspace=work)
    assert K.read_device_status(work) == K.KDA_OK
    ref_o, ref_s = oracle_forward(inp)
    assert_close(out, ref_o, TOL["bf16"], vmax(inp), "prefill after flag-wait probe")
    assert_close(fs, ref_s, TOL["bf16"], vmax(inp), "final state after flag-wait probe")


def test_flag_selftest_rejects_bad_arguments():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KdaError):
        K.selftest_flag_wait(ws, 0)
    with pytest.raises(K.KdaError):
        K.selftest_flag_wait(ws[:128], 1000)
