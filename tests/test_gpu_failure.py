"""Failure handling on the GPU without a fault: bounded waits give up with an
error status the host reads, the context stays usable afterwards, and no
result depends on what a workspace held before the call."""
import pytest
import torch

from parity_util import forward_parity
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASE = MoEConfig("failure_case", T=300, H=512, E=16, top_k=4, I=384, num_shared=1,
                 dtype=torch.bfloat16, x_std=1.0, w_std=0.02, routed_scale=2.827,
                 clip_limit=10.0)


def forward(c, inp, ws):
    p = moe.MoEProblem.from_config(c)
    out = torch.empty(c.T, c.H, dtype=c.dtype, device=DEV)
    idx = torch.empty(c.T, c.top_k, dtype=torch.int32, device=DEV)
    w = torch.empty(c.T, c.top_k, dtype=torch.float32, device=DEV)
    moe.moe_forward(p, inp["x"], inp["gate_w"], inp["logit_bias"], inp["expert_w"],
                    inp["shared_w"], out, idx, w, ws)
    torch.cuda.synchronize()
    return out, idx, w


def test_bounded_waits_time_out_and_report():
    ws = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    # an mbarrier nobody arrives on and a counter nobody increments: both
    # waits give up after their limit instead of hanging
    assert moe.moe_check_wait_timeout(ws) == 3
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_TIMEOUT
    # the context is still usable: clear the word and run a layer
    moe.moe_clear_device_status(ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    inp = make_inputs(CASE, seed=21, device=DEV)
    p = moe.MoEProblem.from_config(CASE)
    ws2 = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD)
    out, idx, w = forward(CASE, inp, ws2)
    assert moe.moe_read_device_status(ws2) == moe.MOE_OK
    forward_parity(inp, CASE, out, idx, w)


@pytest.mark.parametrize("fp8", [False, True])
def test_poisoned_workspace_gives_identical_results(fp8):
    """Every workspace byte the path reads is written first in the same call:
    a workspace filled with 0xFF (NaN in fp32 and bf16, -1 in int32) gives
    bit-identical outputs to a zero-filled one (the path is deterministic)."""
    inp = make_inputs(CASE, seed=22, device=DEV)
    p = moe.MoEProblem.from_config(CASE)
    call = moe.MOE_CALL_FORWARD_FP8 if fp8 else moe.MOE_CALL_FORWARD
    results = []
    for fill in (0x00, 0xFF):
        ws = moe.alloc_workspace(p, call)
        ws.fill_(fill)
        ws[:256].zero_()  # the error word starts clear
        if fp8:
            import test_gpu_fp8 as f8
            q, sg, sd = f8.gpu_quantize(p, inp["expert_w"])
            sq, ssg, ssd = f8.gpu_quantize(p, inp["shared_w"].unsqueeze(0))
            out = torch.empty(CASE.T, CASE.H, dtype=CASE.dtype, device=DEV)
            idx = torch.empty(CASE.T, CASE.top_k, dtype=torch.int32, device=DEV)
            w = torch.empty(CASE.T, CASE.top_k, dtype=torch.float32, device=DEV)
            moe.moe_forward_fp8(p, inp["x"], inp["gate_w"], inp["logit_bias"], q, sg, sd, sq,
                                ssg, ssd, out, idx, w, ws)
            torch.cuda.synchronize()
        else:
            out, idx, w = forward(CASE, inp, ws)
        assert moe.moe_read_device_status(ws) == moe.MOE_OK
        assert torch.isfinite(out.float()).all()
        results.append((out, idx, w))
    (o0, i0, w0), (o1, i1, w1) = results
    assert torch.equal(i0, i1) and torch.equal(w0, w1)
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
