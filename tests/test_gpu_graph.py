"""The forward path allocates nothing and never waits on the host, so it can be
captured in a CUDA graph and replayed: replays reproduce the eager call bit
for bit (bf16 and FP8 weights; fused routing launch included)."""
import pytest
import torch

from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASE = MoEConfig("graph_case", T=300, H=512, E=16, top_k=4, I=384, num_shared=1,
                 dtype=torch.bfloat16, x_std=1.0, w_std=0.02, routed_scale=2.827,
                 clip_limit=10.0)


def _outputs(c):
    return (torch.empty(c.T, c.H, dtype=c.dtype, device=DEV),
            torch.empty(c.T, c.top_k, dtype=torch.int32, device=DEV),
            torch.empty(c.T, c.top_k, dtype=torch.float32, device=DEV))


@pytest.mark.parametrize("fp8", [False, True])
def test_forward_replays_from_a_cuda_graph(fp8):
    c = CASE
    inp = make_inputs(c, seed=31, device=DEV)
    p = moe.MoEProblem.from_config(c)
    if fp8:
        import test_gpu_fp8 as f8
        q, sg, sd = f8.gpu_quantize(p, inp["expert_w"])
        sq, ssg, ssd = f8.gpu_quantize(p, inp["shared_w"].unsqueeze(0))
        ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD_FP8)

        def call(x, out, idx, w, stream=None):
            moe.moe_forward_fp8(p, x, inp["gate_w"], inp["logit_bias"], q, sg, sd, sq, ssg, ssd,
                                out, idx, w, ws, stream)
    else:
        ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD)

        def call(x, out, idx, w, stream=None):
            moe.moe_forward(p, x, inp["gate_w"], inp["logit_bias"], inp["expert_w"],
                            inp["shared_w"], out, idx, w, ws, stream)

    eager = _outputs(c)
    call(inp["x"], *eager)
    torch.cuda.synchronize()

    x_static = inp["x"].clone()
    graph_out = _outputs(c)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm the launch paths outside the capture
        call(x_static, *graph_out, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    for t in graph_out:
        t.zero_()
    with torch.cuda.graph(g):
        call(x_static, *graph_out, stream=torch.cuda.current_stream())
    for _ in range(3):
        for t in graph_out:
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_read_device_status(ws) == moe.MOE_OK
        assert torch.equal(graph_out[1], eager[1]) and torch.equal(graph_out[2], eager[2])
        assert torch.equal(graph_out[0].view(torch.int16), eager[0].view(torch.int16))
    # new inputs copied into the captured buffer are picked up by the replay
    x2 = make_inputs(c, seed=32, device=DEV)["x"]
    x_static.copy_(x2)
    g.replay()
    eager2 = _outputs(c)
    call(x2, *eager2)
    torch.cuda.synchronize()
    assert torch.equal(graph_out[0].view(torch.int16), eager2[0].view(torch.int16))
    del g
