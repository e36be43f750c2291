"""moe_route_noalloc: the router entry point for callers that cannot allocate
device memory (for example code running during a CUDA stream capture, or a
serving loop whose framework allocator owns all device memory).  It keeps its
scratch in a fixed device array inside the library; this file checks it
against moe_route, which takes a caller workspace, and against the CPU
oracle's routing, on two calls in a row with different inputs (so stale
scratch from the first call would show up), and that a problem too large for
the array is refused.  Collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import W_RTOL, check_routing, to_cpu_inputs
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg(T, E, k, H=512):
    return MoEConfig("noalloc", T=T, H=H, E=E, top_k=k, I=128, num_shared=0,
                     dtype=torch.bfloat16, x_std=1.0, w_std=0.02, routed_scale=2.827,
                     clip_limit=10.0)


def _route_both(c, seed, bias=None):
    inp = make_inputs(c, seed=seed, device=DEV)
    p = moe.MoEProblem.from_config(c)
    idx_a = torch.empty(c.T, c.top_k, dtype=torch.int32, device=DEV)
    w_a = torch.empty(c.T, c.top_k, dtype=torch.float32, device=DEV)
    moe.moe_route(p, inp["x"], inp["gate_w"], bias, idx_a, w_a,
                  moe.alloc_workspace(p, moe.MOE_CALL_ROUTE))
    idx_b = torch.full((c.T, c.top_k), -1, dtype=torch.int32, device=DEV)
    w_b = torch.zeros(c.T, c.top_k, dtype=torch.float32, device=DEV)
    moe.moe_route_noalloc(p, inp["x"], inp["gate_w"], bias, idx_b, w_b)
    torch.cuda.synchronize()
    # the no-allocation path against the oracle as well (near-ties validated)
    cpu = to_cpu_inputs(inp)
    orc = oracle.route(cpu["x"], cpu["gate_w"], c.top_k, c.routed_scale,
                       logit_bias=None if bias is None else bias.cpu())
    check_routing(idx_b.cpu().numpy(), w_b.cpu().numpy(), orc, c.top_k)
    return idx_a.cpu(), w_a.cpu(), idx_b.cpu(), w_b.cpu()


def test_noalloc_route_matches_workspace_route_twice():
    # first call: 1000 tokens x 256 experts (close to the capacity);
    # second call: a different, smaller problem with a logit bias
    c1 = _cfg(T=1000, E=256, k=8)
    a_idx, a_w, b_idx, b_w = _route_both(c1, seed=21)
    assert torch.equal(a_idx, b_idx)
    np.testing.assert_allclose(b_w.numpy(), a_w.numpy(), rtol=W_RTOL, atol=0)

    c2 = _cfg(T=77, E=32, k=4, H=256)
    bias = torch.linspace(-0.5, 0.5, 32, device=DEV)
    a_idx, a_w, b_idx, b_w = _route_both(c2, seed=22, bias=bias)
    assert torch.equal(a_idx, b_idx)
    np.testing.assert_allclose(b_w.numpy(), a_w.numpy(), rtol=W_RTOL, atol=0)


def test_noalloc_route_rejects_problems_beyond_capacity():
    c = _cfg(T=1024, E=256, k=8)  # 256 + 4*1024*256 bytes > 1 MiB
    p = moe.MoEProblem.from_config(c)
    x = torch.zeros(c.T, c.H, dtype=c.dtype, device=DEV)
    g = torch.zeros(c.E, c.H, dtype=c.dtype, device=DEV)
    idx = torch.empty(c.T, c.top_k, dtype=torch.int32, device=DEV)
    w = torch.empty(c.T, c.top_k, dtype=torch.float32, device=DEV)
    before = moe.moe_launch_count()
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route_noalloc(p, x, g, None, idx, w)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
    assert moe.moe_launch_count() == before
