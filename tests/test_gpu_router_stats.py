"""GPU parity of moe_router_stats (load-balancing statistics) against the
oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import TIE_REL, to_cpu_inputs
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs, skew_logit_bias

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg(T, H, E, k, dtype=torch.bfloat16):
    return MoEConfig("stats", T=T, H=H, E=E, top_k=k, I=64, num_shared=0, dtype=dtype,
                     x_std=1.0, w_std=0.02, routed_scale=2.827, clip_limit=10.0)


@pytest.mark.parametrize("T,H,E,k,dtype,skew", [
    (300, 256, 16, 4, torch.bfloat16, False),
    (1000, 512, 256, 8, torch.bfloat16, True),
    (77, 256, 33, 5, torch.float32, False),
])
def test_router_stats_match_oracle(T, H, E, k, dtype, skew):
    c = _cfg(T, H, E, k, dtype)
    inp = make_inputs(c, seed=31, device=DEV)
    bias = skew_logit_bias(E).to(DEV) if skew else None
    p = moe.MoEProblem.from_config(c)
    P = torch.empty(E, device=DEV)
    f = torch.empty(E, device=DEV)
    aux = torch.empty(1, device=DEV)
    ema = torch.linspace(0.0, 3.0, E, device=DEV)
    ema_t = torch.tensor([5.0], device=DEV)
    ema0, ema_t0 = ema.cpu().double().numpy(), 5.0
    ws = moe.alloc_workspace(p, moe.MOE_CALL_ROUTER_STATS)
    moe.moe_router_stats(p, inp["x"], inp["gate_w"], bias, P, f, aux, ema, ema_t, 0.9, ws)
    torch.cuda.synchronize()
    ci = to_cpu_inputs(inp)
    ref = oracle.router_stats(ci["x"], ci["gate_w"], k, logit_bias=None if bias is None
                              else bias.cpu(), momentum=0.9, ema_counts=ema0, ema_total=ema_t0)
    # tokens whose k-th / (k+1)-th probabilities tie within TIE_REL may select
    # either expert: each such token can move one count between two experts
    r = oracle.route(ci["x"], ci["gate_w"], k, 1.0,
                     logit_bias=None if bias is None else bias.cpu())
    ps = -np.sort(-r["probs"], axis=1)
    n_tie = int((ps[:, k - 1] - ps[:, k] < TIE_REL * ps[:, k - 1]).sum()) if k < E else 0
    np.testing.assert_allclose(P.cpu().numpy(), ref["P"], rtol=1e-4, atol=1e-7)
    cnt_gpu = np.rint(f.cpu().double().numpy() * T * k).astype(np.int64)
    assert np.abs(cnt_gpu - ref["counts"]).sum() <= 2 * n_tie
    np.testing.assert_allclose(f.cpu().numpy(), cnt_gpu / (T * k), rtol=1e-6)
    assert float(aux.item()) == pytest.approx(ref["aux"], rel=1e-4 + 4.0 * n_tie / (T * k))
    np.testing.assert_allclose(ema.cpu().numpy(), 0.9 * ema0 + 0.1 * cnt_gpu, rtol=1e-5)
    assert float(ema_t.item()) == pytest.approx(ref["ema_total"], rel=1e-6)


def test_router_stats_reproducible_and_uniform_case():
    c = _cfg(128, 256, 8, 3)
    inp = make_inputs(c, seed=32, device=DEV)
    inp["gate_w"].zero_()  # all probabilities 1/E, experts 0..k-1 chosen: aux = 1
    p = moe.MoEProblem.from_config(c)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_ROUTER_STATS)
    outs = []
    for _ in range(2):
        P = torch.empty(8, device=DEV)
        f = torch.empty(8, device=DEV)
        aux = torch.empty(1, device=DEV)
        moe.moe_router_stats(p, inp["x"], inp["gate_w"], None, P, f, aux, None, None, 0.9, ws)
        torch.cuda.synchronize()
        outs.append((P.cpu(), f.cpu(), aux.cpu()))
    assert all(torch.equal(a, b) for a, b in zip(outs[0], outs[1]))
    P, f, aux = outs[0]
    np.testing.assert_allclose(P.numpy(), 1 / 8, rtol=1e-6)
    np.testing.assert_allclose(f.numpy(), [1 / 3] * 3 + [0] * 5, rtol=1e-6)
    assert float(aux) == pytest.approx(1.0, rel=1e-6)
