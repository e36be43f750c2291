"""GPU parity at the five named workload configurations, in the launch
configuration the benchmark times (moe_forward on the whole batch).

Routing is compared with the oracle on every token.  The layer output is
compared on every token of the small batches and, at the large ones, on the
tokens that cover every token tile of both expert GEMMs' schedules: the first
and last row of every chunk of every expert segment and of the shared expert,
derived from the GPU's own routing and the tile widths the launch used
(moe_expert_tile_rows).  The oracle is per-token independent, so a checked
token is checked exactly as in a full run."""
import numpy as np
import pytest
import torch

from parity_util import forward_parity, schedule_cover_tokens, to_cpu_inputs
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import CONFIGS, make_inputs, make_x, sample_tokens

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def hy4_weights():
    """Hy4-shape weights (identical for the three Hy4 configs: same seeds)."""
    c = CONFIGS["hy4_prefill"]
    inp = make_inputs(c.with_tokens(1), seed=0, device=DEV)
    cpu = to_cpu_inputs(inp)
    yield inp, cpu
    del inp, cpu
    torch.cuda.empty_cache()


def _run(c, inp):
    p = moe.MoEProblem.from_config(c)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD)
    out = torch.empty(c.T, c.H, dtype=c.dtype, device=DEV)
    idx = torch.empty(c.T, c.top_k, dtype=torch.int32, device=DEV)
    w = torch.empty(c.T, c.top_k, dtype=torch.float32, device=DEV)
    moe.moe_forward(p, inp["x"], inp["gate_w"], inp["logit_bias"], inp["expert_w"],
                    inp["shared_w"], out, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    del ws
    return out, idx, w


def _check(c, inp, cpu, all_tokens=False):
    out, idx, w = _run(c, inp)
    # routing on every token
    forward_parity_routing_only(inp, c, idx, w, cpu)
    if all_tokens:
        toks = list(range(c.T))
    else:
        widths = moe.moe_expert_tile_rows(moe.MoEProblem.from_config(c))
        toks, tiles = schedule_cover_tokens(idx.cpu().numpy(), c.E, c.num_shared, widths)
        print(f"{c.name}: {len(toks)} tokens cover all tiles (tile widths {widths}: "
              f"{tiles} tiles), coverage 1.0")
    n_ex, err, scale = forward_parity(inp, c, out, idx, w, tokens=toks, cpu_inp=cpu)
    return idx, n_ex, err, scale


def forward_parity_routing_only(inp, c, idx, w, cpu):
    import oracle
    from parity_util import check_routing
    orc = oracle.route(cpu["x"], cpu["gate_w"], c.top_k, c.routed_scale,
                       logit_bias=cpu["logit_bias"])
    exempt = check_routing(idx.cpu().numpy(), w.cpu().numpy(), orc, c.top_k)
    # near-ties are rare: a few per ten thousand tokens at these shapes
    assert len(exempt) <= max(4, c.T // 500), len(exempt)


def test_tiny_config():
    c = CONFIGS["tiny"]
    inp = make_inputs(c, seed=0, device=DEV)
    _check(c, inp, to_cpu_inputs(inp), all_tokens=True)


def test_hy3_config():
    c = CONFIGS["hy3"]
    inp = make_inputs(c, seed=0, device=DEV)
    _check(c, inp, to_cpu_inputs(inp))


@pytest.mark.parametrize("name", ["hy4_decode", "hy4_prefill", "hy4_skew"])
def test_hy4_configs(name, hy4_weights):
    c = CONFIGS[name]
    winp, wcpu = hy4_weights
    x = make_x(c, seed=0, device=DEV)
    inp = dict(winp, x=x)
    inp["logit_bias"] = None
    if c.skew_bias:
        from sparse_moe_layer_06_b200.workloads import skew_logit_bias
        inp["logit_bias"] = skew_logit_bias(c.E).to(DEV)
    cpu = dict(wcpu, x=x.cpu(), logit_bias=None if inp["logit_bias"] is None
               else inp["logit_bias"].cpu())
    idx, n_ex, err, scale = _check(c, inp, cpu, all_tokens=c.T <= 64)
    counts = np.bincount(idx.cpu().numpy().ravel(), minlength=c.E)
    if name == "hy4_decode":
        assert 150 <= (counts > 0).sum() <= 256
    if name == "hy4_prefill":
        assert (counts > 0).all()
    if name == "hy4_skew":
        share = counts / c.T
        assert (share > 0.10).sum() >= 5  # a few experts take >10% of tokens
        assert (counts == 0).sum() >= 20  # and many are idle
