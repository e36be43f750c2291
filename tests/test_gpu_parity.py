"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs, stage by stage and end to end, including edge cases."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (OUT_TOL, assert_close_out, check_routing, forward_parity, out_tol,
                         to_cpu_inputs)
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def cfg(name="case", T=300, H=512, E=16, k=4, I=384, S=1, dtype=torch.bfloat16, scale=2.827,
        clip=10.0, w_std=0.02, x_std=1.0):
    return MoEConfig(name, T=T, H=H, E=E, top_k=k, I=I, num_shared=S, dtype=dtype, x_std=x_std,
                     w_std=w_std, routed_scale=scale, clip_limit=clip)


def run_forward(c: MoEConfig, inp: dict):
    p = moe.MoEProblem.from_config(c)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD)
    out = torch.empty(c.T, c.H, dtype=c.dtype, device=DEV)
    idx = torch.empty(c.T, c.top_k, dtype=torch.int32, device=DEV)
    w = torch.empty(c.T, c.top_k, dtype=torch.float32, device=DEV)
    moe.moe_forward(p, inp["x"], inp["gate_w"], inp["logit_bias"], inp["expert_w"],
                    inp["shared_w"], out, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    return out, idx, w


# ------------------------------------------------------------------ router


@pytest.mark.parametrize("shape", [dict(T=300, H=512, E=16), dict(T=77, H=320, E=256),
                                   dict(T=1, H=64, E=3), dict(T=513, H=1024, E=130)])
def test_router_logits_match_oracle(shape):
    c = cfg(**shape, k=1)
    inp = make_inputs(c, seed=1, device=DEV)
    p = moe.MoEProblem.from_config(c)
    logits = torch.empty(c.T, c.E, dtype=torch.float32, device=DEV)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_ROUTER_LOGITS)
    moe.moe_router_logits(p, inp["x"], inp["gate_w"], logits, ws)
    torch.cuda.synchronize()
    ci = to_cpu_inputs(inp)
    ref = oracle.route(ci["x"], ci["gate_w"], 1, 1.0)["logits"]
    # fp32 accumulation of bf16 products: bound by 1e-4 of sum_h |x_h w_h|
    bound = (ci["x"].double().abs() @ ci["gate_w"].double().abs().T).numpy()
    err = np.abs(logits.cpu().numpy() - ref)
    assert np.all(err <= 1e-4 * bound + 1e-6), float(np.max(err / (bound + 1e-30)))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("E,k", [(16, 2), (256, 8), (8, 8), (33, 5)])
def test_route_matches_oracle(dtype, E, k):
    c = cfg(T=257, H=256, E=E, k=k, dtype=dtype)
    inp = make_inputs(c, seed=2, device=DEV)
    p = moe.MoEProblem.from_config(c)
    idx = torch.empty(c.T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(c.T, k, dtype=torch.float32, device=DEV)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_ROUTE)
    moe.moe_route(p, inp["x"], inp["gate_w"], None, idx, w, ws)
    torch.cuda.synchronize()
    ci = to_cpu_inputs(inp)
    orc = oracle.route(ci["x"], ci["gate_w"], k, c.routed_scale)
    exempt = check_routing(idx.cpu().numpy(), w.cpu().numpy(), orc, k)
    assert len(exempt) <= 2
    np.testing.assert_allclose(w.sum(-1).cpu().numpy(), c.routed_scale, rtol=1e-5)


def test_route_exact_ties_lower_index_first():
    c = cfg(T=64, H=128, E=16, k=3)
    inp = make_inputs(c, seed=3, device=DEV)
    # experts 2, 9 and 13 get identical gate rows -> identical logits
    inp["gate_w"][9] = inp["gate_w"][2]
    inp["gate_w"][13] = inp["gate_w"][2]
    bias = torch.zeros(c.E, device=DEV)
    bias[[2, 9, 13]] = 50.0  # make the tied experts the top three
    p = moe.MoEProblem.from_config(c)
    idx = torch.empty(c.T, 3, dtype=torch.int32, device=DEV)
    w = torch.empty(c.T, 3, dtype=torch.float32, device=DEV)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_ROUTE)
    moe.moe_route(p, inp["x"], inp["gate_w"], bias, idx, w, ws)
    torch.cuda.synchronize()
    assert (idx.cpu() == torch.tensor([2, 9, 13], dtype=torch.int32)).all()
    ci = to_cpu_inputs(inp)
    orc = oracle.route(ci["x"], ci["gate_w"], 3, c.routed_scale, logit_bias=bias.cpu())
    assert (orc["idx"] == np.array([2, 9, 13])).all()
    np.testing.assert_allclose(w.cpu().numpy(), c.routed_scale / 3, rtol=1e-6)


# ------------------------------------------------------------------ dispatch


@pytest.mark.parametrize("T,E,k", [(300, 16, 4), (1, 8, 8), (1000, 256, 8), (40, 64, 2)])
def test_permute_bit_exact(T, E, k):
    c = cfg(T=T, E=E, k=k, H=128)
    inp = make_inputs(c, seed=4, device=DEV)
    ci = to_cpu_inputs(inp)
    orc_route = oracle.route(ci["x"], ci["gate_w"], k, 1.0)
    ref = oracle.permute(orc_route["idx"], E)
    p = moe.MoEProblem.from_config(c)
    idx = torch.from_numpy(orc_route["idx"]).to(DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    pos = torch.empty(T, k, dtype=torch.int32, device=DEV)
    src = torch.empty(T * k, dtype=torch.int32, device=DEV)
    x_perm = torch.empty(T * k, c.H, dtype=c.dtype, device=DEV)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_PERMUTE)
    moe.moe_permute(p, idx, inp["x"], offsets, pos, src, x_perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    np.testing.assert_array_equal(offsets.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(pos.cpu().numpy(), ref["pos"])
    np.testing.assert_array_equal(src.cpu().numpy(), ref["src"])
    assert torch.equal(x_perm.cpu(), ci["x"][torch.from_numpy(ref["src"]).long()])


def test_permute_flags_bad_index_without_fault():
    c = cfg(T=50, E=8, k=2, H=64)
    p = moe.MoEProblem.from_config(c)
    idx = torch.zeros(50, 2, dtype=torch.int32, device=DEV)
    idx[:, 1] = 1
    idx[7, 1] = 8  # out of range
    x = torch.zeros(50, 64, dtype=c.dtype, device=DEV)
    offsets = torch.empty(9, dtype=torch.int32, device=DEV)
    pos = torch.full((50, 2), -1, dtype=torch.int32, device=DEV)
    src = torch.zeros(100, dtype=torch.int32, device=DEV)
    x_perm = torch.zeros(100, 64, dtype=c.dtype, device=DEV)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_PERMUTE)
    moe.moe_permute(p, idx, x, offsets, pos, src, x_perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_BAD_INDEX
    moe.moe_clear_device_status(ws)
    assert moe.moe_read_device_status(ws) == 0


# ------------------------------------------------------------------ grouped FFN


def _ffn_case(c, seed, dtype_out=None):
    inp = make_inputs(c, seed=seed, device=DEV)
    ci = to_cpu_inputs(inp)
    orc_route = oracle.route(ci["x"], ci["gate_w"], c.top_k, 1.0)
    perm = oracle.permute(orc_route["idx"], c.E)
    src = perm["src"]
    row_expert = np.repeat(np.arange(c.E), perm["counts"]).astype(np.int32)
    x_perm = inp["x"][torch.from_numpy(src).long().to(DEV)].contiguous()
    return inp, ci, perm, src, row_expert, x_perm


@pytest.mark.parametrize("shape", [dict(T=300, H=512, E=16, k=4, I=384),
                                   dict(T=64, H=320, E=8, k=2, I=192),
                                   dict(T=700, H=256, E=4, k=2, I=128),
                                   dict(T=20, H=256, E=64, k=6, I=256)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_grouped_ffn_matches_oracle(shape, dtype):
    c = cfg(**shape, dtype=dtype, S=0)
    inp, ci, perm, src, row_expert, x_perm = _ffn_case(c, seed=5)
    p = moe.MoEProblem.from_config(c)
    rows = c.T * c.top_k
    y = torch.zeros(rows, c.H, dtype=dtype, device=DEV)
    offsets = torch.from_numpy(perm["offsets"]).to(DEV)
    ws = torch.zeros(moe.ffn_workspace_size(p, rows, c.E), dtype=torch.uint8, device=DEV)
    moe.moe_grouped_swiglu_ffn(p, x_perm, offsets, c.E, inp["expert_w"], y, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    ref = oracle.expert_rows(ci["x"], ci["expert_w"], None, src, row_expert, c.clip_limit)
    assert_close_out(y.float().cpu().numpy(), ref, "grouped ffn", out_tol(c))


def test_grouped_ffn_clamp_saturated():
    # weights x100: most gate/up pre-activations exceed the +-10 limit
    c = cfg(T=96, H=256, E=4, k=2, I=128, S=0, w_std=2.0)
    inp, ci, perm, src, row_expert, x_perm = _ffn_case(c, seed=6)
    g = ci["x"].double() @ ci["expert_w"][0, 0].double().T
    assert (g.abs() > 10).double().mean() > 0.5
    p = moe.MoEProblem.from_config(c)
    rows = c.T * c.top_k
    y = torch.zeros(rows, c.H, dtype=c.dtype, device=DEV)
    ws = torch.zeros(moe.ffn_workspace_size(p, rows, c.E), dtype=torch.uint8, device=DEV)
    moe.moe_grouped_swiglu_ffn(p, x_perm, torch.from_numpy(perm["offsets"]).to(DEV), c.E,
                               inp["expert_w"], y, ws)
    torch.cuda.synchronize()
    ref = oracle.expert_rows(ci["x"], ci["expert_w"], None, src, row_expert, 10.0)
    assert_close_out(y.float().cpu().numpy(), ref, "clamped ffn")


def test_grouped_ffn_empty_groups_and_single_group():
    c = cfg(T=100, H=256, E=1, k=1, I=128, S=0)
    inp = make_inputs(c, seed=7, device=DEV)
    ci = to_cpu_inputs(inp)
    p = moe.MoEProblem.from_config(c)
    # 5 groups sharing the same weights where groups 0, 2 and 4 are empty
    w5 = inp["expert_w"].expand(5, 3, c.I, c.H).contiguous()
    offsets = torch.tensor([0, 0, 60, 60, 100, 100], dtype=torch.int32, device=DEV)
    y = torch.zeros(100, c.H, dtype=c.dtype, device=DEV)
    ws = torch.zeros(moe.ffn_workspace_size(p, 100, 5), dtype=torch.uint8, device=DEV)
    moe.moe_grouped_swiglu_ffn(p, inp["x"], offsets, 5, w5, y, ws)
    torch.cuda.synchronize()
    ref = oracle.expert_rows(ci["x"], ci["expert_w"], None, np.arange(100), np.zeros(100),
                             c.clip_limit)
    assert_close_out(y.float().cpu().numpy(), ref, "single-group ffn")


# ------------------------------------------------------------------ combine


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("S", [0, 1])
def test_combine_matches_oracle(dtype, S):
    c = cfg(T=129, H=384, E=16, k=4, S=S, dtype=dtype)
    inp = make_inputs(c, seed=8, device=DEV)
    ci = to_cpu_inputs(inp)
    orc_route = oracle.route(ci["x"], ci["gate_w"], c.top_k, c.routed_scale)
    perm = oracle.permute(orc_route["idx"], c.E)
    g = torch.Generator(device="cpu").manual_seed(9)
    y_perm = torch.randn(c.T * c.top_k, c.H, generator=g).to(dtype)
    shared_y = torch.randn(c.T, c.H, generator=g).to(dtype) if S else None
    w32 = torch.from_numpy(orc_route["w"]).float()
    p = moe.MoEProblem.from_config(c)
    out = torch.empty(c.T, c.H, dtype=dtype, device=DEV)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_COMBINE)
    moe.moe_combine(p, y_perm.to(DEV), torch.from_numpy(perm["pos"]).to(DEV), w32.to(DEV),
                    shared_y.to(DEV) if S else None, out, ws)
    torch.cuda.synchronize()
    ref = oracle.combine(y_perm.double().numpy(), perm["pos"], w32.double().numpy(),
                         shared_y.double().numpy() if S else None)
    assert_close_out(out.float().cpu().numpy(), ref, "combine", tol=1e-2)


# ------------------------------------------------------------------ whole layer


@pytest.mark.parametrize("shape", [
    dict(T=300, H=512, E=16, k=4, I=384),           # several tiles, ragged tails
    dict(T=1, H=256, E=16, k=2, I=128),             # single token
    dict(T=8, H=256, E=64, k=2, I=128),             # most experts empty
    dict(T=130, H=256, E=8, k=8, I=128),            # k == E
    dict(T=200, H=320, E=12, k=3, I=192),           # H, I not multiples of 128
    dict(T=64, H=256, E=16, k=2, I=128, S=0, scale=1.0, clip=0.0),  # no shared, no clip
    dict(T=50, H=64, E=1, k=1, I=64),               # one expert, smallest H and I
    dict(T=77, H=192, E=256, k=8, I=64),            # widest router, I below one tile
])
def test_forward_matches_oracle(shape):
    c = cfg(**shape)
    inp = make_inputs(c, seed=10, device=DEV)
    out, idx, w = run_forward(c, inp)
    forward_parity(inp, c, out, idx, w)


def test_forward_fp32_tiny_config():
    from sparse_moe_layer_06_b200.workloads import CONFIGS
    c = CONFIGS["tiny"]
    inp = make_inputs(c, seed=0, device=DEV)
    out, idx, w = run_forward(c, inp)
    assert out.dtype == torch.float32
    # TF32 expert GEMMs: checked to the fp32 bound (a quarter of the bf16 one)
    _, err, scale = forward_parity(inp, c, out, idx, w)
    print(f"tiny fp32 layer: max err {err:.3e} of max |out| {scale:.3e} ({err / scale:.2e})")


def test_forward_all_tokens_to_two_experts():
    c = cfg(T=600, H=256, E=16, k=2, I=128)
    inp = make_inputs(c, seed=11, device=DEV)
    bias = torch.zeros(c.E, device=DEV)
    bias[3] = 40.0
    bias[11] = 30.0  # gap of 10 >> logit spread (std ~0.3): order is fixed
    inp["logit_bias"] = bias
    out, idx, w = run_forward(c, inp)
    assert (idx.cpu()[:, 0] == 3).all() and (idx.cpu()[:, 1] == 11).all()
    forward_parity(inp, c, out, idx, w)


def test_forward_saturating_clamp():
    c = cfg(T=100, H=256, E=8, k=2, I=128, w_std=2.0)
    inp = make_inputs(c, seed=12, device=DEV)
    # keep the router sane: ordinary gate weights
    inp["gate_w"] = (inp["gate_w"].float() * 0.01).to(c.dtype)
    out, idx, w = run_forward(c, inp)
    forward_parity(inp, c, out, idx, w)


def test_forward_empty_batch_is_noop():
    c = cfg(T=0)
    p = moe.MoEProblem.from_config(c)
    # T = 0 tokens, full-size weights: nothing is enqueued
    inp = make_inputs(c.with_tokens(1), seed=1, device=DEV)
    empty = torch.zeros(1, c.H, dtype=c.dtype, device=DEV)  # (a non-null pointer)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD)
    torch.cuda.synchronize()
    before = moe.moe_launch_count()
    moe.moe_forward(p, empty, inp["gate_w"], None, inp["expert_w"], inp["shared_w"], empty, None,
                    None, ws)
    assert moe.moe_launch_count() == before


def test_forward_repeatable_and_staged_path_agrees():
    """The fused path and the staged path (route, permute, FFN, FFN for the
    shared expert, combine) agree within the tolerance; repeated fused calls
    reproduce the routing exactly."""
    c = cfg(T=257, H=384, E=16, k=4, I=256)
    inp = make_inputs(c, seed=13, device=DEV)
    out1, idx1, w1 = run_forward(c, inp)
    out2, idx2, w2 = run_forward(c, inp)
    assert torch.equal(idx1, idx2) and torch.equal(w1, w2)
    p = moe.MoEProblem.from_config(c)
    T, k, H = c.T, c.top_k, c.H
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    moe.moe_route(p, inp["x"], inp["gate_w"], None, idx, w, moe.alloc_workspace(p, 0))
    offsets = torch.empty(c.E + 1, dtype=torch.int32, device=DEV)
    pos = torch.empty(T, k, dtype=torch.int32, device=DEV)
    src = torch.empty(T * k, dtype=torch.int32, device=DEV)
    x_perm = torch.empty(T * k, H, dtype=c.dtype, device=DEV)
    moe.moe_permute(p, idx, inp["x"], offsets, pos, src, x_perm, moe.alloc_workspace(p, 2))
    y_perm = torch.empty(T * k, H, dtype=c.dtype, device=DEV)
    ws = torch.zeros(moe.ffn_workspace_size(p, T * k, c.E), dtype=torch.uint8, device=DEV)
    moe.moe_grouped_swiglu_ffn(p, x_perm, offsets, c.E, inp["expert_w"], y_perm, ws)
    shared_y = torch.empty(T, H, dtype=c.dtype, device=DEV)
    ws1 = torch.zeros(moe.ffn_workspace_size(p, T, 1), dtype=torch.uint8, device=DEV)
    moe.moe_grouped_swiglu_ffn(p, inp["x"], torch.tensor([0, T], dtype=torch.int32, device=DEV),
                               1, inp["shared_w"].unsqueeze(0).contiguous(), shared_y, ws1)
    out_s = torch.empty(T, H, dtype=c.dtype, device=DEV)
    moe.moe_combine(p, y_perm, pos, w, shared_y, out_s, moe.alloc_workspace(p, 4))
    torch.cuda.synchronize()
    assert torch.equal(idx, idx1)
    forward_parity(inp, c, out_s, idx, w)
    ref = out1.float().cpu().numpy()
    assert_close_out(out_s.float().cpu().numpy(), ref.astype(np.float64), "staged vs fused",
                     tol=OUT_TOL)


def test_forward_gather_variants_agree():
    """The permuted token copy instead of the row gather inside the gate/up
    GEMM (MOE_FUSED_GATHER=0), the scatter-add combine (MOE_COMBINE=atomic),
    the rotated K order (MOE_KROT=1), ordinary launches without programmatic
    dependent launch (MOE_PDL=0) give the same layer: each is checked against
    the oracle in a fresh process."""
    import os
    import subprocess
    import sys
    code = (
        "import torch, sys; sys.path.insert(0, '.'); sys.path.insert(0, 'tests');"
        "from test_gpu_parity import cfg, run_forward;"
        "from parity_util import forward_parity;"
        "from sparse_moe_layer_06_b200.workloads import make_inputs;"
        "c = cfg(T=300, H=512, E=16, k=4, I=384);"
        "inp = make_inputs(c, seed=10, device='cuda');"
        "out, idx, w = run_forward(c, inp);"
        "forward_parity(inp, c, out, idx, w); print('ok')")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for env in ({"MOE_FUSED_GATHER": "0"}, {"MOE_COMBINE": "atomic"},
                {"MOE_FUSED_GATHER": "0", "MOE_COMBINE": "atomic"}, {"MOE_KROT": "1"},
                {"MOE_PDL": "0"}, {"MOE_PDL": "0", "MOE_FUSED_GATHER": "0"}):
        r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True,
                           text=True, env={**os.environ, **env}, timeout=600)
        assert r.returncode == 0 and "ok" in r.stdout, (env, r.stdout[-2000:], r.stderr[-2000:])


@pytest.mark.parametrize("env", [
    {"MOE_NMAX": "64"},                                  # 2 chunks per epilogue warp
    {"MOE_NMAX": "32", "MOE_DOWN_NMAX": "16"},           # down tile narrower than gate/up
    {"MOE_NMAX": "256"},                                 # two TMEM batches per sub-tile
    {"MOE_NMAX": "256", "MOE_FUSED_GATHER": "1"},        # gather warps on 256-row tiles
    {"MOE_DOWN_MB": "1"},                                # one 128-row sub-tile per down tile
    {"MOE_NMAX": "160", "MOE_DOWN_MB": "1", "MOE_COMBINE": "atomic"},
])
def test_forward_tile_shape_variants(monkeypatch, env):
    """Forced token-tile widths and down sub-tile counts (the switches are read
    at every call): each selects another instantiation of the expert GEMMs'
    epilogue (chunks per warp, TMEM batches per sub-tile, accumulator buffers)
    on a layer whose experts hold ragged numbers of rows, against the oracle."""
    for k_, v_ in env.items():
        monkeypatch.setenv(k_, v_)
    c = cfg(T=300, H=512, E=16, k=4, I=384)
    inp = make_inputs(c, seed=21, device=DEV)
    out, idx, w = run_forward(c, inp)
    forward_parity(inp, c, out, idx, w)


def test_forward_cta_pair_variant():
    """Expert GEMMs run as CTA pairs (MOE_PAIR=1: cta_group::2 MMAs of
    M = 256, each CTA loading half of the token tile): bf16 layers with an odd
    number of gate/up weight blocks (I = 384) and a ragged H (320), and the
    FP8 layer, each against the oracle in a fresh process."""
    import os
    import subprocess
    import sys
    code = (
        "import torch, sys; sys.path.insert(0, '.'); sys.path.insert(0, 'tests');"
        "from test_gpu_parity import cfg, run_forward;"
        "from parity_util import forward_parity, to_cpu_inputs;"
        "from sparse_moe_layer_06_b200.workloads import make_inputs;"
        "import test_gpu_fp8 as f8;"
        "shapes = [dict(T=300, H=512, E=16, k=4, I=384), dict(T=200, H=320, E=12, k=3, I=192)];"
        "[forward_parity(inp, c, *run_forward(c, inp)) for c, inp in "
        "((c, make_inputs(c, seed=10, device='cuda')) for c in (cfg(**s) for s in shapes))];"
        "inp = make_inputs(f8.SMALL, seed=3, device='cuda');"
        "out, idx, w, _, _ = f8.run_fp8(f8.SMALL, inp);"
        "f8.oracle_fp8_parity(f8.SMALL, to_cpu_inputs(inp), out, idx, w, list(range(f8.SMALL.T)));"
        "print('ok')")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True,
                       env={**os.environ, "MOE_PAIR": "1"}, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, (r.stdout[-2000:], r.stderr[-2000:])
