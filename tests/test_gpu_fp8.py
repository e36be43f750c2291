"""GPU parity of the FP8 (E4M3) expert-weight path against the oracle.

Weight encoding (moe_quantize_weights_fp8): codes bit-exact and scales exact,
since every decision is taken on the same value (weight / power of two, exact
in both precisions) with the same round-to-nearest-even rule.

Layer output (moe_forward_fp8): the oracle's FP8 forward on the same inputs,
with its own codes.  The GPU sums exact code products in fp32 and rounds h to
E4M3 from an fp32 value, the oracle from fp64; an h element whose two values
straddle an E4M3 rounding midpoint changes by one code step (rare), and the
combined rows are bf16 as in the bf16 path, so the bf16 tolerance (2e-2 of the
output's largest magnitude) applies."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_close_out, check_routing, to_cpu_inputs, OUT_TOL
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import CONFIGS, MoEConfig, make_inputs, sample_tokens

pytestmark = pytest.mark.gpu
DEV = "cuda"

SMALL = MoEConfig("fp8_small", T=200, H=256, E=16, top_k=4, I=256, num_shared=1,
                  dtype=torch.bfloat16, x_std=1.0, w_std=0.05, routed_scale=2.827,
                  clip_limit=10.0)


def gpu_quantize(p, w):
    n = w.shape[0]
    q = torch.empty(w.shape, dtype=torch.uint8, device=DEV)
    s_gu = torch.empty(n, 2, p.I, dtype=torch.float32, device=DEV)
    s_d = torch.empty(n, p.H, dtype=torch.float32, device=DEV)
    moe.moe_quantize_weights_fp8(p, w, q, s_gu, s_d)
    torch.cuda.synchronize()
    return q, s_gu, s_d


def assert_same_codes(gpu, ref, what):
    q, s_gu, s_d = (t.cpu().numpy() for t in gpu)
    rq, rs_gu, rs_d = ref
    assert np.array_equal(s_gu.astype(np.float64), rs_gu), f"{what}: gate/up scales"
    assert np.array_equal(s_d.astype(np.float64), rs_d), f"{what}: down scales"
    bad = np.count_nonzero(q != rq)
    assert bad == 0, f"{what}: {bad} codes differ"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_weights_bit_exact(dtype):
    E, I, H = 3, 128, 384
    g = torch.Generator().manual_seed(5)
    w = torch.randn(E, 3, I, H, generator=g) * 0.02
    # rows and columns that exercise the scale choice: all zero, one huge
    # entry, tiny magnitudes, values exactly on powers of two, a row whose
    # maximum is exactly 448 * 2^n
    w[0, 0, 3] = 0.0
    w[0, 1, 5, 17] = 3.0e4
    w[1, 0, 7] *= 1e-6
    w[1, 1, 9, :8] = torch.tensor([1.0, -2.0, 0.5, 0.25, -4.0, 8.0, 1.5, -0.75])
    w[2, 0, 11] = torch.linspace(-448.0 / 64, 448.0 / 64, H)
    w[2, 2, :, 40] = 0.0
    w[2, 2, 64, 41] = -7.5
    w = w.to(dtype)
    p = moe.MoEProblem(T=1, H=H, E=E, I=I, top_k=1, num_shared=0, routed_scale=1.0,
                       clip_limit=10.0, dtype=dtype)
    gpu = gpu_quantize(p, w.to(DEV))
    assert_same_codes(gpu, oracle.quantize_weights_fp8(w), f"{dtype}")


def run_fp8(cfg, inp, T=None):
    T = cfg.T if T is None else T
    p = moe.MoEProblem.from_config(cfg, T=T)
    q, s_gu, s_d = gpu_quantize(p, inp["expert_w"])
    sq = ss_gu = ss_d = None
    if inp["shared_w"] is not None:
        sq, ss_gu, ss_d = gpu_quantize(p, inp["shared_w"].unsqueeze(0))
    ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD_FP8)
    out = torch.full((T, cfg.H), float("nan"), dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(T, cfg.top_k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, cfg.top_k, dtype=torch.float32, device=DEV)
    moe.moe_forward_fp8(p, inp["x"][:T], inp["gate_w"], inp["logit_bias"], q, s_gu, s_d, sq,
                        ss_gu, ss_d, out, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    return out, idx, w, (q, s_gu, s_d), (sq, ss_gu, ss_d)


def oracle_fp8_parity(cfg, cpu, out, idx, w, tokens):
    """Route `tokens` with the oracle, check the GPU's routing (near-ties
    validated), quantize the weights with the oracle and compare the layer
    output with the GPU's expert choice forced."""
    k = cfg.top_k
    r = oracle.route(cpu["x"], cpu["gate_w"], k, cfg.routed_scale,
                     logit_bias=cpu["logit_bias"], tokens=tokens)
    gi = idx.cpu().numpy()[tokens]
    exempt = set(check_routing(gi, w.cpu().numpy()[tokens], r, k))
    rq, rs_gu, rs_d = oracle.quantize_weights_fp8(cpu["expert_w"])
    sq = ss_gu = ss_d = None
    if cpu["shared_w"] is not None:
        sq, ss_gu, ss_d = oracle.quantize_weights_fp8(cpu["shared_w"].unsqueeze(0))
    ref = oracle.forward_fp8(cpu["x"], cpu["gate_w"], rq, rs_gu, rs_d, sq, ss_gu, ss_d, k,
                             cfg.routed_scale, cfg.clip_limit, logit_bias=cpu["logit_bias"],
                             tokens=tokens, forced_idx=gi.astype(np.int32))
    got = out.float().cpu().numpy()[tokens]
    err, scale = assert_close_out(got, ref["out"], f"{cfg.name} fp8 forward", OUT_TOL)
    return len(exempt), err, scale


def test_forward_fp8_small():
    inp = make_inputs(SMALL, seed=3, device=DEV)
    cpu = to_cpu_inputs(inp)
    out, idx, w, gq, gs = run_fp8(SMALL, inp)
    # the kernel's weight codes equal the oracle's
    assert_same_codes(gq, oracle.quantize_weights_fp8(cpu["expert_w"]), "experts")
    assert_same_codes(gs, oracle.quantize_weights_fp8(cpu["shared_w"].unsqueeze(0)), "shared")
    oracle_fp8_parity(SMALL, cpu, out, idx, w, list(range(SMALL.T)))


@pytest.mark.parametrize("T", [1, 37, 129])
def test_forward_fp8_ragged_token_counts(T):
    inp = make_inputs(SMALL, seed=4, device=DEV)
    cpu = to_cpu_inputs(inp)
    out, idx, w, _, _ = run_fp8(SMALL, inp, T=T)
    oracle_fp8_parity(SMALL.with_tokens(T), cpu, out, idx, w, list(range(T)))


def test_forward_fp8_no_shared_expert_and_edge_tokens():
    c = MoEConfig("fp8_noshared", T=96, H=384, E=8, top_k=2, I=128, num_shared=0,
                  dtype=torch.bfloat16, x_std=1.0, w_std=0.05, routed_scale=1.0,
                  clip_limit=7.0)
    inp = make_inputs(c, seed=6, device=DEV)
    # an all-zero token (scale 1, all codes 0), a tiny one and a large one
    inp["x"][0].zero_()
    inp["x"][1].mul_(1e-3)
    inp["x"][2].mul_(300.0)
    cpu = to_cpu_inputs(inp)
    out, idx, w, _, _ = run_fp8(c, inp)
    oracle_fp8_parity(c, cpu, out, idx, w, list(range(c.T)))


def test_forward_fp8_saturating_clamp():
    # large weights: most gate/up values clamp, so h sits near its bound
    # silu(L) * L and the fixed h scale is exercised at its top codes
    c = MoEConfig("fp8_sat", T=64, H=256, E=8, top_k=2, I=128, num_shared=1,
                  dtype=torch.bfloat16, x_std=1.0, w_std=1.5, routed_scale=2.827,
                  clip_limit=10.0)
    inp = make_inputs(c, seed=7, device=DEV)
    cpu = to_cpu_inputs(inp)
    out, idx, w, _, _ = run_fp8(c, inp)
    oracle_fp8_parity(c, cpu, out, idx, w, list(range(c.T)))


@pytest.mark.parametrize("shape", [dict(T=200, E=16, top_k=4, I=256),
                                   dict(T=700, E=8, top_k=2, I=384)])
def test_forward_fp8_row_gather_and_permuted_copy_agree(monkeypatch, shape):
    """The gate/up GEMM takes the E4M3 token rows either straight from the
    per-token codes by the gather warps (MOE_FUSED_GATHER=1; the default for
    tiles of up to 160 rows) or from the permuted copy (MOE_FUSED_GATHER=0).
    The two fill the same shared-memory tiles, so the layers are bit-identical;
    both match the oracle.  The second shape has 175 rows per expert: tiles of
    160 rows and ragged second chunks."""
    c = MoEConfig("fp8_gather", H=512, num_shared=1, dtype=torch.bfloat16, x_std=1.0,
                  w_std=0.05, routed_scale=2.827, clip_limit=10.0, **shape)
    inp = make_inputs(c, seed=12, device=DEV)
    cpu = to_cpu_inputs(inp)
    outs = {}
    for fg in ("1", "0"):
        monkeypatch.setenv("MOE_FUSED_GATHER", fg)
        out, idx, w, _, _ = run_fp8(c, inp)
        oracle_fp8_parity(c, cpu, out, idx, w, list(range(0, c.T, 3)))
        outs[fg] = (out, idx)
    assert torch.equal(outs["1"][1], outs["0"][1])
    assert torch.equal(outs["1"][0], outs["0"][0])


@pytest.mark.parametrize("env", [
    {"MOE_NMAX": "256", "MOE_FUSED_GATHER": "1"},        # E4M3 gather warps on 256-row tiles
    {"MOE_NMAX": "64", "MOE_DOWN_MB": "1"},              # narrow tiles, one down sub-tile
])
def test_forward_fp8_tile_shape_variants(monkeypatch, env):
    """Forced tile shapes of the FP8 expert GEMMs against the oracle."""
    for k_, v_ in env.items():
        monkeypatch.setenv(k_, v_)
    inp = make_inputs(SMALL, seed=13, device=DEV)
    cpu = to_cpu_inputs(inp)
    out, idx, w, _, _ = run_fp8(SMALL, inp)
    oracle_fp8_parity(SMALL, cpu, out, idx, w, list(range(SMALL.T)))


def test_forward_fp8_empty_batch_and_rejections():
    p = moe.MoEProblem.from_config(SMALL, T=0)
    ws = moe.alloc_workspace(moe.MoEProblem.from_config(SMALL, T=1), moe.MOE_CALL_FORWARD_FP8)
    z = torch.zeros(16, dtype=torch.bfloat16, device=DEV)
    gw = torch.zeros(SMALL.E, SMALL.H, dtype=torch.bfloat16, device=DEV)
    q = torch.zeros(SMALL.E, 3, SMALL.I, SMALL.H, dtype=torch.uint8, device=DEV)
    sg = torch.ones(SMALL.E, 2, SMALL.I, device=DEV)
    sd = torch.ones(SMALL.E, SMALL.H, device=DEV)
    shq = torch.zeros(1, 3, SMALL.I, SMALL.H, dtype=torch.uint8, device=DEV)
    shg = torch.ones(1, 2, SMALL.I, device=DEV)
    shd = torch.ones(1, SMALL.H, device=DEV)
    before = moe.moe_launch_count()
    moe.moe_forward_fp8(p, z, gw, None, q, sg, sd, shq, shg, shd, z, None, None, ws)
    assert moe.moe_launch_count() == before
    # no clamp: h is unbounded, so the fixed h scale does not exist
    p2 = moe.MoEProblem.from_config(SMALL, T=1)
    p2 = moe.MoEProblem(**{**p2.__dict__, "clip_limit": 0.0})
    x = torch.zeros(1, SMALL.H, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moe.MoEError):
        moe.moe_forward_fp8(p2, x, gw, None, q, sg, sd, shq, shg, shd, x, None, None, ws)


@pytest.fixture(scope="module")
def hy4():
    c = CONFIGS["hy4_prefill"]
    inp = make_inputs(c, seed=0, device=DEV)
    yield c, inp
    del inp
    torch.cuda.empty_cache()


def test_forward_fp8_hy4_prefill_sampled(hy4):
    """Full Hy4-shape prefill batch (T=4096, 256 experts top-8 + shared) in
    one moe_forward_fp8 call; routing on every token, output on a seeded
    sample, the oracle quantizing the experts those tokens reach."""
    c, inp = hy4
    out, idx, w, gq, _ = run_fp8(c, inp)
    cpu = to_cpu_inputs({k: v for k, v in inp.items() if k != "expert_w"})
    orc = oracle.route(cpu["x"], cpu["gate_w"], c.top_k, c.routed_scale,
                       logit_bias=cpu["logit_bias"])
    check_routing(idx.cpu().numpy(), w.cpu().numpy(), orc, c.top_k)
    toks = sample_tokens(c.T, 6, seed=2)
    gi = idx.cpu().numpy()[toks]
    experts = set(int(e) for e in gi.ravel())
    sel = sorted(experts)
    cpu["expert_w"] = inp["expert_w"][sel].cpu()
    # weight codes of the selected experts: bit-exact
    rq, rs_gu, rs_d = oracle.quantize_weights_fp8(cpu["expert_w"])
    assert_same_codes(tuple(t[sel] for t in gq), (rq, rs_gu, rs_d), "hy4 experts")
    # the oracle runs on the selected experts only, renumbered 0..n-1 (gate
    # rows and bias entries taken along): the GPU's validated choice is
    # forced, and the renormalized routing weights scale * p_j / sum_sel p
    # do not depend on the softmax normalizer over the other experts
    remap = {e: j for j, e in enumerate(sel)}
    forced = np.vectorize(remap.get)(gi).astype(np.int32)
    bias = cpu["logit_bias"][sel] if cpu["logit_bias"] is not None else None
    sq, ss_gu, ss_d = oracle.quantize_weights_fp8(cpu["shared_w"].unsqueeze(0))
    ref = oracle.forward_fp8(cpu["x"], cpu["gate_w"][sel], rq, rs_gu, rs_d, sq, ss_gu, ss_d,
                             c.top_k, c.routed_scale, c.clip_limit, logit_bias=bias,
                             tokens=toks, forced_idx=forced)
    got = out.float().cpu().numpy()[toks]
    assert_close_out(got, ref["out"], "hy4_prefill fp8 forward", OUT_TOL)


def test_forward_fp8_hy4_decode_sampled(hy4):
    """The Hy4-shape decode batch (T=64: about two rows per touched expert,
    the smallest token tiles) with FP8 weights; the oracle checks a seeded
    sample of tokens on the experts they reach."""
    c, inp = hy4
    cd = CONFIGS["hy4_decode"]
    out, idx, w, gq, _ = run_fp8(cd, inp, T=cd.T)
    cpu = to_cpu_inputs({k: v for k, v in inp.items() if k != "expert_w"})
    cpu["x"] = cpu["x"][:cd.T]
    orc = oracle.route(cpu["x"], cpu["gate_w"], cd.top_k, cd.routed_scale,
                       logit_bias=cpu["logit_bias"])
    check_routing(idx.cpu().numpy(), w.cpu().numpy(), orc, cd.top_k)
    toks = sample_tokens(cd.T, 4, seed=5)
    gi = idx.cpu().numpy()[toks]
    sel = sorted(set(int(e) for e in gi.ravel()))
    rq, rs_gu, rs_d = oracle.quantize_weights_fp8(inp["expert_w"][sel].cpu())
    assert_same_codes(tuple(t[sel] for t in gq), (rq, rs_gu, rs_d), "hy4 decode experts")
    remap = {e: j for j, e in enumerate(sel)}
    forced = np.vectorize(remap.get)(gi).astype(np.int32)
    bias = cpu["logit_bias"][sel] if cpu["logit_bias"] is not None else None
    sq, ss_gu, ss_d = oracle.quantize_weights_fp8(cpu["shared_w"].unsqueeze(0))
    ref = oracle.forward_fp8(cpu["x"], cpu["gate_w"][sel], rq, rs_gu, rs_d, sq, ss_gu, ss_d,
                             cd.top_k, cd.routed_scale, cd.clip_limit, logit_bias=bias,
                             tokens=toks, forced_idx=forced)
    got = out.float().cpu().numpy()[toks]
    assert_close_out(got, ref["out"], "hy4_decode fp8 forward", OUT_TOL)
