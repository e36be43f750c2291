"""Pins for the CPU oracle: each test ties the oracle to something other than
itself (a library routine, a closed form, brute force, an invariant, or the
values printed on the pages), so that a dropped term, wrong sign or index, or
transposed operand anywhere in oracle/moe_oracle.c fails at least one test.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from sparse_moe_layer_06_b200.workloads import CONFIGS, MoEConfig, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_cfg(T=48, H=128, E=8, k=3, I=64, S=1, dtype=torch.float32, scale=2.827, clip=10.0,
              w_std=0.05):
    return MoEConfig("small", T=T, H=H, E=E, top_k=k, I=I, num_shared=S, dtype=dtype,
                     x_std=1.0, w_std=w_std, routed_scale=scale, clip_limit=clip)


def f64(t):
    return t.detach().to(torch.float64)


def torch_swiglu(x64, w3, clip):
    """Textbook SwiGLU with torch library ops: down(silu(gate(x)) * up(x))."""
    g = F.linear(x64, w3[0])
    u = F.linear(x64, w3[1])
    if clip > 0:
        g = torch.clamp(g, -clip, clip)
        u = torch.clamp(u, -clip, clip)
    return (F.silu(g) * u) @ w3[2]


# ---------------------------------------------------------------- routing pins

def test_route_logits_and_softmax_match_torch_float64():
    cfg = small_cfg()
    inp = make_inputs(cfg, seed=3)
    r = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, cfg.routed_scale)
    ref_logits = (f64(inp["x"]) @ f64(inp["gate_w"]).T).numpy()
    np.testing.assert_allclose(r["logits"], ref_logits, rtol=0, atol=1e-12)
    ref_p = torch.softmax(torch.from_numpy(ref_logits), dim=-1).numpy()
    np.testing.assert_allclose(r["probs"], ref_p, rtol=1e-12, atol=0)
    vals, ref_idx = torch.topk(torch.from_numpy(ref_p), cfg.top_k, dim=-1)
    np.testing.assert_array_equal(r["idx"], ref_idx.numpy())


def test_route_weights_sum_to_scale():
    for scale in (2.827, 1.0):
        cfg = small_cfg(scale=scale, E=16, k=4)
        inp = make_inputs(cfg, seed=1)
        r = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, cfg.routed_scale)
        np.testing.assert_allclose(r["w"].sum(-1), scale, rtol=1e-13)
        assert (np.diff(r["w"], axis=-1) <= 0).all(), "weights must be in descending order"


def test_renorm_equals_softmax_over_selected_logits():
    # renorm(topk(softmax(l))) * s == s * softmax(l[S]): a different formula for the same weights
    cfg = small_cfg(E=32, k=6)
    inp = make_inputs(cfg, seed=5)
    r = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, cfg.routed_scale)
    sel = np.take_along_axis(r["logits"], r["idx"].astype(np.int64), axis=-1)
    ref = cfg.routed_scale * torch.softmax(torch.from_numpy(sel), dim=-1).numpy()
    np.testing.assert_allclose(r["w"], ref, rtol=1e-12)


def test_route_logit_bias_is_added():
    cfg = small_cfg(E=16, k=2)
    inp = make_inputs(cfg, seed=2)
    bias = torch.linspace(-1.0, 1.0, cfg.E)
    r0 = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, 1.0)
    r1 = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, 1.0, logit_bias=bias)
    np.testing.assert_allclose(r1["logits"] - r0["logits"],
                               np.broadcast_to(bias.double().numpy(), r0["logits"].shape),
                               atol=1e-12)


def test_topk_tie_rule_golden():
    g = json.load(open(os.path.join(GOLDEN, "topk_ties.json")))
    col = torch.tensor(g["gate_col0"], dtype=torch.float32)
    E = col.numel()
    gate_w = torch.zeros(E, 64)
    gate_w[:, 0] = col
    x = torch.zeros(1, 64)
    x[0, 0] = 1.0
    for case in g["cases"]:
        r = oracle.route(x, gate_w, case["k"], 1.0)
        assert r["idx"][0].tolist() == case["idx"], case


def test_topk_matches_bruteforce_sort():
    cfg = small_cfg(E=24, k=5, T=40)
    inp = make_inputs(cfg, seed=9)
    r = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, 1.0)
    for t in range(cfg.T):
        p = r["probs"][t]
        order = sorted(range(cfg.E), key=lambda e: (-p[e], e))
        assert r["idx"][t].tolist() == order[:cfg.top_k]


def test_route_token_subset_matches_full():
    cfg = small_cfg()
    inp = make_inputs(cfg, seed=4)
    full = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, cfg.routed_scale)
    sub = [0, 7, 19, 47]
    part = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, cfg.routed_scale, tokens=sub)
    np.testing.assert_array_equal(part["idx"], full["idx"][sub])
    np.testing.assert_array_equal(part["w"], full["w"][sub])


# ---------------------------------------------------------------- expert FFN pins

def test_expert_rows_match_torch_swiglu():
    cfg = small_cfg(I=96, H=128, E=4)
    inp = make_inputs(cfg, seed=11)
    rows_t = [0, 3, 3, 10, 47]
    rows_e = [0, 1, 3, 2, cfg.E]  # last row: shared expert
    got = oracle.expert_rows(inp["x"], inp["expert_w"], inp["shared_w"], rows_t, rows_e,
                             cfg.clip_limit)
    x64 = f64(inp["x"])
    for r, (t, e) in enumerate(zip(rows_t, rows_e)):
        w3 = f64(inp["shared_w"] if e == cfg.E else inp["expert_w"][e])
        ref = torch_swiglu(x64[t:t + 1], w3, cfg.clip_limit)[0].numpy()
        np.testing.assert_allclose(got[r], ref, rtol=1e-11, atol=1e-13)


def test_clamp_closed_form():
    # one-hot token: g[i] = Wg[i,0], u[i] = Wu[i,0]; identity-like down projection
    gs = [-30.0, -10.0, -3.0, 0.0, 3.0, 10.0, 30.0, 9.5]
    us = [5.0, -20.0, 2.0, 7.0, -1.0, 12.0, 30.0, -10.5]
    I, H = len(gs), 64
    w = torch.zeros(1, 3, I, H)
    for i in range(I):
        w[0, 0, i, 0] = gs[i]
        w[0, 1, i, 0] = us[i]
        w[0, 2, i, i] = 1.0
    x = torch.zeros(1, H)
    x[0, 0] = 1.0
    got = oracle.expert_rows(x, w, None, [0], [0], clip=10.0)[0]
    for i in range(I):
        g = max(-10.0, min(10.0, gs[i]))
        u = max(-10.0, min(10.0, us[i]))
        expect = g / (1.0 + math.exp(-g)) * u
        assert got[i] == pytest.approx(expect, rel=1e-15, abs=1e-300), (i, got[i], expect)
    assert np.all(got[I:] == 0.0)
    # clip off: the raw values go through
    got_off = oracle.expert_rows(x, w, None, [0], [0], clip=0.0)[0]
    for i in range(I):
        expect = gs[i] / (1.0 + math.exp(-gs[i])) * us[i]
        assert got_off[i] == pytest.approx(expect, rel=1e-15, abs=1e-300)


def test_clamp_saturating_weights_match_torch():
    cfg = small_cfg(T=8, H=128, I=64, E=2, w_std=0.05 * 100)
    inp = make_inputs(cfg, seed=12)
    got = oracle.expert_rows(inp["x"], inp["expert_w"], inp["shared_w"], list(range(8)),
                             [t % 2 for t in range(8)], 10.0)
    x64 = f64(inp["x"])
    g = F.linear(x64, f64(inp["expert_w"][0, 0]))
    assert (g.abs() > 10).double().mean() > 0.5, "case must actually saturate the clamp"
    for t in range(8):
        ref = torch_swiglu(x64[t:t + 1], f64(inp["expert_w"][t % 2]), 10.0)[0].numpy()
        np.testing.assert_allclose(got[t], ref, rtol=1e-11, atol=1e-9)


def test_clamp_propagates_nan():
    H, I = 64, 4
    w = torch.zeros(1, 3, I, H)
    w[0, 0, :, 0] = 1.0
    w[0, 1, :, 0] = 1.0
    w[0, 2] = torch.eye(I, H)
    x = torch.zeros(1, H)
    x[0, 0] = float("nan")
    got = oracle.expert_rows(x, w, None, [0], [0], clip=10.0)[0]
    assert np.isnan(got[:I]).all()


# ---------------------------------------------------------------- whole-layer pins

def test_forward_matches_dense_bruteforce():
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=0)
    f = oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], cfg.top_k,
                       cfg.routed_scale, cfg.clip_limit)
    dense = np.zeros((cfg.T, cfg.E))
    for t in range(cfg.T):
        for j in range(cfg.top_k):
            dense[t, f["idx"][t, j]] = f["w"][t, j]
    bf = oracle.dense_bruteforce(inp["x"], inp["expert_w"], inp["shared_w"], dense,
                                 cfg.clip_limit)
    np.testing.assert_allclose(f["out"], bf, rtol=1e-12, atol=1e-14)


def test_forward_token_permutation_equivariance():
    cfg = small_cfg(T=32)
    inp = make_inputs(cfg, seed=6)
    perm = torch.randperm(cfg.T, generator=torch.Generator().manual_seed(1))
    a = oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], cfg.top_k,
                       cfg.routed_scale, cfg.clip_limit)
    b = oracle.forward(inp["x"][perm], inp["gate_w"], inp["expert_w"], inp["shared_w"],
                       cfg.top_k, cfg.routed_scale, cfg.clip_limit)
    np.testing.assert_array_equal(b["out"], a["out"][perm.numpy()])
    np.testing.assert_array_equal(b["idx"], a["idx"][perm.numpy()])


def test_single_expert_reduces_to_textbook_swiglu():
    # E=1, k=1: routing weight is exactly the scale; out = s*FFN(x) + shared(x)
    for clip in (0.0, 10.0):
        cfg = small_cfg(E=1, k=1, T=16, H=128, I=64)
        inp = make_inputs(cfg, seed=7)
        f = oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], 1,
                           cfg.routed_scale, clip)
        assert (f["w"] == cfg.routed_scale).all()
        x64 = f64(inp["x"])
        ref = (cfg.routed_scale * torch_swiglu(x64, f64(inp["expert_w"][0]), clip)
               + torch_swiglu(x64, f64(inp["shared_w"]), clip)).numpy()
        np.testing.assert_allclose(f["out"], ref, rtol=1e-11, atol=1e-13)


def test_forward_without_shared_expert_matches_torch():
    cfg = small_cfg(S=0, scale=1.0, clip=0.0, E=4, k=2, T=12)
    inp = make_inputs(cfg, seed=8)
    f = oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], None, cfg.top_k, 1.0, 0.0)
    x64 = f64(inp["x"])
    logits = x64 @ f64(inp["gate_w"]).T
    p = torch.softmax(logits, -1)
    tv, ti = torch.topk(p, cfg.top_k, -1)
    w = tv / tv.sum(-1, keepdim=True)
    ref = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    for t in range(cfg.T):
        for j in range(cfg.top_k):
            ref[t] += w[t, j] * torch_swiglu(x64[t:t + 1], f64(inp["expert_w"][ti[t, j]]), 0.0)[0]
    np.testing.assert_allclose(f["out"], ref.numpy(), rtol=1e-11, atol=1e-13)


def test_forced_routing_uses_own_weights():
    cfg = small_cfg(E=8, k=2, T=4)
    inp = make_inputs(cfg, seed=13)
    r = oracle.route(inp["x"], inp["gate_w"], 2, cfg.routed_scale)
    forced = np.array([[r["idx"][t, 1], r["idx"][t, 0]] for t in range(4)], np.int32)
    a = oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], 2,
                       cfg.routed_scale, cfg.clip_limit)
    b = oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], 2,
                       cfg.routed_scale, cfg.clip_limit, forced_idx=forced)
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["w"][:, ::-1], a["w"], rtol=1e-14)


def test_bf16_storage_is_widened_exactly():
    cfg = small_cfg(dtype=torch.bfloat16, T=16)
    inp = make_inputs(cfg, seed=14)
    as32 = {k: (v.float() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    a = oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], cfg.top_k,
                       cfg.routed_scale, cfg.clip_limit)
    b = oracle.forward(as32["x"], as32["gate_w"], as32["expert_w"], as32["shared_w"],
                       cfg.top_k, cfg.routed_scale, cfg.clip_limit)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["idx"], b["idx"])


# ---------------------------------------------------------------- dispatch / combine pins

def test_permute_matches_sorted_assignments():
    rng = np.random.default_rng(0)
    T, k, E = 57, 3, 10
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[5] = [9, 0, 4]  # experts 1..3 and 5..8 may be empty: keep one empty on purpose
    idx[idx == 7] = 6
    p = oracle.permute(idx, E)
    np.testing.assert_array_equal(p["counts"], np.bincount(idx.ravel(), minlength=E))
    assert p["counts"][7] == 0
    np.testing.assert_array_equal(p["offsets"], np.concatenate([[0], np.cumsum(p["counts"])]))
    order = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(k))
    for r, (e, t, j) in enumerate(order):
        assert p["pos"][t, j] == r
        assert p["src"][r] == t


def test_combine_matches_python_loops():
    rng = np.random.default_rng(1)
    T, k, H = 9, 2, 5
    rows = T * k
    y = rng.standard_normal((rows, H))
    pos = rng.permutation(rows).reshape(T, k).astype(np.int32)
    w = rng.standard_normal((T, k))
    sh = rng.standard_normal((T, H))
    got = oracle.combine(y, pos, w, sh)
    for t in range(T):
        for h in range(H):
            expect = sum(w[t, j] * y[pos[t, j], h] for j in range(k)) + sh[t, h]
            assert got[t, h] == pytest.approx(expect, rel=1e-14, abs=1e-14)
    got0 = oracle.combine(y, pos, w, None)
    np.testing.assert_allclose(got0, got - sh, rtol=1e-13, atol=1e-13)


def test_near_tie_alternatives():
    p = np.array([0.3, 0.2, 0.2 * (1 + 1e-7), 0.1, 0.2 * (1 - 5e-6), 0.0])
    sets = oracle.near_tie_alternatives(p, 2)
    assert sets[0] == (0, 2)
    assert set(sets) == {(0, 2), (0, 1), (0, 4)}
    assert oracle.near_tie_alternatives(np.array([0.5, 0.3, 0.2]), 2) == [(0, 1)]


# ---------------------------------------------------------------- configuration pins

def test_hy4_config_matches_printed_hyperparameters():
    g = json.load(open(os.path.join(GOLDEN, "hy4_config.json")))
    for name in ("hy4_prefill", "hy4_decode", "hy4_skew"):
        c = CONFIGS[name]
        assert (c.H, c.E, c.top_k, c.I, c.num_shared) == (
            g["hidden_size"], g["n_routed_experts"], g["num_experts_per_tok"],
            g["moe_intermediate_size"], g["n_shared_experts"])
        assert c.routed_scale == g["routed_scaling_factor"]
        assert c.clip_limit == g["swiglu_limit"]
        assert c.w_std == g["initializer_range"]
        assert c.dtype == torch.bfloat16
    # shape sanity: expert parameters of the 77 MoE layers fit inside the
    # printed 770B total / 49B activated
    per_expert = 3 * g["hidden_size"] * g["moe_intermediate_size"]
    experts_total = g["moe_layers"] * (g["n_routed_experts"] + g["n_shared_experts"]) * per_expert
    experts_active = g["moe_layers"] * (g["num_experts_per_tok"] + g["n_shared_experts"]) * per_expert
    assert 0.9 * g["total_params"] < experts_total < g["total_params"]
    assert experts_active < g["activated_params"]
    assert g["moe_layers"] + g["dense_layers"] == g["num_hidden_layers"]


# ---------------------------------------------------------------- router statistics pins

def test_router_stats_uniform_router_closed_form():
    # all-zero gate: every probability is 1/E, ties pick experts 0..k-1 for
    # every token, so P = 1/E, f = 1/k on the first k experts, aux = 1
    E, k, T = 8, 3, 10
    x = torch.randn(T, 64, generator=torch.Generator().manual_seed(0))
    g = torch.zeros(E, 64)
    st = oracle.router_stats(x, g, k)
    np.testing.assert_allclose(st["P"], 1.0 / E, rtol=1e-15)
    np.testing.assert_array_equal(st["counts"], [T] * k + [0] * (E - k))
    assert st["aux"] == pytest.approx(1.0, rel=1e-15)


def test_router_stats_two_token_hand_example():
    # E=2, k=1, one-hot tokens: logits (2, 0) and (0, 1)
    x = torch.zeros(2, 64)
    x[0, 0] = 1.0
    x[1, 1] = 1.0
    g = torch.zeros(2, 64)
    g[0, 0] = 2.0
    g[1, 1] = 1.0
    st = oracle.router_stats(x, g, 1)
    p0 = [math.exp(2) / (math.exp(2) + 1), 1 / (math.exp(2) + 1)]
    p1 = [1 / (1 + math.e), math.e / (1 + math.e)]
    P = [(p0[0] + p1[0]) / 2, (p0[1] + p1[1]) / 2]
    np.testing.assert_allclose(st["P"], P, rtol=1e-14)
    np.testing.assert_array_equal(st["counts"], [1, 1])
    assert st["aux"] == pytest.approx(2 * (P[0] * 0.5 + P[1] * 0.5), rel=1e-14)


def test_router_stats_match_torch_composition_and_ema_closed_form():
    cfg = small_cfg(E=16, k=4, T=64)
    inp = make_inputs(cfg, seed=21)
    st = oracle.router_stats(inp["x"], inp["gate_w"], cfg.top_k)
    logits = f64(inp["x"]) @ f64(inp["gate_w"]).T
    p = torch.softmax(logits, -1)
    _, ti = torch.topk(p, cfg.top_k, -1)
    counts = torch.bincount(ti.reshape(-1), minlength=cfg.E).numpy()
    np.testing.assert_allclose(st["P"], p.mean(0).numpy(), rtol=1e-13)
    np.testing.assert_array_equal(st["counts"], counts)
    assert st["aux"] == pytest.approx(cfg.E * float((p.mean(0).numpy() * counts).sum())
                                      / (cfg.T * cfg.top_k), rel=1e-13)
    # EMA after n identical steps: c_n = m^n c_0 + (1 - m^n) counts
    m, c0 = 0.9, np.linspace(0.0, 5.0, cfg.E)
    ema, tot = c0.copy(), 3.0
    for _ in range(5):
        s2 = oracle.router_stats(inp["x"], inp["gate_w"], cfg.top_k, ema_counts=ema,
                                 ema_total=tot, momentum=m)
        ema, tot = s2["ema_counts"], s2["ema_total"]
    np.testing.assert_allclose(ema, m ** 5 * c0 + (1 - m ** 5) * counts, rtol=1e-12)
    assert tot == pytest.approx(m ** 5 * 3.0 + (1 - m ** 5) * cfg.T, rel=1e-13)


# ---------------------------------------------------------------- FP8 expert weight pins

def _torch_e4m3(v64: torch.Tensor) -> torch.Tensor:
    """Round to E4M3 with torch's float8 conversion (a library routine)."""
    return v64.float().to(torch.float8_e4m3fn).to(torch.float64)


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all() and nan.sum() == 2  # 0x7F, 0xFF
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_torch_rounding():
    g = torch.Generator().manual_seed(5)
    v = torch.cat([torch.randn(4000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 200.0)])
    # exact midpoints between neighbouring codes: ties go to the even code
    mids = torch.tensor([(oracle.e4m3_decode(c) + oracle.e4m3_decode(c + 1)) / 2
                         for c in range(0, 126)], dtype=torch.float64)
    v = torch.cat([v.double(), mids, -mids])
    v = v[v.abs() <= 448.0]  # torch maps out-of-range values to NaN (no saturation)
    got = torch.tensor([oracle.e4m3_decode(oracle.e4m3_encode(float(a))) for a in v],
                       dtype=torch.float64)
    np.testing.assert_array_equal(got.numpy(), _torch_e4m3(v).numpy())
    # saturation: beyond the largest finite value
    assert oracle.e4m3_encode(1000.0) == 0x7E and oracle.e4m3_encode(-449.0) == 0xFE


def test_pow2_scale_closed_form():
    assert oracle.pow2_scale(0.0) == 1.0
    assert oracle.pow2_scale(448.0) == 1.0
    assert oracle.pow2_scale(448.0 * 1.0001) == 2.0
    assert oracle.pow2_scale(1.0) == 2.0 ** -8  # 1/448 -> 2^ceil(-8.8) = 2^-8
    for a in (1e-6, 0.37, 5.0, 1e4):
        s = oracle.pow2_scale(a)
        assert a / s <= 448.0 and a / s > 224.0 and math.log2(s) == round(math.log2(s))


def test_fp8_forward_matches_torch_composition():
    """The FP8 layer against the same steps written with torch float8 rounding
    and float64 matmuls (per-channel power-of-two scales, fixed h scale)."""
    cfg = small_cfg(T=12, H=128, E=4, k=2, I=64, dtype=torch.bfloat16)
    inp = make_inputs(cfg, seed=41)
    q, s_gu, s_d = oracle.quantize_weights_fp8(inp["expert_w"])
    sq, ss_gu, ss_d = oracle.quantize_weights_fp8(inp["shared_w"].unsqueeze(0))
    got = oracle.forward_fp8(inp["x"], inp["gate_w"], q, s_gu, s_d, sq[0], ss_gu[0], ss_d[0],
                             cfg.top_k, cfg.routed_scale, cfg.clip_limit)
    L = cfg.clip_limit

    def p2(a):
        return 2.0 ** math.ceil(math.log2(a / 448.0)) if a > 0 else 1.0

    def q_w(w3):  # [3,I,H] float64 -> dequantized gate, up (row scales), down (col scales)
        g = torch.stack([r / p2(float(r.abs().max())) for r in w3[0]])
        gs = torch.tensor([p2(float(r.abs().max())) for r in w3[0]], dtype=torch.float64)
        u = torch.stack([r / p2(float(r.abs().max())) for r in w3[1]])
        us = torch.tensor([p2(float(r.abs().max())) for r in w3[1]], dtype=torch.float64)
        ds = torch.tensor([p2(float(c.abs().max())) for c in w3[2].T], dtype=torch.float64)
        d = w3[2] / ds
        return _torch_e4m3(g), gs, _torch_e4m3(u), us, _torch_e4m3(d), ds

    s_h = p2(L / (1 + math.exp(-L)) * L)

    def ffn(xq, sx, w3):
        g, gs, u, us, d, ds = q_w(w3)
        gg = torch.clamp((xq @ g.T) * sx * gs, -L, L)
        uu = torch.clamp((xq @ u.T) * sx * us, -L, L)
        hq = _torch_e4m3(F.silu(gg) * uu / s_h)
        return (hq @ d) * s_h * ds

    x64 = f64(inp["x"])
    r = oracle.route(inp["x"], inp["gate_w"], cfg.top_k, cfg.routed_scale)
    assert (got["idx"] == r["idx"]).all()
    for t in range(cfg.T):
        sx = p2(float(x64[t].abs().max()))
        xq = _torch_e4m3(x64[t:t + 1] / sx)
        ref = ffn(xq, sx, f64(inp["shared_w"]))[0]
        for j in range(cfg.top_k):
            ref = ref + r["w"][t, j] * ffn(xq, sx, f64(inp["expert_w"][r["idx"][t, j]]))[0]
        np.testing.assert_allclose(got["out"][t], ref.numpy(), rtol=1e-9, atol=1e-12)


def test_router_inputs_are_the_layer_inputs_draws():
    """make_router_inputs draws exactly the x, gate weight and bias of
    make_inputs (same seeds), without the expert weights."""
    import torch
    from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs, make_router_inputs
    c = MoEConfig("r", T=9, H=64, E=8, top_k=2, I=64, num_shared=1, dtype=torch.bfloat16,
                  x_std=1.0, w_std=0.02, routed_scale=2.827, clip_limit=10.0, skew_bias=True)
    full = make_inputs(c, seed=5)
    r = make_router_inputs(c, seed=5)
    assert torch.equal(full["x"], r["x"]) and torch.equal(full["gate_w"], r["gate_w"])
    assert torch.equal(full["logit_bias"], r["logit_bias"])
