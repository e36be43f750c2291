"""Shared helpers for the GPU parity tests: run the oracle on the same seeded
inputs and compare (routing with the near-tie rule, outputs with the stated
tolerance).  Expected values come only from ``oracle``."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# bf16 storage with fp32 accumulation: max|gpu - oracle| <= 2e-2 * max|oracle|
OUT_TOL = 2e-2
# fp32 problems: the expert GEMMs read fp32 operands as TF32 (10 explicit
# mantissa bits against bf16's 8, a unit roundoff 4x smaller) with fp32 sums
# and fp32 h and output rows: the same arithmetic with every operand rounding
# 4x finer, so the bound is a quarter of the bf16 one
F32_OUT_TOL = 5e-3
# Routing weights: w_j = scale * softmax(selected logits)_j, so a logit error
# dl gives a relative weight error of at most 2*max|dl|.  The kernel's logits
# are fp32 tensor-core sums of exact bf16 products over 8 K-slices of H/8,
# added in slice order; over every token of the five named workloads the
# largest weight error measured is 7.4e-6 (the skewed batch, whose logit bias
# makes the logits largest), 1.0e-6 or less elsewhere, so weights are checked
# to 1e-5 relative (the stated acceptance bound).  Near-tie band between the
# k-th and (k+1)-th probability: 1e-5 relative (the stated routing rule).
W_RTOL = 1e-5
TIE_REL = 1e-5


def to_cpu_inputs(inp: dict) -> dict:
    return {k: (v.detach().cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def check_routing(gpu_idx: np.ndarray, gpu_w: np.ndarray, orc: dict, k: int):
    """Compare GPU top-k (indices, weights) with the oracle's route output.

    Returns the list of row numbers exempted as near-ties (their GPU set must
    be one of the oracle's own valid alternatives).  Raises AssertionError on
    any other difference.
    """
    exempt = []
    n = gpu_idx.shape[0]
    for r in range(n):
        gi = [int(e) for e in gpu_idx[r]]
        oi = [int(e) for e in orc["idx"][r]]
        p = orc["probs"][r]
        assert len(set(gi)) == k, f"row {r}: repeated experts {gi}"
        if set(gi) != set(oi):
            alts = oracle.near_tie_alternatives(p, k, TIE_REL)
            assert tuple(sorted(gi)) in alts, (
                f"row {r}: GPU experts {gi} vs oracle {oi} (not a near-tie)")
            exempt.append(r)
            continue
        # order: descending probability, up to near-ties
        for a, b in zip(gi, gi[1:]):
            assert p[a] >= p[b] * (1 - TIE_REL), f"row {r}: order {gi}"
        # weights, matched by expert
        ow = {int(e): float(w) for e, w in zip(orc["idx"][r], orc["w"][r])}
        for e, w in zip(gi, gpu_w[r]):
            assert abs(float(w) - ow[e]) <= W_RTOL * abs(ow[e]) + 1e-7, (
                f"row {r}: weight of expert {e}: gpu {w} oracle {ow[e]}")
    return exempt


def assert_close_out(gpu: np.ndarray, ref: np.ndarray, what: str, tol: float = OUT_TOL):
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(gpu.astype(np.float64) - ref))) if ref.size else 0.0
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    assert err <= tol * scale, f"{what}: max err {err:.3e} > {tol} * {scale:.3e}"
    return err, scale


def out_tol(cfg) -> float:
    """Output tolerance of a problem: F32_OUT_TOL for fp32 problems (TF32
    tensor-core operands), OUT_TOL for bf16 ones."""
    return F32_OUT_TOL if cfg.dtype == torch.float32 else OUT_TOL


def forward_parity(inp: dict, cfg, gpu_out: torch.Tensor, gpu_idx: torch.Tensor,
                   gpu_w: torch.Tensor, tokens=None, cpu_inp: dict | None = None):
    """Check a GPU forward (out, idx, w) against the oracle on `tokens`
    (all by default), to out_tol(cfg).  Returns (n_exempt, err, scale)."""
    c = cpu_inp or to_cpu_inputs(inp)
    T = cfg.T
    tok = list(range(T)) if tokens is None else list(tokens)
    orc_route = oracle.route(c["x"], c["gate_w"], cfg.top_k, cfg.routed_scale,
                             logit_bias=c["logit_bias"], tokens=tok)
    gi = gpu_idx.cpu().numpy()[tok]
    gw = gpu_w.cpu().numpy()[tok]
    exempt = check_routing(gi, gw, orc_route, cfg.top_k)
    exempt_set = set(exempt)
    ref = oracle.forward(c["x"], c["gate_w"], c["expert_w"], c["shared_w"], cfg.top_k,
                         cfg.routed_scale, cfg.clip_limit, logit_bias=c["logit_bias"],
                         tokens=tok)
    out = gpu_out.float().cpu().numpy()[tok]
    keep = [i for i in range(len(tok)) if i not in exempt_set]
    err, scale = assert_close_out(out[keep], ref["out"][keep], f"{cfg.name} forward", out_tol(cfg))
    if exempt:
        # near-tie rows: the oracle evaluates the GPU's (validated) alternative set
        forced = np.stack([gi[i] for i in exempt]).astype(np.int32)
        ref2 = oracle.forward(c["x"], c["gate_w"], c["expert_w"], c["shared_w"], cfg.top_k,
                              cfg.routed_scale, cfg.clip_limit, logit_bias=c["logit_bias"],
                              tokens=[tok[i] for i in exempt], forced_idx=forced)
        assert_close_out(out[exempt], ref2["out"], f"{cfg.name} near-tie rows", out_tol(cfg))
    return len(exempt), err, scale


def chunk_bounds(rows: int, width: int):
    """[first, last] row of every token chunk of a segment of `rows` rows cut
    for tile width `width` (the rule moe_expert_tile_rows documents:
    c = ceil(rows / width) chunks of ceil16(ceil(rows / c)) rows)."""
    if rows <= 0:
        return []
    c = -(-rows // width)
    cl = (-(-rows // c) + 15) // 16 * 16
    return [(i * cl, min(rows, (i + 1) * cl) - 1) for i in range(c)]


def schedule_cover_tokens(idx: np.ndarray, E: int, num_shared: int, widths):
    """Tokens whose output rows cover every token tile of the expert GEMMs.

    The permuted rows of expert e are the tokens routed to it in ascending
    order (the dispatch orders rows by expert, then token); the shared
    expert's rows are all T tokens in order.  For each tile width in `widths`
    (gate/up and down), every chunk of every segment contributes its first and
    last row's token.  Checking a token's full output row covers all weight
    blocks of the tiles its rows belong to.  Returns (sorted tokens,
    {width: number of tiles}) -- every tile has at least one checked row."""
    T = idx.shape[0]
    by_expert = [[] for _ in range(E)]
    for t in range(T):
        for e in idx[t]:
            by_expert[int(e)].append(t)
    segments = by_expert + ([list(range(T))] if num_shared else [])
    chosen, tiles = set(), {}
    for width in set(widths):
        n_tiles = 0
        for rows in segments:
            for first, last in chunk_bounds(len(rows), width):
                chosen.add(rows[first])
                chosen.add(rows[last])
                n_tiles += 1
        tiles[width] = n_tiles
    return sorted(chosen), tiles
