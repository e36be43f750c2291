"""Expert-parallel layer forward across the ranks of a process group.

Each rank holds every token row of its own batch, the (replicated) router and
shared-expert weights, and the weights of E / world routed experts: rank r
owns experts [r * E/world, (r+1) * E/world).  Per forward:

  1. route the rank's tokens over all E experts (top-k, weights);
  2. permute the token rows by expert.  Expert-major order is rank-major
     order, so the permuted rows already form one contiguous block per
     destination rank;
  3. exchange the per-expert row counts, then the rows (all-to-all);
  4. run the received rows through the local experts, one grouped call per
     source rank (its rows arrive grouped by local expert);
  5. send the expert outputs back (the inverse all-to-all), so they land in
     the rank's own permuted order;
  6. combine: weighted sum of each token's k rows plus the shared expert.

The exchange is the plain collective form of expert parallelism (the baseline
against which a fused dispatch/combine over peer memory would be measured).
Steps 1, 2, 4 and 6 are calls to the CUDA library through ``CudaKernels``;
only the bookkeeping of row counts lives here.  Splits are read on the host
after the counts exchange.
"""
from __future__ import annotations

from dataclasses import replace

import torch
import torch.distributed as dist

from . import moe


class CudaKernels:
    """The per-rank steps, on this rank's GPU, through the C ABI."""

    def __init__(self, problem: moe.MoEProblem, local_experts: int, device):
        self.p = problem
        self.E_local = local_experts
        self.device = torch.device(device)
        self._ws = {}

    def _workspace(self, key, problem, call, rows=None, groups=None):
        if call == moe.MOE_CALL_FFN:
            n = moe.ffn_workspace_size(problem, rows, groups)
        else:
            n = moe.moe_workspace_size(problem, call)
        ws = self._ws.get(key)
        if ws is None or ws.numel() < n:
            ws = torch.empty(n, dtype=torch.uint8, device=self.device)
            ws[:256].zero_()
            self._ws[key] = ws
        return ws

    def route(self, x, gate_w, bias):
        p = replace(self.p, T=x.shape[0])
        idx = torch.empty(p.T, p.top_k, dtype=torch.int32, device=self.device)
        w = torch.empty(p.T, p.top_k, dtype=torch.float32, device=self.device)
        moe.moe_route(p, x, gate_w, bias, idx, w, self._workspace("route", p, moe.MOE_CALL_ROUTE))
        return idx, w

    def permute(self, idx, x):
        p = replace(self.p, T=x.shape[0])
        offsets = torch.empty(p.E + 1, dtype=torch.int32, device=self.device)
        pos = torch.empty_like(idx)
        src = torch.empty(idx.numel(), dtype=torch.int32, device=self.device)
        x_perm = torch.empty(idx.numel(), p.H, dtype=x.dtype, device=self.device)
        moe.moe_permute(p, idx, x, offsets, pos, src, x_perm,
                        self._workspace("permute", p, moe.MOE_CALL_PERMUTE))
        return offsets, pos, src, x_perm

    def ffn(self, rows, offsets, n_groups, expert_w):
        y = torch.empty_like(rows)
        if rows.shape[0] == 0:
            return y
        p = replace(self.p, T=rows.shape[0], E=max(1, n_groups), top_k=1)
        ws = self._workspace(("ffn", n_groups), p, moe.MOE_CALL_FFN, rows.shape[0], n_groups)
        moe.moe_grouped_swiglu_ffn(p, rows, offsets.to(self.device, torch.int32), n_groups,
                                   expert_w, y, ws)
        return y

    def combine(self, y_perm, pos, w, shared_y):
        p = replace(self.p, T=pos.shape[0])
        out = torch.empty(p.T, p.H, dtype=y_perm.dtype, device=self.device)
        moe.moe_combine(p, y_perm, pos, w, shared_y, out,
                        self._workspace("combine", p, moe.MOE_CALL_COMBINE))
        return out


def local_expert_range(num_experts: int, rank: int, world: int):
    """Experts [first, first + count) owned by `rank` (E divisible by world)."""
    if num_experts % world != 0:
        raise ValueError(f"{num_experts} experts do not split evenly over {world} ranks")
    count = num_experts // world
    return rank * count, count


def ep_forward(x, gate_w, logit_bias, local_expert_w, shared_w, problem: moe.MoEProblem,
               kernels, group=None):
    """The layer forward for this rank's tokens `x` with experts spread over
    the ranks of `group` (see the module docstring).  Returns (out, topk_idx,
    topk_w) for the rank's tokens."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    E = problem.E
    _, E_local = local_expert_range(E, rank, world)
    if local_expert_w.shape[0] != E_local:
        raise ValueError("local_expert_w must hold this rank's E/world experts")
    T, H = x.shape

    idx, w = kernels.route(x, gate_w, logit_bias)
    offsets, pos, _, x_perm = kernels.permute(idx, x)

    # rows per (destination rank, its local expert), then what arrives here
    counts = (offsets[1:] - offsets[:-1]).to(torch.int64).reshape(world, E_local)
    recv_counts = torch.empty_like(counts)
    dist.all_to_all_single(recv_counts, counts.contiguous(), group=group)
    counts_h = counts.cpu()
    recv_h = recv_counts.cpu()
    send_splits = counts_h.sum(1).tolist()
    recv_splits = recv_h.sum(1).tolist()

    recv_x = x_perm.new_empty(int(sum(recv_splits)), H)
    dist.all_to_all_single(recv_x, x_perm, recv_splits, send_splits, group=group)

    # the local experts, one grouped call per source rank's block
    recv_y = torch.empty_like(recv_x)
    start = 0
    for s in range(world):
        n = int(recv_splits[s])
        if n:
            offs = torch.zeros(E_local + 1, dtype=torch.int32)
            offs[1:] = torch.cumsum(recv_h[s], 0).to(torch.int32)
            recv_y[start:start + n] = kernels.ffn(recv_x[start:start + n], offs, E_local,
                                                  local_expert_w)
        start += n

    y_perm = torch.empty_like(x_perm)
    dist.all_to_all_single(y_perm, recv_y, send_splits, recv_splits, group=group)

    shared_y = None
    if shared_w is not None:
        shared_y = kernels.ffn(x, torch.tensor([0, T], dtype=torch.int32), 1,
                               shared_w.unsqueeze(0))
    out = kernels.combine(y_perm, pos, w, shared_y)
    return out, idx, w
