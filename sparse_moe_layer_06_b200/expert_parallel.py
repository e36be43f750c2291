"""Expert-parallel layer forward across the ranks of a process group.

Each rank holds every token row of its own batch, the (replicated) router and
shared-expert weights, and the weights of E / world routed experts: rank r
owns experts [r * E/world, (r+1) * E/world).  Per forward:

  1. route the rank's tokens over all E experts (top-k, weights);
  2. permute the token rows by expert.  Expert-major order is rank-major
     order, so the rows for each (destination rank, its local expert) form one
     contiguous block;
  3. exchange the per-(destination, local expert) row counts and copy them to
     pinned host memory without waiting;
  4. launch the shared expert on the rank's own tokens.  The host waits for
     the counts (the one host synchronisation of the step) while the GPU runs
     it;
  5. exchange the rows, one point-to-point transfer per (source, destination,
     local expert) block, each received straight into its place in
     expert-major order (local expert, then source rank);
  6. run all received rows through the local experts in ONE grouped call;
  7. send each output block back to its source, where it lands in the source's
     own permuted order;
  8. combine: weighted sum of each token's k rows plus the shared expert.

Steps 1, 2, 4, 6 and 8 are calls to the CUDA library through ``CudaKernels``.
The exchanges are the communication library's (NCCL point-to-point on GPUs);
on a gloo group the blocks are staged through host memory, which is how the
exchange is tested when only one GPU is available.  This is the plain
collective form of expert parallelism, the baseline a fused dispatch/combine
over peer memory would be measured against.  Deployment context: page "1M上下
文实战：Hy4 preview如何从容处理百万token级长文档", section "最快部署 1M 上下文"
(FP8 weights, 8-card parallel serving).
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


def exchange_layout(send_counts, recv_counts):
    """Block offsets of the row exchange, from host integer tables.

    send_counts[d][e]: rows this rank sends to rank d for d's local expert e
    (consecutive in this rank's permuted order, destination-major);
    recv_counts[s][e]: rows it receives from rank s for its own local expert e.
    Returns (send_off[d][e], recv_off[s][e], group_off[e]): where each sent
    block starts in the permuted rows, where each received block starts in
    the expert-major receive buffer (local expert, then source rank), and the
    local experts' row offsets in that buffer (n_local + 1 entries)."""
    world = len(send_counts)
    n_local = len(send_counts[0]) if world else 0
    send_off, run = [], 0
    for d in range(world):
        row = []
        for e in range(n_local):
            row.append(run)
            run += int(send_counts[d][e])
        send_off.append(row)
    recv_off = [[0] * n_local for _ in range(world)]
    group_off, run = [0], 0
    for e in range(n_local):
        for s in range(world):
            recv_off[s][e] = run
            run += int(recv_counts[s][e])
        group_off.append(run)
    return send_off, recv_off, group_off


def _global_rank(group, r):
    return r if group is None else dist.get_global_rank(group, r)


def _exchange_blocks(src, src_blocks, dst, dst_blocks, group):
    """Point-to-point transfer of row blocks: src_blocks / dst_blocks are
    [(peer, local expert, start row, rows)] in the order both sides post them
    (peer, then local expert).  Blocks to and from this rank itself are local
    copies.  On a gloo group, CUDA rows are staged through host memory."""
    me = dist.get_rank(group)
    host = dist.get_backend(group) == "gloo" and src.is_cuda
    s_buf = src.cpu() if host else src
    d_buf = torch.empty(dst.shape, dtype=dst.dtype) if host else dst
    own_src = [(e, a, n) for p, e, a, n in src_blocks if p == me and n]
    own_dst = [(e, a, n) for p, e, a, n in dst_blocks if p == me and n]
    for (e0, a, n), (e1, b, m) in zip(own_src, own_dst):
        assert e0 == e1 and n == m
        d_buf[b:b + m].copy_(s_buf[a:a + n])
    sends = [(p, e, s_buf[a:a + n]) for p, e, a, n in src_blocks if p != me and n]
    recvs = [(p, e, d_buf[a:a + n]) for p, e, a, n in dst_blocks if p != me and n]
    if dist.get_backend(group) == "nccl":
        ops = [dist.P2POp(dist.isend, t, _global_rank(group, p), group) for p, _, t in sends]
        ops += [dist.P2POp(dist.irecv, t, _global_rank(group, p), group) for p, _, t in recvs]
        reqs = dist.batch_isend_irecv(ops) if ops else []
    else:
        # tag = local expert: the blocks between one pair of ranks match by tag
        reqs = [dist.isend(t, _global_rank(group, p), group=group, tag=e) for p, e, t in sends]
        reqs += [dist.irecv(t, _global_rank(group, p), group=group, tag=e) for p, e, t in recvs]
    for r in reqs:
        r.wait()
    if host:
        dst.copy_(d_buf)


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
    on_gpu = x.is_cuda

    idx, w = kernels.route(x, gate_w, logit_bias)
    offsets, pos, _, x_perm = kernels.permute(idx, x)

    # rows per (destination rank, its local expert), and what arrives here
    counts = (offsets[1:] - offsets[:-1]).to(torch.int64).reshape(world, E_local).contiguous()
    if dist.get_backend(group) == "nccl":
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts, group=group)
        both = torch.stack([counts, recv_counts])
    else:
        both = counts
    # start the copy of the counts to the host, launch the shared expert (its
    # GPU time covers the host's wait), then wait for the counts
    both_h = torch.empty(both.shape, dtype=both.dtype, pin_memory=on_gpu)
    both_h.copy_(both, non_blocking=on_gpu)
    ready = None
    if on_gpu:
        ready = torch.cuda.Event()
        ready.record()
    shared_y = None
    if shared_w is not None:
        shared_y = kernels.ffn(x, torch.tensor([0, T], dtype=torch.int32), 1,
                               shared_w.unsqueeze(0))
    if ready is not None:
        ready.synchronize()
    if dist.get_backend(group) == "nccl":
        send_h, recv_h = both_h[0], both_h[1]
    else:
        send_h = both_h
        recv_h = torch.empty_like(send_h)
        dist.all_to_all_single(recv_h, send_h, group=group)
    send_c, recv_c = send_h.tolist(), recv_h.tolist()
    send_off, recv_off, group_off = exchange_layout(send_c, recv_c)

    # rows out, received in expert-major order
    fwd_src = [(d, e, send_off[d][e], send_c[d][e]) for d in range(world) for e in range(E_local)]
    fwd_dst = [(s, e, recv_off[s][e], recv_c[s][e]) for s in range(world) for e in range(E_local)]
    recv_x = x_perm.new_empty(group_off[-1], H)
    _exchange_blocks(x_perm, fwd_src, recv_x, fwd_dst, group)

    # every local expert in one grouped call
    if group_off[-1]:
        recv_y = kernels.ffn(recv_x, torch.tensor(group_off, dtype=torch.int32), E_local,
                             local_expert_w)
    else:
        recv_y = torch.empty_like(recv_x)

    # outputs back to their sources, into the sources' permuted order
    y_perm = torch.empty_like(x_perm)
    _exchange_blocks(recv_y, fwd_dst, y_perm, fwd_src, group)

    out = kernels.combine(y_perm, pos, w, shared_y)
    return out, idx, w
