"""Expert-parallel exchange logic (sparse_moe_layer_06_b200.expert_parallel) on
two gloo ranks on CPU.  The per-rank compute steps (route, permute, grouped
expert FFN, combine) are the oracle's, so the test checks exactly what the
module adds: the row counts, the block layout (each receiver gets its rows
expert-major: local expert, then source rank), the point-to-point exchange of
the blocks and the inverse exchange.  Each rank's output must equal the oracle's
single-process layer on that rank's tokens with all experts."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleKernels:
    """The four per-rank steps, computed by the oracle (test only)."""

    def __init__(self, cfg, shared_w):
        self.cfg = cfg
        self.shared_w = shared_w

    def route(self, x, gate_w, bias):
        import oracle
        r = oracle.route(x, gate_w, self.cfg.top_k, self.cfg.routed_scale, logit_bias=bias)
        return torch.from_numpy(r["idx"]), torch.from_numpy(r["w"])

    def permute(self, idx, x):
        import oracle
        d = oracle.permute(idx.numpy(), self.cfg.E)
        src = torch.from_numpy(d["src"]).long()
        return (torch.from_numpy(d["offsets"]), torch.from_numpy(d["pos"]), src, x[src])

    def ffn(self, rows, offsets, n_groups, expert_w):
        import oracle
        offs = offsets.numpy().astype(np.int64)
        row_expert = np.zeros(rows.shape[0], np.int32)
        for g in range(n_groups):
            row_expert[offs[g]:offs[g + 1]] = g
        y = oracle.expert_rows(rows.contiguous(), expert_w, self.shared_w,
                               np.arange(rows.shape[0], dtype=np.int32), row_expert,
                               self.cfg.clip_limit)
        return torch.from_numpy(y).to(rows.dtype)

    def combine(self, y_perm, pos, w, shared_y):
        import oracle
        out = oracle.combine(y_perm.double().numpy(), pos.numpy(), w.double().numpy(),
                             None if shared_y is None else shared_y.double().numpy())
        return torch.from_numpy(out)


def _rank_main(rank, world, port, skew, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import oracle
    from sparse_moe_layer_06_b200 import expert_parallel as ep
    from sparse_moe_layer_06_b200 import moe
    from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs, make_x
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = MoEConfig("ep", T=37 + 11 * rank, H=64, E=8, top_k=2, I=64, num_shared=1,
                        dtype=torch.float32, x_std=1.0, w_std=0.05, routed_scale=2.827,
                        clip_limit=10.0)
        w = make_inputs(cfg.with_tokens(1), seed=3)
        x = make_x(cfg, seed=100 + rank)
        bias = None
        if skew:
            # most rows go to rank 0's experts; some source/destination blocks are empty
            bias = torch.tensor([4.0, 3.0, 2.0, 1.0, -6.0, -6.0, -6.0, -6.0])
        first, count = ep.local_expert_range(cfg.E, rank, world)
        p = moe.MoEProblem.from_config(cfg)
        kern = OracleKernels(cfg, w["shared_w"])
        out, idx, wt = ep.ep_forward(x, w["gate_w"], bias, w["expert_w"][first:first + count],
                                     w["shared_w"], p, kern)
        ref = oracle.forward(x, w["gate_w"], w["expert_w"], w["shared_w"], cfg.top_k,
                             cfg.routed_scale, cfg.clip_limit, logit_bias=bias)
        err = float(np.max(np.abs(out.double().numpy() - ref["out"])))
        scale = float(np.max(np.abs(ref["out"])))
        same_idx = bool(np.array_equal(idx.numpy(), ref["idx"]))
        q.put((rank, err, scale, same_idx))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("skew", [False, True])
def test_two_rank_expert_parallel_matches_single_process_oracle(skew):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, skew, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert len(results) == world
    for rank, err, scale, same_idx in results:
        assert same_idx, rank
        # rows cross the exchange as fp32: relative rounding of the expert outputs
        assert err <= 1e-5 * scale, (rank, err, scale)


def test_local_expert_range():
    from sparse_moe_layer_06_b200.expert_parallel import local_expert_range
    assert local_expert_range(256, 3, 8) == (96, 32)
    with pytest.raises(ValueError):
        local_expert_range(10, 0, 4)


def test_exchange_layout_expert_major():
    from sparse_moe_layer_06_b200.expert_parallel import exchange_layout
    send = [[2, 0, 1], [3, 4, 0]]          # to rank 0: experts 0..2; to rank 1: 0..2
    recv = [[1, 5, 0], [2, 0, 7]]          # from rank 0 / rank 1 for my experts 0..2
    send_off, recv_off, group_off = exchange_layout(send, recv)
    assert send_off == [[0, 2, 2], [3, 6, 10]]          # destination-major, consecutive
    # expert-major receive buffer: e0 (s0: 1, s1: 2), e1 (s0: 5, s1: 0), e2 (s0: 0, s1: 7)
    assert recv_off == [[0, 3, 8], [1, 8, 8]]
    assert group_off == [0, 3, 8, 15]
