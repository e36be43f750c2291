"""The multi-process (one rank per GPU) host logic of bench.py, run as two
gloo ranks on CPU: per-rank token seeds with shared weights, max-over-ranks
timing, and the whole-job rate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs, make_x
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = MoEConfig("t", T=8, H=64, E=4, top_k=2, I=64, num_shared=1,
                        dtype=torch.float32, x_std=1.0, w_std=0.02, routed_scale=2.827,
                        clip_limit=10.0)
        w = make_inputs(cfg.with_tokens(1), seed=0)
        x = make_x(cfg, seed=bench.rank_token_seed(rank))
        # gather the per-rank tensors on rank 0 for comparison
        ws = [torch.zeros_like(w["expert_w"]) for _ in range(world)]
        xs = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(ws, w["expert_w"])
        dist.all_gather(xs, x)
        slowest = bench.max_over_ranks(10.0 + rank, dist)
        rate = bench.whole_job_rate(cfg.T, world, slowest / 1e3)
        q.put((rank, slowest, rate, bool(torch.equal(ws[0], ws[1])),
               bool(torch.equal(xs[0], xs[1]))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_weights_and_reduce_max():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, rate, same_w, same_x in results:
        assert slowest == 11.0            # the max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 8 / 0.011)
        assert same_w                     # every replica holds the same weights
        assert not same_x                 # and its own token batch


def test_single_process_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_token_seed(0) != bench.rank_token_seed(1)
    assert bench.whole_job_rate(4096, 1, 0.004) == pytest.approx(1.024e6)
