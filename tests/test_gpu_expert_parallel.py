"""The expert-parallel forward with its CUDA steps (CudaKernels).

One GPU is available per run here, so two forms are tested:
- a one-rank NCCL group, where every exchange block is a local copy: the CUDA
  wiring of the staged calls (route, permute, one grouped FFN over the local
  experts, combine) against the oracle;
- two gloo ranks as two processes sharing the GPU, each running the CUDA
  library on its own tokens and half of the experts, the row blocks crossing
  ranks through host memory: CUDA-produced rows go through the real
  exchange, and each rank's output is checked against the oracle's
  single-process layer on that rank's tokens.  No kernel of one process waits
  on the other's (the processes meet only in the host-side exchange), and the
  router runs as two ordinary launches (no cross-CTA wait) while the two
  contexts share the GPU."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from parity_util import forward_parity
from sparse_moe_layer_06_b200 import expert_parallel as ep
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs, make_x

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg(T=300):
    return MoEConfig("ep_gpu", T=T, H=512, E=16, top_k=4, I=384, num_shared=1,
                     dtype=torch.bfloat16, x_std=1.0, w_std=0.02, routed_scale=2.827,
                     clip_limit=10.0)


def test_one_rank_expert_parallel_forward_matches_oracle():
    cfg = _cfg()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=dev)
    try:
        inp = make_inputs(cfg, seed=41, device=dev)
        p = moe.MoEProblem.from_config(cfg)
        kern = ep.CudaKernels(p, cfg.E, dev)
        out, idx, w = ep.ep_forward(inp["x"], inp["gate_w"], inp["logit_bias"],
                                    inp["expert_w"], inp["shared_w"], p, kern)
        torch.cuda.synchronize()
        for ws in kern._ws.values():
            assert moe.moe_read_device_status(ws) == moe.MOE_OK
        forward_parity(inp, cfg, out, idx, w)
    finally:
        dist.destroy_process_group()


def _rank_main(rank, world, port, skew, q):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ["MOE_FUSED_ROUTE"] = "0"  # no cross-CTA wait while two contexts share the GPU
    from parity_util import forward_parity as parity
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        cfg = _cfg(T=200 + 37 * rank)
        wts = make_inputs(cfg.with_tokens(1), seed=43, device=dev)
        x = make_x(cfg, seed=500 + rank, device=dev)
        bias = None
        if skew:
            # most rows go to rank 0's experts: uneven and some empty blocks
            bias = torch.tensor([3.0] * 4 + [1.0] * 4 + [-8.0] * 8, device=dev)
        first, count = ep.local_expert_range(cfg.E, rank, world)
        p = moe.MoEProblem.from_config(cfg)
        kern = ep.CudaKernels(p, count, dev)
        out, idx, w = ep.ep_forward(x, wts["gate_w"], bias, wts["expert_w"][first:first + count],
                                    wts["shared_w"], p, kern)
        torch.cuda.synchronize()
        status = [moe.moe_read_device_status(ws) for ws in kern._ws.values()]
        inp = dict(wts, x=x, logit_bias=bias)
        n_ex, err, scale = parity(inp, cfg, out, idx, w)
        q.put((rank, "ok", status, err, scale))
    except Exception as e:  # reported to the parent
        q.put((rank, repr(e)[:2000], [], 0.0, 0.0))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("skew", [False, True])
def test_two_rank_gloo_expert_parallel_with_cuda_kernels(skew):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, skew, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=300) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    assert len(results) == world
    for rank, msg, status, err, scale in results:
        assert msg == "ok", (rank, msg)
        assert all(s == moe.MOE_OK for s in status), (rank, status)
