"""The expert-parallel forward with its CUDA steps (CudaKernels) on one GPU, as
a one-rank NCCL group: every exchange is then a copy, so the result checks the
CUDA wiring of the staged calls (route, permute, grouped FFN per source block,
combine) against the oracle.  The cross-rank exchange itself is covered by the
two-rank gloo test on CPU; every GPU run available here has one GPU."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

from parity_util import forward_parity
from sparse_moe_layer_06_b200 import expert_parallel as ep
from sparse_moe_layer_06_b200 import moe
from sparse_moe_layer_06_b200.workloads import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_expert_parallel_forward_matches_oracle():
    cfg = MoEConfig("ep_gpu", T=300, H=512, E=16, top_k=4, I=384, num_shared=1,
                    dtype=torch.bfloat16, x_std=1.0, w_std=0.02, routed_scale=2.827,
                    clip_limit=10.0)
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
