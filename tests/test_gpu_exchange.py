"""The sequence-parallel exchange on the GPU path: libcf codecs, NCCL
all-gather on a communication stream.  The test runs a world of one rank on
one GPU (the collective degenerates to a copy); the multi-rank host logic is
covered on the CPU by test_exchange.py."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("mode,kw", [("q2", {}), ("sign1", {}),
                                     ("blocksel", {"bs_grid_h": 16, "bs_block": 8, "bs_k": 1, "bs_warm": 2})])
def test_single_rank_exchange_on_nccl(mode, kw):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    from activation_residual_compression_b200.exchange import SPExchange
    ex = SPExchange(256, 512, mode, n_tensors=2, **kw)
    try:
        g = torch.Generator(device="cuda").manual_seed(3)
        a = [torch.randn(256, 512, generator=g, device="cuda").to(torch.bfloat16) for _ in range(2)]
        for t in range(5):
            shards = [(x.float() + 0.1 * t).to(torch.bfloat16) for x in a]
            outs = ex.step(shards)
            torch.cuda.synchronize()
            for i in range(2):
                assert outs[i].shape == (1, 256, 512)
                assert torch.equal(outs[i][0], shards[i])
        assert ex.status() == 0
    finally:
        ex.close()
        dist.destroy_process_group()
