"""The sequence-parallel exchange on the GPU path.

* Two ranks as two processes sharing the one GPU, on a gloo group (payloads
  staged through host memory): every rank's libcf receivers decode the peer's
  payloads, and each peer's reconstructed shard is checked bit for bit against
  an oracle replay of that peer's seeded stream -- 1-bit, 2-bit, N:M and block
  selection, two tensors per step, warm-up steps included.  The two processes'
  kernels never wait on each other (the only exchange is on the host).
* A world of one rank on NCCL, all-gather on a communication stream (the
  collective degenerates to a copy).
The multi-rank host logic is also covered on the CPU by test_exchange.py."""
import datetime
import os
import queue
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

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


ROWS, COLS, STEPS = 64, 128, 8
GPU_CASES = [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}), ("nm", {"nm_n": 2, "nm_m": 16}),
             ("blocksel", {"bs_grid_h": 8, "bs_block": 4, "bs_k": 1, "bs_warm": 3})]


def _shard(rank, tensor, t):
    g = torch.Generator().manual_seed(1000 * rank + 17 * tensor)
    base = torch.randn(ROWS, COLS, generator=g)
    walk = torch.zeros(ROWS, COLS)
    for _ in range(t + 1):
        walk += 0.1 * torch.randn(ROWS, COLS, generator=g)
    return (base + walk).to(torch.bfloat16)


def _gpu_worker(rank, world, port, mode, kw, q):
    try:
        torch.cuda.set_device(0)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
        from activation_residual_compression_b200.exchange import SPExchange
        from test_exchange import OracleCodec
        ex = SPExchange(ROWS, COLS, mode, n_tensors=2, device="cuda:0", **kw)   # libcf codecs
        assert ex.host_staged
        replay = {(p, i): (OracleCodec(ROWS, COLS, mode, 0, **kw), OracleCodec(ROWS, COLS, mode, 1, **kw))
                  for p in range(world) if p != rank for i in range(2)}
        for t in range(STEPS):
            shards = [_shard(rank, i, t).cuda() for i in range(2)]
            outs = ex.step(shards)
            torch.cuda.synchronize()
            for i in range(2):
                got = outs[i].cpu()
                assert torch.equal(got[rank], shards[i].cpu())
                for p in range(world):
                    if p == rank:
                        continue
                    s, r = replay[(p, i)]
                    P = s.payload_bytes(s.next_is_warm())
                    buf = torch.empty(P, dtype=torch.uint8)
                    s.encode(_shard(p, i, t), buf)
                    rec = torch.empty(ROWS, COLS, dtype=torch.bfloat16)
                    r.decode(buf, rec)
                    a = got[p].view(torch.int16).numpy()
                    b = rec.view(torch.int16).numpy()
                    assert np.array_equal(a, b), (rank, p, i, t, int((a != b).sum()))
        assert ex.status() == 0
        ex.close()
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except BaseException as e:  # report to the parent instead of hanging it
        q.put((rank, repr(e)))


@pytest.mark.parametrize("mode,kw", GPU_CASES)
def test_two_ranks_on_one_gpu_decode_peers_bit_exactly(mode, kw):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gpu_worker, args=(r, 2, port, mode, kw, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        # the first rank that fails reports at once; its peer may then wait in
        # a collective until its group timeout, so stop collecting there
        while len(results) < len(procs):
            try:
                r, msg = q.get(timeout=300)
            except queue.Empty:
                pytest.fail(f"no report from a rank within 300 s; reports so far: {results}")
            results[r] = msg
            if msg != "ok":
                break
    finally:
        ok = len(results) == len(procs) and all(v == "ok" for v in results.values())
        for p in procs:
            p.join(timeout=60 if ok else 5)
            if p.is_alive():
                p.kill()
    assert results == {0: "ok", 1: "ok"}, results
