"""Host logic of the sequence-parallel payload exchange
(``activation_residual_compression_b200.exchange``), on CPU with two and three gloo ranks.

The exchange is codec-agnostic; here each rank drives it with the CPU oracle
as the codec (test infrastructure), so no GPU is needed.  Every rank checks
that the reconstruction it received for each peer's shard is bit-identical
to an independent replay of that peer's seeded stream through a local
sender/receiver pair, and that its own slot is its exact shard -- for two
tensors per step, warm-up steps included -- and that a payload corrupted in
transit is reported by the receiving rank's status.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROWS, COLS, STEPS = 64, 64, 9
CASES = [("q2", {}), ("blocksel", {"bs_grid_h": 8, "bs_block": 4, "bs_k": 1, "bs_warm": 3})]


class OracleCodec:
    """The exchange's codec interface over the CPU oracle (one role used)."""

    def __init__(self, rows, cols, mode, role, **params):
        import oracle
        kw = dict(params)
        if "bs_grid_h" in kw:
            kw["bs_h"] = kw.pop("bs_grid_h")
        self.o = oracle.Oracle(rows, cols, mode, dtype="bf16", **kw)
        self.kw = kw
        self.role = role

    def payload_bytes(self, warm):
        return self.o.payload_bytes(warm)

    def next_is_warm(self):
        return self.o.next_is_warm(receiver=False)

    def encode(self, a, payload, stream=None):
        p = self.o.encode(a.view(torch.int16).numpy().view(np.uint16))
        payload.copy_(torch.from_numpy(p))

    def decode(self, payload, recon, stream=None):
        r, st = self.o.decode(payload.numpy())
        assert st == 0
        recon.copy_(torch.from_numpy(r.reshape(recon.shape).view(np.int16)).view(torch.bfloat16))

    def status(self, stream=None):
        return self.o.status()

    def reset(self):
        import oracle
        o = self.o
        self.o = oracle.Oracle(o.rows, o.cols, o.mode, dtype="bf16", **self.kw)

    def close(self):
        pass


def _shard(rank, tensor, t):
    g = torch.Generator().manual_seed(1000 * rank + 17 * tensor)
    base = torch.randn(ROWS, COLS, generator=g)
    walk = torch.zeros(ROWS, COLS)
    for _ in range(t + 1):
        walk += 0.1 * torch.randn(ROWS, COLS, generator=g)
    return (base + walk).to(torch.bfloat16)


def _worker(rank, world, port, mode, kw, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        from activation_residual_compression_b200.exchange import SPExchange
        ex = SPExchange(ROWS, COLS, mode, n_tensors=2, device="cpu", codec_factory=OracleCodec, **kw)
        # independent replay of every peer's stream: a local sender/receiver pair per (peer, tensor)
        replay = {(p, i): (OracleCodec(ROWS, COLS, mode, 0, **kw), OracleCodec(ROWS, COLS, mode, 1, **kw))
                  for p in range(world) if p != rank for i in range(2)}
        for t in range(STEPS):
            shards = [_shard(rank, i, t) for i in range(2)]
            outs = ex.step(shards)
            for i in range(2):
                assert torch.equal(outs[i][rank], shards[i])
                for p in range(world):
                    if p == rank:
                        continue
                    s, r = replay[(p, i)]
                    a = _shard(p, i, t)
                    P = s.payload_bytes(s.next_is_warm())
                    buf = torch.empty(P, dtype=torch.uint8)
                    s.encode(a, buf)
                    rec = torch.empty(ROWS, COLS, dtype=torch.bfloat16)
                    r.decode(buf, rec)
                    assert torch.equal(outs[i][p], rec), (rank, p, i, t)
        assert ex.status() == 0
        ex.close()
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except BaseException as e:  # report to the parent instead of hanging it
        q.put((rank, repr(e)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(world, mode, kw):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, kw, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert results == {r: "ok" for r in range(world)}, results


@pytest.mark.parametrize("mode,kw", CASES)
def test_two_rank_exchange_matches_independent_replay(mode, kw):
    _run(2, mode, kw)


def test_three_rank_exchange_matches_independent_replay():
    """An odd world: every rank receives two peers' shards per tensor."""
    _run(3, "sign1", {})


T_FAULT = 4


class CorruptingCodec(OracleCodec):
    """Rank 1's sender flips a byte of the payload header at step T_FAULT (a
    host-made fault in transit); receivers record the decode status instead of
    asserting it."""

    rank = 0

    def __init__(self, *a, **kw):
        super().__init__(*a, **kw)
        self.t = 0
        self.statuses = []

    def encode(self, a, payload, stream=None):
        super().encode(a, payload, stream)
        if self.rank == 1 and self.t == T_FAULT:
            payload[0] ^= 0x5A
        self.t += 1

    def decode(self, payload, recon, stream=None):
        r, st = self.o.decode(payload.numpy())
        self.statuses.append(st)
        if st == 0:
            recon.copy_(torch.from_numpy(r.reshape(recon.shape).view(np.int16)).view(torch.bfloat16))


def _fault_worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        from activation_residual_compression_b200.exchange import SPExchange
        CorruptingCodec.rank = rank
        ex = SPExchange(ROWS, COLS, "q2", n_tensors=1, device="cpu", codec_factory=CorruptingCodec)
        seen = []
        for t in range(STEPS):
            ex.step([_shard(rank, 0, t)])
            seen.append(ex.status())
        rx = ex.channels[0].receivers
        per_step = {p: c.statuses for p, c in rx.items()}
        ex.close()
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, (seen, per_step)))
    except BaseException as e:  # report to the parent instead of hanging it
        q.put((rank, repr(e)))


def test_corrupted_payload_is_reported_by_the_receiving_rank_only():
    """A payload whose header was altered in transit fails that step's decode
    on the receiving rank (the receiver keeps its state) and sets its status,
    which stays set: later payloads decode, but the exchange's status reports
    the desync at every following step.  The sending rank sees nothing."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fault_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert all(isinstance(v, tuple) for v in results.values()), results
    seen0, dec0 = results[0]
    seen1, dec1 = results[1]
    assert dec0 == {1: [0] * T_FAULT + [1] + [0] * (STEPS - T_FAULT - 1)}, dec0
    assert seen0[:T_FAULT] == [0] * T_FAULT
    assert all(st != 0 for st in seen0[T_FAULT:]), seen0
    assert seen1 == [0] * STEPS and dec1 == {0: [0] * STEPS}


def _bench_worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import bench
        from activation_residual_compression_b200.exchange import SPExchange
        ex = SPExchange(ROWS, COLS, "q2", n_tensors=2, device="cpu", codec_factory=OracleCodec)
        res = bench.exchange_bench(ex, lambda t: [_shard(rank, i, t) for i in range(2)], 4, 3, "cpu")
        # the exchange still works after the bench's resets: a fresh request decodes every peer exactly
        outs = ex.step([_shard(rank, i, 0) for i in range(2)])
        for i in range(2):
            for p in range(world):
                assert torch.equal(outs[i][p], _shard(p, i, 0))      # warm-up step: raw activations
        ex.close()
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, res))
    except BaseException as e:  # report to the parent instead of hanging it
        q.put((rank, repr(e)))


def test_exchange_bench_on_two_gloo_ranks():
    """bench.py's exchange timing (the --exchange leg) on two CPU ranks with the
    oracle as the codec: it runs, agrees across ranks (times are maxima over
    ranks), reports positive step and codec times, no error status, and leaves
    the exchange usable."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert all(isinstance(v, dict) for v in results.values()), results
    r0, r1 = results[0], results[1]
    assert r0["ms_per_step"] == r1["ms_per_step"] and r0["codec_ms_per_step"] == r1["codec_ms_per_step"]
    assert r0["ms_per_step"] > 0 and r0["codec_ms_per_step"] > 0 and r0["status"] == 0
    assert r0["activation_gbs_per_rank"] > 0
    assert r0["payload_bytes_per_tensor"] == 64 + 16 * ((ROWS * 2 + 15) // 16) + ROWS * COLS // 4
