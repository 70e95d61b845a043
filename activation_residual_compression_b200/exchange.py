"""Sequence-parallel payload exchange (the communication layer the compressor
plugs into: "Overall framework" -- the method wraps the collective, each device
transmits its compressed residual and the receivers rebuild the activation;
"Key design: system co-design" -- compression overlaps communication).

Every rank owns one token shard of each exchanged tensor (rows x cols, the
same shape on every rank).  Per step and tensor:

1. the rank's sender state encodes its shard into a packed payload
   (libcf kernels, on the compute stream);
2. the payloads of all ranks are gathered with one ``all_gather_into_tensor``
   (NCCL over NVLink on GPUs) issued on a separate communication stream as
   soon as that tensor's encode has finished, so the gather of tensor i runs
   while tensors i+1, ... are being encoded;
3. one receiver state per peer decodes that peer's payload (libcf kernels,
   compute stream, after the gather) into the peer's slot of the output; the
   rank's own slot is its exact shard.

The host logic (payload sizes, warm-up steps, ordering, per-peer states) is
independent of the codec: ``codec_factory`` builds the per-tensor codec; the
default is the CUDA library (``CfCodec``).  Payloads travel as uint8 tensors;
no TMA multicast or peer-memory loads are involved (NCCL moves the bytes).
On a group whose backend cannot gather device tensors (gloo), device payloads
are staged through host memory: copied to the host, gathered there, and
copied back before the peers' decodes (a synchronous transport, used when
several ranks share one GPU or have no NVLink path).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import _cf as cf


class CfCodec:
    """One sender or receiver state of libcf for a (rows, cols) tensor."""

    def __init__(self, rows, cols, mode, role, dtype=cf.CF_BF16, **params):
        self.rows, self.cols = int(rows), int(cols)
        self.h = cf.cf_create(rows, cols, cf.MODE_NAMES[mode] if isinstance(mode, str) else mode,
                              cf.cf_params_init(role=role, dtype=dtype, **params))
        # leading steps whose payload is the raw activation
        self.warm_steps = int(params.get("bs_warm", 5)) if mode == "blocksel" else 1

    def payload_bytes(self, warm: bool) -> int:
        return cf.cf_payload_bytes(self.h, warm)

    def next_is_warm(self) -> bool:
        """The next payload is a full-size warm-up payload."""
        return cf.cf_step(self.h) < self.warm_steps

    def encode(self, a: torch.Tensor, payload: torch.Tensor, stream=None):
        cf.cf_encode(self.h, a, payload, stream)

    def decode(self, payload: torch.Tensor, recon: torch.Tensor, stream=None):
        cf.cf_decode(self.h, payload, recon, stream)

    def status(self, stream=None) -> int:
        return cf.cf_status(self.h, stream)

    def reset(self):
        """New request: the next call is the warm-up step again."""
        cf.cf_reset(self.h)

    def close(self):
        if self.h is not None:
            cf.cf_destroy(self.h)
            self.h = None


def cf_codec_factory(rows, cols, mode, role, **params):
    return CfCodec(rows, cols, mode, role, **params)


@dataclass
class _Channel:
    sender: object
    receivers: dict            # peer rank -> codec
    send_buf: torch.Tensor     # uint8 [max payload]
    gather_buf: torch.Tensor   # uint8 [world, max payload]


class SPExchange:
    """Payload exchange for ``n_tensors`` tensors of shape (rows, cols) per rank."""

    def __init__(self, rows, cols, mode, n_tensors=1, group=None, device=None, codec_factory=None,
                 act_dtype=torch.bfloat16, **params):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.rows, self.cols, self.mode = int(rows), int(cols), mode
        self.device = torch.device(device) if device is not None else (
            torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu"))
        self.act_dtype = act_dtype
        self.cuda = self.device.type == "cuda"
        make = codec_factory or cf_codec_factory
        self.channels = []
        for _ in range(n_tensors):
            s = make(rows, cols, mode, cf.CF_SENDER, **params)
            rx = {p: make(rows, cols, mode, cf.CF_RECEIVER, **params) for p in range(self.world) if p != self.rank}
            n = max(s.payload_bytes(True), s.payload_bytes(False))
            self.channels.append(_Channel(
                s, rx, torch.empty(n, dtype=torch.uint8, device=self.device),
                torch.empty(self.world, n, dtype=torch.uint8, device=self.device)))
        # device payloads over a backend without device collectives go through the host
        self.host_staged = self.cuda and dist.get_backend(group) == "gloo"
        self.comm = torch.cuda.Stream(self.device) if self.cuda and not self.host_staged else None
        self.t = 0

    def step(self, shards):
        """One step: ``shards`` is a list of ``n_tensors`` local (rows, cols)
        tensors.  Returns a list of (world, rows, cols) tensors: the full
        activation of every exchanged tensor (own shard exact, peers' shards
        reconstructed from their payloads)."""
        assert len(shards) == len(self.channels)
        outs = [torch.empty(self.world, self.rows, self.cols, dtype=self.act_dtype, device=self.device)
                for _ in shards]
        compute = torch.cuda.current_stream(self.device) if self.cuda else None
        sizes, gathered = [], []
        # encode every tensor, issuing each gather as soon as its payload is ready
        for ch, a in zip(self.channels, shards):
            warm = ch.sender.next_is_warm()
            P = ch.sender.payload_bytes(warm)
            sizes.append(P)
            ch.sender.encode(a, ch.send_buf[:P], compute)
            if self.host_staged:
                work = _host_staged_gather(_flat(ch.gather_buf, P), ch.send_buf[:P], self.world, self.group)
            elif self.cuda:
                self.comm.wait_stream(compute)
                with torch.cuda.stream(self.comm):
                    work = dist.all_gather_into_tensor(_flat(ch.gather_buf, P), ch.send_buf[:P], group=self.group,
                                                       async_op=True)
            else:
                work = dist.all_gather_into_tensor(_flat(ch.gather_buf, P), ch.send_buf[:P], group=self.group,
                                                   async_op=True)
            gathered.append(work)
        # decode the peers' payloads of each tensor once its gather is complete
        for ch, a, out, P, work in zip(self.channels, shards, outs, sizes, gathered):
            work.wait()
            if self.comm is not None:
                compute.wait_stream(self.comm)
            flat = _flat(ch.gather_buf, P).view(self.world, P)
            for p, rx in ch.receivers.items():
                rx.decode(flat[p], out[p], compute)
            out[self.rank].copy_(a)
        self.t += 1
        return outs

    def reset(self):
        """Start a new request on every state of this rank (the next step is a
        warm-up step again); every rank must reset before the same step."""
        for ch in self.channels:
            for c in [ch.sender] + list(ch.receivers.values()):
                c.reset()
        self.t = 0

    def status(self) -> int:
        """First nonzero device status of this rank's states (libcf codes)."""
        for ch in self.channels:
            for c in [ch.sender] + list(ch.receivers.values()):
                st = c.status()
                if st != 0:
                    return st
        return 0

    def close(self):
        for ch in self.channels:
            for c in [ch.sender] + list(ch.receivers.values()):
                c.close()
        self.channels = []


class _Done:
    """A completed collective (the synchronous host-staged transport)."""

    def wait(self):
        return True


def _host_staged_gather(out: torch.Tensor, send: torch.Tensor, world: int, group) -> _Done:
    """All-gather of device bytes through host memory: the device-to-host copy
    waits for the encode on the current stream; the gathered bytes are copied
    back on the current stream, ahead of the decodes enqueued after it."""
    h_send = send.cpu()
    h_out = torch.empty(world * h_send.numel(), dtype=torch.uint8)
    dist.all_gather_into_tensor(h_out, h_send, group=group)
    out.copy_(h_out.to(out.device, non_blocking=False))
    return _Done()


def _flat(gather_buf: torch.Tensor, P: int) -> torch.Tensor:
    """The first world * P bytes of the gather buffer as one contiguous vector
    (rank r's payload at [r * P, (r + 1) * P))."""
    return gather_buf.view(-1)[: gather_buf.shape[0] * P]
