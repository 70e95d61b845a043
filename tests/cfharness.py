"""Test-side helpers: drive the CUDA codec through the C-ABI binding and read
its outputs back to the host.  No compression arithmetic lives here."""
from __future__ import annotations

import numpy as np
import torch

import activation_residual_compression_b200 as cf

GUARD = 4096
CANARY = 0xA5


def to_np(t: torch.Tensor) -> np.ndarray:
    """Host copy; bf16 tensors come back as uint16 bit patterns."""
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def guarded(nbytes: int, device="cuda") -> tuple[torch.Tensor, torch.Tensor]:
    """A uint8 device buffer with GUARD canary bytes on both sides; returns (whole, inner)."""
    whole = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device=device)
    return whole, whole[GUARD:GUARD + nbytes]


def canaries_intact(whole: torch.Tensor) -> bool:
    h = whole.cpu().numpy()
    return bool((h[:GUARD] == CANARY).all() and (h[-GUARD:] == CANARY).all())


class GpuPair:
    """A sender and a receiver state of the CUDA codec plus guarded device buffers."""

    def __init__(self, rows, cols, mode, dtype="bf16", ef="explicit", nm_n=1, nm_m=16, batch=1,
                 rank=70, iters=1, lr_int4=1, seed=0, **extra):
        self.rows, self.cols, self.batch = rows, cols, batch
        self.mode = cf.MODE_NAMES[mode]
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        bf16_state = extra.get("state_dtype") == "bf16"
        if "state_dtype" in extra:
            extra["state_dtype"] = cf.CF_BF16 if bf16_state else cf.CF_F32
        kw = dict(dtype=cf.CF_BF16 if dtype == "bf16" else cf.CF_F32,
                  ef={"explicit": cf.CF_EF_EXPLICIT, "implicit": cf.CF_EF_IMPLICIT, "off": cf.CF_EF_OFF}[ef],
                  nm_n=nm_n, nm_m=nm_m, batch=batch, rank=rank, iters=iters, lr_int4=lr_int4, seed=seed, **extra)
        self.has_err = mode != "blocksel"       # block selection keeps no error term
        # block selection keeps its state (raw activations) in the activation dtype;
        # the bf16-state option stores ahat and e as bf16
        self.state_esz = (2 if dtype == "bf16" else 4) if mode == "blocksel" else (2 if bf16_state else 4)
        self.S = cf.cf_create(rows, cols, self.mode, cf.cf_params_init(role=cf.CF_SENDER, **kw))
        self.R = cf.cf_create(rows, cols, self.mode, cf.cf_params_init(role=cf.CF_RECEIVER, **kw))
        self.pb_warm = cf.cf_payload_bytes(self.S, True)
        self.pb = cf.cf_payload_bytes(self.S, False)
        self.pay_whole, self.payload = guarded(max(self.pb_warm, self.pb))
        esz = 2 if dtype == "bf16" else 4
        self.rec_whole, rec_bytes = guarded(batch * rows * cols * esz)
        self.recon = rec_bytes.view(self.tdtype).view(batch, rows, cols)
        self.t = 0

    def step(self, a: torch.Tensor, stream=None):
        cf.cf_encode(self.S, a, self.payload, stream)
        cf.cf_decode(self.R, self.payload, self.recon, stream)
        self.t += 1

    def payload_np(self, warm: bool) -> np.ndarray:
        n = self.pb_warm if warm else self.pb
        return self.payload[:n].cpu().numpy()

    def export(self, which="S") -> np.ndarray:
        st = self.S if which == "S" else self.R
        buf = np.zeros(cf.cf_state_bytes(st), dtype=np.uint8)
        cf.cf_state_export(st, buf)
        return buf

    def state(self, which="S", with_vprev=False):
        """(ahat, err or None) as float32 arrays of shape (batch, rows, cols); with
        with_vprev the sender's low-rank warm start (batch, cols, rank) is appended."""
        buf = self.export(which)
        tb = int(buf[80:88].view(np.uint64)[0])
        ten = buf[len(buf) - tb:]
        n = self.batch * self.rows * self.cols
        z = self.state_esz

        def tensor(k):
            raw = ten[k * z * n:(k + 1) * z * n]
            if z == 2:
                return (raw.view(np.uint16).astype(np.uint32) << 16).view(np.float32).reshape(
                    self.batch, self.rows, self.cols)
            return raw.view(np.float32).reshape(self.batch, self.rows, self.cols)

        ahat = tensor(0)
        err = None
        if which == "S" and self.has_err:
            err = tensor(1)
        if with_vprev:
            vp = ten[2 * z * n:].view(np.float32).reshape(self.batch, self.cols, -1)
            return ahat, err, vp
        return ahat, err

    def sent_flags(self) -> np.ndarray:
        """Block selection (sender): the per-block 'sent this round' flags (the export's tail)."""
        buf = self.export("S")
        tb = int(buf[80:88].view(np.uint64)[0])
        ten = buf[len(buf) - tb:]
        return ten[self.state_esz * self.batch * self.rows * self.cols:].copy()

    def guards_ok(self) -> bool:
        return canaries_intact(self.pay_whole) and canaries_intact(self.rec_whole)

    def close(self):
        for h in (self.S, self.R):
            if h is not None:
                cf.cf_destroy(h)
        self.S = self.R = None
