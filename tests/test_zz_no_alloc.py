"""The allocation-free low-rank decode, cf_lowrank_decode_noalloc.

Some callers cannot allocate device memory when they decode: a process whose
framework owns every allocation, a fixed-memory serving deployment, or code
that must not call cudaMalloc on that path.  For them the library offers one
decode entry point with no state object and no allocation; its scratch is a
fixed array inside the library.  These tests call it through the C ABI and
check that it reproduces cf_decode (the stateful receiver) bit for bit on two
consecutive steps, that a mismatched payload is reported through the caller's
status word, and that a problem beyond the fixed scratch is refused.

This file is collected last and is self-contained: it passes alone in a fresh
process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import activation_residual_compression_b200 as cf
from activation_residual_compression_b200 import inputs
from cfharness import GpuPair, to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


EF = {"explicit": cf.CF_EF_EXPLICIT, "implicit": cf.CF_EF_IMPLICIT, "off": cf.CF_EF_OFF}


def _noalloc_io(rows, cols, dtype, a0):
    """Caller-owned receiver state (after the warm-up step), output and status word."""
    ahat = a0[0].float().contiguous()
    recon = torch.empty(rows, cols, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    return ahat, recon, status


def _same_as_stateful(pair, ahat, recon, step):
    ref_ahat, _ = pair.state("R")
    assert np.array_equal(ahat.cpu().numpy().view(np.uint32), ref_ahat[0].view(np.uint32)), step
    assert np.array_equal(to_np(recon), to_np(pair.recon)[0]), step


@pytest.mark.parametrize("dtype,ef,int4,iters", [
    ("bf16", "explicit", 1, 1), ("bf16", "explicit", 0, 1), ("f32", "explicit", 1, 1), ("f32", "explicit", 0, 1),
    ("bf16", "implicit", 1, 1), ("f32", "implicit", 0, 1), ("bf16", "off", 1, 1), ("f32", "off", 0, 1),
    ("bf16", "explicit", 1, 2), ("f32", "implicit", 0, 2)])
def test_noalloc_decode_matches_stateful_decode(dtype, ef, int4, iters):
    """Bit for bit the stateful receiver's ahat and recon on two calls in a row, for
    bf16 and fp32 activations, every error-feedback form (carried in the payload
    header the entry point checks), INT4 and fp32 factors, one and two sweeps."""
    rows, cols, rank = 1024, 768, 70
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    pair = GpuPair(rows, cols, "lowrank", dtype=dtype, ef=ef, rank=rank, iters=iters, lr_int4=int4, seed=3)
    s = inputs.ar1("cuda", rows=rows, cols=cols, seed=11, dtype=tdt)
    params = cf.cf_params_init(dtype=cf.CF_BF16 if dtype == "bf16" else cf.CF_F32, ef=EF[ef], rank=rank,
                               iters=iters, lr_int4=int4)
    try:
        a0 = s.next()
        pair.step(a0)                                        # warm-up: raw activations
        ahat, recon, status = _noalloc_io(rows, cols, dtype, a0)
        for step in (1, 2):                                  # two calls in a row
            a = s.next()
            cf.cf_encode(pair.S, a, pair.payload)
            cf.cf_decode(pair.R, pair.payload, pair.recon)
            cf.cf_lowrank_decode_noalloc(rows, cols, params, step, pair.payload, ahat, recon, status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            _same_as_stateful(pair, ahat, recon, step)
        # a payload for another step is reported and leaves the caller's tensors alone
        a = s.next()
        cf.cf_encode(pair.S, a, pair.payload)
        before = ahat.clone()
        rec_before = recon.clone()
        cf.cf_lowrank_decode_noalloc(rows, cols, params, 7, pair.payload, ahat, recon, status)
        torch.cuda.synchronize()
        assert int(status.item()) & 1
        assert torch.equal(before, ahat) and torch.equal(rec_before, recon)
    finally:
        pair.close()


def test_noalloc_decode_survives_a_smaller_rank_state():
    """Setting up a low-rank state of a smaller rank between two calls must not lower
    the shared kernels' shared-memory limit below what this entry point launches
    with (rank 70 with fp32 factors: the largest reconstruction tile)."""
    rows, cols, rank = 1024, 768, 70
    pair = GpuPair(rows, cols, "lowrank", dtype="bf16", rank=rank, iters=1, lr_int4=0, seed=5)
    s = inputs.ar1("cuda", rows=rows, cols=cols, seed=12)
    params = cf.cf_params_init(dtype=cf.CF_BF16, rank=rank, iters=1, lr_int4=0)
    small = None
    try:
        a0 = s.next()
        pair.step(a0)
        ahat, recon, status = _noalloc_io(rows, cols, "bf16", a0)
        for step in (1, 2):
            if step == 2:   # a rank-32 state in between: its set-up must leave the limits alone
                small = cf.cf_create(rows, cols, cf.CF_LOWRANK,
                                     cf.cf_params_init(role=cf.CF_RECEIVER, dtype=cf.CF_BF16, rank=32, lr_int4=1))
            a = s.next()
            cf.cf_encode(pair.S, a, pair.payload)
            cf.cf_decode(pair.R, pair.payload, pair.recon)
            assert cf.cf_lowrank_decode_noalloc(rows, cols, params, step, pair.payload, ahat, recon, status) == cf.CF_OK
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            _same_as_stateful(pair, ahat, recon, step)
    finally:
        if small is not None:
            cf.cf_destroy(small)
        pair.close()


def test_noalloc_decode_refuses_problems_beyond_its_scratch():
    buf = torch.zeros(64, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    P = ctypes.c_void_p
    p = cf.cf_params_init(dtype=cf.CF_BF16, rank=128, iters=1, lr_int4=0)
    fn = cf.raw("cf_lowrank_decode_noalloc")
    rc = fn(16384, 8192, ctypes.byref(p), 1, P(buf.data_ptr()), P(buf.data_ptr()), P(buf.data_ptr()),
            P(status.data_ptr()), None)
    assert rc == cf.CF_ERR_TOO_LARGE
    assert "fixed scratch" in cf.cf_strerror(rc)
    rc = fn(1000, 768, ctypes.byref(p), 1, P(buf.data_ptr()), P(buf.data_ptr()), P(buf.data_ptr()),
            P(status.data_ptr()), None)
    assert rc == cf.CF_ERR_SHAPE
    assert int(status.item()) == 0
