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


@pytest.mark.parametrize("int4", [1, 0])
def test_noalloc_decode_matches_stateful_decode(int4):
    rows, cols, rank = 1024, 768, 70
    pair = GpuPair(rows, cols, "lowrank", dtype="bf16", rank=rank, iters=1, lr_int4=int4, seed=3)
    s = inputs.ar1("cuda", rows=rows, cols=cols, seed=11)
    params = cf.cf_params_init(dtype=cf.CF_BF16, rank=rank, iters=1, lr_int4=int4)
    try:
        a0 = s.next()
        pair.step(a0)                                        # warm-up: raw activations
        ahat = a0[0].float().contiguous()                    # the caller-owned receiver state
        recon = torch.empty(rows, cols, dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for step in (1, 2):                                  # two calls in a row
            a = s.next()
            cf.cf_encode(pair.S, a, pair.payload)
            cf.cf_decode(pair.R, pair.payload, pair.recon)
            cf.cf_lowrank_decode_noalloc(rows, cols, params, step, pair.payload, ahat, recon, status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            ref_ahat, _ = pair.state("R")
            assert np.array_equal(ahat.cpu().numpy().view(np.uint32), ref_ahat[0].view(np.uint32)), step
            assert np.array_equal(to_np(recon), to_np(pair.recon)[0]), step
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
