"""Host-made faults and state management on the GPU path: every failure is
injected on the host (a corrupted header, a skipped step, a wrong role, a
misaligned or missing pointer, a destroyed handle) or is a bounded device wait
made to run out with nothing in flight; no kernel traps, spins without a limit
or faults.  Also checkpoint/resume and reset."""
import ctypes

import numpy as np
import pytest
import torch

import activation_residual_compression_b200 as cf
import oracle
from activation_residual_compression_b200 import inputs
from cfharness import GpuPair, to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _pair_after(steps, mode="sign1", rows=40, cols=256):
    s = inputs.ActivationStream(rows, cols, dtype=torch.bfloat16, device="cuda", seed=3)
    pair = GpuPair(rows, cols, mode, dtype="bf16")
    for _ in range(steps):
        pair.step(s.next())
    torch.cuda.synchronize()
    return pair, s


@pytest.mark.parametrize("corrupt", ["step", "mode", "magic", "rows", "skip"])
def test_header_mismatch_sets_desync_and_leaves_receiver(corrupt):
    pair, s = _pair_after(3)
    try:
        assert cf.cf_status(pair.R) == cf.CF_OK
        before_ah, _ = pair.state("R")
        before_rec = to_np(pair.recon).copy()
        a = s.next()
        cf.cf_encode(pair.S, a, pair.payload)
        if corrupt == "skip":
            cf.cf_encode(pair.S, s.next(), pair.payload)   # receiver misses a step
        else:
            off = {"step": 16, "mode": 4, "magic": 0, "rows": 24}[corrupt]
            pair.payload[off:off + 1] ^= 1
        cf.cf_decode(pair.R, pair.payload, pair.recon)
        assert cf.cf_status(pair.R) == cf.CF_ERR_DESYNC
        after_ah, _ = pair.state("R")
        assert np.array_equal(before_ah.view(np.uint32), after_ah.view(np.uint32))
        assert np.array_equal(before_rec, to_np(pair.recon))
        # still usable: reset both sides and run a clean request
        cf.cf_reset(pair.S)
        cf.cf_reset(pair.R)
        assert cf.cf_status(pair.R) == cf.CF_OK
        pair.step(s.next())
        pair.step(s.next())
        assert cf.cf_status(pair.R) == cf.CF_OK
    finally:
        pair.close()


@pytest.mark.parametrize("role", ["receiver", "sender"])
def test_lowrank_bounded_wait_runs_out(role):
    """The low-rank reconstruction kernel's bounded wait for its operand copies,
    made to run out by the test hook (no copy is issued, so nothing is in flight;
    a limit of 256 polls): the kernel returns, cf_status reports CF_ERR_TIMEOUT
    for that state only, and the state it would have updated (receiver: ahat and
    recon; sender: ahat and e) is unchanged.  In the sender's encode the
    orthonormalisation kernel's first grid barrier runs out as well (one block
    withholds its arrival): every block leaves before Q is formed, so the U
    scales of the payload stay zero (the column maxima are zeroed at the start
    of each encode).  With the hook off and both states reset, a clean request
    runs and reports no error."""
    rows, cols = 256, 256
    pair = GpuPair(rows, cols, "lowrank", dtype="bf16", rank=16, iters=1, lr_int4=1, seed=3)
    s = inputs.ar1("cuda", rows=rows, cols=cols)
    try:
        pair.step(s.next())
        pair.step(s.next())
        torch.cuda.synchronize()
        hooked, other = (pair.R, pair.S) if role == "receiver" else (pair.S, pair.R)
        which = "R" if role == "receiver" else "S"
        before = pair.state(which)
        rec_before = to_np(pair.recon).copy()
        cf.cf_test_wait_timeout(hooked, 256)
        a = s.next()
        cf.cf_encode(pair.S, a, pair.payload)
        if role == "receiver":
            cf.cf_decode(pair.R, pair.payload, pair.recon)
        assert cf.cf_status(hooked) == cf.CF_ERR_TIMEOUT
        assert cf.cf_status(other) == cf.CF_OK
        u_scales = to_np(pair.payload[64:64 + 4 * 16]).view(np.float32)  # header, then the r U scales
        if role == "sender":
            assert np.all(u_scales == 0.0), u_scales
        else:
            assert np.all(u_scales > 0.0), u_scales
        after = pair.state(which)
        assert np.array_equal(before[0].view(np.uint32), after[0].view(np.uint32))
        if role == "sender":
            assert np.array_equal(before[1].view(np.uint32), after[1].view(np.uint32))
        assert np.array_equal(rec_before, to_np(pair.recon))
        # the context is still usable: hook off, both sides reset, a clean request
        cf.cf_test_wait_timeout(hooked, 0)
        cf.cf_reset(pair.S)
        cf.cf_reset(pair.R)
        for _ in range(3):
            pair.step(s.next())
        assert cf.cf_status(pair.S) == cf.CF_OK and cf.cf_status(pair.R) == cf.CF_OK
        ah_s, _ = pair.state("S")
        ah_r, _ = pair.state("R")
        assert np.array_equal(ah_s.view(np.uint32), ah_r.view(np.uint32))
        assert cf.raw("cf_test_wait_timeout")(pair.S, 0) == cf.CF_OK
    finally:
        pair.close()


def test_wait_timeout_hook_is_lowrank_only():
    pair, _ = _pair_after(1)
    try:
        assert cf.raw("cf_test_wait_timeout")(pair.S, 16) == cf.CF_ERR_UNSUPPORTED
    finally:
        pair.close()


def test_role_alignment_and_handle_errors():
    pair, s = _pair_after(1)
    try:
        a = s.next()
        enc, dec = cf.raw("cf_encode"), cf.raw("cf_decode")
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        P = ctypes.c_void_p
        assert enc(pair.R, P(a.data_ptr()), P(pair.payload.data_ptr()), st) == cf.CF_ERR_ROLE
        assert dec(pair.S, P(pair.payload.data_ptr()), P(pair.recon.data_ptr()), st) == cf.CF_ERR_ROLE
        assert enc(pair.S, P(a.data_ptr() + 2), P(pair.payload.data_ptr()), st) == cf.CF_ERR_ALIGN
        assert enc(pair.S, None, P(pair.payload.data_ptr()), st) == cf.CF_ERR_ARG
        assert dec(pair.R, P(pair.payload.data_ptr() + 8), P(pair.recon.data_ptr()), st) == cf.CF_ERR_ALIGN
        assert cf.cf_step(pair.S) == 1 and cf.cf_step(pair.R) == 1   # rejected calls do not advance
        dead = pair.S
        cf.cf_destroy(dead)
        pair.S = None
        assert enc(dead, P(a.data_ptr()), P(pair.payload.data_ptr()), st) == cf.CF_ERR_STATE
        assert cf.raw("cf_destroy")(dead) == cf.CF_ERR_STATE
    finally:
        pair.close()


def test_export_import_resume_is_bit_identical():
    rows, cols = 64, 3072
    s1 = inputs.ActivationStream(rows, cols, dtype=torch.bfloat16, device="cuda", seed=21)
    s2 = inputs.ActivationStream(rows, cols, dtype=torch.bfloat16, device="cuda", seed=21)
    full = GpuPair(rows, cols, "q2", dtype="bf16")
    part = GpuPair(rows, cols, "q2", dtype="bf16")
    try:
        for _ in range(10):
            full.step(s1.next())
            part.step(s2.next())
        bS, bR = part.export("S"), part.export("R")
        part.close()
        resumed = GpuPair(rows, cols, "q2", dtype="bf16")
        cf.cf_state_import(resumed.S, bS)
        cf.cf_state_import(resumed.R, bR)
        assert cf.cf_step(resumed.S) == 10
        for t in range(5):
            full.step(s1.next())
            resumed.step(s2.next())
            torch.cuda.synchronize()
            assert np.array_equal(full.payload_np(False), resumed.payload_np(False)), t
            assert np.array_equal(to_np(full.recon), to_np(resumed.recon)), t
        bad = bytearray(bS)
        bad[8] ^= 1
        assert cf.raw("cf_state_import")(resumed.S, ctypes.c_char_p(bytes(bad)), len(bad), None) == cf.CF_ERR_ARG
        assert cf.raw("cf_state_import")(resumed.S, ctypes.c_char_p(bytes(bS)), len(bS) - 1, None) == cf.CF_ERR_SIZE
        resumed.close()
    finally:
        full.close()


def test_reset_restarts_with_warmup():
    rows, cols = 8, 64
    pair, s = _pair_after(4, rows=rows, cols=cols)
    try:
        cf.cf_reset(pair.S)
        cf.cf_reset(pair.R)
        a = s.next()
        pair.step(a)
        torch.cuda.synchronize()
        p = pair.payload_np(True)
        assert p[8:12].view(np.uint32)[0] == 1
        assert np.array_equal(to_np(pair.recon)[0], to_np(a)[0])
    finally:
        pair.close()


def test_caller_workspace():
    rows, cols = 33, 1920
    p = cf.cf_params_init(role=cf.CF_SENDER)
    need = cf.cf_workspace_bytes(rows, cols, cf.CF_Q2, p)
    ws = torch.zeros(need + 256, dtype=torch.uint8, device="cuda")
    base = (ws.data_ptr() + 255) // 256 * 256
    p.workspace = base
    p.workspace_bytes = need
    S = cf.cf_create(rows, cols, cf.CF_Q2, p)
    R = cf.cf_create(rows, cols, cf.CF_Q2, cf.cf_params_init(role=cf.CF_RECEIVER))
    orc = oracle.Oracle(rows, cols, "q2", dtype="bf16")
    s = inputs.ActivationStream(rows, cols, dtype=torch.bfloat16, device="cuda", seed=2)
    pay = torch.empty(cf.cf_payload_bytes(S, True), dtype=torch.uint8, device="cuda")
    rec = torch.empty(rows, cols, dtype=torch.bfloat16, device="cuda")
    try:
        for t in range(3):
            a = s.next()
            cf.cf_encode(S, a, pay)
            cf.cf_decode(R, pay, rec)
            torch.cuda.synchronize()
            p_o = orc.encode(to_np(a))
            assert np.array_equal(pay[:len(p_o)].cpu().numpy(), p_o)
        small = cf.cf_params_init(role=cf.CF_SENDER)
        small.workspace = base
        small.workspace_bytes = need - 1
        h = ctypes.c_void_p()
        assert cf.raw("cf_create")(rows, cols, cf.CF_Q2, ctypes.byref(small), ctypes.byref(h)) == cf.CF_ERR_NOMEM
    finally:
        cf.cf_destroy(S)
        cf.cf_destroy(R)
