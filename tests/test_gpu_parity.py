"""GPU <-> oracle parity for the streaming modes, through the C-ABI.

Payload bytes, sender ahat and e, receiver ahat and recon must be
bit-identical to the CPU oracle on the same seeded inputs at every step (a
stronger bar than 1e-3 relative L2).  Method: "Accelerating Parallel
Diffusion Model Serving with Residual Compression" -- overall framework,
error feedback, residual 1-bit/2-bit quantisation, N:M block sparsifier,
warm-up of the first step.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_residual_compression_b200 import inputs
from cfharness import GpuPair, to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _np_act(a: torch.Tensor):
    return to_np(a)


def _run_and_compare(pair: GpuPair, orc: oracle.Oracle, stream_next, steps, check_state_every=1,
                     sender_tracks_receiver=True):
    for t in range(steps):
        a = stream_next()
        pair.step(a)
        torch.cuda.synchronize()
        a_h = _np_act(a)
        p_o = orc.encode(a_h)
        rec_o, st = orc.decode(p_o)
        assert st == 0
        p_g = pair.payload_np(warm=(t == 0))
        assert p_g.shape == p_o.shape, (t, p_g.shape, p_o.shape)
        if not np.array_equal(p_g, p_o):
            diff = np.nonzero(p_g != p_o)[0]
            raise AssertionError(f"step {t}: payload differs at {diff.size} bytes, first {diff[:8]}")
        assert np.array_equal(to_np(pair.recon).reshape(rec_o.shape), rec_o), f"recon differs at step {t}"
        if t % check_state_every == 0 or t == steps - 1:
            ah_s, e_s = pair.state("S")
            ah_r, _ = pair.state("R")
            assert np.array_equal(ah_s.view(np.uint32), orc.ahat_s.view(np.uint32)), f"ahat_S differs at step {t}"
            assert np.array_equal(e_s.view(np.uint32), orc.err.view(np.uint32)), f"e differs at step {t}"
            assert np.array_equal(ah_r.view(np.uint32), orc.ahat_r.view(np.uint32)), f"ahat_R differs at step {t}"
            if sender_tracks_receiver:
                assert np.array_equal(ah_s.view(np.uint32), ah_r.view(np.uint32))
    assert pair.guards_ok(), "a kernel wrote outside its buffers"


# ----------------------------------------------------------------------------- tiny config

@pytest.mark.parametrize("mode", ["sign1", "q2"])
def test_tiny_config_bit_exact(mode):
    """256 x 64 fp32 random walk, 8 steps, sigma 0.1, CPU generator seed 0."""
    s = inputs.tiny("cpu")
    pair = GpuPair(256, 64, mode, dtype="f32")
    orc = oracle.Oracle(256, 64, mode, dtype="f32")
    try:
        _run_and_compare(pair, orc, lambda: s.next().cuda(), 8)
    finally:
        pair.close()


# ----------------------------------------------------------------------------- shapes / modes

CASES = [
    ("identity", {}, [64, 200, 3072, 8192]),
    ("sign1", {}, [32, 96, 640, 1920, 3072, 8192]),
    ("q2", {}, [16, 48, 1920, 3072, 8192]),
    ("nm", {"nm_n": 1, "nm_m": 16}, [128, 1920, 3072, 8192]),
    ("nm", {"nm_n": 2, "nm_m": 16}, [64, 1920, 3072]),
    ("nm", {"nm_n": 1, "nm_m": 4}, [64, 640, 3072]),
    ("nm", {"nm_n": 2, "nm_m": 4}, [32, 96, 3072]),
]


def _param_cases():
    out = []
    for mode, kw, cols_list in CASES:
        for cols in cols_list:
            for rows in (1, 7, 33):
                out.append(pytest.param(mode, kw, rows, cols, id=f"{mode}{kw.get('nm_n', '')}{kw.get('nm_m', '')}-{rows}x{cols}"))
    return out


@pytest.mark.parametrize("mode,kw,rows,cols", _param_cases())
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_modes_and_shapes_bit_exact(mode, kw, rows, cols, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    s = inputs.ActivationStream(rows, cols, dtype=tdt, device="cuda", seed=rows * 7 + cols, sigma=0.1,
                                outlier_frac=0.01)
    pair = GpuPair(rows, cols, mode, dtype=dtype, **kw)
    orc = oracle.Oracle(rows, cols, mode, dtype=dtype, **kw)
    try:
        _run_and_compare(pair, orc, s.next, 4)
    finally:
        pair.close()


@pytest.mark.parametrize("ef", ["implicit", "off"])
@pytest.mark.parametrize("mode,kw", [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 2, "nm_m": 16}),
                                     ("nm", {"nm_n": 1, "nm_m": 4}), ("identity", {})])
def test_other_error_feedback_forms_bit_exact(mode, kw, ef):
    """Implicit feedback, and no feedback (the sender's state is the previous
    activation, e stays zero): payloads and both states bit-identical."""
    rows, cols = 65, 3072
    s = inputs.ActivationStream(rows, cols, dtype=torch.bfloat16, device="cuda", seed=5)
    pair = GpuPair(rows, cols, mode, dtype="bf16", ef=ef, **kw)
    orc = oracle.Oracle(rows, cols, mode, dtype="bf16", ef=ef, **kw)
    try:
        _run_and_compare(pair, orc, s.next, 5, sender_tracks_receiver=ef != "off")
        if ef == "off":
            _, e_s = pair.state("S")
            assert not np.any(e_s)
    finally:
        pair.close()


@pytest.mark.parametrize("mode,kw", [("sign1", {}), ("q2", {})])
def test_error_feedback_off_batched_fp32_bit_exact(mode, kw):
    """No feedback in the batched launch with fp32 activations."""
    rows, cols, batch = 40, 512, 3
    s = inputs.ActivationStream(rows, cols, dtype=torch.float32, device="cuda", seed=8, batch=batch)
    pair = GpuPair(rows, cols, mode, dtype="f32", ef="off", batch=batch, **kw)
    orc = oracle.Oracle(rows, cols, mode, dtype="f32", ef="off", batch=batch, **kw)
    try:
        _run_and_compare(pair, orc, s.next, 4, sender_tracks_receiver=False)
    finally:
        pair.close()


@pytest.mark.parametrize("ef", ["explicit", "implicit", "off"])
@pytest.mark.parametrize("mode,kw", [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}),
                                     ("nm", {"nm_n": 2, "nm_m": 4}), ("identity", {})])
def test_bf16_state_bit_exact(mode, kw, ef):
    """The bf16-state option: every state update rounds to bf16 on both sides."""
    rows, cols = 33, 1920
    s = inputs.ActivationStream(rows, cols, dtype=torch.bfloat16, device="cuda", seed=12)
    pair = GpuPair(rows, cols, mode, dtype="bf16", ef=ef, state_dtype="bf16", **kw)
    orc = oracle.Oracle(rows, cols, mode, dtype="bf16", ef=ef, state_dtype="bf16", **kw)
    try:
        _run_and_compare(pair, orc, s.next, 6, sender_tracks_receiver=ef != "off")
    finally:
        pair.close()


@pytest.mark.parametrize("mode,kw", [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 2, "nm_m": 16})])
def test_bf16_state_batched_bit_exact(mode, kw):
    rows, cols, B = 24, 3072, 3
    s = inputs.ActivationStream(rows, cols, batch=B, dtype=torch.bfloat16, device="cuda", seed=13)
    pair = GpuPair(rows, cols, mode, dtype="bf16", batch=B, state_dtype="bf16", **kw)
    orc = oracle.Oracle(rows, cols, mode, dtype="bf16", batch=B, state_dtype="bf16", **kw)
    try:
        _run_and_compare(pair, orc, s.next, 4)
    finally:
        pair.close()


def test_degenerate_inputs_bit_exact():
    """Constant activations (all-zero residual), exact zeros, sign flips, huge and tiny values."""
    rows, cols = 16, 256
    g = torch.Generator().manual_seed(9)
    seq = [torch.zeros(rows, cols), torch.zeros(rows, cols), torch.full((rows, cols), -0.0),
           torch.randn(rows, cols, generator=g) * 1e-30, torch.randn(rows, cols, generator=g) * 1e30,
           torch.randn(rows, cols, generator=g).sign(), torch.zeros(rows, cols)]
    for mode, kw in [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}), ("nm", {"nm_n": 2, "nm_m": 4}),
                     ("identity", {})]:
        pair = GpuPair(rows, cols, mode, dtype="f32", **kw)
        orc = oracle.Oracle(rows, cols, mode, dtype="f32", **kw)
        it = iter(seq)
        try:
            _run_and_compare(pair, orc, lambda: next(it).float().cuda().unsqueeze(0), len(seq))
        finally:
            pair.close()


# ----------------------------------------------------------------------------- full-size FLUX stream

@pytest.mark.parametrize("mode,kw", [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}),
                                     ("nm", {"nm_n": 2, "nm_m": 16})])
def test_flux_full_size_bit_exact(mode, kw):
    """4608 x 3072 bf16, 28 steps, 1% outlier channels: every payload byte, every step."""
    rows, cols, T = 4608, 3072, 28
    s = inputs.flux("cuda")
    pair = GpuPair(rows, cols, mode, dtype="bf16", **kw)
    orc = oracle.Oracle(rows, cols, mode, dtype="bf16", **kw)
    try:
        _run_and_compare(pair, orc, s.next, T, check_state_every=9)
    finally:
        pair.close()


# ----------------------------------------------------------------------------- batched launch

@pytest.mark.parametrize("mode,kw", [("q2", {}), ("sign1", {}), ("nm", {"nm_n": 1, "nm_m": 16})])
def test_batched_pointer_table_matches_oracle(mode, kw):
    """Separate tensors through the pointer-table entry points: one launch per step."""
    import activation_residual_compression_b200 as cf
    B, rows, cols, T = 5, 37, 1920, 4
    s = inputs.ActivationStream(rows, cols, batch=B, dtype=torch.bfloat16, device="cuda", seed=11,
                                sigma_per_tensor=[0.05, 0.1, 0.2, 0.07, 0.15])
    pair = GpuPair(rows, cols, mode, dtype="bf16", batch=B, **kw)
    orc = oracle.Oracle(rows, cols, mode, dtype="bf16", batch=B, **kw)
    recs = [torch.empty(rows, cols, dtype=torch.bfloat16, device="cuda") for _ in range(B)]
    try:
        for t in range(T):
            a = s.next()
            parts = [a[b].clone() for b in range(B)]   # separate allocations
            cf.cf_encode_batched(pair.S, parts, pair.payload)
            cf.cf_decode_batched(pair.R, pair.payload, recs)
            torch.cuda.synchronize()
            p_o = orc.encode(to_np(a))
            rec_o, _ = orc.decode(p_o)
            assert np.array_equal(pair.payload_np(t == 0), p_o), t
            for b in range(B):
                assert np.array_equal(to_np(recs[b]), rec_o[b]), (t, b)
        assert pair.guards_ok()
    finally:
        pair.close()


def test_cogvideox_full_step_sampled_rows():
    """60 x 17550 x 1920 bf16, Q2, 50 steps, one batched launch per encode/decode.
    Rows are independent in this mode, so sampled rows of three tensors run through
    the oracle as small tensors and must match the GPU payload rows and recon rows."""
    import activation_residual_compression_b200 as cf
    B, rows, cols, T = 60, 17550, 1920, 50
    s = inputs.cogvideox("cuda")
    pair = GpuPair(rows, cols, "q2", dtype="bf16", batch=B)
    g = np.random.default_rng(0)
    tens = [0, 31, 59]
    sel = {b: np.sort(np.concatenate([[0, rows - 1], g.choice(rows, 14, replace=False)])) for b in tens}
    orcs = {b: oracle.Oracle(len(sel[b]), cols, "q2", dtype="bf16") for b in tens}
    sec1 = ((rows * 2 + 15) // 16) * 16
    body = sec1 + rows * cols // 4
    body = ((body + 15) // 16) * 16
    try:
        for t in range(T):
            a = s.next()
            parts = [a[b] for b in range(B)]
            recs = [pair.recon[b] for b in range(B)]
            cf.cf_encode_batched(pair.S, parts, pair.payload)
            cf.cf_decode_batched(pair.R, pair.payload, recs)
            torch.cuda.synchronize()
            warm = t == 0
            for b in tens:
                rr = torch.as_tensor(sel[b], device="cuda")
                sub = a[b].index_select(0, rr)
                p_o = orcs[b].encode(to_np(sub))
                rec_o, _ = orcs[b].decode(p_o)
                assert np.array_equal(to_np(pair.recon[b].index_select(0, rr)), rec_o[0]), (t, b)
                if warm:
                    continue
                n = len(sel[b])
                base = 64 + b * body
                pb = pair.payload[base:base + body].cpu().numpy()
                sc_g = pb[:rows * 2].view(np.uint16)[sel[b]]
                cw_g = pb[sec1:sec1 + rows * cols // 4].view(np.uint32).reshape(rows, cols // 16)[sel[b]]
                ob = p_o[64:]
                osec1 = ((n * 2 + 15) // 16) * 16
                sc_o = ob[:n * 2].view(np.uint16)
                cw_o = ob[osec1:osec1 + n * cols // 4].view(np.uint32).reshape(n, cols // 16)
                assert np.array_equal(sc_g, sc_o), (t, b)
                assert np.array_equal(cw_g, cw_o), (t, b)
            del a, parts
        assert pair.guards_ok()
    finally:
        pair.close()


def test_q2_decision_boundaries_bit_exact():
    """Residuals at and a few ulps around the 2-bit decision boundaries (-2S/3, 0,
    +2S/3), where the kernel's fast code path hands over to the exact division
    chain, must still match the oracle bit for bit."""
    rows, cols = 24, 256
    rng = np.random.default_rng(31)
    a1 = np.zeros((rows, cols), np.float32)
    for r in range(rows):
        S = np.float32(rng.choice([1.5, 0.75, 3.0, 1.0, 0.1, 7.0, 2.0 ** -60, 2.0 ** 60]))
        a1[r, 0] = S                                  # the row maximum: S = bf16(S) = S
        two3 = np.float32(2.0 * float(S) / 3.0)
        cand = []
        for base in (two3, -two3, np.float32(0.0)):
            x = base
            for _ in range(6):
                x = np.nextafter(x, np.float32(-np.inf))
            for _ in range(13):
                cand.append(x)
                x = np.nextafter(x, np.float32(np.inf))
        cand = np.array(cand, np.float32)
        a1[r, 1:1 + len(cand)] = cand
        a1[r, 1 + len(cand):] = (rng.uniform(-1, 1, cols - 1 - len(cand)) * float(S)).astype(np.float32)
    seq = [np.zeros((rows, cols), np.float32), a1, a1 * np.float32(0.5)]
    pair = GpuPair(rows, cols, "q2", dtype="f32")
    orc = oracle.Oracle(rows, cols, "q2", dtype="f32")
    it = iter(seq)
    try:
        _run_and_compare(pair, orc, lambda: torch.from_numpy(next(it)).cuda().unsqueeze(0), len(seq))
    finally:
        pair.close()
