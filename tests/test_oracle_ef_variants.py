"""Pins for the error-feedback variants of the CPU oracle (CPU only).

Source: "Accelerating Parallel Diffusion Model Serving with Residual
Compression" -- "Key design: error feedback": the untransmitted error is kept
and added to the next residual; without it the total error of residual
compression grows linearly with the step count; with it the error settles to
a bounded steady state, and (Proposition 3.1) the steady-state error of
residual compression is the naive (direct) compression error scaled by
sigma_Delta^2 / sigma_a^2, far below it.

CF_EF_OFF is read as residual compression against the previous activation
with the error dropped: D_t = a_t - a_{t-1}, sender state ahat_S = fp32(a_t).
Each test checks the oracle against something outside its own EF code: the
explicit codec after a warm-up, exact arithmetic on a ramp, or the naive
codec reached by zeroing the state.
"""
import numpy as np
import pytest


def _ar1(rows, cols, steps, seed, ratio=0.1):
    """Stationary AR(1): a_t = rho a_{t-1} + ratio * N(0, 1), rho = sqrt(1 - ratio^2),
    so sigma_a = 1 and sigma_Delta / sigma_a ~ ratio."""
    rng = np.random.default_rng(seed)
    rho = np.sqrt(1.0 - ratio * ratio)
    a = rng.standard_normal((rows, cols))
    out = [a.astype(np.float32)]
    for _ in range(steps - 1):
        a = rho * a + ratio * rng.standard_normal((rows, cols))
        out.append(a.astype(np.float32))
    return out


MODES = [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 2, "nm_m": 16}), ("nm", {"nm_n": 1, "nm_m": 4})]


@pytest.mark.parametrize("mode,kw", MODES)
def test_ef_off_residual_is_the_consecutive_difference(orc, mode, kw):
    """Every EF-off payload body equals the payload body of an explicit codec
    that was warmed up on a_{t-1} (ahat = fp32(a_{t-1}), e = 0) and then
    encodes a_t: the residual is a_t - a_{t-1}, with no error term."""
    rows, cols, T = 12, 64, 6
    s = _ar1(rows, cols, T, 3)
    off = orc.Oracle(rows, cols, mode, dtype="f32", ef="off", **kw)
    off.encode(s[0])
    for t in range(1, T):
        p = off.encode(s[t])
        ref = orc.Oracle(rows, cols, mode, dtype="f32", ef="explicit", **kw)
        ref.encode(s[t - 1])
        q = ref.encode(s[t])
        assert np.array_equal(p[64:], q[64:]), t


@pytest.mark.parametrize("mode,kw", MODES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ef_off_sender_state_is_the_activation(orc, mode, kw, dtype):
    rows, cols, T = 8, 64, 5
    s = _ar1(rows, cols, T, 4)
    o = orc.Oracle(rows, cols, mode, dtype=dtype, ef="off", **kw)
    for t in range(T):
        a = s[t]
        if dtype == "bf16":
            import torch
            a = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            a32 = (a.astype(np.uint32) << 16).view(np.float32)
        else:
            a32 = a
        p = o.encode(a)
        _, st = o.decode(p)
        assert st == 0
        assert np.array_equal(o.ahat_s[0].view(np.uint32), a32.view(np.uint32)), t
        assert not np.any(o.err)


@pytest.mark.parametrize("mode,kw", [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16})])
def test_ef_off_error_grows_linearly_on_a_ramp(orc, mode, kw):
    """a_t = a_0 + t g with g a power-of-two multiple of small integers, so
    every a_t and every difference a_t - a_{t-1} = g is exact in fp32.  EF off
    then sends enc(g) every step and the receiver error after t steps is
    t (g - C(g)), up to the rounding of the receiver's fp32 sum: the linear
    growth the page names."""
    rows, cols, T = 8, 64, 17
    rng = np.random.default_rng(5)
    a0 = (rng.integers(-64, 65, (rows, cols)) * 2.0 ** -6).astype(np.float32)
    g = (rng.integers(-16, 17, (rows, cols)) * 2.0 ** -10).astype(np.float32)
    ramp = [(a0 + t * g).astype(np.float32) for t in range(T)]
    for t in range(T):
        assert np.array_equal(ramp[t].astype(np.float64), a0.astype(np.float64) + t * g.astype(np.float64))
    off = orc.Oracle(rows, cols, mode, dtype="f32", ef="off", **kw)
    err = []
    for t in range(T):
        _, st = off.decode(off.encode(ramp[t]))
        assert st == 0
        err.append(off.ahat_r[0].astype(np.float64) - ramp[t].astype(np.float64))
    one = err[1]
    assert np.abs(one).max() > 0
    # the receiver's running fp32 sum rounds by at most 2^-24 |ahat| per step
    # (zero for SIGN1 and N:M here, whose C values add exactly)
    amax = max(np.abs(x).max() for x in ramp) + np.abs(one).max() * T
    for t in range(1, T):
        assert np.abs(err[t] - t * one).max() <= t * 2.0 ** -24 * amax, t
        if mode != "q2":
            assert np.array_equal(err[t], t * one), t


def _rel_errors(orc, stream, mode, kw, ef):
    rows, cols = stream[0].shape
    o = orc.Oracle(rows, cols, mode, dtype="f32", ef=ef, **kw)
    rel = []
    for a in stream:
        _, st = o.decode(o.encode(a))
        assert st == 0
        rel.append(float(np.linalg.norm(o.ahat_r[0].astype(np.float64) - a) / np.linalg.norm(a)))
    return rel


STUDY = [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}), ("nm", {"nm_n": 2, "nm_m": 16})]


@pytest.mark.parametrize("mode,kw", STUDY)
def test_feedback_bounds_the_error_and_its_absence_does_not(orc, mode, kw):
    """On a stationary stream (sigma_Delta / sigma_a = 0.1) feedback, in the
    form where the residual is taken against the reconstruction, settles: the
    error over steps 25..49 stays within 1.25x of its level over steps 10..24.
    Without feedback it keeps growing (a random walk of per-step errors)."""
    s = _ar1(64, 3072, 50, 1)
    imp = _rel_errors(orc, s, mode, kw, "implicit")
    off = _rel_errors(orc, s, mode, kw, "off")
    assert max(imp[25:]) <= 1.25 * max(imp[10:25]), imp
    assert off[49] > 1.5 * off[10], off
    assert off[49] > 2.0 * imp[49]


@pytest.mark.parametrize("mode,kw", STUDY)
def test_explicit_form_feeds_the_error_back_twice(orc, mode, kw):
    """The recurrence as literally specified, D_t = (a_t - ahat_{t-1}) + e_{t-1},
    adds e to a residual that already contains it (a_t - ahat_t = e_t - e_{t-1}).
    On the stationary stream its error ends above the implicit form's in every
    mode, and for the N:M sparsifier (most coordinates pass into e unchanged,
    so e_t ~ 2 e_{t-1} - e_{t-2}) it diverges."""
    s = _ar1(64, 3072, 50, 1)
    imp = _rel_errors(orc, s, mode, kw, "implicit")
    exp = _rel_errors(orc, s, mode, kw, "explicit")
    assert exp[1] == imp[1]          # identical on the first compressed step (e_0 = 0)
    assert exp[49] > 2.0 * imp[49], (exp[49], imp[49])
    if mode == "nm":
        assert exp[49] > 100.0 and exp[49] > 10 * exp[25]


def _steady_error(orc, stream, mode, kw, ef, naive=False):
    """Mean squared receiver error over the second half of the stream.  The
    naive codec compresses a_t itself: its state is zeroed before each step,
    so D = a_t and the receiver's reconstruction is C(a_t)."""
    rows, cols = stream[0].shape
    o = orc.Oracle(rows, cols, mode, dtype="f32", ef=ef, **kw)
    errs = []
    for t, a in enumerate(stream):
        if naive and t > 0:
            o.ahat_s[:] = 0.0
            o.err[:] = 0.0
            p = o.encode(a)
            rec = o.meaning(p).astype(np.float64)
        else:
            _, st = o.decode(o.encode(a))
            assert st == 0
            rec = o.ahat_r[0].astype(np.float64)
        if t >= len(stream) // 2:
            errs.append(np.mean((rec - a.astype(np.float64)) ** 2))
    return float(np.mean(errs))


@pytest.mark.parametrize("mode,kw", STUDY)
def test_prop31_residual_error_far_below_naive(orc, mode, kw):
    """Proposition 3.1: v_residual / v_naive is of order sigma_Delta^2 / sigma_a^2
    (here 0.01) times a compressor-dependent ratio, far below 1; checked for
    the feedback form whose error is bounded."""
    ratio = 0.1
    s = _ar1(64, 256, 24, 6, ratio)
    v_naive = _steady_error(orc, s, mode, kw, "implicit", naive=True)
    v_res = _steady_error(orc, s, mode, kw, "implicit")
    assert v_res / v_naive < 0.1, (v_res, v_naive)
    assert v_res / v_naive > 0.1 * ratio * ratio, (v_res, v_naive)  # the same order as the scaling
