"""Pins for the oracle's bf16-state option (CPU only).

The option stores ahat and e in bf16: every state update of the recurrence
("Overall framework", "Key design: error feedback") rounds its fp32 result to
bf16 (nearest even), on the sender and the receiver alike.  Checked against
torch's bfloat16 cast applied to the fp32-state oracle's update from the same
pre-step state, and for boundedness of the feedback loop.
"""
import numpy as np
import pytest
import torch


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(h):
    return (np.asarray(h, dtype=np.uint32) << 16).view(np.float32)


def _walk(rows, cols, T, seed):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((rows, cols))
    out = []
    for _ in range(T):
        out.append(_bf16(a))
        a = a + 0.1 * rng.standard_normal((rows, cols))
    return out


MODES = [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 2, "nm_m": 16}), ("nm", {"nm_n": 1, "nm_m": 4}), ("identity", {})]


@pytest.mark.parametrize("mode,kw", MODES)
@pytest.mark.parametrize("ef", ["explicit", "implicit", "off"])
def test_state_update_is_the_bf16_rounding_of_the_fp32_update(orc, mode, kw, ef):
    rows, cols, T = 16, 128, 6
    s = _walk(rows, cols, T, 1)
    o16 = orc.Oracle(rows, cols, mode, dtype="bf16", ef=ef, state_dtype="bf16", **kw)
    o32 = orc.Oracle(rows, cols, mode, dtype="bf16", ef=ef, **kw)
    for t in range(T):
        if t > 0:          # the fp32 oracle starts from the bf16 oracle's state
            o32.ahat_s[...] = o16.ahat_s
            o32.err[...] = o16.err
            o32.ahat_r[...] = o16.ahat_r
        p16 = o16.encode(s[t])
        p32 = o32.encode(s[t])
        assert np.array_equal(p16, p32), t                       # same residual, same payload
        r16, st16 = o16.decode(p16)
        o32.decode(p32)
        assert st16 == 0
        for a16, a32 in ((o16.ahat_s, o32.ahat_s), (o16.err, o32.err), (o16.ahat_r, o32.ahat_r)):
            assert np.array_equal(a16.view(np.uint32), _f32(_bf16(a32)).view(np.uint32)), t
        assert np.array_equal(o16.ahat_s.view(np.uint32), o16.ahat_r.view(np.uint32)) or ef == "off"
        assert np.array_equal(r16.reshape(-1), _bf16(o16.ahat_r).reshape(-1))


def test_bf16_state_feedback_stays_bounded(orc):
    """Implicit feedback on a stationary stream: the bf16 state's error settles
    within 5 % of the fp32 state's."""
    rng = np.random.default_rng(3)
    rho = np.sqrt(0.99)
    a = rng.standard_normal((32, 512))
    seq = []
    for _ in range(40):
        seq.append(_bf16(a))
        a = rho * a + 0.1 * rng.standard_normal(a.shape)
    errs = {}
    for sd in ("f32", "bf16"):
        o = orc.Oracle(32, 512, "q2", dtype="bf16", ef="implicit", state_dtype=sd)
        e = []
        for x in seq:
            o.decode(o.encode(x))
            xf = _f32(x)
            e.append(np.linalg.norm(o.ahat_r[0] - xf) / np.linalg.norm(xf))
        errs[sd] = e
    assert max(errs["bf16"][20:]) <= 1.25 * max(errs["bf16"][10:20])
    assert abs(np.mean(errs["bf16"][20:]) - np.mean(errs["f32"][20:])) <= 0.05 * np.mean(errs["f32"][20:])


def test_bf16_state_needs_bf16_activations_and_a_streaming_mode(orc):
    with pytest.raises(ValueError):
        orc.Oracle(8, 64, "q2", dtype="f32", state_dtype="bf16")
    with pytest.raises(ValueError):
        orc.Oracle(128, 128, "lowrank", dtype="bf16", rank=4, state_dtype="bf16")
