"""Pins for the oracle's block-selection mode (CPU only).

Source: the Otil page ("Square sub-block partition", "Informative sub-block
selection", "Dynamic round-robin", warm-up: the first step plus 4 more sent in
full).  The token grid H x W (rows = H*W, raster order) is cut into b x b
blocks spanning all channels; each selective step sends, raw, the k blocks of
largest cosine dissimilarity d = 1 - <x_{t-1}, x_t>_F / (||x_{t-1}|| ||x_t||)
among the blocks not yet sent in the current round (lower index first on
equal d); the round restarts when every block has been sent.

Every check uses an independent computation: numpy block reshapes for d and
the payload data, Python's sort for the selection, and a numpy model of the
receiver's stale blocks.
"""
import math

import numpy as np
import pytest
import torch

NONE = 0xFFFFFFFF


def _blocks(x, H, b):
    """(K, b*b*C) view of a [H*W][C] activation: block-major, tokens raster within a block."""
    W = x.shape[0] // H
    C = x.shape[1]
    v = x.reshape(H // b, b, W // b, b, C).transpose(0, 2, 1, 3, 4)
    return v.reshape((H // b) * (W // b), b * b * C)


def _stream(H, W, C, T, seed, dtype="f32"):
    """Per-block innovation scales (log-uniform), so the changes concentrate in a few blocks."""
    rng = np.random.default_rng(seed)
    b = 8 if H % 8 == 0 and W % 8 == 0 else 4
    K = (H // b) * (W // b)
    scale = np.exp(rng.uniform(np.log(0.01), np.log(0.3), K))
    sc = np.repeat(np.repeat(scale.reshape(H // b, W // b), b, 0), b, 1).reshape(H * W, 1)
    a = rng.standard_normal((H * W, C))
    out = []
    for _ in range(T):
        out.append(a.astype(np.float32))
        a = a + sc * rng.standard_normal((H * W, C))
    if dtype == "bf16":
        out = [torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16) for x in out]
    return out


def _f32(x):
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32)
    return x


def _np_dissim(p, a, H, b):
    P = _blocks(p.astype(np.float64), H, b)
    A = _blocks(a.astype(np.float64), H, b)
    d = np.empty(P.shape[0])
    for i in range(P.shape[0]):
        if np.array_equal(P[i], A[i]):
            d[i] = 0.0
        elif not P[i].any() or not A[i].any():
            d[i] = 1.0
        else:
            d[i] = 1.0 - float(P[i] @ A[i]) / (np.linalg.norm(P[i]) * np.linalg.norm(A[i]))
    return d


@pytest.mark.parametrize("H,W,C,b", [(16, 16, 64, 8), (24, 40, 32, 8), (12, 8, 16, 4)])
def test_dissimilarity_matches_numpy(orc, H, W, C, b):
    s = _stream(H, W, C, 2, 1)
    o = orc.Oracle(H * W, C, "blocksel", dtype="f32", bs_h=H, bs_block=b, bs_warm=1)
    d_o = o.dissimilarity(s[0], s[1])
    d_n = _np_dissim(s[0], s[1], H, b)
    assert np.allclose(d_o, d_n, rtol=1e-10, atol=1e-14)
    # special cases: an unchanged block, a block that becomes zero, a zero block that stays zero
    p, a = s[0].copy(), s[1].copy()
    Bp, Ba = _blocks(p, H, b), _blocks(a, H, b)
    Ba[0] = Bp[0]
    Ba[1] = 0.0
    Bp[2] = 0.0
    Ba[2] = 0.0
    W_ = H * W // H
    back = lambda B: B.reshape(H // b, W_ // b, b, b, C).transpose(0, 2, 1, 3, 4).reshape(H * W, C)  # noqa: E731
    p2, a2 = back(Bp), back(Ba)
    d2 = o.dissimilarity(p2, a2)
    assert d2[0] == 0.0 and d2[1] == 1.0 and d2[2] == 0.0
    # scaling leaves every cosine at 1 (d ~ 0); a sign flip gives d = 2
    assert np.abs(o.dissimilarity(s[0], 2.0 * s[0])).max() < 1e-12
    assert np.abs(o.dissimilarity(s[0], -s[0]) - 2.0).max() < 1e-12


@pytest.mark.parametrize("H,W,C,b,k,dtype", [(16, 16, 64, 8, 1, "f32"), (32, 32, 32, 8, 0, "bf16"),
                                             (24, 40, 32, 8, 4, "f32"), (12, 8, 16, 4, 2, "bf16")])
def test_selection_payload_and_receiver(orc, H, W, C, b, k, dtype):
    """Brute-force top-k over the unsent blocks, raw block bytes, the round-robin
    flags, and the receiver's stale blocks, step by step."""
    warm, T = 3, 16
    s = _stream(H, W, C, T, 2, dtype)
    o = orc.Oracle(H * W, C, "blocksel", dtype=dtype, bs_h=H, bs_block=b, bs_k=k, bs_warm=warm)
    K, k = o.bs_K, o.bs_k
    if k == 0:
        raise AssertionError
    assert k == (k if k else max(1, K // 4))
    asz = 2 if dtype == "bf16" else 4
    sent = np.zeros(K, dtype=bool)
    model = None                         # the receiver's values, per the reading
    for t in range(T):
        a = s[t]
        p = o.encode(a)
        recon, st = o.decode(p)
        assert st == 0
        a32 = _f32(a)
        if t < warm:
            assert p[8] == 1                                  # warm-up flag: raw payload
            assert np.array_equal(p[64:64 + a.nbytes], a.reshape(-1).view(np.uint8))
            model = a32.copy()
            assert np.array_equal(recon.reshape(a.shape), a)
            continue
        assert p[8] == 0
        prev = _f32(s[t - 1])
        d = o.dissimilarity(prev, a32)                        # the oracle's own d, pinned above
        cand = sorted((i for i in range(K) if not sent[i]), key=lambda i: (-d[i], i))
        m = min(k, len(cand))
        want = sorted(cand[:m])
        idx = p[64:64 + 4 * k].view(np.uint32)
        assert list(idx[:m]) == want and all(x == NONE for x in idx[m:])
        off = 64 + (4 * k + 15) // 16 * 16
        blk = b * b * C * asz
        raw = _blocks(a.reshape(H * W, C), H, b)
        for j in range(k):
            chunk = p[off + j * blk: off + (j + 1) * blk]
            if j < m:
                assert np.array_equal(chunk, raw[idx[j]].view(np.uint8)), (t, j)
                mb = _blocks(model, H, b)
                mb[idx[j]] = _blocks(a32, H, b)[idx[j]]
                model = mb.reshape(H // b, W // b, b, b, C).transpose(0, 2, 1, 3, 4).reshape(H * W, C)
            else:
                assert not chunk.any()
        sent[want] = True
        if sent.all():
            sent[:] = False
        assert np.array_equal(o.sent.astype(bool), sent)
        assert np.array_equal(o.ahat_s[0].view(np.uint32), a32.view(np.uint32))  # sender keeps a_t
        assert np.array_equal(o.ahat_r[0], model)
        r = recon.reshape(H * W, C)
        assert np.array_equal(_f32(r), model)


def test_round_robin_covers_every_block_once_per_round(orc):
    H = W = 32
    C, b = 16, 8
    s = _stream(H, W, C, 20, 3)
    o = orc.Oracle(H * W, C, "blocksel", dtype="f32", bs_h=H, bs_block=b, bs_k=3, bs_warm=1)
    K, k = o.bs_K, o.bs_k
    assert (K, k) == (16, 3)
    rounds, cur = [], []
    for t, a in enumerate(s):
        p = o.encode(a)
        o.decode(p)
        if t == 0:
            continue
        idx = [int(x) for x in p[64:64 + 4 * k].view(np.uint32) if x != NONE]
        cur += idx
        if len(cur) == K:
            rounds.append(cur)
            cur = []
    assert len(rounds) >= 3
    for r in rounds:
        assert sorted(r) == list(range(K))       # each block exactly once per round
    # a round of K = 16 blocks at k = 3 takes ceil(16 / 3) = 6 steps, the last with one block
    assert math.ceil(K / k) == 6


def test_quarter_of_the_blocks_is_the_default(orc):
    o = orc.Oracle(64 * 64, 32, "blocksel", dtype="bf16")
    assert (o.bs_h, o.bs_b, o.bs_K, o.bs_k, o.bs_warm) == (64, 8, 64, 16, 5)
    assert o.payload_bytes(False) == 64 + 16 * 4 + 16 * 64 * 32 * 2


def test_rejects_grids_not_cut_into_blocks(orc):
    with pytest.raises(ValueError):
        orc.Oracle(10 * 12, 16, "blocksel", dtype="f32", bs_h=10, bs_block=8)
    with pytest.raises(ValueError):
        orc.Oracle(16 * 16, 16, "blocksel", dtype="f32", bs_h=16, bs_block=8, bs_k=5)  # k > K = 4
