"""GPU <-> oracle parity for the block-selection mode (Otil page: "Informative
sub-block selection", "Dynamic round-robin"), through the C ABI.

Payload bytes (selected indices and raw blocks), the receiver's ahat and
recon, the sender's state (fp32 of the previous activation) and the
round-robin flags must be bit-identical to the oracle at every step.  The
selection is an integer decision taken from fp64 dissimilarities whose sums
the two sides form in different orders; on these random streams no two
blocks come within rounding of each other at the selection boundary (the
test reports the margin when a selection differs).  Exact ties (unchanged or
zero blocks) are exact on both sides by the mode's readings.
"""
import numpy as np
import pytest
import torch

import activation_residual_compression_b200 as cf
import oracle
from cfharness import GpuPair, to_np

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _stream(H, W, C, T, seed, b):
    rng = np.random.default_rng(seed)
    K = (H // b) * (W // b)
    scale = np.exp(rng.uniform(np.log(0.01), np.log(0.3), K))
    sc = np.repeat(np.repeat(scale.reshape(H // b, W // b), b, 0), b, 1).reshape(H * W, 1)
    a = rng.standard_normal((H * W, C))
    out = []
    for _ in range(T):
        out.append(a.astype(np.float32))
        a = a + sc * rng.standard_normal((H * W, C))
    return out


def _run(H, W, C, b, k, dtype, T, seq=None, warm=3, seed=1):
    kw = dict(bs_grid_h=H, bs_block=b, bs_k=k, bs_warm=warm)
    pair = GpuPair(H * W, C, "blocksel", dtype=dtype, **kw)
    orc = oracle.Oracle(H * W, C, "blocksel", dtype=dtype, bs_h=H, bs_block=b, bs_k=k, bs_warm=warm)
    seq = seq if seq is not None else _stream(H, W, C, T, seed, b)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    try:
        for t, a32 in enumerate(seq):
            a = torch.from_numpy(a32).to(tdt).cuda().unsqueeze(0)
            a_np = to_np(a)
            pair.step(a)
            torch.cuda.synchronize()
            p_o = orc.encode(a_np)
            rec_o, st = orc.decode(p_o)
            assert st == 0
            warm_step = t < warm
            p_g = pair.payload[:len(p_o)].cpu().numpy()
            if not np.array_equal(p_g, p_o):
                kk = orc.bs_k
                ig = p_g[64:64 + 4 * kk].view(np.uint32)
                io = p_o[64:64 + 4 * kk].view(np.uint32)
                msg = f"step {t}: payload differs"
                if not warm_step and not np.array_equal(ig, io):
                    prev = oracle.f32_from_bf16(to_np(torch.from_numpy(seq[t - 1]).to(tdt))) \
                        if dtype == "bf16" else seq[t - 1]
                    d = orc.dissimilarity(prev, oracle.f32_from_bf16(a_np[0]) if dtype == "bf16" else a32)
                    msg += f"; selections GPU {list(ig)} oracle {list(io)}; d {d}"
                raise AssertionError(msg)
            assert np.array_equal(to_np(pair.recon).reshape(rec_o.shape), rec_o), f"recon differs at step {t}"
            ah_s, e_s = pair.state("S")
            ah_r, _ = pair.state("R")
            assert e_s is None
            assert np.array_equal(ah_s.view(np.uint32), orc.ahat_s.view(np.uint32)), t
            assert np.array_equal(ah_r.view(np.uint32), orc.ahat_r.view(np.uint32)), t
            assert np.array_equal(pair.sent_flags(), orc.sent), t
        assert pair.guards_ok()
        assert cf.cf_status(pair.R) == cf.CF_OK
    finally:
        pair.close()


@pytest.mark.parametrize("H,W,C,b,k,dtype", [(16, 16, 64, 8, 1, "f32"), (32, 32, 64, 8, 0, "bf16"),
                                             (24, 40, 32, 8, 4, "f32"), (12, 8, 16, 4, 2, "bf16"),
                                             (48, 32, 1920, 16, 0, "bf16"), (64, 64, 256, 8, 3, "bf16"),
                                             # around the switch from all-pairs ranking (K <= 256) to the sort
                                             (80, 160, 32, 8, 0, "f32"), (128, 128, 32, 8, 50, "bf16"),
                                             (136, 128, 16, 8, 7, "bf16")])
def test_block_selection_bit_exact(H, W, C, b, k, dtype):
    _run(H, W, C, b, k, dtype, T=14)


def test_full_size_grid_bit_exact():
    """64 x 64 token grid x 3072 channels bf16 (K = 64 blocks of 8 x 8, k = 16), 10 steps."""
    _run(64, 64, 3072, 8, 16, "bf16", T=10, warm=5)


def test_largest_block_count_bit_exact():
    """K = 4096 blocks (the limit of the in-CTA sort): a 512 x 512 grid of 8 x 8
    blocks, 16 channels, k = 1000 (not a divisor of K: rounds end with fewer
    blocks and unused slots)."""
    _run(512, 512, 16, 8, 1000, "bf16", T=9, warm=1)


def test_ties_and_zero_blocks_bit_exact():
    """Unchanged activations (every d = 0: the lowest unsent indices win), blocks
    that become or stay zero (d = 1 / d = 0), then ordinary steps."""
    H = W = 32
    C, b = 64, 8
    rng = np.random.default_rng(4)
    a = rng.standard_normal((H * W, C)).astype(np.float32)
    z = a.copy()
    z[:8 * C] = 0.0                          # block 0's first token row becomes zero
    seq = [a, a, a.copy(), a.copy(), z, z.copy(), np.zeros_like(a), np.zeros_like(a)]
    seq += _stream(H, W, C, 6, 5, b)
    _run(H, W, C, b, 3, "f32", T=len(seq), seq=seq, warm=1)


def test_export_import_resumes_the_round():
    """The round-robin flags are part of the state: a receiver/sender restored
    from an export mid-round continues bit-identically."""
    H = W = 32
    C, b, k = 64, 8, 3
    kw = dict(bs_grid_h=H, bs_block=b, bs_k=k, bs_warm=1)
    seq = _stream(H, W, C, 10, 6, b)
    A = GpuPair(H * W, C, "blocksel", dtype="f32", **kw)
    B = GpuPair(H * W, C, "blocksel", dtype="f32", **kw)
    try:
        for t in range(4):
            A.step(torch.from_numpy(seq[t]).cuda().unsqueeze(0))
        torch.cuda.synchronize()
        cf.cf_state_import(B.S, A.export("S"))
        cf.cf_state_import(B.R, A.export("R"))
        for t in range(4, 10):
            a = torch.from_numpy(seq[t]).cuda().unsqueeze(0)
            A.step(a)
            B.step(a)
            torch.cuda.synchronize()
            assert np.array_equal(A.payload_np(False), B.payload_np(False)), t
            assert torch.equal(A.recon, B.recon), t
    finally:
        A.close()
        B.close()


def test_desynchronised_payload_is_reported():
    """A payload decoded twice (the receiver then expects the next step) is
    refused on the device: the status reports it and recon / ahat keep their values."""
    H = W = 16
    C = 32
    pair = GpuPair(H * W, C, "blocksel", dtype="f32", bs_grid_h=H, bs_block=8, bs_k=1, bs_warm=1)
    seq = _stream(H, W, C, 3, 7, 8)
    try:
        for t in range(3):
            pair.step(torch.from_numpy(seq[t]).cuda().unsqueeze(0))
        torch.cuda.synchronize()
        assert cf.cf_status(pair.R) == cf.CF_OK
        rec = to_np(pair.recon).copy()
        ah = pair.state("R")[0].copy()
        cf.cf_decode(pair.R, pair.payload, pair.recon)       # step 2's payload; the receiver is at step 3
        torch.cuda.synchronize()
        assert cf.cf_status(pair.R) == cf.CF_ERR_DESYNC
        assert np.array_equal(to_np(pair.recon), rec)
        assert np.array_equal(pair.state("R")[0], ah)
    finally:
        pair.close()


def test_rejected_configurations():
    p = cf.cf_params_init(dtype=cf.CF_F32, bs_grid_h=10, bs_block=8)
    with pytest.raises(cf.CFError):
        cf.cf_create(10 * 12, 16, cf.CF_BLOCKSEL, p)
    p = cf.cf_params_init(dtype=cf.CF_F32, bs_grid_h=16, bs_block=8, bs_k=5)   # k > K = 4
    with pytest.raises(cf.CFError):
        cf.cf_create(16 * 16, 16, cf.CF_BLOCKSEL, p)
    p = cf.cf_params_init(dtype=cf.CF_F32, bs_grid_h=16, bs_block=6)
    with pytest.raises(cf.CFError):
        cf.cf_create(16 * 16, 16, cf.CF_BLOCKSEL, p)
