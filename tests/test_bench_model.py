"""bench.py's byte model, checked on the CPU.

The roofline fractions bench.py reports divide algorithmic bytes by kernel
time, so the byte model must describe the real payload format: its payload
sizes (header + body, written out per mode in bench.py) are compared with the
sizes the CPU oracle's payload writer produces, at the benchmark shapes and at
small ones, and the FLUX figures with the per-element counts of the streaming
kernels (encode: read a, ahat, e and write ahat, e, payload; decode: read
payload, ahat and write ahat, recon).
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402

STREAMING = [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}), ("nm", {"nm_n": 2, "nm_m": 16}),
             ("identity", {})]


@pytest.mark.parametrize("rows,cols", [(4608, 3072), (4096, 3072), (130, 512)])
@pytest.mark.parametrize("mode,kw", STREAMING)
def test_streaming_payload_model_matches_the_oracle(mode, kw, rows, cols):
    o = oracle.Oracle(rows, cols, mode, dtype="bf16", **kw)
    assert bench._payload_body(mode, rows, cols, kw) + 64 == o.payload_bytes(False)


def test_blocksel_payload_model_matches_the_oracle():
    kw = dict(bench.WORKLOADS["blocksel"]["codecs"][0][1])
    o = oracle.Oracle(4096, 3072, "blocksel", dtype="bf16", bs_h=kw["bs_grid_h"], bs_block=kw["bs_block"],
                      bs_k=kw["bs_k"], bs_warm=kw["bs_warm"])
    assert bench._payload_body("blocksel", 4096, 3072, kw) + 64 == o.payload_bytes(False) == 6291584


def test_flux_step_bytes():
    E = 4608 * 3072
    for mode, P in (("sign1", 1778752), ("q2", 3548224)):
        assert bench._payload_body(mode, 4608, 3072, {}) + 64 == P
        assert bench.encode_bytes(mode, 4608, 3072, {}) == 18 * E + P
        assert bench.decode_bytes(mode, 4608, 3072, {}) == 10 * E + P
        assert bench.step_bytes(mode, 4608, 3072, {}, P) == 28 * E + 2 * P
    assert bench.encode_bytes("sign1", 4608, 3072, {}) == 256582720
    assert bench.decode_bytes("sign1", 4608, 3072, {}) == 143336512
    # bf16 state: 2-byte ahat and e; implicit feedback reads no e; without feedback e is not touched
    P = 1778752
    assert bench.encode_bytes("sign1", 4608, 3072, {}, state_size=2) == 10 * E + P
    assert bench.encode_bytes("sign1", 4608, 3072, {}, ef="implicit") == 14 * E + P
    assert bench.encode_bytes("sign1", 4608, 3072, {}, ef="off") == 10 * E + P


def test_lowrank_payload_sizes():
    """The rank-70 INT4 and rank-9 fp32 payloads of the low-rank sweep carry about
    the same bytes (the pages' "coverage over precision" comparison)."""
    assert oracle.Oracle(4096, 3072, "lowrank", dtype="bf16", rank=70, iters=1, lr_int4=1).payload_bytes(False) \
        == 251504
    assert oracle.Oracle(4096, 3072, "lowrank", dtype="bf16", rank=9, iters=1, lr_int4=0).payload_bytes(False) \
        == 258112
