"""bench.py's grouped per-call timing, checked on the CPU with torch's CUDA
events and streams replaced by a recording fake.

The per-kernel figures (per_mode, the dominant kernel's roofline, the suite)
come from grouped loops: per sender/receiver pair, n encodes back to back into
their own payload slots between two events, then the decodes of those slots
between two more; several pairs of one configuration are cycled where a
decode's state is not much larger than the L2.  These tests pin the order of
the calls (each payload decoded after it was written and before its slot is
reused, every pair's calls in step order), the arithmetic of the mean, the
grouping under a slot budget, and the pair counts of the benchmark workloads.
"""
import contextlib
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _Clock:
    """A device clock that advances by the cost of every recorded call."""

    def __init__(self):
        self.t = 0.0
        self.log = []


@pytest.fixture
def fake_cuda(monkeypatch):
    clk = _Clock()

    class Ev:
        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            self.t = clk.t
            clk.log.append(("event",))

        def elapsed_time(self, other):
            return other.t - self.t

    monkeypatch.setattr(torch.cuda, "Event", Ev)
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "_sleep", lambda n: clk.log.append(("sleep",)))
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: clk.log.append(("sync",)))
    return clk


def _pairs(clk, n_pairs, enc_ms, dec_ms, pay_bytes=64):
    """Fake pairs whose calls cost enc_ms / dec_ms of device time and check
    the payload protocol: a decode reads the slot its encode wrote, once."""
    reps, state = [], []
    for r in range(n_pairs):
        st = {"enc": [], "dec": [], "slot_of": {}}
        state.append(st)

        def enc(j, p, r=r, st=st):
            assert all(q.data_ptr() != p.data_ptr() for k, q in st["slot_of"].items() if k not in st["dec"])
            p.fill_(j % 251)
            st["slot_of"][j] = p
            st["enc"].append(j)
            clk.t += enc_ms
            clk.log.append(("enc", r, j))

        def dec(j, p, r=r, st=st):
            assert st["slot_of"][j] is p and int(p[0]) == j % 251
            st["dec"].append(j)
            clk.t += dec_ms
            clk.log.append(("dec", r, j))

        reps.append((enc, dec, torch.empty(pay_bytes, dtype=torch.uint8)))
    return reps, state


@pytest.mark.parametrize("n,n_pairs,slot_bytes", [(5, 1, 1 << 30), (7, 3, 1 << 30), (7, 3, 3 * 64 * 2),
                                                  (1, 2, 1)])
def test_grouped_order_and_mean(fake_cuda, n, n_pairs, slot_bytes):
    enc_ms, dec_ms = 0.05, 0.03
    reps, state = _pairs(fake_cuda, n_pairs, enc_ms, dec_ms)
    e, d = bench.grouped_times(reps, n, stream=None, slot_bytes=slot_bytes)
    assert e == pytest.approx(enc_ms) and d == pytest.approx(dec_ms)
    for st in state:  # every call once, in step order, each decode after its encode
        assert st["enc"] == list(range(n)) and st["dec"] == list(range(n))
    calls = [x for x in fake_cuda.log if x[0] in ("enc", "dec")]
    # within a group: encodes of call j of every pair, then call j + 1, ...; then
    # the decodes in the same order; no event between two calls of a group
    g = max(1, min(n, slot_bytes // (64 * n_pairs)))
    expect = []
    for j0 in range(0, n, g):
        js = range(j0, min(n, j0 + g))
        expect += [("enc", r, j) for j in js for r in range(n_pairs)]
        expect += [("dec", r, j) for j in js for r in range(n_pairs)]
    assert calls == expect
    seq = [x[0] for x in fake_cuda.log]
    for i in range(1, len(seq)):
        if seq[i - 1] == "enc" and seq[i] == "enc" or seq[i - 1] == "dec" and seq[i] == "dec":
            continue
        if seq[i] in ("enc", "dec") and seq[i - 1] in ("enc", "dec"):
            pytest.fail("an encode and a decode with no event between them")
    # a device-side spin ahead of every group's first event
    for i, x in enumerate(fake_cuda.log):
        if x == ("event",) and (i == 0 or fake_cuda.log[i - 1] == ("sync",)):
            pytest.fail("a group's first event without the spin before it")


def test_pair_counts_of_the_benchmark_workloads():
    E_flux, E_lr = 4608 * 3072, 4096 * 3072
    assert bench.n_replicas(E_flux * 10) == 3         # FLUX: ahat read + written, recon written
    assert bench.n_replicas(E_lr * 10) == 4           # low-rank receiver
    assert bench.n_replicas(E_lr * 6) == 6            # block selection (bf16 state), capped
    assert bench.n_replicas(60 * 17550 * 1920 * 10) == 1   # CogVideoX batch: far beyond the L2
    # the cycle of pairs moves at least three L2s of decode traffic (up to the cap)
    for b in (1e6, 5e7, 1e8, 2e8, 4e8, 1e9):
        k = bench.n_replicas(b)
        assert 1 <= k <= 6 and (k == 6 or k * b >= 3 * bench.L2_BYTES)
