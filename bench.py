#!/usr/bin/env python
"""Benchmark of the residual codec on B200: activation GB/s and ms/step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cf,reference}]

Workload: the FLUX.1-dev-shaped activation stream (4608 x 3072 bf16, 1%
outlier channels x20, random walk with sigma/sigma_a = 0.1) compressed with
residual compression + explicit error feedback in the 1-bit and the 2-bit
modes ("Accelerating Parallel Diffusion Model Serving with Residual
Compression": experiments, main table).  Each mode is a sender/receiver pair
of its own on its own seeded stream; one step = encode + decode of one
activation in every mode.  Inputs are pre-generated in HBM (a fresh tensor
per step; the per-kernel working set exceeds the 126 MB L2).

value  = activation bytes (rows*cols*2 per mode) / device time per step,
         CUDA events on the launching stream, max over ranks.
e2e    = the same metric with the activation in pinned host memory: each
         step copies a_t host->device, encodes, decodes and copies the
         reconstruction device->host, inside the timed region; the copies
         run on their own streams (two buffer slots), so step i's compute
         overlaps step i+1's upload and step i-1's download.
Timed region: after the barrier and synchronize, a short device-side spin
runs ahead of the first event so that the host has queued the first steps
(without it the first step's events also time the host's launch latency).
roofline = the encode kernel of the first mode: algorithmic bytes per launch
         (read a, ahat, e; write ahat, e, payload) / its mean event-timed
         duration, against the measured copy bandwidth.

With --gpus N (torchrun) every rank runs an independent replica on its own
GPU (the method needs no exchange here); value sums all ranks' activation
bytes over the slowest rank's time.  --impl reference times the CPU oracle
(rank 0 only) on a row sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

ROWS, COLS = 4608, 3072
MODES = [("sign1", {}), ("q2", {})]
WORKLOAD = "flux1dev-4608x3072-bf16"
SEQ_STEPS = 27          # compressed steps of a 28-step request (one warm-up step + 27)
DATASHEET_GBS = 8000.0  # B200 HBM3e datasheet bandwidth (context beside the measured copy peak)
METRIC = "activation GB/s and ms/step per mode (encode+EF+decode), % of B200 HBM roofline"

# Timed workloads (--workload): shape, batch, seeded stream and the codecs one
# step runs (each codec has its own sender/receiver pair and its own stream).
WORKLOADS = {
    "flux": dict(name=WORKLOAD, rows=ROWS, cols=COLS, batch=1, stream="flux", codecs=MODES),
    "nm": dict(name="flux1dev-4608x3072-bf16-nm16", rows=ROWS, cols=COLS, batch=1, stream="flux",
               codecs=[("nm", {"nm_n": 1, "nm_m": 16}), ("nm", {"nm_n": 2, "nm_m": 16})]),
    "lowrank": dict(name="ar1-4096x3072-bf16-rank70-int4-k1", rows=4096, cols=3072, batch=1, stream="ar1",
                    codecs=[("lowrank", {"rank": 70, "iters": 1, "lr_int4": 1, "seed": 7})]),
    "lowrank2": dict(name="ar1-4096x3072-bf16-rank70-int4-k2", rows=4096, cols=3072, batch=1, stream="ar1",
                     codecs=[("lowrank", {"rank": 70, "iters": 2, "lr_int4": 1, "seed": 7})]),
    "cogvideox": dict(name="cogvideox2b-60x17550x1920-bf16", rows=17550, cols=1920, batch=60, stream="cogvideox",
                      codecs=[("q2", {})]),
    "blocksel": dict(name="otil-grid64x64-3072ch-bf16-b8-k16", rows=4096, cols=3072, batch=1, stream="blocksel",
                     codecs=[("blocksel", {"bs_grid_h": 64, "bs_block": 8, "bs_k": 16, "bs_warm": 5})]),
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _payload_body(mode, rows, cols, kw):
    pad = lambda b: (b + 15) // 16 * 16  # noqa: E731
    if mode == "sign1":
        return pad(rows * 2) + pad(rows * cols // 8)
    if mode == "q2":
        return pad(rows * 2) + pad(rows * cols // 4)
    if mode == "nm":
        n, m = kw["nm_n"], kw["nm_m"]
        return pad(rows * cols // m * n * 2) + pad(rows * (cols // m * n * (m.bit_length() - 1) // 32) * 4)
    if mode == "identity":
        return rows * cols * 4
    if mode == "blocksel":
        b, k = kw["bs_block"], kw["bs_k"]
        return pad(4 * k) + k * b * b * cols * 2
    raise ValueError(mode)


def _bs_frac(rows, kw):
    H = kw["bs_grid_h"]
    K = (H // kw["bs_block"]) * ((rows // H) // kw["bs_block"])
    return kw["bs_k"] / K


def encode_bytes(mode, rows, cols, kw, act_size=2, ef="explicit", state_size=4):
    """Algorithmic bytes of one encode launch: read a, ahat, e; write ahat, e, payload.
    Implicit feedback does not read e; without feedback e is neither read nor written.
    Block selection: read a and the previous activation (kept in the
    activation dtype), write it, and read + write the sent fraction f of a into
    the payload."""
    E = rows * cols
    if mode == "blocksel":
        return int(E * 3 * act_size + 2 * _bs_frac(rows, kw) * E * act_size) + 64 + 16
    z = state_size
    e_rd = z if ef == "explicit" else 0
    e_wr = 0 if ef == "off" else z
    return E * (act_size + z + e_rd + z + e_wr) + 64 + _payload_body(mode, rows, cols, kw)


def decode_bytes(mode, rows, cols, kw, act_size=2, state_size=4):
    """Algorithmic bytes of one decode launch: read payload, ahat; write ahat, recon.
    Block selection (state in the activation dtype): unsent blocks read ahat and
    write recon; sent blocks read the payload and write ahat and recon."""
    E = rows * cols
    if mode == "blocksel":
        f = _bs_frac(rows, kw)
        return int(E * ((1 - f) * 2 * act_size + f * 3 * act_size)) + 64
    return E * (2 * state_size + act_size) + 64 + _payload_body(mode, rows, cols, kw)


def _kernel_sources_sha256():
    """Hash of the streaming kernels' sources (the ncu traffic figure is only
    valid for the kernels it was taken on)."""
    csrc = os.path.join(ROOT, "activation_residual_compression_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(csrc)):
        if f.startswith("cf_stream"):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()


def _traffic_record():
    """dram read+write bytes per encode launch from the committed ncu summary,
    valid only while the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "encode_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    h = _kernel_sources_sha256()
    if d.get("source_sha256") != h:
        return None
    return d


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            self.path = f"/tmp/cf_clocks_{os.getpid()}.csv"
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu_index)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm

EF_CODES = {"explicit": 0, "implicit": 1, "off": 2}


def _codec_name(mode, kw):
    if mode == "blocksel":
        return f"blocksel_b{kw['bs_block']}_k{kw['bs_k']}"
    if mode == "nm":
        return f"nm{kw['nm_n']}_{kw['nm_m']}"
    if mode == "lowrank":
        return f"lowrank_r{kw['rank']}_k{kw['iters']}"
    return mode


def _make_stream(kind, wl, seed, device="cuda"):
    from activation_residual_compression_b200 import inputs
    if kind == "flux":
        return inputs.flux(device, rows=wl["rows"], cols=wl["cols"], seed=seed)
    if kind == "ar1":
        return inputs.ar1(device, rows=wl["rows"], cols=wl["cols"], seed=seed)
    if kind == "cogvideox":
        return inputs.cogvideox(device, rows=wl["rows"], cols=wl["cols"], n_tensors=wl["batch"])
    if kind == "blocksel":
        return inputs.blocksel(device, H=64, W=wl["rows"] // 64, cols=wl["cols"], seed=seed)
    raise ValueError(kind)


def step_bytes(mode, rows, cols, kw, payload, ef="explicit", state_size=4):
    """Algorithmic bytes of one encode + decode of one tensor (low-rank: the
    explicit-feedback figure)."""
    if mode == "lowrank":
        return _lr_alg_bytes(rows, cols, kw["iters"], payload)
    return (encode_bytes(mode, rows, cols, kw, ef=ef, state_size=state_size) +
            decode_bytes(mode, rows, cols, kw, state_size=state_size))


def workload_config(args, wl, world):
    """The `config` keys both arms report for a workload."""
    return {"workload": wl["name"], "rows": wl["rows"], "cols": wl["cols"], "tensors": wl["batch"],
            "activation_dtype": "bf16", "modes": [_codec_name(m, k) for m, k in wl["codecs"]],
            **({"selection": "raw blocks, no error feedback, state in the activation dtype"}
               if args.workload == "blocksel" else {"error_feedback": args.ef, "state_dtype": args.state}),
            "parallelism": f"replicas{world}" if world > 1 else "single"}


def state_bytes_per_elem(args):
    """Sender + receiver state bytes per element of one codec pair."""
    if args.workload == "blocksel":
        return 2 + 2                               # previous activation (sender), values (receiver), bf16
    esz = 2 if args.state == "bf16" else 4
    return esz * (3 if args.ef == "explicit" or args.ef == "implicit" else 2)  # ahat + e (sender), ahat (receiver)


def launches_per_call(mode, kw, encode):
    """libcf kernels one steady-state cf_encode / cf_decode call launches."""
    if mode == "blocksel":
        return 2 if encode else 1                 # block sums with the selection in the last CTA, pack; decode
    if mode != "lowrank":
        return 1
    if not encode:
        return 2                                   # dequantise, reconstruction
    return 1 + 4 * kw["iters"] + 2                 # residual with the V preparation; per sweep: 2 GEMMs, the
                                                   # orthonormalisation (one persistent kernel), V sum; pack,
                                                   # reconstruction


L2_BYTES = 126e6  # B200 L2


def n_replicas(dec_bytes):
    """Sender/receiver pairs a grouped loop cycles through so that between two
    calls of one pair the others move more than twice the L2: a decode's
    state is smaller than the L2 on some workloads, and back-to-back decodes
    of one receiver would find part of it there."""
    return int(min(6, max(1, math.ceil(3 * L2_BYTES / max(1, dec_bytes)))))


def grouped_times(reps, n, stream, slot_bytes=4 << 30):
    """Mean device time per encode and per decode with no event between two
    kernels.  reps: one (enc_j, dec_j, pay) per sender/receiver pair of the
    same configuration; enc_j(j, p) makes the pair's call j into payload slot
    p, dec_j(j, p) decodes it, pay is a payload buffer to copy the slot size
    from.  Per group: the encodes (call j of every pair, then call j + 1 ...)
    back to back between two events, each into its own slot, then the decodes
    of those slots in the same order between two more.  Groups hold as many
    slots as fit in slot_bytes; the mean is over n calls of every pair."""
    import torch

    per_call = sum(p.numel() for _, _, p in reps)
    g = max(1, min(n, slot_bytes // max(1, per_call)))
    slots = [[torch.empty_like(p) for _ in range(g)] for _, _, p in reps]
    t_enc = t_dec = 0.0
    j = 0
    with torch.cuda.stream(stream):
        while j < n:
            m = min(g, n - j)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            # a device-side spin first, so the group's first call does not
            # time the host's launch latency into an empty queue
            torch.cuda._sleep(1_000_000)
            ev[0].record(stream)
            for u in range(m):
                for r, (enc_j, _, _) in enumerate(reps):
                    enc_j(j + u, slots[r][u])
            ev[1].record(stream)
            for u in range(m):
                for r, (_, dec_j, _) in enumerate(reps):
                    dec_j(j + u, slots[r][u])
            ev[2].record(stream)
            torch.cuda.synchronize()
            t_enc += ev[0].elapsed_time(ev[1])
            t_dec += ev[1].elapsed_time(ev[2])
            j += m
    del slots
    return t_enc / (n * len(reps)), t_dec / (n * len(reps))


def run_cf(args, rank, world, device):
    import torch

    import activation_residual_compression_b200 as cf

    wl = WORKLOADS[args.workload]
    R_, C_, B_ = wl["rows"], wl["cols"], wl["batch"]
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream()
    K, W = args.steps, args.warmup
    in_bytes = B_ * R_ * C_ * 2
    want = max(W + K + 1, SEQ_STEPS + 1 if args.sequences > 0 else 0)
    n_inputs = max(2, min(want, args.max_resident, int(args.resident_gb * 1e9 // (in_bytes * len(wl["codecs"])))))
    batched = B_ > 1
    codecs = []
    for mi, (mode, kw) in enumerate(wl["codecs"]):
        s = _make_stream(wl["stream"], wl, seed=1 + 100 * mi + 1000 * rank)
        acts = [s.next() for _ in range(n_inputs)]
        del s
        base = dict(dtype=cf.CF_BF16, batch=B_, ef=EF_CODES[args.ef], **kw)
        if args.state == "bf16":
            base["state_dtype"] = cf.CF_BF16
        S = cf.cf_create(R_, C_, cf.MODE_NAMES[mode], cf.cf_params_init(role=cf.CF_SENDER, **base))
        R = cf.cf_create(R_, C_, cf.MODE_NAMES[mode], cf.cf_params_init(role=cf.CF_RECEIVER, **base))
        pay = torch.empty(max(cf.cf_payload_bytes(S, True), cf.cf_payload_bytes(S, False)), dtype=torch.uint8,
                          device="cuda")
        rec = torch.empty(B_, R_, C_, dtype=torch.bfloat16, device="cuda")
        codecs.append(dict(mode=mode, kw=kw, name=_codec_name(mode, kw), S=S, R=R, pay=pay, rec=rec, acts=acts,
                           P=cf.cf_payload_bytes(S, False), params=base))
    torch.cuda.empty_cache()
    torch.cuda.synchronize()

    def enc(c, a, pay=None):
        pay = c["pay"] if pay is None else pay
        if batched:
            cf.cf_encode_batched(c["S"], [a[b] for b in range(B_)], pay, stream)
        else:
            cf.cf_encode(c["S"], a, pay, stream)

    def dec(c, out=None, pay=None):
        out = c["rec"] if out is None else out
        pay = c["pay"] if pay is None else pay
        if batched:
            cf.cf_decode_batched(c["R"], pay, [out[b] for b in range(B_)], stream)
        else:
            cf.cf_decode(c["R"], pay, out, stream)

    def step(i, evs=None):
        for c in codecs:
            a = c["acts"][i % n_inputs]
            if evs is not None:
                evs.append(torch.cuda.Event(enable_timing=True)); evs[-1].record(stream)
            enc(c, a)
            if evs is not None:
                evs.append(torch.cuda.Event(enable_timing=True)); evs[-1].record(stream)
            dec(c)
        if evs is not None:
            evs.append(torch.cuda.Event(enable_timing=True)); evs[-1].record(stream)

    dist = None
    if world > 1:
        import torch.distributed as dist

    # untimed steps: at least the warm-up, and past every codec's full-size
    # leading steps (block selection sends bs_warm steps in full)
    W_run = max([W] + [kw.get("bs_warm", 1) for _, kw in wl["codecs"]])
    with torch.cuda.stream(stream):
        for i in range(W_run):
            step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(device)
    clocks.start()
    time.sleep(0.3)
    # The timed region: K steps between two events and nothing else on the
    # stream, the way a caller runs them back to back.  An event recorded
    # between two kernels costs ~2.7 us of device time on this pool (an empty
    # kernel between two events reads 6.1-6.5 us), so the per-kernel times come
    # from a second loop of K steps with an event around every encode and decode
    # (the per-mode figures and the roofline of the dominant kernel), reported
    # beside it as ms_per_step_instrumented.
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        # a ~0.5 ms device-side spin ahead of the first event: the host enqueues
        # the first steps meanwhile, so the timed region measures the kernels
        # rather than the launch latency of an empty queue after the synchronize
        torch.cuda._sleep(1_000_000)
        t0.record(stream)
        for i in range(W_run, W_run + K):
            step(i)
        t1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    evs = []
    u0 = torch.cuda.Event(enable_timing=True)
    u1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(1_000_000)
        u0.record(stream)
        for i in range(W_run + K, W_run + 2 * K):
            step(i, evs)
        u1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    instr_ms = u0.elapsed_time(u1)
    # events per step: for each codec (before encode, before decode), then one at the end
    nm = len(codecs)
    stride = 2 * nm + 1
    per = {c["name"]: {"enc": [], "dec": []} for c in codecs}
    for k in range(K):
        base = k * stride
        for mi, c in enumerate(codecs):
            per[c["name"]]["enc"].append(evs[base + 2 * mi].elapsed_time(evs[base + 2 * mi + 1]))
            per[c["name"]]["dec"].append(evs[base + 2 * mi + 1].elapsed_time(evs[base + 2 * mi + 2]))
    for c in codecs:
        if cf.cf_status(c["R"], stream) != cf.CF_OK or cf.cf_status(c["S"], stream) != cf.CF_OK:
            raise RuntimeError(f"codec {c['name']} reported an error status")

    # Per-kernel times without events between kernels: per codec, K encodes
    # back to back (each into its own payload slot) between two events, then
    # the K decodes of those payloads between two more.  Both states advance
    # exactly as in the interleaved loops.  Where a decode's state is not much
    # larger than the L2, the loop cycles through several sender/receiver
    # pairs of the same configuration (each warmed up like the first), so that
    # no call finds its state left in the L2 by its own previous call.
    grouped = {}
    i0 = W_run + 2 * K
    for c in codecs:
        zs = 2 if (args.state == "bf16" or c["mode"] == "blocksel") else 4
        nrep = n_replicas(B_ * R_ * C_ * (2 * zs + 2))
        reps = [c]
        for _ in range(nrep - 1):
            x = dict(c, S=cf.cf_create(R_, C_, cf.MODE_NAMES[c["mode"]],
                                       cf.cf_params_init(role=cf.CF_SENDER, **c["params"])),
                     R=cf.cf_create(R_, C_, cf.MODE_NAMES[c["mode"]],
                                    cf.cf_params_init(role=cf.CF_RECEIVER, **c["params"])),
                     pay=torch.empty_like(c["pay"]), rec=torch.empty_like(c["rec"]))
            with torch.cuda.stream(stream):
                for i in range(W_run):
                    enc(x, x["acts"][i % n_inputs])
                    dec(x)
            reps.append(x)
        torch.cuda.synchronize()
        ms_e, ms_d = grouped_times(
            [(lambda j, p, x=x: enc(x, x["acts"][(i0 + j) % n_inputs], p),
              lambda j, p, x=x: dec(x, None, p), x["pay"]) for x in reps], K, stream)
        grouped[c["name"]] = {"enc": ms_e, "dec": ms_d, "pairs": nrep}
        for x in reps:
            if cf.cf_status(x["R"], stream) != cf.CF_OK or cf.cf_status(x["S"], stream) != cf.CF_OK:
                raise RuntimeError(f"codec {c['name']} reported an error status in the grouped loop")
        for x in reps[1:]:
            cf.cf_destroy(x["S"]); cf.cf_destroy(x["R"])
        del reps
        torch.cuda.empty_cache()

    # full sequences: each a new request (both states reset, the warm-up step
    # untimed) of SEQ_STEPS compressed steps, every encode and decode bracketed
    # by events; the median over sequences of the mean step time
    seq = None
    if args.sequences > 0:
        W_seq = max(kw.get("bs_warm", 1) for _, kw in wl["codecs"])
        seq_step, seq_per = [], {c["name"]: [] for c in codecs}
        for q in range(args.sequences):
            for c in codecs:
                cf.cf_reset(c["S"]); cf.cf_reset(c["R"])
            sev = []
            with torch.cuda.stream(stream):
                for i in range(W_seq):
                    step(i)
                for i in range(W_seq, W_seq + SEQ_STEPS):
                    step(i, sev)
            torch.cuda.synchronize()
            tot = 0.0
            for mi, c in enumerate(codecs):
                ms_c = sum(sev[k * stride + 2 * mi].elapsed_time(sev[k * stride + 2 * mi + 2])
                           for k in range(SEQ_STEPS)) / SEQ_STEPS
                seq_per[c["name"]].append(ms_c)
                tot += ms_c
            seq_step.append(tot)
        for c in codecs:
            if cf.cf_status(c["R"], stream) != cf.CF_OK or cf.cf_status(c["S"], stream) != cf.CF_OK:
                raise RuntimeError(f"codec {c['name']} reported an error status in the sequence runs")
        seq = dict(n=args.sequences, steps=SEQ_STEPS, step_ms=seq_step, per=seq_per)

    # e2e: pinned host activations in, pinned host reconstruction out, every
    # step.  Three streams and two buffer slots: the host-to-device copy of
    # step i+1 and the device-to-host copy of step i-1 run while step i is
    # encoded and decoded (PCIe is full duplex); each slot is reused only
    # after its previous contents were consumed.
    e2e = None
    if args.e2e_steps > 0:
        nslot = 2
        host_in = [[c["acts"][sl % n_inputs].cpu().pin_memory() for c in codecs] for sl in range(nslot)]
        host_out = [[torch.empty_like(c["rec"], device="cpu").pin_memory() for c in codecs] for sl in range(nslot)]
        dev_in = [[torch.empty_like(c["acts"][0]) for c in codecs] for _ in range(nslot)]
        dev_out = [[torch.empty_like(c["rec"]) for c in codecs] for _ in range(nslot)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nslot)]     # the slot's inputs are on the device
        ev_done = [torch.cuda.Event() for _ in range(nslot)]   # encode + decode of the slot finished
        ev_out = [torch.cuda.Event() for _ in range(nslot)]    # the slot's outputs are on the host
        for c in codecs:
            cf.cf_reset(c["S"]); cf.cf_reset(c["R"])

        def e2e_step(i):
            sl = i % nslot
            with torch.cuda.stream(h2d):
                if i >= nslot:
                    h2d.wait_event(ev_done[sl])
                for ci in range(len(codecs)):
                    dev_in[sl][ci].copy_(host_in[sl][ci], non_blocking=True)
                ev_in[sl].record(h2d)
            stream.wait_event(ev_in[sl])
            if i >= nslot:
                stream.wait_event(ev_out[sl])
            with torch.cuda.stream(stream):
                for ci, c in enumerate(codecs):
                    enc(c, dev_in[sl][ci])
                    dec(c, dev_out[sl][ci])
                ev_done[sl].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_done[sl])
                for ci in range(len(codecs)):
                    host_out[sl][ci].copy_(dev_out[sl][ci], non_blocking=True)
                ev_out[sl].record(d2h)

        n_warm = max(3, W_run)
        for i in range(n_warm):
            e2e_step(i)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(h2d)
        for i in range(n_warm, n_warm + args.e2e_steps):
            e2e_step(i)
        # the last device-to-host copy depends on every earlier copy and step
        a1.record(d2h)
        torch.cuda.synchronize()
        e2e_ms = a0.elapsed_time(a1) / args.e2e_steps
        e2e = dict(ms=e2e_ms, h2d=sum(t.numel() * t.element_size() for t in host_in[0]),
                   d2h=sum(t.numel() * t.element_size() for t in host_out[0]))
        for c in codecs:
            if cf.cf_status(c["R"], stream) != cf.CF_OK or cf.cf_status(c["S"], stream) != cf.CF_OK:
                raise RuntimeError(f"codec {c['name']} reported an error status in the e2e run")

    info = [dict(mode=c["mode"], kw=c["kw"], name=c["name"], P=c["P"]) for c in codecs]
    for c in codecs:
        cf.cf_destroy(c["S"]); cf.cf_destroy(c["R"])
    del codecs
    torch.cuda.empty_cache()

    ms_step = total_ms / K
    stats = dict(ms_step=ms_step, ms_step_instr=instr_ms / K, grouped=grouped,
                 per={m: {k: statistics.mean(v) for k, v in d.items()} for m, d in per.items()},
                 per_steps=per, e2e=e2e, clocks=clk, codecs=info, seq=seq)
    return stats


def _lr_alg_bytes(rows, cols, iters, payload, ef="explicit"):
    """Low-rank step's algorithmic bytes: read a, ahat, e and write ahat, e once
    (sender; implicit feedback reads no e), re-read the residual as one bf16
    copy per GEMM (2 per iteration), read and write the receiver's ahat and
    write recon, plus the payload twice."""
    E = rows * cols
    sender = 2 + 4 + (4 if ef == "explicit" else 0) + 4 + 4
    return E * (sender + 4 * iters) + E * (4 + 4 + 2) + 2 * payload


def run_suite(args, device):
    """The other workloads, timed the same way (inputs resident; per workload
    K encodes back to back then their K decodes, between CUDA events on the
    launching stream, beside a loop with an event around every call)."""
    import torch

    import activation_residual_compression_b200 as cf
    from activation_residual_compression_b200 import inputs

    peak, _ = _peaks()
    stream = torch.cuda.Stream()
    out = {}

    def timed(S, R, pay, recs, acts, steps, warm, batched, mk=None, dec_ws=0):
        """Evented loop on (S, R), then the grouped loop over (S, R) and, when
        mk is given, the extra pairs n_replicas(dec_ws) asks for: mk() makes
        one (S, R, pay, recs), warmed up here and destroyed after."""
        def one(S, R, pay, recs, i, evs=None, p=None):
            a = acts[i % len(acts)]
            p = pay if p is None else p
            if evs is not None:
                evs.append(torch.cuda.Event(enable_timing=True)); evs[-1].record(stream)
            if batched:
                cf.cf_encode_batched(S, [a[b] for b in range(a.shape[0])], p, stream)
            else:
                cf.cf_encode(S, a, p, stream)
            if evs is not None:
                evs.append(torch.cuda.Event(enable_timing=True)); evs[-1].record(stream)
            if batched:
                cf.cf_decode_batched(R, p, recs, stream)
            else:
                cf.cf_decode(R, p, recs, stream)
            if evs is not None:
                evs.append(torch.cuda.Event(enable_timing=True)); evs[-1].record(stream)
        with torch.cuda.stream(stream):
            for i in range(warm):
                one(S, R, pay, recs, i)
            evs = []
            for i in range(warm, warm + steps):
                one(S, R, pay, recs, i, evs)
        torch.cuda.synchronize()
        enc = [evs[3 * k].elapsed_time(evs[3 * k + 1]) for k in range(steps)]
        dec = [evs[3 * k + 1].elapsed_time(evs[3 * k + 2]) for k in range(steps)]

        # the same number of calls grouped: encodes back to back, then their decodes
        pairs = [(S, R, pay, recs)]
        if mk is not None:
            for _ in range(n_replicas(dec_ws) - 1):
                x = mk()
                with torch.cuda.stream(stream):
                    for i in range(warm + steps):
                        one(*x, i)
                pairs.append(x)
            torch.cuda.synchronize()
        j0 = warm + steps
        reps = []
        for (S_, R_, pay_, recs_) in pairs:
            def genc(j, p, S_=S_):
                a = acts[(j0 + j) % len(acts)]
                if batched:
                    cf.cf_encode_batched(S_, [a[b] for b in range(a.shape[0])], p, stream)
                else:
                    cf.cf_encode(S_, a, p, stream)

            def gdec(j, p, R_=R_, recs_=recs_):
                if batched:
                    cf.cf_decode_batched(R_, p, recs_, stream)
                else:
                    cf.cf_decode(R_, p, recs_, stream)
            reps.append((genc, gdec, pay_))
        g_enc, g_dec = grouped_times(reps, steps, stream)
        for (S_, R_, _, _) in pairs:
            if cf.cf_status(R_, stream) != cf.CF_OK or cf.cf_status(S_, stream) != cf.CF_OK:
                raise RuntimeError("suite: a codec reported an error status")
        for (S_, R_, _, _) in pairs[1:]:
            cf.cf_destroy(S_); cf.cf_destroy(R_)
        del pairs, reps
        return g_enc, g_dec, statistics.mean(enc), statistics.mean(dec)

    def make(rows, cols, mode, kw, batch=1):
        base = dict(dtype=cf.CF_BF16, batch=batch, **kw)
        S = cf.cf_create(rows, cols, cf.MODE_NAMES[mode], cf.cf_params_init(role=cf.CF_SENDER, **base))
        R = cf.cf_create(rows, cols, cf.MODE_NAMES[mode], cf.cf_params_init(role=cf.CF_RECEIVER, **base))
        pay = torch.empty(max(cf.cf_payload_bytes(S, True), cf.cf_payload_bytes(S, False)), dtype=torch.uint8,
                          device="cuda")
        return S, R, pay

    def entry(times, alg, act_bytes, P, **extra):
        e_ms, d_ms, ee_ms, de_ms = times
        t = (e_ms + d_ms) / 1e3
        return {"ms_per_step": round(e_ms + d_ms, 5), "encode_ms": round(e_ms, 5), "decode_ms": round(d_ms, 5),
                "activation_gbs": round(act_bytes / t / 1e9, 2), "roofline_frac": round(alg / t / 1e9 / peak, 4),
                "roofline_frac_datasheet": round(alg / t / 1e9 / DATASHEET_GBS, 4),
                "encode_ms_evented": round(ee_ms, 5), "decode_ms_evented": round(de_ms, 5),
                "roofline_frac_evented": round(alg / ((ee_ms + de_ms) / 1e3) / 1e9 / peak, 4),
                "payload_bytes": P, "ratio_vs_bf16": round(act_bytes / P, 2), **extra}

    # implicit error feedback on the FLUX-shaped stream: the form that settles to a
    # bounded steady state in every mode (the explicit recurrence diverges for N:M)
    for mode, kw in (("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}), ("nm", {"nm_n": 2, "nm_m": 16})):
        s = inputs.flux("cuda", rows=ROWS, cols=COLS, seed=6)
        acts = [s.next() for _ in range(24)]
        S, R, pay = make(ROWS, COLS, mode, dict(kw, ef=EF_CODES["implicit"]))
        rec = torch.empty(ROWS, COLS, dtype=torch.bfloat16, device="cuda")
        tt = timed(S, R, pay, rec, acts, 20, 4, False,
                   mk=lambda mode=mode, kw=kw: (*make(ROWS, COLS, mode, dict(kw, ef=EF_CODES["implicit"])),
                                                torch.empty_like(rec)),
                   dec_ws=ROWS * COLS * 10)
        alg = encode_bytes(mode, ROWS, COLS, kw, ef="implicit") + decode_bytes(mode, ROWS, COLS, kw)
        out[f"{_codec_name(mode, kw)}_flux_implicit"] = entry(tt, alg, ROWS * COLS * 2,
                                                              cf.cf_payload_bytes(S, False))
        cf.cf_destroy(S); cf.cf_destroy(R)
        del acts
    # block selection (the Otil page): 64 x 64 token grid x 3072 channels, 8 x 8 blocks, k/K = 16/64
    bkw = {"bs_grid_h": 64, "bs_block": 8, "bs_k": 16, "bs_warm": 5}
    s = inputs.blocksel("cuda", seed=1)
    acts = [s.next() for _ in range(28)]
    S, R, pay = make(4096, 3072, "blocksel", bkw)
    rec = torch.empty(4096, 3072, dtype=torch.bfloat16, device="cuda")
    tt = timed(S, R, pay, rec, acts, 20, bkw["bs_warm"] + 2, False,
               mk=lambda: (*make(4096, 3072, "blocksel", bkw), torch.empty_like(rec)), dec_ws=4096 * 3072 * 6)
    alg = encode_bytes("blocksel", 4096, 3072, bkw) + decode_bytes("blocksel", 4096, 3072, bkw)
    out["blocksel_grid64x64_3072_b8_k16"] = entry(tt, alg, 4096 * 3072 * 2, cf.cf_payload_bytes(S, False),
                                                  launches_per_step=3)
    cf.cf_destroy(S); cf.cf_destroy(R)
    del acts

    # N:M 1:16 and 2:16 on the FLUX-shaped stream
    for n in (1, 2):
        kw = {"nm_n": n, "nm_m": 16}
        s = inputs.flux("cuda", rows=ROWS, cols=COLS, seed=5)
        acts = [s.next() for _ in range(24)]
        S, R, pay = make(ROWS, COLS, "nm", kw)
        rec = torch.empty(ROWS, COLS, dtype=torch.bfloat16, device="cuda")
        tt = timed(S, R, pay, rec, acts, 20, 4, False,
                   mk=lambda kw=kw: (*make(ROWS, COLS, "nm", kw), torch.empty_like(rec)), dec_ws=ROWS * COLS * 10)
        alg = encode_bytes("nm", ROWS, COLS, kw) + decode_bytes("nm", ROWS, COLS, kw)
        P = 64 + _payload_body("nm", ROWS, COLS, kw)
        out[f"nm{n}_16_flux"] = entry(tt, alg, ROWS * COLS * 2, P)
        cf.cf_destroy(S); cf.cf_destroy(R)
        del acts
    # low-rank ~100x on 4096 x 3072, rank 70, INT4, 1 and 2 iterations (explicit
    # feedback, as specified), and 1 iteration with implicit feedback
    lr_rows, lr_cols = 4096, 3072
    for it, ef in ((1, "explicit"), (2, "explicit"), (1, "implicit")):
        s = inputs.ar1("cuda", rows=lr_rows, cols=lr_cols)
        acts = [s.next() for _ in range(28)]
        lkw = {"rank": 70, "iters": it, "lr_int4": 1, "seed": 7, "ef": EF_CODES[ef]}
        S, R, pay = make(lr_rows, lr_cols, "lowrank", lkw)
        rec = torch.empty(lr_rows, lr_cols, dtype=torch.bfloat16, device="cuda")
        tt = timed(S, R, pay, rec, acts, 20, 5, False,
                   mk=lambda lkw=lkw: (*make(lr_rows, lr_cols, "lowrank", lkw), torch.empty_like(rec)),
                   dec_ws=lr_rows * lr_cols * 10)
        P = cf.cf_payload_bytes(S, False)
        alg = _lr_alg_bytes(lr_rows, lr_cols, it, P, ef=ef)
        name = f"lowrank_r70_k{it}" + ("" if ef == "explicit" else "_implicit")
        out[name] = entry(tt, alg, lr_rows * lr_cols * 2, P,
                          launches_per_step=launches_per_call("lowrank", {"iters": it}, True) + 2,
                          budget_note="pages quote a ~1 ms compression budget")
        cf.cf_destroy(S); cf.cf_destroy(R)
        del acts
    # CogVideoX-2b-shaped full step: 60 tensors of 17550 x 1920, Q2, one launch each way
    if not args.no_cogvideox:
        B, cr, cc = 60, 17550, 1920
        s = inputs.cogvideox("cuda")
        acts = [s.next() for _ in range(3)]
        del s
        torch.cuda.empty_cache()
        S, R, pay = make(cr, cc, "q2", {}, batch=B)
        recs = [torch.empty(cr, cc, dtype=torch.bfloat16, device="cuda") for _ in range(B)]
        tt = timed(S, R, pay, recs, acts, 6, 2, True)
        E = B * cr * cc
        alg = B * (encode_bytes("q2", cr, cc, {}) + decode_bytes("q2", cr, cc, {}))
        out["cogvideox_q2_60x17550x1920"] = entry(tt, alg, E * 2, cf.cf_payload_bytes(S, False),
                                                  launches_per_step=2)
        cf.cf_destroy(S); cf.cf_destroy(R)
        del acts, recs
    torch.cuda.empty_cache()
    return out


EF_STUDY_MODES = [("sign1", {}), ("q2", {}), ("nm", {"nm_n": 1, "nm_m": 16}), ("nm", {"nm_n": 2, "nm_m": 16}),
                  ("lowrank", {"rank": 70, "iters": 1, "lr_int4": 1, "seed": 7})]
EF_STUDY_STEPS = (1, 2, 5, 10, 20, 27, 40, 49)


def run_ef_study(args, device, T=50):
    """Receiver error ||recon_t - a_t|| / ||a_t|| of the CUDA codec (C ABI) over
    T steps of the stationary AR(1) stream (rho = sqrt(0.99), innovations
    0.1 N(0, 1), so sigma_Delta / sigma_a ~ 0.1) for every mode and feedback
    form: explicit (the recurrence as specified), implicit (residual against
    the reconstruction only) and off (residual against the previous
    activation).  Streaming modes on 4608 x 3072 bf16, low-rank on 4096 x 3072."""
    import torch

    import activation_residual_compression_b200 as cf
    from activation_residual_compression_b200 import inputs
    torch.cuda.set_device(device)
    out = {}
    for mode, kw in EF_STUDY_MODES:
        rows, cols = (4096, 3072) if mode == "lowrank" else (ROWS, COLS)
        row = {}
        for ef in ("explicit", "implicit", "off"):
            base = dict(dtype=cf.CF_BF16, ef=EF_CODES[ef], **kw)
            S = cf.cf_create(rows, cols, cf.MODE_NAMES[mode], cf.cf_params_init(role=cf.CF_SENDER, **base))
            R = cf.cf_create(rows, cols, cf.MODE_NAMES[mode], cf.cf_params_init(role=cf.CF_RECEIVER, **base))
            pay = torch.empty(max(cf.cf_payload_bytes(S, True), cf.cf_payload_bytes(S, False)), dtype=torch.uint8,
                              device="cuda")
            rec = torch.empty(1, rows, cols, dtype=torch.bfloat16, device="cuda")
            s = inputs.ar1("cuda", rows=rows, cols=cols, seed=1)
            rel = []
            for _ in range(T):
                a = s.next()
                cf.cf_encode(S, a, pay)
                cf.cf_decode(R, pay, rec)
                af = a.float()
                rel.append(float(torch.linalg.vector_norm(rec.float() - af) / torch.linalg.vector_norm(af)))
            if cf.cf_status(R) != cf.CF_OK or cf.cf_status(S) != cf.CF_OK:
                raise RuntimeError(f"{mode} {ef}: codec reported an error status")
            cf.cf_destroy(S)
            cf.cf_destroy(R)
            row[ef] = {str(t): (round(rel[t], 5) if rel[t] < 1e6 else float(f"{rel[t]:.3e}")) for t in EF_STUDY_STEPS}
        out[_codec_name(mode, kw)] = row
    print(json.dumps({"ef_study": out, "metric": "receiver relative L2 error ||recon_t - a_t|| / ||a_t|| at step t",
                      "stream": "ar1 rho=sqrt(0.99) sigma=0.1 (stationary, sigma_Delta/sigma_a ~ 0.1)",
                      "steps": T, "data": "synthetic"}), flush=True)


# Low-rank settings at (about) one payload: INT4 factors at rank 70 against fp32
# factors at rank 9 (the rank that fits the same bytes), one and two sweeps,
# plus INT4 at rank 128 as the larger-payload point.
LR_SWEEP = [(70, 1, 1), (70, 2, 1), (9, 1, 0), (9, 2, 0), (128, 1, 1), (128, 2, 1), (35, 2, 1)]


def run_lr_sweep(args, device, T=50, ef="implicit"):
    """Low-rank quality sweep ("coverage over precision"): receiver error of
    the CUDA codec on the stationary AR(1) stream (4096 x 3072 bf16) for rank,
    sweeps and factor precision, with the payload bytes and the encode time."""
    import torch

    import activation_residual_compression_b200 as cf
    from activation_residual_compression_b200 import inputs
    torch.cuda.set_device(device)
    rows, cols = 4096, 3072
    out = []
    for rank, iters, int4 in LR_SWEEP:
        base = dict(dtype=cf.CF_BF16, ef=EF_CODES[ef], rank=rank, iters=iters, lr_int4=int4, seed=7)
        S = cf.cf_create(rows, cols, cf.MODE_NAMES["lowrank"], cf.cf_params_init(role=cf.CF_SENDER, **base))
        R = cf.cf_create(rows, cols, cf.MODE_NAMES["lowrank"], cf.cf_params_init(role=cf.CF_RECEIVER, **base))
        P = cf.cf_payload_bytes(S, False)
        pay = torch.empty(max(cf.cf_payload_bytes(S, True), P), dtype=torch.uint8, device="cuda")
        rec = torch.empty(1, rows, cols, dtype=torch.bfloat16, device="cuda")
        s = inputs.ar1("cuda", rows=rows, cols=cols, seed=1)
        rel, enc_ms = [], []
        for t in range(T):
            a = s.next()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            cf.cf_encode(S, a, pay)
            e1.record()
            cf.cf_decode(R, pay, rec)
            af = a.float()
            rel.append(float(torch.linalg.vector_norm(rec.float() - af) / torch.linalg.vector_norm(af)))
            torch.cuda.synchronize()
            if t >= 3:
                enc_ms.append(e0.elapsed_time(e1))
        if cf.cf_status(R) != cf.CF_OK or cf.cf_status(S) != cf.CF_OK:
            raise RuntimeError(f"rank {rank} iters {iters}: codec reported an error status")
        cf.cf_destroy(S)
        cf.cf_destroy(R)
        out.append({"rank": rank, "iters": iters, "factors": "int4" if int4 else "fp32", "payload_bytes": P,
                    "ratio_vs_bf16": round(rows * cols * 2 / P, 1),
                    "rel_err": {str(t): round(rel[t], 5) for t in EF_STUDY_STEPS},
                    "steady_rel_err": round(statistics.mean(rel[T // 2:]), 5),
                    "encode_ms": round(statistics.median(enc_ms), 4)})
    print(json.dumps({"lr_sweep": out, "metric": "receiver relative L2 error ||recon_t - a_t|| / ||a_t||",
                      "stream": "ar1 4096x3072 bf16 rho=sqrt(0.99) sigma=0.1", "error_feedback": ef,
                      "steps": T, "data": "synthetic"}), flush=True)


# Sequence-parallel exchange: one token shard per rank of the FLUX-shaped activation
# (4608 tokens over the pages' 4 GPUs: 1152 rows x 3072 channels bf16), the per-rank
# shard fixed as ranks are added (weak scaling), several exchanged tensors per step.
EXCHANGE = dict(rows=1152, cols=3072, tensors=4, mode="q2", kw={})


def exchange_bench(ex, shards_at, steps, warmup, device, group=None):
    """Time the exchange `ex` (an SPExchange) over `steps` steps after `warmup`
    untimed ones; `shards_at(t)` gives the rank's shards of step t.  Two timed
    passes on the same inputs: the exchange step itself, and the same codec
    work with no collective (the rank's encodes and one decode per peer from
    its own payload), so that exposed communication = step - codec work.
    Times are the max over ranks (CUDA events on a GPU, wall clock on a CPU)."""
    import torch
    import torch.distributed as dist

    cuda = torch.device(device).type == "cuda"

    def clock(fn, n, t0):
        if cuda:
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for t in range(t0, t0 + n):
                fn(t)
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b)
        else:
            t = time.perf_counter()
            for k in range(t0, t0 + n):
                fn(k)
            ms = (time.perf_counter() - t) * 1e3
        m = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(m, op=dist.ReduceOp.MAX, group=group)
        return float(m[0]) / n

    def codec_only(t):
        for ch, a in zip(ex.channels, shards_at(t)):
            P = ch.sender.payload_bytes(ch.sender.next_is_warm())
            ch.sender.encode(a, ch.send_buf[:P], torch.cuda.current_stream() if cuda else None)
            for p, rx in ch.receivers.items():
                rx.decode(ch.send_buf[:P], ch.scratch_out, torch.cuda.current_stream() if cuda else None)

    for t in range(warmup):
        ex.step(shards_at(t))
    step_ms = clock(lambda t: ex.step(shards_at(t)), steps, warmup)
    st = ex.status()
    # the codec-only pass runs fresh states (receivers fed by this rank's own payloads)
    ex.reset()
    for ch in ex.channels:
        ch.scratch_out = torch.empty(ex.rows, ex.cols, dtype=ex.act_dtype, device=device)
    for t in range(warmup):
        codec_only(t)
    codec_ms = clock(codec_only, steps, warmup)
    ex.reset()
    world = ex.world
    act = len(ex.channels) * world * ex.rows * ex.cols * 2
    return {"ms_per_step": round(step_ms, 5), "codec_ms_per_step": round(codec_ms, 5),
            "exposed_comm_ms": round(max(step_ms - codec_ms, 0.0), 5),
            "activation_gbs_per_rank": round(act / (step_ms / 1e3) / 1e9, 3),
            "activation_gbs_all_ranks": round(world * act / (step_ms / 1e3) / 1e9, 3),
            "payload_bytes_per_tensor": ex.channels[0].sender.payload_bytes(False),
            "status": st}


def run_exchange(args, rank, world, local):
    """The payload exchange over NCCL on this node's GPUs (one rank per GPU)."""
    import torch
    import torch.distributed as dist

    from activation_residual_compression_b200 import inputs
    from activation_residual_compression_b200.exchange import SPExchange

    X = EXCHANGE
    streams = [inputs.flux("cuda", rows=X["rows"], cols=X["cols"], seed=11 + 100 * i + 1000 * rank)
               for i in range(X["tensors"])]
    n = args.warmup + args.steps
    acts = [[s.next()[0] for _ in range(n)] for s in streams]
    del streams
    ex = SPExchange(X["rows"], X["cols"], X["mode"], n_tensors=X["tensors"], **X["kw"])
    try:
        res = exchange_bench(ex, lambda t: [a[t % n] for a in acts], args.steps, args.warmup, f"cuda:{local}")
    finally:
        ex.close()
    res.update({"ranks": world, "transport": "nccl all_gather_into_tensor on a communication stream",
                "shard": f"{X['rows']}x{X['cols']} bf16 per rank per tensor", "tensors": X["tensors"],
                "mode": X["mode"], "scaling": "weak (fixed shard per rank)"})
    return res


def _oracle_kw(mode, kw):
    """The oracle's names for a codec's parameters."""
    if mode == "blocksel":
        return {"bs_h": kw["bs_grid_h"], "bs_block": kw["bs_block"], "bs_k": kw["bs_k"], "bs_warm": kw["bs_warm"]}
    return kw


BS_STUDY_K = (4, 8, 16, 32, 64)   # of K = 64 blocks: k/K = 1/16, 1/8, 1/4, 1/2, 1


def run_bs_study(args, device, T=50):
    """Block selection (Otil page, "Ablation: transmitted fraction k/K"): receiver
    error and step time of the CUDA codec on the block-scaled random walk
    (64 x 64 tokens x 3072 channels bf16, 8 x 8 blocks) for several k."""
    import torch

    import activation_residual_compression_b200 as cf
    from activation_residual_compression_b200 import inputs
    torch.cuda.set_device(device)
    rows, cols = 4096, 3072
    out = []
    for k in BS_STUDY_K:
        kw = {"bs_grid_h": 64, "bs_block": 8, "bs_k": k, "bs_warm": 5}
        base = dict(dtype=cf.CF_BF16, **kw)
        S = cf.cf_create(rows, cols, cf.MODE_NAMES["blocksel"], cf.cf_params_init(role=cf.CF_SENDER, **base))
        R = cf.cf_create(rows, cols, cf.MODE_NAMES["blocksel"], cf.cf_params_init(role=cf.CF_RECEIVER, **base))
        P = cf.cf_payload_bytes(S, False)
        pay = torch.empty(max(cf.cf_payload_bytes(S, True), P), dtype=torch.uint8, device="cuda")
        rec = torch.empty(1, rows, cols, dtype=torch.bfloat16, device="cuda")
        s = inputs.blocksel("cuda", seed=1)
        rel, ms = [], []
        for t in range(T):
            a = s.next()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            cf.cf_encode(S, a, pay)
            cf.cf_decode(R, pay, rec)
            e1.record()
            af = a.float()
            rel.append(float(torch.linalg.vector_norm(rec.float() - af) / torch.linalg.vector_norm(af)))
            torch.cuda.synchronize()
            if t >= kw["bs_warm"] + 2:
                ms.append(e0.elapsed_time(e1))
        if cf.cf_status(R) != cf.CF_OK:
            raise RuntimeError(f"k {k}: codec reported an error status")
        cf.cf_destroy(S)
        cf.cf_destroy(R)
        out.append({"k": k, "k_over_K": f"{k}/64", "payload_bytes": P, "ratio_vs_bf16": round(rows * cols * 2 / P, 2),
                    "rel_err": {str(t): round(rel[t], 5) for t in EF_STUDY_STEPS},
                    "steady_rel_err": round(statistics.mean(rel[T // 2:]), 5),
                    "ms_per_step": round(statistics.median(ms), 4)})
    print(json.dumps({"bs_study": out, "metric": "receiver relative L2 error ||recon_t - a_t|| / ||a_t||",
                      "stream": "random walk, per-8x8-block innovation scale log-uniform in [0.01, 0.3]",
                      "steps": T, "data": "synthetic"}), flush=True)


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_leg(wl, max_seconds, max_steps=SEQ_STEPS):
    """The CPU oracle, as it stands, on full-size tensors of a workload's stream
    (for a many-tensor step its first tensor only: tensors are independent);
    compressed steps until max_seconds of oracle time, at least one (the
    leading full-size steps untimed).  Returns (activation GB/s, steps, seconds)."""
    import numpy as np
    import torch

    import oracle
    from activation_residual_compression_b200 import inputs

    R_, C_, B_ = wl["rows"], wl["cols"], wl["batch"]
    orcs = []
    for mi, (mode, kw) in enumerate(wl["codecs"]):
        if wl["stream"] == "cogvideox":   # the first tensor of the step (seed and sigma of layer 0)
            s = inputs.ActivationStream(R_, C_, dtype=torch.bfloat16, device="cpu", seed_per_tensor=[1000],
                                        sigma_per_tensor=inputs.cogvideox_sigmas(B_)[:1])
        else:
            s = _make_stream(wl["stream"], wl, seed=1 + 100 * mi, device="cpu")
        o = oracle.Oracle(R_, C_, mode, dtype="bf16", batch=1, **_oracle_kw(mode, kw))
        for _ in range(kw.get("bs_warm", 1)):     # the full-size leading steps, untimed
            a = s.next().view(torch.int16).numpy().view(np.uint16)
            o.decode(o.encode(a))
        orcs.append((s, o))
    spent, steps = 0.0, 0
    while steps < 1 or (spent < max_seconds and steps < max_steps):
        ins = [s.next().view(torch.int16).numpy().view(np.uint16) for s, _ in orcs]
        t = time.perf_counter()
        for (s, o), a in zip(orcs, ins):
            o.decode(o.encode(a))
        spent += time.perf_counter() - t
        steps += 1
    return steps * len(orcs) * R_ * C_ * 2 / spent / 1e9, steps, spent


def cpu_baseline(wl=None, max_seconds=10.0, per_workload_seconds=4.0):
    """The oracle timed on the host cores, as a baseline (not the target): the
    timed workload with every core and with one thread, and a bounded sample of
    each other workload (every core)."""
    import oracle

    wl = wl or WORKLOADS["flux"]
    cores = oracle.set_threads(int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)))
    val, steps, spent = _oracle_leg(wl, max_seconds)
    oracle.set_threads(1)
    val1, steps1, spent1 = _oracle_leg(wl, max_seconds)
    oracle.set_threads(cores)
    modes = "+".join(_codec_name(m, k) for m, k in wl["codecs"])
    others = {}
    for key in ("nm", "lowrank", "cogvideox", "blocksel"):
        w = WORKLOADS[key]
        if w["name"] == wl["name"]:
            continue
        v, n, t = _oracle_leg(w, per_workload_seconds)
        others[w["name"]] = {"value": round(v, 5), "unit": "GB/s", "steps": n, "seconds": round(t, 2),
                             "modes": "+".join(_codec_name(m, k) for m, k in w["codecs"]),
                             **({"tensors_of_step": f"1 of {w['batch']}"} if w["batch"] > 1 else {})}
    return {"value": round(val, 5), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{steps} compressed steps of one full {wl['rows']}x{wl['cols']} bf16 tensor"
                      + (f" (of the {wl['batch']}-tensor step)" if wl["batch"] > 1 else "")
                      + f", modes {modes} (encode+decode), {spent:.1f} s of oracle time",
            "ms_per_step": round(spent / steps * 1e3, 2), "cpu_model": _cpu_model(),
            "single_thread": {"value": round(val1, 5), "unit": "GB/s", "cores": 1, "steps": steps1,
                              "seconds": round(spent1, 2)},
            "other_workloads": others}


def run_reference(args):
    """The oracle as the reference arm, on the workload's codecs.  Streaming
    modes: each step is encode + decode of a 1152-row sample of the stream
    (rows are independent in these modes, so a row sample is the same per-row
    work); the low-rank mode couples all rows, so its steps are full tensors."""
    import numpy as np
    import torch

    import oracle
    from activation_residual_compression_b200 import inputs

    wl = WORKLOADS[args.workload]
    R_, C_ = wl["rows"], wl["cols"]
    coupled = any(m in ("lowrank", "blocksel") for m, _ in wl["codecs"])   # rows not independent
    rows = R_ if coupled else 1152
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    orcs = []
    for mi, (mode, kw) in enumerate(wl["codecs"]):
        sub = dict(wl, rows=rows)
        if wl["stream"] == "cogvideox":
            s = inputs.ActivationStream(rows, C_, dtype=torch.bfloat16, device="cpu", seed_per_tensor=[1000],
                                        sigma_per_tensor=inputs.cogvideox_sigmas(wl["batch"])[:1])
        else:
            s = _make_stream(wl["stream"], sub, seed=1 + 100 * mi, device="cpu")
        okw = dict(_oracle_kw(mode, kw))
        if mode != "blocksel":
            okw["ef"] = args.ef
            if args.state == "bf16" and mode != "lowrank":
                okw["state_dtype"] = "bf16"
        orcs.append((s, oracle.Oracle(rows, C_, mode, dtype="bf16", **okw)))

    def one():
        ins = [s.next().view(torch.int16).numpy().view(np.uint16) for s, _ in orcs]
        t = time.perf_counter()
        for (s, o), a in zip(orcs, ins):
            o.decode(o.encode(a))
        return time.perf_counter() - t

    for _ in range(max([1] + [kw.get("bs_warm", 1) for _, kw in wl["codecs"]])):
        one()  # the stream's full-size leading steps
    for _ in range(args.warmup):
        one()
    spent = sum(one() for _ in range(args.steps))
    ms = spent / args.steps * 1e3
    val = len(orcs) * rows * C_ * 2 / (ms / 1e3) / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {**workload_config(args, wl, args.gpus), "sample_rows": rows},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} of {R_} rows x {C_} bf16 per step, "
                                       f"{'+'.join(_codec_name(m, k) for m, k in wl['codecs'])}"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cf", choices=["cf", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--sequences", type=int, default=5,
                    help="full request sequences (27 compressed steps each) timed after the main region; 0: none")
    ap.add_argument("--max-resident", type=int, default=400, help="pre-generated inputs per mode (cycled)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-suite", action="store_true", help="skip the supplementary workloads")
    ap.add_argument("--workload", default="flux", choices=sorted(WORKLOADS),
                    help="timed workload (default: the FLUX-shaped 1-bit + 2-bit step)")
    ap.add_argument("--resident-gb", type=float, default=12.0, help="device memory for pre-generated inputs")
    ap.add_argument("--no-cogvideox", action="store_true", help="skip the 60-tensor CogVideoX-shaped step")
    ap.add_argument("--ef", default="explicit", choices=sorted(EF_CODES),
                    help="error-feedback form of the timed codecs (default: explicit)")
    ap.add_argument("--state", default="f32", choices=["f32", "bf16"],
                    help="state dtype of the timed streaming codecs (default fp32; bf16: the bf16-state option)")
    ap.add_argument("--ef-study", action="store_true",
                    help="instead of timing: receiver error per step of every mode and feedback form")
    ap.add_argument("--lr-sweep", action="store_true",
                    help="instead of timing: low-rank receiver error over rank, sweeps and factor precision")
    ap.add_argument("--exchange", action="store_true",
                    help="also time the sequence-parallel payload exchange (always on with several GPUs)")
    ap.add_argument("--bs-study", action="store_true",
                    help="instead of timing: block-selection receiver error and step time over k/K")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU fallback)")
    if args.ef_study or args.lr_sweep or args.bs_study:
        if rank == 0:
            (run_ef_study if args.ef_study else run_lr_sweep if args.lr_sweep else run_bs_study)(args, local)
        return
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    st = run_cf(args, rank, world, local)
    wl = WORKLOADS[args.workload]
    R_, C_, B_ = wl["rows"], wl["cols"], wl["batch"]
    ms = st["ms_step"]
    ms_instr = st["ms_step_instr"]
    e2e_ms = st["e2e"]["ms"] if st["e2e"] else None
    if dist:
        t = torch.tensor([ms, e2e_ms or 0.0, ms_instr], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, e2e_ms, ms_instr = float(t[0]), float(t[1]), float(t[2])
    n_codecs = len(st["codecs"])
    act_bytes = n_codecs * B_ * R_ * C_ * 2 * world
    value = act_bytes / (ms / 1e3) / 1e9
    peak, peak_kind = _peaks()
    c0 = st["codecs"][0]
    enc_ms = st["grouped"][c0["name"]]["enc"]
    if c0["mode"] == "lowrank":
        E = R_ * C_
        enc_alg = E * (2 + 16 + 4 * c0["kw"]["iters"]) + c0["P"]
        kern = f"cf_encode low-rank ({launches_per_call(c0['mode'], c0['kw'], True)} launches)"
        tr = None
    elif c0["mode"] == "blocksel":
        enc_alg = encode_bytes(c0["mode"], R_, C_, c0["kw"])
        kern = f"cf_encode block selection ({launches_per_call(c0['mode'], c0['kw'], True)} launches)"
        tr = None
    else:
        zs = 2 if args.state == "bf16" else 4
        enc_alg = B_ * encode_bytes(c0["mode"], R_, C_, c0["kw"], ef=args.ef, state_size=zs)
        kern = f"encode_kernel<{c0['name']}, bf16" + (", bf16 state>" if zs == 2 else ">")
        tr = _traffic_record() if args.workload == "flux" and args.ef == "explicit" and zs == 4 else None
    achieved = enc_alg / (enc_ms / 1e3) / 1e9
    per_mode = {}
    for c in st["codecs"]:
        pm = st["grouped"][c["name"]]
        pe = st["per"][c["name"]]
        step_ms = pm["enc"] + pm["dec"]
        alg = B_ * step_bytes(c["mode"], R_, C_, c["kw"], c["P"], ef=args.ef,
                              state_size=2 if args.state == "bf16" else 4)
        per_mode[c["name"]] = {"ms_per_step": round(step_ms, 5), "encode_ms": round(pm["enc"], 5),
                               "decode_ms": round(pm["dec"], 5),
                               "encode_ms_evented": round(pe["enc"], 5), "decode_ms_evented": round(pe["dec"], 5),
                               "roofline_frac_evented": round(alg / ((pe["enc"] + pe["dec"]) / 1e3) / 1e9 / peak, 4),
                               "activation_gbs": round(B_ * R_ * C_ * 2 / (step_ms / 1e3) / 1e9, 2),
                               "hbm_gbs": round(alg / (step_ms / 1e3) / 1e9, 1),
                               "roofline_frac": round(alg / (step_ms / 1e3) / 1e9 / peak, 4),
                               "roofline_frac_datasheet": round(alg / (step_ms / 1e3) / 1e9 / DATASHEET_GBS, 4),
                               "payload_bytes": c["P"],
                               "ratio_vs_bf16": round(B_ * R_ * C_ * 2 / c["P"], 2)}
    in_mb = B_ * R_ * C_ * 2 / 1e6
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "ms_per_step_instrumented": round(ms_instr, 5),
        "timing": "value and ms_per_step: K steps between two CUDA events; per_mode and roofline: per codec K "
                  "encodes back to back (one payload slot each) between two events, then their K decodes between "
                  "two more, so no event sits between two kernels; *_evented and ms_per_step_instrumented: a loop "
                  "of K steps with an event around every encode and decode (each such event adds ~2.7 us of device "
                  "time between two kernels)",
        "config": {**workload_config(args, wl, world),
                   "l2": f"inputs larger than L2: a fresh {in_mb:.0f} MB input per codec per step, state "
                         f"{B_ * R_ * C_ * state_bytes_per_elem(args) / 1e6:.0f} MB per codec",
                   "inputs_resident": True},
        "per_mode": per_mode,
        "roofline": {"bound": "hbm", "kernel": kern, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": (tr["bytes_per_launch"] if tr else None),
                     "algorithmic_bytes": enc_alg, "peak_source": peak_kind,
                     "datasheet_peak": DATASHEET_GBS, "frac_of_datasheet": round(achieved / DATASHEET_GBS, 4)},
        "gpu_launches": sum(launches_per_call(c["mode"], c["kw"], True) + launches_per_call(c["mode"], c["kw"], False)
                            for c in st["codecs"]) * args.steps,
        "clocks": st["clocks"],
    }
    if st["seq"]:
        sq = st["seq"]
        med = statistics.median(sq["step_ms"])
        line["sequences"] = {
            "n": sq["n"], "compressed_steps_each": sq["steps"],
            "what": "each a new request (states reset, warm-up step untimed); per sequence the mean "
                    "encode+decode time per step over all codecs",
            "ms_per_step_median": round(med, 5), "ms_per_step_min": round(min(sq["step_ms"]), 5),
            "ms_per_step_max": round(max(sq["step_ms"]), 5),
            "activation_gbs_median": round(n_codecs * B_ * R_ * C_ * 2 / (med / 1e3) / 1e9, 2),
            "per_mode_ms_median": {m: round(statistics.median(v), 5) for m, v in sq["per"].items()},
            "per_mode_roofline_frac_median": {
                c["name"]: round(B_ * step_bytes(c["mode"], R_, C_, c["kw"], c["P"], ef=args.ef,
                                                 state_size=2 if args.state == "bf16" else 4)
                                 / (statistics.median(sq["per"][c["name"]]) / 1e3) / 1e9 / peak, 4)
                for c in st["codecs"]}}
    if e2e_ms:
        line["e2e"] = {"value": round(act_bytes / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                       "h2d_bytes_per_step": st["e2e"]["h2d"], "d2h_bytes_per_step": st["e2e"]["d2h"],
                       "ms_per_step": round(e2e_ms, 4)}
    if args.exchange or world > 1:
        own_group = dist is None
        if own_group:   # a one-rank NCCL group for the exchange on this GPU
            import datetime
            import socket

            import torch.distributed as dist
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ["MASTER_PORT"] = str(port)
            dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        line["exchange"] = run_exchange(args, rank, world, local)
        if own_group:
            dist.destroy_process_group()
            dist = None
    if world == 1 and not args.no_suite and args.workload == "flux" and args.ef == "explicit" and args.state == "f32":
        line["suite"] = run_suite(args, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
