"""CPU oracle for residual compression with error feedback -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and this package never imports the
product: the two share no code.

The arithmetic lives in ``cf_oracle.c`` (plain scalar C, compiled with
``-ffp-contract=off``); this module only builds it and marshals numpy arrays.
Source of the method: "Accelerating Parallel Diffusion Model Serving with
Residual Compression" (NeurIPS 2025 paper notes), sections "Overall framework",
"Key design" (residual compression, error feedback, low-rank strategy) and
"Limitations" (first step sent in full).

Activations are numpy arrays: float32, or uint16 holding bfloat16 bit patterns.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cf_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

MODES = {"identity": 0, "sign1": 1, "q2": 2, "nm": 3, "lowrank": 4, "blocksel": 5}
DTYPES = {"f32": 0, "bf16": 1}
EFS = {"explicit": 0, "implicit": 1, "off": 2}


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to the source (gcc, -O2, no FP contraction)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        c = ctypes
        P = c.c_void_p
        L.orc_create.restype = P
        L.orc_create.argtypes = [c.c_int64, c.c_int64, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int,
                                 c.c_int, c.c_int, c.c_int, c.c_int, c.c_uint64]
        L.orc_destroy.argtypes = [P]
        L.orc_payload_bytes.restype = c.c_size_t
        L.orc_payload_bytes.argtypes = [P, c.c_int]
        L.orc_tensor_body_bytes.restype = c.c_size_t
        L.orc_tensor_body_bytes.argtypes = [P]
        L.orc_encode.restype = c.c_int
        L.orc_encode.argtypes = [P, P, P]
        L.orc_decode.restype = c.c_int
        L.orc_decode.argtypes = [P, P, P]
        L.orc_payload_meaning.restype = c.c_int
        L.orc_payload_meaning.argtypes = [P, P, c.c_int, P]
        L.orc_buffer.restype = P
        L.orc_buffer.argtypes = [P, c.c_int]
        L.orc_step.restype = c.c_uint64
        L.orc_step.argtypes = [P, c.c_int]
        L.orc_status.restype = c.c_int
        L.orc_status.argtypes = [P]
        L.orc_set_vprev_valid.argtypes = [P, c.c_int]
        L.orc_set_step.argtypes = [P, c.c_uint64, c.c_uint64]
        L.orc_bf16_from_f32.restype = c.c_uint16
        L.orc_bf16_from_f32.argtypes = [c.c_float]
        L.orc_f32_from_bf16.restype = c.c_float
        L.orc_f32_from_bf16.argtypes = [c.c_uint16]
        L.orc_bf16_from_f32_array.argtypes = [P, P, c.c_int64]
        L.orc_f32_from_bf16_array.argtypes = [P, P, c.c_int64]
        L.orc_sign1_scale.restype = c.c_uint16
        L.orc_sign1_scale.argtypes = [P, c.c_int64]
        L.orc_q2_scale.restype = c.c_uint16
        L.orc_q2_scale.argtypes = [P, c.c_int64]
        L.orc_q2_code.restype = c.c_int
        L.orc_q2_code.argtypes = [c.c_float, c.c_float]
        L.orc_q2_level.restype = c.c_float
        L.orc_q2_level.argtypes = [c.c_int, c.c_float]
        L.orc_nm_select.argtypes = [P, c.c_int, c.c_int, P]
        L.orc_set_threads.restype = c.c_int
        L.orc_set_threads.argtypes = [c.c_int]
        L.orc_splitmix64.restype = c.c_uint64
        L.orc_splitmix64.argtypes = [c.c_uint64]
        L.orc_lr_v0.restype = c.c_float
        L.orc_lr_v0.argtypes = [c.c_uint64, c.c_int64, c.c_int, c.c_int]
        L.orc_householder_qr.argtypes = [P, c.c_int64, c.c_int, c.c_double, P, P, P]
        L.orc_subspace_iteration.argtypes = [P, c.c_int64, c.c_int64, c.c_int, c.c_int, P, P]
        L.orc_set_state_bf16.restype = c.c_int
        L.orc_set_state_bf16.argtypes = [P, c.c_int]
        L.orc_next_is_warm.restype = c.c_int
        L.orc_next_is_warm.argtypes = [P, c.c_int]
        L.orc_set_blocksel.restype = c.c_int
        L.orc_set_blocksel.argtypes = [P, c.c_int, c.c_int, c.c_int, c.c_int]
        L.orc_blocksel_sent.restype = P
        L.orc_blocksel_sent.argtypes = [P]
        L.orc_blocksel_dissimilarity.restype = c.c_int
        L.orc_blocksel_dissimilarity.argtypes = [P, P, P, P]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalar pieces

def bf16_from_f32(x) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 values, round-to-nearest-even."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_bf16_from_f32_array(_ptr(x), _ptr(out), x.size)
    return out


def f32_from_bf16(h) -> np.ndarray:
    h = np.ascontiguousarray(np.asarray(h, dtype=np.uint16))
    out = np.empty(h.shape, dtype=np.float32)
    lib().orc_f32_from_bf16_array(_ptr(h), _ptr(out), h.size)
    return out


def sign1_scale(d) -> int:
    d = np.ascontiguousarray(d, dtype=np.float32)
    return int(lib().orc_sign1_scale(_ptr(d), d.size))


def q2_scale(d) -> int:
    d = np.ascontiguousarray(d, dtype=np.float32)
    return int(lib().orc_q2_scale(_ptr(d), d.size))


def q2_code(d: float, S: float) -> int:
    return int(lib().orc_q2_code(float(d), float(S)))


def q2_level(q: int, S: float) -> float:
    return float(lib().orc_q2_level(int(q), float(S)))


def nm_select(d, n: int) -> list[int]:
    d = np.ascontiguousarray(d, dtype=np.float32)
    out = np.zeros(n, dtype=np.int32)
    lib().orc_nm_select(_ptr(d), d.size, n, _ptr(out))
    return [int(v) for v in out]


def set_threads(n: int) -> int:
    """Threads of the oracle's row-parallel loops (timing only); returns the count in effect."""
    return int(lib().orc_set_threads(int(n)))


def splitmix64(x: int) -> int:
    return int(lib().orc_splitmix64(x & (2 ** 64 - 1)))


def lr_v0(seed: int, cols: int, r: int) -> np.ndarray:
    out = np.empty((cols, r), dtype=np.float32)
    L = lib()
    for j in range(cols):
        for k in range(r):
            out[j, k] = L.orc_lr_v0(seed, j, r, k)
    return out


def householder_qr(Y: np.ndarray, tol: float = 1e-6):
    Y = np.ascontiguousarray(Y, dtype=np.float64)
    m, r = Y.shape
    Q = np.empty((m, r), dtype=np.float64)
    rd = np.empty(r, dtype=np.float64)
    dead = np.empty(r, dtype=np.int32)
    lib().orc_householder_qr(_ptr(Y), m, r, tol, _ptr(Q), _ptr(rd), _ptr(dead))
    return Q, rd, dead.astype(bool)


def subspace_iteration(D: np.ndarray, V0: np.ndarray, iters: int):
    D = np.ascontiguousarray(D, dtype=np.float32)
    V = np.ascontiguousarray(V0, dtype=np.float64).copy()
    m, n = D.shape
    r = V.shape[1]
    Q = np.empty((m, r), dtype=np.float64)
    lib().orc_subspace_iteration(_ptr(D), m, n, r, iters, _ptr(V), _ptr(Q))
    return Q, V


# ---------------------------------------------------------------- stateful codec

class Oracle:
    """One compression stream (sender and receiver state) on the CPU.

    ``a`` passed to :meth:`encode` has shape ``(batch, rows, cols)`` (or
    ``(rows, cols)`` when batch == 1): float32, or uint16 bf16 patterns.
    """

    def __init__(self, rows, cols, mode, dtype="bf16", ef="explicit", nm_n=1, nm_m=16,
                 rank=1, iters=1, lr_int4=1, batch=1, seed=0, bs_h=0, bs_block=8, bs_k=0, bs_warm=5,
                 state_dtype="f32"):
        self.rows, self.cols, self.batch = int(rows), int(cols), int(batch)
        self.mode = mode
        self.dtype = dtype
        self.rank = int(rank)
        self._h = lib().orc_create(self.rows, self.cols, MODES[mode], DTYPES[dtype], EFS[ef],
                                   nm_n, nm_m, rank, iters, lr_int4, batch, seed)
        if not self._h:
            raise ValueError("oracle rejected the configuration")
        if state_dtype != "f32" and lib().orc_set_state_bf16(self._h, 1) != 0:
            raise ValueError("the bf16 state needs a streaming mode on bf16 activations")
        if mode == "blocksel":
            # the grid defaults to square; k to a quarter of the blocks ("k/K = 1/4")
            h = int(bs_h) or math.isqrt(self.rows)
            K = (h // bs_block) * ((self.rows // h) // bs_block) if h else 0
            self.bs_h, self.bs_w, self.bs_b = h, (self.rows // h if h else 0), int(bs_block)
            self.bs_K = K
            self.bs_k = int(bs_k) or max(1, K // 4)
            self.bs_warm = int(bs_warm)
            if lib().orc_set_blocksel(self._h, h, self.bs_b, self.bs_k, self.bs_warm) != 0:
                raise ValueError("oracle rejected the block-selection configuration")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._h = None
            try:
                lib().orc_destroy(h)
            except TypeError:   # interpreter shutdown: the module globals are gone
                pass

    @property
    def np_act(self):
        return np.uint16 if self.dtype == "bf16" else np.float32

    def next_is_warm(self, receiver: bool = False) -> bool:
        """The next encode (receiver: decode) is a full-size warm-up step."""
        return lib().orc_next_is_warm(self._h, 1 if receiver else 0) != 0

    def payload_bytes(self, warmup: bool) -> int:
        return int(lib().orc_payload_bytes(self._h, 1 if warmup else 0))

    def body_bytes(self) -> int:
        return int(lib().orc_tensor_body_bytes(self._h))

    def step(self, receiver=False) -> int:
        return int(lib().orc_step(self._h, 1 if receiver else 0))

    def status(self) -> int:
        return int(lib().orc_status(self._h))

    def encode(self, a) -> np.ndarray:
        a = np.ascontiguousarray(a, dtype=self.np_act)
        assert a.size == self.batch * self.rows * self.cols
        warm = lib().orc_next_is_warm(self._h, 0) != 0
        out = np.zeros(self.payload_bytes(warm), dtype=np.uint8)
        lib().orc_encode(self._h, _ptr(a), _ptr(out))
        return out

    def decode(self, payload: np.ndarray):
        payload = np.ascontiguousarray(payload, dtype=np.uint8)
        recon = np.zeros((self.batch, self.rows, self.cols), dtype=self.np_act)
        st = lib().orc_decode(self._h, _ptr(payload), _ptr(recon))
        return recon, int(st)

    def meaning(self, payload: np.ndarray, b: int = 0) -> np.ndarray:
        """C(Delta) that tensor b of a steady-state payload stands for."""
        payload = np.ascontiguousarray(payload, dtype=np.uint8)
        C = np.empty((self.rows, self.cols), dtype=np.float32)
        lib().orc_payload_meaning(self._h, _ptr(payload), b, _ptr(C))
        return C

    def _buf(self, which: int, shape):
        p = lib().orc_buffer(self._h, which)
        n = int(np.prod(shape))
        arr = np.ctypeslib.as_array((ctypes.c_float * n).from_address(p))
        return arr.reshape(shape)

    # live views of the state (writable: tests use them to teacher-force)
    @property
    def ahat_s(self):
        return self._buf(0, (self.batch, self.rows, self.cols))

    @property
    def err(self):
        return self._buf(1, (self.batch, self.rows, self.cols))

    @property
    def ahat_r(self):
        return self._buf(2, (self.batch, self.rows, self.cols))

    @property
    def vprev(self):
        return self._buf(3, (self.batch, self.cols, self.rank))

    @property
    def sent(self):
        """BLOCKSEL: live view of the per-block 'sent this round' flags."""
        p = lib().orc_blocksel_sent(self._h)
        return np.ctypeslib.as_array((ctypes.c_uint8 * self.bs_K).from_address(p))

    def dissimilarity(self, prev: np.ndarray, cur: np.ndarray) -> np.ndarray:
        """BLOCKSEL: cosine dissimilarity of every block between two fp32 activations."""
        prev = np.ascontiguousarray(prev, dtype=np.float32)
        cur = np.ascontiguousarray(cur, dtype=np.float32)
        d = np.empty(self.bs_K, dtype=np.float64)
        assert lib().orc_blocksel_dissimilarity(self._h, _ptr(prev), _ptr(cur), _ptr(d)) == 0
        return d

    def set_vprev_valid(self, v: bool):
        lib().orc_set_vprev_valid(self._h, 1 if v else 0)

    def set_step(self, send: int, recv: int):
        lib().orc_set_step(self._h, send, recv)
