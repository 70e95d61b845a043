"""ctypes binding of libcf (include/cf.h): the same entry points, argument
marshalling only.  Every step of the codec runs in libcf's CUDA kernels; this
module has no compute path of its own and raises if the library is missing.

Tensors are torch CUDA tensors (their ``data_ptr()`` is passed), streams are
``torch.cuda.Stream`` objects or raw ``cudaStream_t`` integers (None = the
current torch stream).
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcf.so")

CF_OK = 0
CF_ERR_ARG = -1
CF_ERR_SHAPE = -2
CF_ERR_ROLE = -3
CF_ERR_UNSUPPORTED = -4
CF_ERR_CUDA = -5
CF_ERR_NOMEM = -6
CF_ERR_DESYNC = -7
CF_ERR_ALIGN = -8
CF_ERR_STATE = -9
CF_ERR_SIZE = -10
CF_ERR_TIMEOUT = -11
CF_ERR_TOO_LARGE = -12

CF_IDENTITY, CF_SIGN1, CF_Q2, CF_NM, CF_LOWRANK, CF_BLOCKSEL = 0, 1, 2, 3, 4, 5
CF_F32, CF_BF16 = 0, 1
CF_SENDER, CF_RECEIVER = 0, 1
CF_EF_EXPLICIT, CF_EF_IMPLICIT, CF_EF_OFF = 0, 1, 2
CF_T_RECON, CF_T_ERROR, CF_T_VPREV = 0, 1, 2

MODE_NAMES = {"identity": CF_IDENTITY, "sign1": CF_SIGN1, "q2": CF_Q2, "nm": CF_NM, "lowrank": CF_LOWRANK,
              "blocksel": CF_BLOCKSEL}


class cf_params(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("role", ctypes.c_int),
        ("ef", ctypes.c_int),
        ("nm_n", ctypes.c_int),
        ("nm_m", ctypes.c_int),
        ("rank", ctypes.c_int),
        ("iters", ctypes.c_int),
        ("lr_int4", ctypes.c_int),
        ("batch", ctypes.c_int),
        ("seed", ctypes.c_uint64),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("bs_grid_h", ctypes.c_int),
        ("bs_block", ctypes.c_int),
        ("bs_k", ctypes.c_int),
        ("bs_warm", ctypes.c_int),
        ("state_dtype", ctypes.c_int),
        ("lr_qr2_tol", ctypes.c_double),
    ]


class CFError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({cf_strerror(code)})")


_lib = None

EXPORTS = ["cf_version", "cf_strerror", "cf_params_init", "cf_workspace_bytes", "cf_create", "cf_payload_bytes",
           "cf_encode", "cf_decode", "cf_encode_batched", "cf_decode_batched", "cf_status", "cf_tensor",
           "cf_step", "cf_reset", "cf_state_bytes", "cf_state_export", "cf_state_import", "cf_destroy",
           "cf_lowrank_decode_noalloc", "cf_test_wait_timeout"]


def load(path: str = LIB_PATH):
    """Load libcf.so (built by ``activation_residual_compression_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libcf.so not found at {path}: build it with "
                          "`python -m activation_residual_compression_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(path)
    c = ctypes
    P = c.c_void_p
    PP = c.POINTER(c.c_void_p)
    L.cf_version.restype = c.c_char_p
    L.cf_version.argtypes = []
    L.cf_strerror.restype = c.c_char_p
    L.cf_strerror.argtypes = [c.c_int]
    L.cf_params_init.argtypes = [c.POINTER(cf_params)]
    L.cf_workspace_bytes.argtypes = [c.c_int64, c.c_int64, c.c_int, c.POINTER(cf_params), c.POINTER(c.c_size_t)]
    L.cf_create.argtypes = [c.c_int64, c.c_int64, c.c_int, c.POINTER(cf_params), PP]
    L.cf_payload_bytes.argtypes = [P, c.c_int, c.POINTER(c.c_size_t)]
    L.cf_encode.argtypes = [P, P, P, P]
    L.cf_decode.argtypes = [P, P, P, P]
    L.cf_encode_batched.argtypes = [P, PP, P, P]
    L.cf_decode_batched.argtypes = [P, P, PP, P]
    L.cf_status.argtypes = [P, P]
    L.cf_tensor.argtypes = [P, c.c_int, PP, c.POINTER(c.c_size_t)]
    L.cf_step.argtypes = [P, c.POINTER(c.c_uint64)]
    L.cf_reset.argtypes = [P]
    L.cf_state_bytes.argtypes = [P, c.POINTER(c.c_size_t)]
    L.cf_state_export.argtypes = [P, P, c.c_size_t, P]
    L.cf_state_import.argtypes = [P, P, c.c_size_t, P]
    L.cf_destroy.argtypes = [P]
    L.cf_lowrank_decode_noalloc.argtypes = [c.c_int64, c.c_int64, c.POINTER(cf_params), c.c_uint64, P, P, P, P, P]
    L.cf_test_wait_timeout.argtypes = [P, c.c_uint32]
    for name in EXPORTS:
        if name not in ("cf_version", "cf_strerror"):
            getattr(L, name).restype = c.c_int
    _lib = L
    return L


def _check(fn, rc):
    if rc != CF_OK:
        raise CFError(fn, rc)
    return rc


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


# ------------------------------------------------------------------ entry points

def cf_version() -> str:
    return load().cf_version().decode()


def cf_strerror(code: int) -> str:
    return load().cf_strerror(code).decode()


def cf_params_init(**overrides) -> cf_params:
    p = cf_params()
    _check("cf_params_init", load().cf_params_init(ctypes.byref(p)))
    for k, v in overrides.items():
        setattr(p, k, v)
    return p


def cf_workspace_bytes(rows: int, cols: int, mode: int, params: cf_params) -> int:
    out = ctypes.c_size_t()
    _check("cf_workspace_bytes", load().cf_workspace_bytes(rows, cols, mode, ctypes.byref(params), ctypes.byref(out)))
    return out.value


def cf_create(rows: int, cols: int, mode: int, params: cf_params) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check("cf_create", load().cf_create(rows, cols, mode, ctypes.byref(params), ctypes.byref(h)))
    return h


def cf_payload_bytes(state, warmup: bool) -> int:
    out = ctypes.c_size_t()
    _check("cf_payload_bytes", load().cf_payload_bytes(state, 1 if warmup else 0, ctypes.byref(out)))
    return out.value


def cf_encode(state, a, payload, stream=None) -> int:
    return _check("cf_encode", load().cf_encode(state, _ptr(a), _ptr(payload), _stream(stream)))


def cf_decode(state, payload, recon, stream=None) -> int:
    return _check("cf_decode", load().cf_decode(state, _ptr(payload), _ptr(recon), _stream(stream)))


def _ptr_array(tensors):
    arr = (ctypes.c_void_p * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = t if isinstance(t, int) else t.data_ptr()
    return arr


def cf_encode_batched(state, a_list, payload, stream=None) -> int:
    arr = _ptr_array(a_list)
    return _check("cf_encode_batched", load().cf_encode_batched(
        state, ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)), _ptr(payload), _stream(stream)))


def cf_decode_batched(state, payload, recon_list, stream=None) -> int:
    arr = _ptr_array(recon_list)
    return _check("cf_decode_batched", load().cf_decode_batched(
        state, _ptr(payload), ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)), _stream(stream)))


def cf_status(state, stream=None) -> int:
    """Device status after synchronising the stream: CF_OK, CF_ERR_DESYNC or CF_ERR_TIMEOUT (not raised)."""
    rc = load().cf_status(state, _stream(stream))
    if rc not in (CF_OK, CF_ERR_DESYNC, CF_ERR_TIMEOUT):
        raise CFError("cf_status", rc)
    return rc


def cf_tensor(state, which: int):
    p = ctypes.c_void_p()
    n = ctypes.c_size_t()
    _check("cf_tensor", load().cf_tensor(state, which, ctypes.byref(p), ctypes.byref(n)))
    return p.value, n.value


def cf_step(state) -> int:
    out = ctypes.c_uint64()
    _check("cf_step", load().cf_step(state, ctypes.byref(out)))
    return out.value


def cf_reset(state) -> int:
    return _check("cf_reset", load().cf_reset(state))


def cf_state_bytes(state) -> int:
    out = ctypes.c_size_t()
    _check("cf_state_bytes", load().cf_state_bytes(state, ctypes.byref(out)))
    return out.value


def cf_state_export(state, host_buf, stream=None) -> int:
    """host_buf: a writable buffer (bytearray / numpy uint8 array) of cf_state_bytes() bytes."""
    n = len(host_buf) if not hasattr(host_buf, "nbytes") else host_buf.nbytes
    addr = ctypes.addressof((ctypes.c_char * n).from_buffer(host_buf))
    return _check("cf_state_export", load().cf_state_export(state, ctypes.c_void_p(addr), n, _stream(stream)))


def cf_state_import(state, host_buf, stream=None) -> int:
    n = len(host_buf) if not hasattr(host_buf, "nbytes") else host_buf.nbytes
    addr = ctypes.addressof((ctypes.c_char * n).from_buffer(host_buf))
    return _check("cf_state_import", load().cf_state_import(state, ctypes.c_void_p(addr), n, _stream(stream)))


def cf_destroy(state) -> int:
    return _check("cf_destroy", load().cf_destroy(state))


def cf_lowrank_decode_noalloc(rows: int, cols: int, params: cf_params, step: int, payload, ahat, recon, status,
                              stream=None) -> int:
    """Allocation-free low-rank decode (see include/cf.h); all tensors caller-owned."""
    return _check("cf_lowrank_decode_noalloc", load().cf_lowrank_decode_noalloc(
        rows, cols, ctypes.byref(params), step, _ptr(payload), _ptr(ahat), _ptr(recon), _ptr(status),
        _stream(stream)))


def cf_test_wait_timeout(state, polls: int) -> int:
    """Low-rank failure-detection test hook (see include/cf.h): polls > 0 makes the
    reconstruction kernel's bounded operand wait run out; 0 restores it."""
    return _check("cf_test_wait_timeout", load().cf_test_wait_timeout(state, polls))


def raw(name: str):
    """The raw ctypes function (tests that check return codes without raising)."""
    return getattr(load(), name)
