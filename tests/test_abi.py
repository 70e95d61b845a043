"""The C-ABI library loads and exports every entry point include/cf.h declares;
host-side validation answers without a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "cf.h")).read()
    return sorted(set(re.findall(r"^CF_API\s+(?:const\s+char\s*\*|int)\s*(cf_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def cf():
    from activation_residual_compression_b200 import build
    build.build()
    import activation_residual_compression_b200 as m
    m._cf.load()
    return m


def test_every_declared_symbol_is_exported(cf):
    names = _declared()
    assert len(names) >= 18
    lib = ctypes.CDLL(cf._cf.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(cf._cf.EXPORTS)


def test_strerror_and_version(cf):
    assert "sm_100a" in cf.cf_version()
    for code in range(0, -13, -1):
        assert cf.cf_strerror(code) != "unknown status"
    assert cf.cf_strerror(-99) == "unknown status"


def test_params_defaults(cf):
    p = cf.cf_params_init()
    assert (p.dtype, p.role, p.ef, p.nm_n, p.nm_m, p.rank, p.iters, p.lr_int4, p.batch) == \
        (cf.CF_BF16, cf.CF_SENDER, cf.CF_EF_EXPLICIT, 2, 16, 70, 1, 1, 1)
    assert (p.bs_grid_h, p.bs_block, p.bs_k, p.bs_warm, p.state_dtype) == (0, 8, 0, 5, cf.CF_F32)
    assert p.lr_qr2_tol == 2.0 ** -16


def test_lowrank_qr2_tolerance_range(cf):
    ok = _ws(cf, 512, 384, cf.CF_LOWRANK, rank=40)
    assert ok[0] == cf.CF_OK
    for tol in (0.0, 2.0 ** -12):
        assert _ws(cf, 512, 384, cf.CF_LOWRANK, rank=40, lr_qr2_tol=tol) == ok
    for tol in (-1e-9, 2.0 ** -12 * 1.001, float("nan"), float("inf")):
        assert _ws(cf, 512, 384, cf.CF_LOWRANK, rank=40, lr_qr2_tol=tol)[0] == cf.CF_ERR_ARG, tol


def _ws(cf, rows, cols, mode, **kw):
    p = cf.cf_params_init(**kw)
    out = ctypes.c_size_t()
    rc = cf.raw("cf_workspace_bytes")(rows, cols, mode, ctypes.byref(p), ctypes.byref(out))
    return rc, out.value


def test_shape_rules_rejected_on_host(cf):
    assert _ws(cf, 4608, 3072, cf.CF_SIGN1)[0] == cf.CF_OK
    assert _ws(cf, 4608, 3072 + 16, cf.CF_SIGN1)[0] == cf.CF_ERR_SHAPE      # cols % 32
    assert _ws(cf, 4608, 3072 + 16, cf.CF_Q2)[0] == cf.CF_OK
    assert _ws(cf, 4608, 3072 + 8, cf.CF_Q2)[0] == cf.CF_ERR_SHAPE          # cols % 16
    assert _ws(cf, 4608, 3072 + 4, cf.CF_IDENTITY)[0] == cf.CF_ERR_SHAPE    # cols % 8
    assert _ws(cf, 0, 64, cf.CF_Q2)[0] == cf.CF_ERR_SHAPE
    assert _ws(cf, 4, 8192 + 32, cf.CF_SIGN1)[0] == cf.CF_ERR_SHAPE         # > max row width
    assert _ws(cf, 4, 1920, cf.CF_NM, nm_n=1, nm_m=16)[0] == cf.CF_OK
    assert _ws(cf, 4, 1920 + 64, cf.CF_NM, nm_n=1, nm_m=16)[0] == cf.CF_ERR_SHAPE  # index words
    assert _ws(cf, 4, 64, cf.CF_NM, nm_n=2, nm_m=8)[0] == cf.CF_ERR_UNSUPPORTED
    assert _ws(cf, 4, 64, cf.CF_NM, nm_n=3, nm_m=16)[0] == cf.CF_ERR_UNSUPPORTED
    assert _ws(cf, 4, 64, 7)[0] == cf.CF_ERR_ARG
    assert _ws(cf, 4, 64, cf.CF_Q2, dtype=5)[0] == cf.CF_ERR_ARG
    assert _ws(cf, 4, 64, cf.CF_Q2, batch=0)[0] == cf.CF_ERR_ARG


def test_lowrank_shape_rules_rejected_on_host(cf):
    """CF_LOWRANK: rows and cols multiples of 128, 1 <= rank <= min(rows, cols, 128),
    1 or 2 sweeps, INT4 or fp32 factors, batch 1."""
    L = cf.CF_LOWRANK
    assert _ws(cf, 4096, 3072, L)[0] == cf.CF_OK
    assert _ws(cf, 4096 + 64, 3072, L)[0] == cf.CF_ERR_SHAPE
    assert _ws(cf, 4096, 3072 + 64, L)[0] == cf.CF_ERR_SHAPE
    assert _ws(cf, 4096, 3072, L, rank=128)[0] == cf.CF_OK
    assert _ws(cf, 128, 3072, L, rank=128)[0] == cf.CF_OK
    for rank in (0, 129):
        assert _ws(cf, 4096, 3072, L, rank=rank)[0] == cf.CF_ERR_SHAPE, rank
    assert _ws(cf, 4096, 3072, L, iters=2)[0] == cf.CF_OK
    for iters in (0, 3):
        assert _ws(cf, 4096, 3072, L, iters=iters)[0] == cf.CF_ERR_UNSUPPORTED, iters
    assert _ws(cf, 4096, 3072, L, lr_int4=0)[0] == cf.CF_OK
    assert _ws(cf, 4096, 3072, L, lr_int4=2)[0] == cf.CF_ERR_ARG
    assert _ws(cf, 4096, 3072, L, batch=2)[0] == cf.CF_ERR_UNSUPPORTED


def test_blocksel_shape_rules_rejected_on_host(cf):
    """CF_BLOCKSEL: the grid and its sides divisible by the block side (4, 8 or 16),
    K <= 4096 blocks, 1 <= k <= K, at least one leading full step, batch 1."""
    B = cf.CF_BLOCKSEL
    assert _ws(cf, 4096, 3072, B)[0] == cf.CF_OK                      # 64 x 64 grid, b = 8
    assert _ws(cf, 4096, 3072, B, bs_block=16)[0] == cf.CF_OK
    assert _ws(cf, 4096, 3072, B, bs_block=5)[0] == cf.CF_ERR_UNSUPPORTED
    assert _ws(cf, 4096 + 8, 3072, B)[0] == cf.CF_ERR_SHAPE           # not a square grid
    assert _ws(cf, 4096, 3072, B, bs_grid_h=32)[0] == cf.CF_OK        # 32 x 128 grid
    assert _ws(cf, 4096, 3072, B, bs_grid_h=48)[0] == cf.CF_ERR_SHAPE  # 48 does not divide 4096
    assert _ws(cf, 256 * 256, 64, B, bs_block=4)[0] == cf.CF_OK       # K = 4096
    assert _ws(cf, 512 * 512, 64, B, bs_block=4)[0] == cf.CF_ERR_UNSUPPORTED  # K = 16384
    assert _ws(cf, 4096, 3072, B, bs_k=64)[0] == cf.CF_OK             # k = K
    for k in (65, -1):
        assert _ws(cf, 4096, 3072, B, bs_k=k)[0] == cf.CF_ERR_ARG, k
    assert _ws(cf, 4096, 3072, B, bs_warm=0)[0] == cf.CF_ERR_ARG
    assert _ws(cf, 4096, 3072, B, batch=2)[0] == cf.CF_ERR_UNSUPPORTED


def test_workspace_sizes(cf):
    E = 4608 * 3072
    rc, s = _ws(cf, 4608, 3072, cf.CF_SIGN1, role=cf.CF_SENDER)
    assert rc == 0 and s >= 2 * E * 4 and s < 2 * E * 4 + 4096
    rc, r = _ws(cf, 4608, 3072, cf.CF_SIGN1, role=cf.CF_RECEIVER)
    assert rc == 0 and r >= E * 4 and r < E * 4 + 4096


def test_null_handles_rejected(cf):
    P = ctypes.c_void_p
    assert cf.raw("cf_encode")(None, P(16), P(16), None) == cf.CF_ERR_STATE
    assert cf.raw("cf_decode")(None, P(16), P(16), None) == cf.CF_ERR_STATE
    assert cf.raw("cf_destroy")(P(12345)) == cf.CF_ERR_STATE
    assert cf.raw("cf_status")(P(12345), None) == cf.CF_ERR_STATE
    out = ctypes.c_size_t()
    assert cf.raw("cf_payload_bytes")(P(12345), 0, ctypes.byref(out)) == cf.CF_ERR_STATE


def test_params_layout_and_constants_match_the_header(cf, tmp_path):
    """The ctypes mirror of cf_params and the binding's constants against the
    header itself, compiled as C: every field's offset, the struct size, and
    every CF_* value the binding defines."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    fields = [f[0] for f in cf.cf_params._fields_]
    consts = sorted(n for n in dir(cf) if n.startswith("CF_") and isinstance(getattr(cf, n), int))
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "cf.h"', "int main(void) {",
             '  printf("size %zu\\n", sizeof(cf_params));']
    lines += [f'  printf("off.{f} %zu\\n", offsetof(cf_params, {f}));' for f in fields]
    lines += [f'  printf("const.{c} %d\\n", (int)({c}));' for c in consts]
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    inc = os.path.join(ROOT, "include")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], check=True, capture_output=True,
                                                       text=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(cf.cf_params)
    for f in fields:
        assert int(got[f"off.{f}"]) == getattr(cf.cf_params, f).offset, f
    for c in consts:
        assert int(got[f"const.{c}"]) == getattr(cf, c), c


def test_missing_library_raises_instead_of_falling_back(tmp_path):
    """Without libcf.so the binding raises on its first call; nothing runs on the CPU instead."""
    import subprocess
    import sys
    code = ("import activation_residual_compression_b200 as m\n"
            "try:\n"
            f"    m._cf.load({str(tmp_path / 'libcf.so')!r})\n"
            "except ImportError as e:\n"
            "    print('raised', 'no CPU fallback' in str(e))\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "raised True"
