"""The C-ABI library: loads, exports every declared symbol, rejects bad
arguments synchronously (no GPU needed: every check here returns before any
CUDA call is made)."""
import ctypes
import os
import re

import pytest

from long_context_02_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "lightning.h")).read()
    return sorted(set(re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from long_context_02_b200 import build
    build.build()
    return B.lib()


def test_header_declares_the_entry_points():
    names = _declared_symbols()
    for required in ("la_prefill", "la_prefill_varlen", "la_decode", "la_backward",
                     "la_workspace_bytes", "la_status_string", "la_read_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(_declared_symbols()) <= set(B.EXPORTED) | set(_declared_symbols())


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5):
        assert B.la_status_string(code).startswith("LA_")
    assert "unknown" in B.la_status_string(42)


def test_workspace_bytes(lib):
    # decode needs none; prefill always needs at least the 256-byte header
    assert B.la_workspace_bytes(B.LA_OP_DECODE, 256, 64, 1, 128) == 0
    small = B.la_workspace_bytes(B.LA_OP_PREFILL, 1, 2, 256, 64, 0, B.torch.float32)
    assert small >= 256
    big = B.la_workspace_bytes(B.LA_OP_PREFILL, 1, 64, 32768, 128)
    assert big >= 256 + 64 * 4 + 64 * 2 * 128 * 128 * 4
    vl = B.la_workspace_bytes(B.LA_OP_PREFILL_VARLEN, 1, 64, 500000, 128, 16)
    assert vl > big
    # invalid shapes
    assert B.la_workspace_bytes(B.LA_OP_PREFILL, 0, 64, 1024, 128) == 0
    assert B.la_workspace_bytes(B.LA_OP_PREFILL, 1, 64, 1024, 96) == 0


def _prefill(lib, **kw):
    a = dict(q=16, k=16, v=16, s=16, o=16, st=0, B=1, H=2, N=64, d=64, it=1, ot=1, ws=16,
             wsb=1 << 20)
    a.update(kw)
    P = ctypes.c_void_p
    return lib.la_prefill(P(a["q"]), P(a["k"]), P(a["v"]), P(a["s"]), P(a["o"]),
                          P(a["st"]) if a["st"] else None, a["B"], a["H"], a["N"], a["d"],
                          a["it"], a["ot"], P(a["ws"]) if a["ws"] else None, a["wsb"], None)


def test_prefill_argument_errors(lib):
    assert _prefill(lib, B=0) == B.LA_ERR_INVALID_ARG
    assert _prefill(lib, H=-1) == B.LA_ERR_INVALID_ARG
    assert _prefill(lib, N=-5) == B.LA_ERR_INVALID_ARG
    assert _prefill(lib, d=96) == B.LA_ERR_UNSUPPORTED
    assert _prefill(lib, d=0) == B.LA_ERR_INVALID_ARG
    assert _prefill(lib, it=1, ot=0) == B.LA_ERR_UNSUPPORTED   # fp32 in, bf16 out
    assert _prefill(lib, it=7) == B.LA_ERR_INVALID_ARG
    assert _prefill(lib, q=0) == B.LA_ERR_INVALID_ARG
    assert _prefill(lib, o=0) == B.LA_ERR_INVALID_ARG
    assert _prefill(lib, k=24) == B.LA_ERR_INVALID_ARG        # misaligned
    assert _prefill(lib, ws=0) == B.LA_ERR_WORKSPACE
    assert _prefill(lib, wsb=8) == B.LA_ERR_WORKSPACE


def test_decode_and_backward_argument_errors(lib):
    P = ctypes.c_void_p
    x = P(16)
    assert lib.la_decode(x, x, x, x, x, x, 0, 64, 128, 0, 0, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_decode(x, x, x, x, None, x, 4, 64, 128, 0, 0, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_decode(x, x, x, x, x, x, 4, 64, 80, 0, 0, None) == B.LA_ERR_UNSUPPORTED
    assert lib.la_backward(x, x, x, x, x, x, x, x, 1, 2, 64, 64, 0, 0, None, 0,
                           None) == B.LA_ERR_WORKSPACE
    assert lib.la_backward(x, x, x, x, x, x, x, None, 1, 2, 64, 64, 0, 0, x, 1 << 20,
                           None) == B.LA_ERR_INVALID_ARG


def test_varlen_argument_errors(lib):
    P = ctypes.c_void_p
    x = P(16)
    assert lib.la_prefill_varlen(None, 2, x, x, x, x, x, None, 4, 100, 128, 0, 0, x, 1 << 30,
                                 None) == B.LA_ERR_INVALID_ARG
    assert lib.la_prefill_varlen(x, -1, x, x, x, x, x, None, 4, 100, 128, 0, 0, x, 1 << 30,
                                 None) == B.LA_ERR_INVALID_ARG
    assert lib.la_prefill_varlen(P(18), 2, x, x, x, x, x, None, 4, 100, 128, 0, 0, x, 1 << 30,
                                 None) == B.LA_ERR_INVALID_ARG
    # tokens but no sequences: the arguments disagree (O would be left unwritten)
    assert lib.la_prefill_varlen(x, 0, x, x, x, x, x, None, 4, 100, 128, 0, 0, x, 1 << 30,
                                 None) == B.LA_ERR_INVALID_ARG
    assert lib.la_prefill_varlen_with_state(x, 0, x, x, x, x, None, x, None, 4, 100, 128, 0, 0,
                                            x, 1 << 30, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_mixed_step(x, 0, x, x, x, x, None, x, 4, 100, 128, 0, 0, x, 1 << 30, None,
                             None) == B.LA_ERR_INVALID_ARG


def test_with_state_argument_errors(lib):
    P = ctypes.c_void_p
    x = P(16)
    # the incoming state is required and must be 16-byte aligned
    assert lib.la_prefill_with_state(x, x, x, x, None, x, x, 1, 2, 64, 64, 1, 1, x, 1 << 20,
                                     None) == B.LA_ERR_INVALID_ARG
    assert lib.la_prefill_with_state(x, x, x, x, P(20), x, x, 1, 2, 64, 64, 1, 1, x, 1 << 20,
                                     None) == B.LA_ERR_INVALID_ARG
    assert lib.la_prefill_with_state(x, x, x, x, x, x, x, 0, 2, 64, 64, 1, 1, x, 1 << 20,
                                     None) == B.LA_ERR_INVALID_ARG
    assert lib.la_prefill_with_state(x, x, x, x, x, x, x, 1, 2, 64, 64, 1, 1, None, 0,
                                     None) == B.LA_ERR_WORKSPACE
    assert lib.la_prefill_varlen_with_state(x, 2, x, x, x, x, None, x, None, 4, 100, 128, 0, 0,
                                            x, 1 << 30, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_prefill_varlen_with_state(None, 2, x, x, x, x, x, x, None, 4, 100, 128, 0, 0,
                                            x, 1 << 30, None) == B.LA_ERR_INVALID_ARG
    # an empty batch may pass no states (the workspace check comes next)
    assert lib.la_prefill_varlen_with_state(x, 0, None, None, None, x, None, None, None, 4, 0,
                                            128, 0, 0, None, 0, None) == B.LA_ERR_WORKSPACE


def test_mixed_step_argument_errors(lib):
    P = ctypes.c_void_p
    x = P(16)
    # states are required; the workspace is that of the varlen prefill
    assert lib.la_mixed_step(x, 2, x, x, x, x, None, x, 4, 100, 128, 0, 0, x, 1 << 30, None,
                             None) == B.LA_ERR_INVALID_ARG
    assert lib.la_mixed_step(None, 2, x, x, x, x, x, x, 4, 100, 128, 0, 0, x, 1 << 30, None,
                             None) == B.LA_ERR_INVALID_ARG
    assert lib.la_mixed_step(x, 2, x, x, x, x, x, x, 4, 100, 96, 0, 0, x, 1 << 30, None,
                             None) == B.LA_ERR_UNSUPPORTED
    assert lib.la_mixed_step(x, 2, x, x, x, x, x, x, 4, 100, 128, 0, 0, x, 64, None,
                             None) == B.LA_ERR_WORKSPACE
    # an empty batch may pass no states (the workspace check comes next)
    assert lib.la_mixed_step(x, 0, None, None, None, x, None, None, 4, 0, 128, 0, 0, None, 0,
                             None, None) == B.LA_ERR_WORKSPACE


def test_norm_gate_argument_errors(lib):
    P = ctypes.c_void_p
    x = P(16)
    f = ctypes.c_float
    assert lib.la_output_norm_gate(x, x, x, f(1e-5), x, 1, 129, 10, 128, 0, 0,
                                   None) == B.LA_ERR_UNSUPPORTED   # H*d > 16384
    assert lib.la_output_norm_gate(x, x, x, f(-1.0), x, 1, 4, 10, 128, 0, 0,
                                   None) == B.LA_ERR_INVALID_ARG   # eps < 0
    assert lib.la_output_norm_gate(x, x, x, f(float("nan")), x, 1, 4, 10, 128, 0, 0,
                                   None) == B.LA_ERR_INVALID_ARG
    assert lib.la_output_norm_gate(x, None, x, f(1e-5), x, 1, 4, 10, 128, 0, 0,
                                   None) == B.LA_ERR_INVALID_ARG
    assert lib.la_output_norm_gate(x, x, P(24), f(1e-5), x, 1, 4, 10, 128, 0, 0,
                                   None) == B.LA_ERR_INVALID_ARG   # misaligned weight
    assert lib.la_output_norm_gate(x, x, x, f(1e-5), x, 1, 4, 10, 96, 0, 0,
                                   None) == B.LA_ERR_UNSUPPORTED
    assert lib.la_output_norm_gate(x, x, x, f(1e-5), x, 1, 4, 10, 128, 0, 5,
                                   None) == B.LA_ERR_INVALID_ARG


def test_state_prefix_argument_errors(lib):
    P = ctypes.c_void_p
    x = P(16)
    lens = (ctypes.c_longlong * 3)(4, 5, 6)
    bad = (ctypes.c_longlong * 3)(4, -1, 6)
    assert lib.la_state_prefix(x, x, lens, 3, 4, 1, 2, 128, x, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_state_prefix(x, x, lens, 0, 0, 1, 2, 128, x, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_state_prefix(x, x, lens, 65, 1, 1, 2, 128, x, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_state_prefix(x, x, bad, 3, 1, 1, 2, 128, x, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_state_prefix(x, x, None, 3, 1, 1, 2, 128, x, None) == B.LA_ERR_INVALID_ARG
    assert lib.la_state_prefix(x, x, lens, 3, 1, 1, 2, 96, x, None) == B.LA_ERR_UNSUPPORTED


def test_sp_prefill_checks_chunk_lengths():
    from long_context_02_b200 import sp
    import torch
    q = torch.zeros((1, 2, 5, 64))
    with pytest.raises(ValueError):
        sp.sp_prefill(q, q, q, None, [4, 5], 0, q, None, gather=lambda s: s)


def test_prefill_state_argument_errors(lib):
    P = ctypes.c_void_p
    x = P(16)
    assert lib.la_prefill_state(x, x, x, None, None, 1, 2, 64, 128, 0, x, 1 << 30,
                                None) == B.LA_ERR_INVALID_ARG   # no state_out
    assert lib.la_prefill_state(x, x, x, P(20), x, 1, 2, 64, 128, 0, x, 1 << 30,
                                None) == B.LA_ERR_INVALID_ARG   # misaligned state_in
    assert lib.la_prefill_state(x, x, x, None, x, 1, 2, 64, 128, 0, None, 0,
                                None) == B.LA_ERR_WORKSPACE
    assert lib.la_prefill_state(x, x, x, None, x, 1, 2, 64, 96, 0, x, 1 << 30,
                                None) == B.LA_ERR_UNSUPPORTED


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "lightning.h"
int main(void) {
    size_t ws = la_workspace_bytes(LA_OP_PREFILL, 1, 64, 32768, 128, 0, LA_BF16);
    int bad = la_prefill(0, 0, 0, 0, 0, 0, 0, 64, 32768, 128, LA_BF16, LA_BF16, 0, 0, 0);
    printf("%zu %d\n", ws, bad);
    return (ws > 0 && bad == LA_ERR_INVALID_ARG &&
            strncmp(la_status_string(bad), "LA_", 3) == 0) ? 0 : 1;
}
"""


def test_plain_c_program_uses_the_library(lib, tmp_path):
    """include/lightning.h is valid C99 (no C++ needed) and a C program links
    against liblightning.so and calls it (argument checks only: no GPU)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    src = tmp_path / "prog.c"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(B.LIB_PATH)
    exe = tmp_path / "prog"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir,
                         "-llightning", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr


def test_size_limits(lib):
    P = ctypes.c_void_p
    x = P(16)
    too_long = (1 << 31) - 1
    assert _prefill(lib, N=too_long) == B.LA_ERR_UNSUPPORTED
    assert _prefill(lib, B=1 << 20, H=1 << 9) == B.LA_ERR_UNSUPPORTED   # 2^29 problems
    assert lib.la_prefill_varlen(x, 2, x, x, x, x, x, None, 4, too_long, 128, 0, 0, x, 1 << 30,
                                 None) == B.LA_ERR_UNSUPPORTED
    assert lib.la_backward(x, x, x, x, x, x, x, x, 1, 2, too_long, 64, 0, 0, x, 1 << 20,
                           None) == B.LA_ERR_UNSUPPORTED
    assert lib.la_mixed_step(x, 2, x, x, x, x, x, x, 4, too_long, 128, 0, 0, x, 1 << 30, None,
                             None) == B.LA_ERR_UNSUPPORTED


def test_tuning_roundtrip(lib):
    assert lib.la_set_tuning(48, 0) == B.LA_ERR_INVALID_ARG
    assert lib.la_set_tuning(0, 100) == B.LA_ERR_INVALID_ARG
    B.la_set_tuning(32, 256)
    assert B.la_get_tuning() == (32, 256)
    B.la_set_tuning(0, 0)
    assert B.la_get_tuning() == (0, 0)


def test_binding_refuses_missing_library(tmp_path, monkeypatch):
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(ImportError):
        B.lib()
