"""The C-ABI library builds, loads and exports what include/mxattn.h declares;
host-side argument checks (no GPU: every call here returns before any CUDA call)."""
import ctypes
import subprocess

import pytest

from mxfp4_microscaled_quantization_b200 import build as build_mod
from mxfp4_microscaled_quantization_b200 import mxattn as mx


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return mx.lib()


def test_header_declares_the_boundary():
    syms = mx.declared_symbols()
    for name in ("mxattn_quantize", "mxattn_quantize_vt", "mxattn_workspace_size", "mxattn_forward",
                 "mxattn_forward_quantized", "mxattn_workspace_status", "mxattn_status_string", "mxattn_prepare",
                 "mxattn_attend", "mxattn_nvfp4_forward", "mxattn_nvfp4_quantize", "mxattn_nvfp4_workspace_size",
                 "mxattn_mxf4_mma_loop"):
        assert name in syms


def test_library_exports_every_declared_symbol(L):
    for name in mx.declared_symbols():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", mx.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(mx.declared_symbols()) <= exported
    # nothing but the C ABI is exported from the library's own code
    assert not [s for s in exported if s.startswith("_ZN6mxattn")]


def test_status_strings(L):
    for s in range(5):
        assert isinstance(mx.status_string(s), str) and mx.status_string(s)
    assert mx.status_string(99) == "unknown status"


def test_workspace_size_matches_documented_layout(L):
    for shape in ((1, 1, 256, 64), (1, 8, 4096, 128), (1, 40, 32760, 128), (2, 3, 1, 64), (1, 1, 129, 128)):
        assert mx.mxattn_workspace_size(*shape) == mx.workspace_layout(*shape)["total"]
    assert mx.mxattn_workspace_size(1, 1, 256, 96) == 0
    assert mx.mxattn_workspace_size(1, 1, 0, 64) == 0
    assert mx.mxattn_workspace_size(0, 1, 16, 64) == 0


def _p(x):
    return ctypes.c_void_p(x)


def test_quantize_rejects_bad_arguments_before_launching(L):
    fake = _p(1 << 20)
    assert L.mxattn_quantize(fake, 4, 48, 1, fake, fake, None) == 1        # cols % 32 != 0
    assert L.mxattn_quantize(fake, -1, 64, 1, fake, fake, None) == 1       # negative rows
    assert L.mxattn_quantize(fake, 4, 64, 7, fake, fake, None) == 1        # unknown rule
    assert L.mxattn_quantize(None, 4, 64, 1, fake, fake, None) == 1        # null input
    assert L.mxattn_quantize(_p((1 << 20) + 8), 4, 64, 1, fake, fake, None) == 1  # misaligned input
    assert L.mxattn_quantize(None, 0, 64, 1, None, None, None) == 0        # empty is a no-op
    assert L.mxattn_quantize_vt(fake, 1, 16, 96, 1, fake, fake, None) == 2  # d unsupported
    assert L.mxattn_quantize_vt(fake, 1, 0, 64, 1, fake, fake, None) == 1   # N < 1


def test_forward_rejects_bad_arguments_before_launching(L):
    fake = _p(1 << 20)
    ws_ok = mx.mxattn_workspace_size(1, 1, 256, 64)
    args = lambda d=64, t=64, pnq=1, rule=1, N=256, ws=ws_ok, o=fake: (  # noqa: E731
        fake, fake, fake, 1, 1, N, d, t, pnq, rule, ctypes.c_float(0.0), o, fake, ws, None)
    assert L.mxattn_forward(*args(d=96)) == 2
    assert L.mxattn_forward(*args(t=32)) == 2
    assert L.mxattn_forward(*args(pnq=2)) == 1
    assert L.mxattn_forward(*args(rule=3)) == 1
    assert L.mxattn_forward(*args(N=0)) == 1
    assert L.mxattn_forward(*args(ws=ws_ok - 1)) == 1
    assert L.mxattn_forward(*args(o=None)) == 1
    assert L.mxattn_forward(*args(N=(1 << 24) + 1, ws=1 << 40)) == 2
    q = (fake,) * 6
    assert L.mxattn_forward_quantized(*q, 1, 1, 256, 64, 96, 1, 1, ctypes.c_float(0), fake, fake, ws_ok, None) == 2


def test_forward_host_rejects_bad_arguments_before_launching(L):
    """mxattn_forward_host checks everything before it creates a stream or copies a byte."""
    fake = _p(1 << 20)
    ws = mx.forward_host_workspace_size(1, 4, 256, 64)
    ok = dict(d=64, t=64, pnq=1, rule=1, N=256, H=4, o=fake, dev=fake, ws=fake, wsb=ws, groups=None, ng=0)

    def call(**kw):
        a = {**ok, **kw}
        return L.mxattn_forward_host(fake, fake, fake, 1, a["H"], a["N"], a["d"], a["t"], a["pnq"], a["rule"],
                                     ctypes.c_float(0.0), a["o"], a["dev"], fake, fake, fake, a["ws"], a["wsb"],
                                     a["groups"], a["ng"], None)
    assert call(d=96) == 2
    assert call(t=32) == 2
    assert call(N=(1 << 24) + 1, wsb=1 << 40) == 2
    assert call(pnq=2) == 1
    assert call(rule=5) == 1
    assert call(o=None) == 1
    assert call(dev=None) == 1
    assert call(dev=_p((1 << 20) + 4)) == 1          # misaligned staging buffer
    assert call(ws=_p((1 << 20) + 16)) == 1          # misaligned workspace
    assert call(wsb=ws - 1) == 1                      # workspace too small for the largest group
    bad = (ctypes.c_int * 2)(3, 2)                     # sums to 5, B*H = 4
    assert call(groups=bad, ng=2) == 1
    zero = (ctypes.c_int * 2)(4, 0)
    assert call(groups=zero, ng=2) == 1
    assert call(ng=-1) == 1


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mx, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mx, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        mx.lib()


def test_qmax_entry_points_reject_boundaries_outside_the_family(L):
    """A scale boundary outside (4, 8] (or NaN) is an argument error, caught before any launch."""
    fake = _p(1 << 20)
    f = ctypes.c_float
    ws_ok = mx.mxattn_workspace_size(1, 1, 256, 64)
    for q in (4.0, 3.0, 8.5, float("nan"), -7.25):
        assert L.mxattn_quantize_qmax(fake, 4, 64, f(q), fake, fake, None) == 1
        assert L.mxattn_forward_qmax(fake, fake, fake, 1, 1, 256, 64, 64, 1, f(q), f(0.0), fake, fake, ws_ok,
                                     None) == 1
        assert L.mxattn_prepare_qmax(fake, fake, fake, 1, 1, 256, 64, f(q), fake, ws_ok, None) == 1
        assert L.mxattn_attend_qmax(1, 1, 256, 64, 64, 1, f(q), f(0.0), fake, fake, ws_ok, None) == 1
    assert L.mxattn_quantize_qmax(None, 0, 64, f(6.0), None, None, None) == 0  # empty, valid boundary


def test_nvfp4_workspace_size_matches_documented_layout(L):
    for shape in ((1, 1, 256, 64), (1, 8, 4096, 128), (1, 40, 32760, 128), (2, 3, 1, 64), (1, 1, 129, 128)):
        assert mx.nvfp4_workspace_size(*shape) == mx.nvfp4_workspace_layout(*shape)["total"]
    assert mx.nvfp4_workspace_size(1, 1, 256, 96) == 0
    assert mx.nvfp4_workspace_size(1, 1, 0, 64) == 0


def test_nvfp4_entry_points_reject_bad_arguments_before_launching(L):
    fake = _p(1 << 20)
    f = ctypes.c_float
    assert L.mxattn_nvfp4_quantize(fake, 4, 40, fake, fake, fake, None) == 1   # cols % 16 != 0
    assert L.mxattn_nvfp4_quantize(fake, -1, 64, fake, fake, fake, None) == 1  # negative rows
    assert L.mxattn_nvfp4_quantize(None, 4, 64, fake, fake, fake, None) == 1   # null input
    assert L.mxattn_nvfp4_quantize(fake, 4, 64, fake, fake, None, None) == 1   # null gs
    assert L.mxattn_nvfp4_quantize(_p((1 << 20) + 8), 4, 64, fake, fake, fake, None) == 1  # misaligned
    assert L.mxattn_nvfp4_quantize(None, 0, 64, None, None, None, None) == 0   # empty is a no-op
    ws_ok = mx.nvfp4_workspace_size(1, 1, 256, 64)
    args = lambda d=64, t=64, pnq=1, N=256, ws=ws_ok, o=fake, H=1: (  # noqa: E731
        fake, fake, fake, 1, H, N, d, t, pnq, f(0.0), o, fake, ws, None)
    assert L.mxattn_nvfp4_forward(*args(d=96)) == 2
    assert L.mxattn_nvfp4_forward(*args(t=32)) == 2
    assert L.mxattn_nvfp4_forward(*args(pnq=2)) == 1
    assert L.mxattn_nvfp4_forward(*args(N=0)) == 1
    assert L.mxattn_nvfp4_forward(*args(ws=ws_ok - 1)) == 1
    assert L.mxattn_nvfp4_forward(*args(o=None)) == 1
    assert L.mxattn_nvfp4_forward(*args(H=65536, ws=1 << 40)) == 2
    # an MXFP4-sized workspace is too small for the NVFP4 layout of the same shape
    assert mx.mxattn_workspace_size(1, 1, 256, 128) < mx.nvfp4_workspace_size(1, 1, 256, 128)
    assert L.mxattn_nvfp4_prepare(fake, fake, fake, 1, 1, 256, 128, fake, mx.mxattn_workspace_size(1, 1, 256, 128),
                                  None) == 1
    assert L.mxattn_nvfp4_attend(1, 1, 256, 64, 64, 1, f(0.0), fake, fake, ws_ok - 1, None) == 1


def test_p_selftest_rejects_bad_arguments_before_launching(L):
    fake = _p(1 << 20)
    f = ctypes.c_float
    assert L.mxattn_p_selftest(6, fake, 8, f(7.25), fake, None) == 1    # unknown path
    assert L.mxattn_p_selftest(0, fake, 12, f(7.25), fake, None) == 1   # n % 8 != 0
    assert L.mxattn_p_selftest(3, fake, 8, f(9.0), fake, None) == 1     # boundary outside (4, 8]
    assert L.mxattn_p_selftest(0, None, 8, f(7.25), fake, None) == 1    # null input
    assert L.mxattn_p_selftest(0, _p((1 << 20) + 2), 8, f(7.25), fake, None) == 1  # misaligned
    assert L.mxattn_p_selftest(1, None, 0, f(7.25), None, None) == 0    # empty is a no-op


def test_mma_loop_rejects_bad_arguments_before_launching(L):
    fake = _p(1 << 20)
    assert L.mxattn_mxf4_mma_loop(0, 10, fake, None, None) == 1          # no CTAs
    assert L.mxattn_mxf4_mma_loop(5000, 10, fake, None, None) == 1       # too many CTAs
    assert L.mxattn_mxf4_mma_loop(148, 0, fake, None, None) == 1         # no iterations
    assert L.mxattn_mxf4_mma_loop(148, 200001, fake, None, None) == 1    # a launch would run too long
    assert L.mxattn_mxf4_mma_loop(148, 10, None, None, None) == 1        # null status
    assert L.mxattn_mxf4_mma_loop(148, 10, _p((1 << 20) + 2), None, None) == 1  # misaligned status
    assert L.mxattn_mxf4_mma_loop(148, 10, fake, _p((1 << 20) + 4), None) == 1  # misaligned cycles


def test_header_compiles_as_c_and_links(L, tmp_path):
    """include/mxattn.h is plain C (C99, no torch or CUDA headers needed): a C program
    includes it, links against libmxattn.so and calls the host-only entry points."""
    import os

    src = tmp_path / "abi.c"
    src.write_text(
        "#include <stdio.h>\n#include \"mxattn.h\"\n"
        "int main(void) {\n"
        "  size_t ws = mxattn_workspace_size(1, 40, 32760, 128);\n"
        "  size_t nv = mxattn_nvfp4_workspace_size(1, 40, 32760, 128);\n"
        "  size_t hw = mxattn_forward_host_workspace_size(1, 40, 32760, 128, 0, 0);\n"
        "  mxattn_status st = mxattn_quantize(0, 4, 48, MXATTN_RULE_UOS, 0, 0, 0);\n"
        "  printf(\"%zu %zu %d %s %zu\\n\", ws, nv, (int)st, mxattn_status_string(st), hw);\n"
        "  return 0;\n}\n")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(mx.LIB_PATH)
    inc = os.path.join(os.path.dirname(libdir), "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe), f"-L{libdir}",
                    "-l:libmxattn.so", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert int(out[0]) == mx.mxattn_workspace_size(1, 40, 32760, 128)
    assert int(out[1]) == mx.nvfp4_workspace_size(1, 40, 32760, 128)
    assert out[2] == "1" and " ".join(out[3:-1]) == mx.status_string(1)
    assert int(out[-1]) == mx.forward_host_workspace_size(1, 40, 32760, 128)
