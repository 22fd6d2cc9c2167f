"""Host-side checks of the C ABI that need no GPU.

* libr2l.so loads and exports every function declared in include/r2l.h;
* the ctypes mirror of r2l_scan_args has the C layout (checked against gcc);
* argument validation happens on the host, before any CUDA call;
* without a usable GPU a compute call fails loudly (no CPU fallback).
"""

import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "r2l.h")
CUDA_INC = "/usr/local/cuda/include"


@pytest.fixture(scope="module")
def r2l():
    from reverse_mamba_selective_b200 import _build

    _build.build()
    import reverse_mamba_selective_b200 as pkg

    pkg.load()
    return pkg


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*R2L_API\s+(?:r2l_status|const char \*|int)\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(["r2l_scan_block", "fwd_scan_from_state", "r2l_residual_apply",
                                           "r2l_status_string", "r2l_device_status", "r2l_last_error",
                                           "r2l_abi_version"])


def test_library_exports_every_declared_symbol(r2l):
    lib = ctypes.CDLL(r2l.r2l.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"libr2l.so does not export {name}"
    out = subprocess.run(["nm", "-D", "--defined-only", r2l.r2l.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    # nothing but the C ABI leaks out of the shared object
    assert exported == set(declared_functions())


def test_struct_layout_matches_c(r2l, tmp_path):
    fields = [f for f, _ in r2l.ScanArgs._fields_]
    prog = tmp_path / "layout.c"
    prog.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"r2l.h\"\nint main(void){\n"
                    "printf(\"%zu\\n\", sizeof(r2l_scan_args));\n"
                    + "".join(f"printf(\"%zu\\n\", offsetof(r2l_scan_args, {f}));\n" for f in fields)
                    + "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.dirname(HEADER), "-I", CUDA_INC, "-o", str(exe), str(prog)])
    vals = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    assert vals[0] == ctypes.sizeof(r2l.ScanArgs)
    assert vals[1:] == [getattr(r2l.ScanArgs, f).offset for f in fields]


def test_status_strings_and_version(r2l):
    for code in range(5):
        s = r2l.status_string(code)
        assert s.startswith("R2L_")
    assert r2l.r2l_abi_version() == 100


def _args(r2l, **over):
    a = dict(batch=2, seqlen=32, block_len=32, d_inner=64, d_state=16, conv_width=0, in_dtype=r2l.R2L_BF16,
             x=256, dt=512, B=768, C=1024, z=None, A=1280, D=1536, dt_bias=1792, conv_w=None, conv_b=None)
    a.update(over)
    return r2l.ScanArgs(**a)


@pytest.mark.parametrize("over,code", [
    (dict(d_state=8), "R2L_ERR_UNSUPPORTED"),
    (dict(conv_width=3), "R2L_ERR_UNSUPPORTED"),
    (dict(conv_width=4), "R2L_ERR_INVALID_ARG"),        # conv weights missing
    (dict(block_len=5), "R2L_ERR_INVALID_ARG"),         # does not divide seqlen
    (dict(block_len=0), "R2L_ERR_INVALID_ARG"),
    (dict(batch=-1), "R2L_ERR_INVALID_ARG"),
    (dict(d_inner=12), "R2L_ERR_INVALID_ARG"),          # rows not a multiple of 16 bytes
    (dict(x=None), "R2L_ERR_INVALID_ARG"),
    (dict(x=258), "R2L_ERR_INVALID_ARG"),               # misaligned
    (dict(in_dtype=7), "R2L_ERR_INVALID_ARG"),
])
def test_scan_validation_is_host_side(r2l, over, code):
    st = r2l.load().r2l_scan_block(ctypes.byref(_args(r2l, **over)), 4096, r2l.R2L_F32, None)
    assert r2l.status_string(st).startswith(code)


def test_empty_inputs_are_noops(r2l):
    lib = r2l.load()
    for over in (dict(batch=0), dict(seqlen=0), dict(d_inner=0)):
        assert lib.r2l_scan_block(ctypes.byref(_args(r2l, **over)), None, r2l.R2L_F32, None) == r2l.R2L_OK
        assert lib.fwd_scan_from_state(ctypes.byref(_args(r2l, **over)), None, None, None, None, r2l.R2L_F32,
                                       None) == r2l.R2L_OK
    assert lib.r2l_residual_apply(None, None, None, 0.5, 0, 64, 64, r2l.R2L_BF16, None) == r2l.R2L_OK


def test_residual_s0_is_identity_without_launch(r2l):
    # s == 0 returns before any CUDA call: hidden is left untouched by construction
    assert r2l.load().r2l_residual_apply(4096, 8192, 12288, 0.0, 128, 64, 64, r2l.R2L_BF16, None) == r2l.R2L_OK


def test_fused_reverse_validation(r2l):
    lib = r2l.load()
    fwd = _args(r2l)
    bad = [(_args(r2l, x=4096), "R2L_ERR_INVALID_ARG"),              # x must be shared
           (_args(r2l, seqlen=128, block_len=128), "R2L_ERR_INVALID_ARG"),  # shape mismatch
           ]
    for rev, code in bad:
        st = lib.fwd_scan_from_state(ctypes.byref(fwd), ctypes.byref(rev), None, None, 8192, r2l.R2L_F32, None)
        assert r2l.status_string(st).startswith(code)
    long_fwd = _args(r2l, seqlen=256, block_len=256)
    long_rev = _args(r2l, seqlen=256, block_len=128)
    st = lib.fwd_scan_from_state(ctypes.byref(long_fwd), ctypes.byref(long_rev), None, None, 8192, r2l.R2L_F32, None)
    assert r2l.status_string(st).startswith("R2L_ERR_UNSUPPORTED")


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour on a machine without a GPU")
def test_no_cpu_fallback_without_gpu(r2l):
    """A valid call on a host without a usable GPU reports R2L_ERR_CUDA (pointers are never
    dereferenced on the host)."""
    st = r2l.load().r2l_scan_block(ctypes.byref(_args(r2l)), 4096, r2l.R2L_F32, None)
    assert st == r2l.R2L_ERR_CUDA
    assert r2l.load().r2l_last_error().decode() != ""


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import reverse_mamba_selective_b200.r2l as b

    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        b.load()
