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
    return sorted(set(re.findall(r"^\s*R2L_API\s+(?:r2l_status|const char \*|int|size_t)\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(["r2l_scan_block", "fwd_scan_from_state", "r2l_residual_apply", "r2l_decode_step",
                                           "r2l_in_proj", "r2l_x_proj_workspace_size", "r2l_x_proj", "r2l_x_proj_noalloc",
                                           "r2l_dt_proj", "r2l_sidecar_workspace_size", "r2l_sidecar_forward",
                                           "r2l_bidir_scan_workspace_size", "r2l_bidir_scan", "r2l_scan_block_bwd",
                                           "r2l_status_string", "r2l_device_status", "r2l_last_error",
                                           "r2l_wait_selftest", "r2l_abi_version"])


def test_library_exports_every_declared_symbol(r2l):
    lib = ctypes.CDLL(r2l.r2l.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"libr2l.so does not export {name}"
    out = subprocess.run(["nm", "-D", "--defined-only", r2l.r2l.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    # nothing but the C ABI leaks out of the shared object
    assert exported == set(declared_functions())


@pytest.mark.parametrize("cname,pyname", [("r2l_scan_args", "ScanArgs"), ("r2l_sidecar_weights", "SidecarWeights")])
def test_struct_layout_matches_c(r2l, tmp_path, cname, pyname):
    cls = getattr(r2l, pyname)
    fields = [f for f, _ in cls._fields_]
    prog = tmp_path / "layout.c"
    prog.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"r2l.h\"\nint main(void){\n"
                    f"printf(\"%zu\\n\", sizeof({cname}));\n"
                    + "".join(f"printf(\"%zu\\n\", offsetof({cname}, {f}));\n" for f in fields)
                    + "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.dirname(HEADER), "-I", CUDA_INC, "-o", str(exe), str(prog)])
    vals = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    assert vals[0] == ctypes.sizeof(cls)
    assert vals[1:] == [getattr(cls, f).offset for f in fields]


def test_status_strings_and_version(r2l):
    for code in range(5):
        s = r2l.status_string(code)
        assert s.startswith("R2L_")
    assert r2l.r2l_abi_version() == 102


def _args(r2l, **over):
    a = dict(batch=2, seqlen=32, block_len=32, d_inner=64, d_state=16, conv_width=0, in_dtype=r2l.R2L_BF16,
             x=256, dt=512, B=768, C=1024, z=None, A=1280, D=1536, dt_bias=1792, conv_w=None, conv_b=None,
             conv_state=None, conv_state_out=None)
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
    (dict(conv_width=4, conv_w=2048, conv_b=2304, conv_state=2560), "R2L_ERR_INVALID_ARG"),  # reverse: no conv state
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


def test_decode_step_validation_is_host_side(r2l):
    lib = r2l.load()
    code = lambda st: r2l.status_string(st).split(":")[0]
    cases = [(_args(r2l, block_len=5), 8192, 12288, 0.5, r2l.R2L_BF16),   # scan arguments first
             (_args(r2l), 8194, 12288, 0.5, r2l.R2L_BF16),                 # misaligned hidden
             (_args(r2l), 8192, None, 0.5, r2l.R2L_BF16),                  # W_out missing
             (_args(r2l), 8192, 12288, 0.5, 7)]                            # unknown dtype
    for a, hidden, w, s, dt in cases:
        assert code(lib.r2l_decode_step(ctypes.byref(a), 4096, hidden, w, s, 64, dt, None)) == "R2L_ERR_INVALID_ARG"
    # empty problems return before any launch
    for over in (dict(batch=0), dict(seqlen=0), dict(d_inner=0)):
        assert lib.r2l_decode_step(ctypes.byref(_args(r2l, **over)), None, None, None, 0.5, 64, r2l.R2L_BF16,
                                   None) == r2l.R2L_OK


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
    conv = dict(conv_width=4, conv_w=2048, conv_b=2304)
    for fa, code in [(_args(r2l, conv_state=2560), "R2L_ERR_INVALID_ARG"),          # no convolution to carry
                     (_args(r2l, conv_state_out=2560), "R2L_ERR_INVALID_ARG"),
                     (_args(r2l, **conv, conv_state=2562), "R2L_ERR_INVALID_ARG"),  # misaligned fp32
                     ]:
        st = lib.fwd_scan_from_state(ctypes.byref(fa), None, None, None, 8192, r2l.R2L_F32, None)
        assert r2l.status_string(st).startswith(code)
    # the two-pass bidirectional scan takes any reverse block length, but needs its workspace
    fa, ra = _args(r2l, seqlen=256, block_len=256), _args(r2l, seqlen=256, block_len=128)
    need = lib.r2l_bidir_scan_workspace_size(ctypes.byref(fa))
    assert need == 2 * 2 * 256 * 64 * 4
    st = lib.r2l_bidir_scan(ctypes.byref(fa), ctypes.byref(ra), None, None, 8192, r2l.R2L_F32, 1 << 20, need - 1, None)
    assert r2l.status_string(st).startswith("R2L_ERR_INVALID_ARG")
    st = lib.r2l_bidir_scan(ctypes.byref(fa), ctypes.byref(_args(r2l, seqlen=256, block_len=96)), None, None, 8192,
                            r2l.R2L_F32, 1 << 20, need, None)
    assert r2l.status_string(st).startswith("R2L_ERR_INVALID_ARG")  # 96 does not divide 256
    long_fwd = _args(r2l, seqlen=256, block_len=256)
    long_rev = _args(r2l, seqlen=256, block_len=128)
    st = lib.fwd_scan_from_state(ctypes.byref(long_fwd), ctypes.byref(long_rev), None, None, 8192, r2l.R2L_F32, None)
    assert r2l.status_string(st).startswith("R2L_ERR_UNSUPPORTED")


def _weights(r2l, **over):
    a = dict(d_model=256, d_inner=256, d_state=16, dt_rank=16, conv_width=4, W_in=4096, conv_w=8192, conv_b=8448,
             W_x=12288, W_dt=16384, A=20480, D=24576, dt_bias=28672, W_out=32768)
    a.update(over)
    return r2l.SidecarWeights(**a)


def test_scan_bwd_validation_is_host_side(r2l):
    lib = r2l.load()
    code = lambda st: r2l.status_string(st).split(":")[0]
    outs = [65536 + 4096 * i for i in range(8)]
    dconv = [65536 + 4096 * 8, 65536 + 4096 * 9]
    for over, want in [(dict(block_len=128, seqlen=128), "R2L_ERR_UNSUPPORTED"),   # longer than 64 tokens
                       (dict(d_inner=40), "R2L_ERR_UNSUPPORTED")]:                  # not a multiple of 16
        st = lib.r2l_scan_block_bwd(ctypes.byref(_args(r2l, **over)), 4096, r2l.R2L_F32, *outs, None, None, None)
        assert code(st) == want, over
    # dz must be given exactly when z is
    st = lib.r2l_scan_block_bwd(ctypes.byref(_args(r2l, z=2816)), 4096, r2l.R2L_F32, *outs[:4], None, *outs[5:],
                                None, None, None)
    assert code(st) == "R2L_ERR_INVALID_ARG"
    # dconv_w and dconv_b must be given exactly when the convolution is
    st = lib.r2l_scan_block_bwd(ctypes.byref(_args(r2l, conv_width=4, conv_w=2048, conv_b=2304)), 4096, r2l.R2L_F32,
                                *outs, None, None, None)
    assert code(st) == "R2L_ERR_INVALID_ARG"
    st = lib.r2l_scan_block_bwd(ctypes.byref(_args(r2l)), 4096, r2l.R2L_F32, *outs, *dconv, None)
    assert code(st) == "R2L_ERR_INVALID_ARG"


def test_front_end_validation_is_host_side(r2l):
    lib = r2l.load()
    code = lambda st: r2l.status_string(st).split(":")[0]
    # in_proj: d_inner must be a multiple of 64, d_model of 8, block_len must divide seqlen
    assert code(lib.r2l_in_proj(4096, 8192, None, None, 2, 32, 32, 256, 96, 12288, 16384, None)) == "R2L_ERR_INVALID_ARG"
    assert code(lib.r2l_in_proj(4096, 8192, None, None, 2, 32, 32, 250, 128, 12288, 16384, None)) == "R2L_ERR_INVALID_ARG"
    assert code(lib.r2l_in_proj(4096, 8192, 256, 512, 2, 32, 24, 256, 128, 12288, 16384, None)) == "R2L_ERR_INVALID_ARG"
    assert code(lib.r2l_in_proj(4096, 8192, 256, None, 2, 32, 32, 256, 128, 12288, 16384, None)) == "R2L_ERR_INVALID_ARG"
    assert lib.r2l_in_proj(None, None, None, None, 0, 32, 32, 256, 128, None, None, None) == r2l.R2L_OK  # empty
    # x_proj: N = dt_rank + 2 d_state must fit one 256-wide tile; the workspace must be large enough
    assert code(lib.r2l_x_proj(4096, 8192, 64, 256, 240, 16, 12288, 16384, 20480, 24576, 1 << 30, None)) == \
        "R2L_ERR_INVALID_ARG"
    need = lib.r2l_x_proj_workspace_size(2048, 2048, 128, 16)
    assert need >= 2048 * 160 * 4
    assert code(lib.r2l_x_proj(4096, 8192, 2048, 2048, 128, 16, 12288, 16384, 20480, 24576, need - 1, None)) == \
        "R2L_ERR_INVALID_ARG"
    assert code(lib.r2l_dt_proj(4096, 8192, 64, 12, 256, 12288, None)) == "R2L_ERR_INVALID_ARG"
    # the library-scratch x_proj: same checks; inputs beyond its 16 MiB scratch are refused on the host
    assert code(lib.r2l_x_proj_noalloc(4096, 8192, 64, 256, 240, 16, 12288, 16384, 20480, None)) == "R2L_ERR_INVALID_ARG"
    assert code(lib.r2l_x_proj_noalloc(4096, 8192, 65536, 2048, 128, 16, 12288, 16384, 20480, None)) == \
        "R2L_ERR_UNSUPPORTED"
    # the whole sidecar
    sw = _weights(r2l)
    ws = lib.r2l_sidecar_workspace_size(ctypes.byref(sw), 4, 32)
    assert ws >= 4 * 32 * 256 * 2 * 4
    for bad, want in [(dict(d_state=8), "R2L_ERR_UNSUPPORTED"), (dict(conv_width=3), "R2L_ERR_UNSUPPORTED"),
                      (dict(conv_w=None), "R2L_ERR_INVALID_ARG"), (dict(W_x=12290), "R2L_ERR_INVALID_ARG"),
                      (dict(dt_rank=24), "R2L_ERR_INVALID_ARG"), (dict(d_inner=96), "R2L_ERR_INVALID_ARG")]:
        st = lib.r2l_sidecar_forward(ctypes.byref(_weights(r2l, **bad)), 4, 32, 32, 0.05, 65536, 1 << 20, ws, None)
        assert code(st) == want, bad
    assert code(lib.r2l_sidecar_forward(ctypes.byref(sw), 4, 32, 32, 0.05, 65536, 1 << 20, ws - 1, None)) == \
        "R2L_ERR_INVALID_ARG"
    assert code(lib.r2l_sidecar_forward(ctypes.byref(sw), 4, 32, 32, 0.05, 65536, (1 << 20) + 16, ws, None)) == \
        "R2L_ERR_INVALID_ARG"  # workspace must be 256-byte aligned
    # s == 0 returns before any CUDA call
    assert lib.r2l_sidecar_forward(ctypes.byref(sw), 4, 32, 32, 0.0, 65536, None, 0, None) == r2l.R2L_OK


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
