"""The C ABI without a GPU: the library loads, exports every entry point that
include/hm.h declares, the ctypes mirrors match the C struct layouts, and
host-side argument validation rejects bad calls before anything is launched."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hm.h")


@pytest.fixture(scope="module")
def hm():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import selective_ssm_sequence_b200 as mod
    return mod


def _declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"HM_API\s+[\w\s\*]*?\b(hm_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(hm):
    names = _declared_functions()
    assert len(names) >= 11
    out = subprocess.run(["nm", "-D", "--defined-only", hm.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(hm.lib, n)
    assert set(hm.EXPORTED) == set(names)


def test_library_has_no_cpu_fallback_dependencies(hm):
    out = subprocess.run(["ldd", hm.LIB_PATH], capture_output=True, text=True).stdout
    # the CUDA runtime is linked statically; nothing links the oracle
    assert "hm_oracle" not in out
    assert "libtorch" not in out


def _c_layout(struct, fields):
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"hm.h\"\nint main(void){\n"
    prog += 'printf("%%zu\\n", sizeof(%s));\n' % struct
    for f in fields:
        prog += 'printf("%%zu\\n", offsetof(%s, %s));\n' % (struct, f)
    prog += "return 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True,
                                               check=True).stdout.split()]
    return vals[0], vals[1:]


@pytest.mark.parametrize("cname,pyname", [("hm_scan_args", "ScanArgs"),
                                          ("hm_decode_args", "DecodeArgs"),
                                          ("hm_mixer_args", "MixerArgs"),
                                          ("hm_scan_bwd_args", "ScanBwdArgs"),
                                          ("hm_combine_args", "CombineArgs"),
                                          ("hm_block_args", "BlockArgs")])
def test_struct_layouts_match_the_header(hm, cname, pyname):
    cls = getattr(hm, pyname)
    fields = [f[0] for f in cls._fields_]
    size, offs = _c_layout(cname, fields)
    assert ctypes.sizeof(cls) == size
    assert [getattr(cls, f).offset for f in fields] == offs


def test_status_strings(hm):
    for s in range(6):
        assert hm.lib.hm_status_string(s)
    assert b"sm_100a" in hm.lib.hm_version()


def _args(hm, **kw):
    a = hm.ScanArgs()
    a.B, a.L, a.H, a.d, a.p, a.dv = 4, 2048, 8, 256, 128, 256
    a.io_dtype = hm.HM_BF16
    fake = 1 << 20  # an aligned address; validation never dereferences it
    a.q = a.k = a.v = a.o = a.W_q = a.W_k = fake
    a.dt = a.A_log = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_workspace_size_is_linear_in_length(hm):
    sizes = [hm.hm_scan_workspace_size(_args(hm, L=L)) for L in (1024, 2048, 4096)]
    assert all(s > 0 for s in sizes)
    # never quadratic: doubling L at most doubles the scratch (plus a constant)
    assert sizes[2] - sizes[1] <= 2 * (sizes[1] - sizes[0]) + 4096
    assert sizes[2] <= 4 * sizes[0] + (1 << 20)


def test_validation_rejects_bad_calls_before_launch(hm):
    def call(a):
        return hm.lib.hm_scan_chunked_fwd(ctypes.byref(a), None)
    assert call(_args(hm, B=-1)) == hm.HM_ERR_INVALID_ARG
    assert call(_args(hm, W_k=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_args(hm, q=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_args(hm, q=(1 << 20) + 2)) == hm.HM_ERR_INVALID_ARG
    assert call(_args(hm, A_log=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_args(hm, p=300)) == hm.HM_ERR_UNSUPPORTED
    assert call(_args(hm, dv=6)) == hm.HM_ERR_UNSUPPORTED
    # missing workspace
    assert call(_args(hm)) == hm.HM_ERR_INVALID_ARG
    assert b"workspace" in hm.lib.hm_last_error_detail()
    d = hm.DecodeArgs()
    d.B, d.H, d.d, d.p, d.dv = 2, 8, 256, 128, 256
    assert hm.lib.hm_step_decode(ctypes.byref(d), None) == hm.HM_ERR_INVALID_ARG  # null q
    assert hm.lib.hm_featmap(None, 1, 10, 1, 256, 128, None, 0, None, None, 1, None) == \
        hm.HM_ERR_INVALID_ARG
    m = hm.MixerArgs()
    m.B, m.L, m.d_model, m.H, m.E, m.p, m.conv_k = 1, 16, 2048, 8, 2050, 128, 4
    assert hm.lib.hm_mixer_fwd(ctypes.byref(m), None, 0, None) in (hm.HM_ERR_INVALID_ARG,
                                                                   hm.HM_ERR_UNSUPPORTED)


def _block(hm, **kw):
    fake = 1 << 20
    b = hm.BlockArgs()
    m = b.mixer
    m.B, m.L, m.d_model, m.H, m.E, m.p, m.conv_k = 2, 300, 512, 2, 512, 128, 4
    m.x = m.out = m.W_q = m.W_k = m.W_v = m.W_g = m.W_dt = m.conv_w = fake
    m.W_hq = m.W_hk = m.A_log = m.W_o = fake
    b.eps, b.d_ff, b.W_fc1, b.W_fc2 = 1e-5, 2048, fake, fake
    for k, v in kw.items():
        setattr(b, k, v)
    return b


def test_block_sizes_and_validation(hm):
    def call(b, ws=None, n=0):
        return hm.lib.hm_block_fwd(ctypes.byref(b), ws, n, None)
    size = hm.hm_block_workspace_size(_block(hm))
    M, D, dff = 600, 512, 2048
    # h1, h2 (bf16), the fp32 residual sum and the MLP's hidden activations, plus the mixer's own
    assert size >= M * D * (2 + 2 + 4) + M * dff * 2 + hm.hm_mixer_workspace_size(_block(hm).mixer)
    assert call(_block(hm)) == hm.HM_ERR_INVALID_ARG                    # no workspace
    assert b"workspace" in hm.lib.hm_last_error_detail()
    assert call(_block(hm, eps=0.0)) == hm.HM_ERR_INVALID_ARG
    assert call(_block(hm, d_ff=100)) == hm.HM_ERR_UNSUPPORTED
    assert call(_block(hm, W_fc2=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_block(hm, ln1_w=(1 << 20) + 4)) == hm.HM_ERR_INVALID_ARG   # misaligned
    assert hm.hm_block_workspace_size(_block(hm, d_ff=100)) == 0


def test_variant_flags_are_validated_before_launch(hm):
    def call(a):
        return hm.lib.hm_scan_chunked_fwd(ctypes.byref(a), None)
    assert call(_args(hm, flags=8)) == hm.HM_ERR_INVALID_ARG           # unknown bit
    assert b"flag" in hm.lib.hm_last_error_detail()
    assert call(_args(hm, flags=hm.HM_FLAG_ROPE)) == hm.HM_ERR_INVALID_ARG   # no rope_base
    assert call(_args(hm, flags=hm.HM_FLAG_ROPE, rope_base=1e4, pos0=-1)) == hm.HM_ERR_INVALID_ARG
    assert hm.hm_scan_workspace_size(_args(hm, flags=hm.HM_FLAG_ROPE, rope_base=1e4)) > 0
    assert call(_args(hm, flags=hm.HM_FLAG_DT_SCALED_INPUT, dt=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_args(hm, flags=hm.HM_FLAG_PER_FEATURE_DECAY, dt=None)) == hm.HM_ERR_INVALID_ARG
    # valid flags size a workspace like the plain call (CUDA-core path for the per-feature decay)
    assert hm.hm_scan_workspace_size(_args(hm, flags=hm.HM_FLAG_DT_SCALED_INPUT)) > 0
    assert hm.hm_scan_workspace_size(_args(hm, flags=hm.HM_FLAG_PER_FEATURE_DECAY)) > 0
    d = hm.DecodeArgs()
    d.B, d.H, d.d, d.p, d.dv = 2, 8, 256, 128, 256
    d.q = d.k = d.v = d.o = d.S = d.z = 1 << 20
    d.flags = 8
    assert hm.lib.hm_step_decode(ctypes.byref(d), None) == hm.HM_ERR_INVALID_ARG
    d.flags, d.rope_base = hm.HM_FLAG_ROPE, 1e4                             # needs positions
    assert hm.lib.hm_step_decode(ctypes.byref(d), None) == hm.HM_ERR_INVALID_ARG
    d.rope_base = 0.0
    d.flags = hm.HM_FLAG_DT_SCALED_INPUT                                    # needs dt
    assert hm.lib.hm_step_decode(ctypes.byref(d), None) == hm.HM_ERR_INVALID_ARG


def _bwd(hm, **kw):
    a = hm.ScanBwdArgs()
    a.B, a.L, a.H, a.d, a.p, a.dv = 4, 2048, 8, 256, 128, 256
    a.io_dtype = hm.HM_BF16
    fake = 1 << 20  # an aligned address; validation never dereferences it
    for n in ("q", "k", "v", "dout", "W_q", "W_k", "dt", "A_log", "grad_q", "grad_k", "grad_v", "grad_W_q",
              "grad_W_k", "grad_dt", "grad_A_log"):
        setattr(a, n, fake)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_backward_sizes_and_validation(hm):
    size = lambda a: hm.hm_scan_bwd_workspace_size(a)
    rows, F, p, d, ns = 4 * 2048 * 8, 256, 128, 256, 8
    s_bf16 = size(_bwd(hm))
    # the fp32 features, the value slices' shares (plus the denominator's) of
    # dphiq and dphik, and du as bf16 hi | lo segments for the tensor cores
    assert s_bf16 >= 2 * rows * F * 4 + 2 * (ns + 1) * rows * F * 4 + rows * 2 * p * 2
    # fp32 inputs carry W's rounding remainder too: one more segment of du and of W^T
    assert size(_bwd(hm, io_dtype=hm.HM_F32)) - s_bf16 == rows * p * 2 + d * p * 2
    # a width the tensor-core GEMMs do not take (d = 250) has no segments
    assert size(_bwd(hm, d=250)) < s_bf16
    sizes = [size(_bwd(hm, L=L)) for L in (512, 1024, 2048)]
    assert sizes[2] - sizes[1] <= 2 * (sizes[1] - sizes[0]) + 4096
    call = lambda a: hm.lib.hm_scan_bwd(ctypes.byref(a), None)
    assert call(_bwd(hm, W_k=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_bwd(hm, grad_q=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_bwd(hm, grad_dt=None)) == hm.HM_ERR_INVALID_ARG
    assert call(_bwd(hm, S0=1 << 20)) == hm.HM_ERR_INVALID_ARG          # S0 without z0
    assert call(_bwd(hm, q=(1 << 20) + 2)) == hm.HM_ERR_INVALID_ARG     # misaligned
    assert call(_bwd(hm, p=300)) == hm.HM_ERR_UNSUPPORTED
    assert size(_bwd(hm, p=300)) == 0
    assert call(_bwd(hm)) == hm.HM_ERR_INVALID_ARG                      # no workspace
    assert b"workspace" in hm.lib.hm_last_error_detail()
