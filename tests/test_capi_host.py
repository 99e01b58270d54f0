"""Host-side checks of the C-ABI library (no GPU needed, nothing is launched).

The library must load on a machine without a GPU, export every entry point that
include/convrot.h declares, compute padded K on the host, name every status code, and reject
bad arguments before touching the device.
"""

import ctypes
import os
import re

import pytest

from oracle import convrot_oracle as O
from rotation_w4a4_quantized_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def b():
    build.build()
    from rotation_w4a4_quantized_b200 import binding
    return binding


def header_names():
    text = open(os.path.join(ROOT, "include", "convrot.h")).read()
    return sorted(set(re.findall(r"\b(convrot_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol(b):
    names = header_names()
    assert len(names) == 26
    assert b.exported_names() == names
    for n in names:
        assert hasattr(b.lib, n), n
    # the ctypes table covers exactly the header
    assert sorted(b._SIGNATURES) == names


def test_padded_k_matches_oracle(b):
    for K in (0, 1, 15, 16, 17, 255, 256, 257, 3000, 3072, 15360):
        for g in (16, 64, 256, 1024):
            assert b.lib.convrot_padded_k(K, g) == O.padded_k(K, g)
    for g in (0, 4, 8, 32, 4096, -16):
        assert b.lib.convrot_padded_k(100, g) == -1
    assert b.lib.convrot_padded_k(-1, 16) == -1


def test_status_strings(b):
    for code in range(8):
        s = b.status_string(code)
        assert s.startswith("CONVROT_")
    assert b.status_string(99) == "CONVROT_ERR_UNKNOWN"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case below fails validation


def rq(b, X=FAKE, M=4, K=64, ldx=64, g=16, q=FAKE, ldq=32, s=FAKE):
    return b.lib.convrot_rotate_quant_act(X, M, K, ldx, g, q, ldq, s, None)


def test_quant_argument_validation(b):
    assert rq(b, g=17) == 1 and rq(b, g=4) == 1 and rq(b, g=4096) == 1
    assert rq(b, M=-1) == 2 and rq(b, K=-1) == 2
    assert rq(b, ldx=32) == 2                           # ldx < K
    assert rq(b, ldq=16) == 2                           # ldq < K_pad / 2
    assert rq(b, K=40000, ldx=40000, ldq=20480) == 2    # K_pad above the kernel limit
    assert rq(b, s=None) == 3 and rq(b, X=None) == 3 and rq(b, q=None) == 3
    assert rq(b, X=FAKE + 2) == 4 and rq(b, q=FAKE + 8) == 4 and rq(b, s=FAKE + 2) == 4
    assert rq(b, ldx=68, K=64) == 4                     # ldx not a multiple of 8
    assert rq(b, ldq=40) == 4                           # ldq not a multiple of 16
    assert rq(b, M=0) == 0                              # no-op, nothing touched
    assert b.lib.convrot_prepack_weight(FAKE, 4, 64, 64, 48, FAKE, 32, FAKE, None) == 1


def lin(b, qx=FAKE, ldqx=32, sx=FAKE, qw=FAKE, ldqw=32, sw=FAKE, bias=None, Y=FAKE, ldy=64,
        M=8, N=64, K_pad=64):
    return b.lib.convrot_w4a4_linear(qx, ldqx, sx, qw, ldqw, sw, bias, Y, ldy, M, N, K_pad, None)


def test_gemm_argument_validation(b):
    assert lin(b, M=-1) == 2 and lin(b, K_pad=0) == 2 and lin(b, K_pad=40) == 2
    assert lin(b, K_pad=262144, ldqx=131072, ldqw=131072) == 2
    assert lin(b, ldqx=16) == 2 and lin(b, ldy=32) == 2
    assert lin(b, qx=None) == 3 and lin(b, sx=None) == 3 and lin(b, Y=None) == 3
    assert lin(b, qw=FAKE + 4) == 4 and lin(b, ldqx=40) == 4 and lin(b, Y=FAKE + 1) == 4
    assert lin(b, bias=FAKE + 1) == 4 and lin(b, sx=FAKE + 2) == 4
    assert lin(b, M=0) == 0 and lin(b, N=0) == 0
    s32 = b.lib.convrot_w4a4_gemm_s32
    assert s32(FAKE, 32, FAKE, 32, FAKE + 2, 66, 8, 64, 64, None) == 4   # acc alignment
    assert s32(None, 32, FAKE, 32, FAKE, 64, 8, 64, 64, None) == 3
    assert b.lib.convrot_make_rht(17, FAKE, None) == 1
    assert b.lib.convrot_make_rht(16, None, None) == 3
    assert b.lib.convrot_device_status(None, 0) == 3
    assert b.lib.convrot_selftest_bounded_wait(0, None) == 2
    assert b.lib.convrot_selftest_bounded_wait(-5, None) == 2


def rq8(b, X=FAKE, M=4, K=64, ldx=64, g=16, q=FAKE, ldq=64, s=FAKE):
    return b.lib.convrot_rotate_quant_i8(X, M, K, ldx, g, q, ldq, s, None)


def lin8(b, qx=FAKE, ldqx=64, sx=FAKE, qw=FAKE, ldqw=64, sw=FAKE, bias=None, Y=FAKE, ldy=64,
         M=8, N=64, K_pad=64):
    return b.lib.convrot_w8a8_linear(qx, ldqx, sx, qw, ldqw, sw, bias, Y, ldy, M, N, K_pad, None)


def test_int8_argument_validation(b):
    # int8 code rows hold K_pad bytes (not K_pad / 2)
    assert rq8(b, ldq=32) == 2 and rq8(b, ldq=48) == 2
    assert rq8(b, g=32) == 1 and rq8(b, s=None) == 3 and rq8(b, ldq=72) == 4
    assert rq8(b, K=40000, ldx=40000, ldq=40960) == 2
    assert rq8(b, M=0) == 0
    assert lin8(b, ldqx=32) == 2 and lin8(b, ldqw=48) == 2 and lin8(b, K_pad=40) == 2
    assert lin8(b, K_pad=262144, ldqx=262144, ldqw=262144) == 2
    assert lin8(b, sw=None) == 3 and lin8(b, qx=FAKE + 8) == 4 and lin8(b, ldqw=72) == 4
    assert lin8(b, M=0) == 0
    s32 = b.lib.convrot_w8a8_gemm_s32
    assert s32(FAKE, 32, FAKE, 64, FAKE, 64, 8, 64, 64, None) == 2      # ldqx < K_pad
    assert s32(FAKE, 64, FAKE, 64, FAKE + 2, 66, 8, 64, 64, None) == 4  # acc alignment


def test_nvfp4_host_helpers_and_validation(b):
    for K in (0, 1, 40, 100, 256, 3000, 3072, 15360):
        for g in (16, 64, 256, 1024):
            K4 = -(-O.padded_k(K, g) // 64) * 64
            assert b.lib.convrot_nvfp4_k(K, g) == K4
            for rows in (1, 128, 129, 224, 4608):
                assert b.lib.convrot_nvfp4_scale_bytes(rows, K, g, 0) == \
                    -(-rows // 128) * ((K4 // 64 + 1) // 2 * 2) * 512   # atoms, even count
                assert b.lib.convrot_nvfp4_scale_bytes(rows, K, g, 1) == \
                    -(-rows // 192) * (K4 // 64) * 4096              # one image per chunk
    assert b.lib.convrot_nvfp4_k(10, 32) == -1 and b.lib.convrot_nvfp4_scale_bytes(4, 64, 16, 2) == -1
    q4 = b.lib.convrot_rotate_quant_act_nvfp4
    assert q4(FAKE, 4, 64, 64, 16, FAKE, 16, FAKE, FAKE, None) == 2      # ldq < K4 / 2
    assert q4(FAKE, 4, 64, 64, 16, FAKE, 32, None, FAKE, None) == 3      # no scale buffer
    assert q4(FAKE, 4, 64, 64, 16, FAKE, 32, FAKE + 8, FAKE, None) == 4  # scales misaligned
    assert q4(FAKE, 4, 64, 64, 12, FAKE, 32, FAKE, FAKE, None) == 1
    l4 = b.lib.convrot_nvfp4_linear
    args = [FAKE, 32, FAKE, FAKE, FAKE, 32, FAKE, FAKE, None, FAKE, 64, 8, 64, 64, None]
    assert l4(*args[:13], 48, None) == 2                                  # K4 not a multiple of 64
    bad = list(args); bad[2] = FAKE + 4
    assert l4(*bad) == 4
    bad = list(args); bad[3] = None
    assert l4(*bad) == 3
    assert b.lib.convrot_nvfp4_gemm_f32(FAKE, 16, FAKE, FAKE, 32, FAKE, FAKE, 64, 8, 64, 64, None) == 2


def test_mxfp4_host_helpers_and_validation(b):
    for K in (0, 1, 40, 100, 256, 3000, 3072, 15360):
        for g in (16, 64, 256, 1024):
            K4 = -(-O.padded_k(K, g) // 64) * 64
            kc = -(-K4 // 128)                                     # 128-K chunks of 4 scales
            for rows in (1, 128, 129, 224, 4608):
                assert b.lib.convrot_mxfp4_scale_bytes(rows, K, g, 0) == \
                    -(-rows // 128) * ((kc + 1) // 2 * 2) * 512
                assert b.lib.convrot_mxfp4_scale_bytes(rows, K, g, 1) == -(-rows // 224) * kc * 4096
    assert b.lib.convrot_mxfp4_scale_bytes(4, 64, 16, 2) == -1
    assert b.lib.convrot_mxfp4_scale_bytes(4, 64, 12, 0) == -1
    q = b.lib.convrot_rotate_quant_act_mxfp4
    assert q(FAKE, 4, 64, 64, 16, FAKE, 16, FAKE, None) == 2           # ldq < K4 / 2
    assert q(FAKE, 4, 64, 64, 16, FAKE, 32, None, None) == 3           # no scale buffer
    assert q(FAKE, 4, 64, 64, 16, FAKE, 32, FAKE + 8, None) == 4       # scales misaligned
    assert q(FAKE, 4, 64, 64, 12, FAKE, 32, FAKE, None) == 1
    assert q(FAKE, 0, 64, 64, 16, FAKE, 32, FAKE, None) == 0            # nothing to do
    lin = b.lib.convrot_mxfp4_linear
    args = [FAKE, 32, FAKE, FAKE, 32, FAKE, None, FAKE, 64, 8, 64, 64, None]
    assert lin(*args[:11], 48, None) == 2                                # K4 not a multiple of 64
    bad = list(args); bad[2] = FAKE + 4
    assert lin(*bad) == 4
    bad = list(args); bad[3] = None
    assert lin(*bad) == 3
    assert b.lib.convrot_mxfp4_gemm_f32(FAKE, 16, FAKE, FAKE, 32, FAKE, FAKE, 64, 8, 64, 64, None) == 2


def test_valid_call_without_device_reports_device_error(b):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # arguments pass validation; the device check then fails cleanly (nothing launched)
    assert rq(b) == 5 and rq8(b) == 5 and lin8(b) == 5
    assert b.lib.convrot_make_rht(16, FAKE, None) == 5
    v = ctypes.c_int(0)
    assert b.lib.convrot_device_status(ctypes.byref(v), 0) == 5


def test_binding_fails_loudly_without_the_library(b, monkeypatch, tmp_path):
    """No CPU fallback: with the shared library absent, loading the binding raises."""
    monkeypatch.setattr(b._build, "LIBPATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError, match="not built"):
        b._load()


def fused(b, X=FAKE, M=4, K=64, ldx=64, g=16, qw=FAKE, ldqw=32, sw=FAKE, bias=None, Y=FAKE,
          ldy=64, N=64, ws=FAKE, wsb=None):
    if wsb is None:
        wsb = b.lib.convrot_w4a4_fused_workspace_bytes(M, K, g) if g in (16, 64, 256, 1024) else 0
    return b.lib.convrot_w4a4_linear_fused(X, M, K, ldx, g, qw, ldqw, sw, bias, Y, ldy, N, ws,
                                           wsb, None)


def test_fused_workspace_and_argument_validation(b):
    # packed codes [M, round_up(K_pad / 2, 16)], then the row scales at the next 256-byte boundary
    ws = b.lib.convrot_w4a4_fused_workspace_bytes
    assert ws(4, 64, 16) == 256 + 256
    assert ws(4608, 3072, 256) == 4608 * 1536 + 4608 * 4 // 256 * 256
    assert ws(37, 3000, 1024) == -(-37 * 1536 // 256) * 256 + 256
    assert ws(4, 64, 48) == -1 and ws(-1, 64, 16) == -1
    assert fused(b, g=48) == 1
    assert fused(b, K=0) == 2
    assert fused(b, K=40000, ldx=40000, ldqw=20480) == 2  # K_pad above the quantisation limit
    assert fused(b, wsb=100) == 2                         # workspace too small
    assert fused(b, ws=FAKE + 16) == 4                    # workspace not 256-byte aligned
    assert fused(b, X=FAKE + 2) == 4 and fused(b, ldx=68) == 4
    assert fused(b, X=None) == 3 and fused(b, sw=None) == 3 and fused(b, qw=None) == 3
    assert fused(b, ws=None) == 3
    assert fused(b, ldy=32) == 2                          # ldy < N
    assert fused(b, M=0) == 0 and fused(b, N=0) == 0      # no-ops, nothing touched
