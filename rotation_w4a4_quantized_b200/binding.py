"""Python binding of the ConvLinear4bit C ABI (argument marshalling only).

Each function takes torch tensors that already live on the current CUDA device, allocates the
outputs with torch (the library itself never allocates), and calls the C entry point of the
same name on torch's current stream. Every step of the hot path runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback. If the shared library is missing, importing this
module raises.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_c_ptr = ctypes.c_void_p

# argtypes of every exported entry point (kept in the order of include/convrot.h)
_SIGNATURES = {
    "convrot_status_string": ([_c_int], ctypes.c_char_p),
    "convrot_padded_k": ([_c_i64, _c_int], _c_i64),
    "convrot_make_rht": ([_c_int, _c_ptr, _c_ptr], _c_int),
    "convrot_rotate_quant_act": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64, _c_ptr,
                                  _c_ptr], _c_int),
    "convrot_prepack_weight": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64, _c_ptr,
                                _c_ptr], _c_int),
    "convrot_w4a4_linear": ([_c_ptr, _c_i64, _c_ptr, _c_ptr, _c_i64, _c_ptr, _c_ptr, _c_ptr,
                             _c_i64, _c_i64, _c_i64, _c_i64, _c_ptr], _c_int),
    "convrot_w4a4_gemm_s32": ([_c_ptr, _c_i64, _c_ptr, _c_i64, _c_ptr, _c_i64, _c_i64, _c_i64,
                               _c_i64, _c_ptr], _c_int),
    "convrot_rotate_quant_i8": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64, _c_ptr,
                                 _c_ptr], _c_int),
    "convrot_w8a8_linear": ([_c_ptr, _c_i64, _c_ptr, _c_ptr, _c_i64, _c_ptr, _c_ptr, _c_ptr,
                             _c_i64, _c_i64, _c_i64, _c_i64, _c_ptr], _c_int),
    "convrot_w8a8_gemm_s32": ([_c_ptr, _c_i64, _c_ptr, _c_i64, _c_ptr, _c_i64, _c_i64, _c_i64,
                               _c_i64, _c_ptr], _c_int),
    "convrot_nvfp4_k": ([_c_i64, _c_int], _c_i64),
    "convrot_nvfp4_scale_bytes": ([_c_i64, _c_i64, _c_int, _c_int], _c_i64),
    "convrot_mxfp4_scale_bytes": ([_c_i64, _c_i64, _c_int, _c_int], _c_i64),
    "convrot_rotate_quant_act_nvfp4": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64,
                                        _c_ptr, _c_ptr, _c_ptr], _c_int),
    "convrot_prepack_weight_nvfp4": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64,
                                      _c_ptr, _c_ptr, _c_ptr], _c_int),
    "convrot_nvfp4_linear": ([_c_ptr, _c_i64, _c_ptr, _c_ptr, _c_ptr, _c_i64, _c_ptr, _c_ptr,
                              _c_ptr, _c_ptr, _c_i64, _c_i64, _c_i64, _c_i64, _c_ptr], _c_int),
    "convrot_nvfp4_gemm_f32": ([_c_ptr, _c_i64, _c_ptr, _c_ptr, _c_i64, _c_ptr, _c_ptr, _c_i64,
                                _c_i64, _c_i64, _c_i64, _c_ptr], _c_int),
    "convrot_rotate_quant_act_mxfp4": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64,
                                        _c_ptr, _c_ptr], _c_int),
    "convrot_prepack_weight_mxfp4": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64,
                                      _c_ptr, _c_ptr], _c_int),
    "convrot_mxfp4_linear": ([_c_ptr, _c_i64, _c_ptr, _c_ptr, _c_i64, _c_ptr, _c_ptr, _c_ptr,
                              _c_i64, _c_i64, _c_i64, _c_i64, _c_ptr], _c_int),
    "convrot_mxfp4_gemm_f32": ([_c_ptr, _c_i64, _c_ptr, _c_ptr, _c_i64, _c_ptr, _c_ptr, _c_i64,
                                _c_i64, _c_i64, _c_i64, _c_ptr], _c_int),
    "convrot_w4a4_fused_workspace_bytes": ([_c_i64, _c_i64, _c_int], _c_i64),
    "convrot_w4a4_linear_fused": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr, _c_i64, _c_ptr,
                                   _c_ptr, _c_ptr, _c_i64, _c_i64, _c_ptr, _c_i64, _c_ptr],
                                  _c_int),
    "convrot_w4a4_linear_fused_noalloc": ([_c_ptr, _c_i64, _c_i64, _c_i64, _c_int, _c_ptr,
                                           _c_i64, _c_ptr, _c_ptr, _c_ptr, _c_i64, _c_i64,
                                           _c_ptr], _c_int),
    "convrot_selftest_bounded_wait": ([_c_int, _c_ptr], _c_int),
    "convrot_device_status": ([ctypes.POINTER(_c_int), _c_int], _c_int),
}

GROUPS = (16, 64, 256, 1024)


class ConvRotError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)}")


def _load() -> ctypes.CDLL:
    path = _build.LIBPATH
    if not os.path.exists(path):
        raise ImportError(
            f"ConvLinear4bit CUDA library not built ({path} missing); run "
            "`python -m rotation_w4a4_quantized_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(path)
    for name, (args, res) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def exported_names():
    """Names of the C entry points declared in include/convrot.h."""
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                       "convrot.h")
    text = open(hdr).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*]+\s+\*?(convrot_\w+)\s*\(", text,
                                 flags=re.M)))


def status_string(status: int) -> str:
    return lib.convrot_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise ConvRotError(fn, status)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def padded_k(K: int, group: int) -> int:
    v = lib.convrot_padded_k(int(K), int(group))
    if v < 0:
        raise ConvRotError("convrot_padded_k", 1 if group not in GROUPS else 2)
    return int(v)


def packed_stride(K_pad: int) -> int:
    """Row stride (bytes) used for packed code buffers: K_pad / 2 rounded up to 16."""
    return ((K_pad // 2 + 15) // 16) * 16


def int8_stride(K_pad: int) -> int:
    """Row stride (bytes) used for int8 code buffers: K_pad rounded up to 16."""
    return ((K_pad + 15) // 16) * 16


def make_rht(group: int, out: torch.Tensor | None = None) -> torch.Tensor:
    if out is None:
        out = torch.empty(group, group, dtype=torch.float32, device="cuda")
    _check("convrot_make_rht", lib.convrot_make_rht(int(group), _ptr(out), _stream()))
    return out


def _rotate_quant(fn_name, X, group, q=None, s=None, int8=False):
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a 2-D bf16 tensor with unit column stride")
    M, K = X.shape
    K_pad = padded_k(K, group)
    if q is None:
        width = int8_stride(K_pad) if int8 else packed_stride(K_pad)
        q = torch.empty(M, width, dtype=torch.uint8, device=X.device)
    if s is None:
        s = torch.empty(M, dtype=torch.float32, device=X.device)
    fn = getattr(lib, fn_name)
    _check(fn_name, fn(_ptr(X), M, K, X.stride(0), int(group), _ptr(q), q.stride(0), _ptr(s),
                       _stream()))
    return q, s


def rotate_quant_act(X: torch.Tensor, group: int, qx=None, sx=None):
    """Returns (qx uint8 [M, ldq], sx float32 [M]); only qx[:, :K_pad/2] is defined."""
    return _rotate_quant("convrot_rotate_quant_act", X, group, qx, sx)


def prepack_weight(W: torch.Tensor, group: int, qw=None, sw=None):
    """Returns (qw uint8 [N, ldq], sw float32 [N]); only qw[:, :K_pad/2] is defined."""
    return _rotate_quant("convrot_prepack_weight", W, group, qw, sw)


def w4a4_linear(qx, sx, qw, sw, K_pad: int, bias=None, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device)
    _check("convrot_w4a4_linear",
           lib.convrot_w4a4_linear(_ptr(qx), qx.stride(0), _ptr(sx), _ptr(qw), qw.stride(0),
                                   _ptr(sw), _ptr(bias), _ptr(out), out.stride(0), M, N,
                                   int(K_pad), _stream()))
    return out


def w4a4_gemm_s32(qx, qw, K_pad: int, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.int32, device=qx.device)
    _check("convrot_w4a4_gemm_s32",
           lib.convrot_w4a4_gemm_s32(_ptr(qx), qx.stride(0), _ptr(qw), qw.stride(0), _ptr(out),
                                     out.stride(0), M, N, int(K_pad), _stream()))
    return out


def rotate_quant_i8(X: torch.Tensor, group: int, q=None, s=None):
    """W8A8 variant: returns (q uint8 [rows, ldq] holding int8 codes, s float32 [rows]);
    only q[:, :K_pad] is defined. Serves activations and weights alike."""
    return _rotate_quant("convrot_rotate_quant_i8", X, group, q, s, int8=True)


def w8a8_linear(qx, sx, qw, sw, K_pad: int, bias=None, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device)
    _check("convrot_w8a8_linear",
           lib.convrot_w8a8_linear(_ptr(qx), qx.stride(0), _ptr(sx), _ptr(qw), qw.stride(0),
                                   _ptr(sw), _ptr(bias), _ptr(out), out.stride(0), M, N,
                                   int(K_pad), _stream()))
    return out


def w8a8_gemm_s32(qx, qw, K_pad: int, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.int32, device=qx.device)
    _check("convrot_w8a8_gemm_s32",
           lib.convrot_w8a8_gemm_s32(_ptr(qx), qx.stride(0), _ptr(qw), qw.stride(0), _ptr(out),
                                     out.stride(0), M, N, int(K_pad), _stream()))
    return out


def nvfp4_k(K: int, group: int) -> int:
    v = lib.convrot_nvfp4_k(int(K), int(group))
    if v < 0:
        raise ConvRotError("convrot_nvfp4_k", 1 if group not in GROUPS else 2)
    return int(v)


def nvfp4_scale_bytes(rows: int, K: int, group: int, weights: bool) -> int:
    v = lib.convrot_nvfp4_scale_bytes(int(rows), int(K), int(group), 1 if weights else 0)
    if v < 0:
        raise ConvRotError("convrot_nvfp4_scale_bytes", 2)
    return int(v)


def _rotate_quant_fp4(fn_name, X, group, weights, q=None, sf=None, g=None):
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a 2-D bf16 tensor with unit column stride")
    rows, K = X.shape
    K4 = nvfp4_k(K, group)
    if q is None:
        q = torch.empty(rows, packed_stride(K4), dtype=torch.uint8, device=X.device)
    if sf is None:
        sf = torch.empty(max(nvfp4_scale_bytes(rows, K, group, weights), 16), dtype=torch.uint8,
                         device=X.device)
    if g is None:
        g = torch.empty(rows, dtype=torch.float32, device=X.device)
    fn = getattr(lib, fn_name)
    _check(fn_name, fn(_ptr(X), rows, K, X.stride(0), int(group), _ptr(q), q.stride(0), _ptr(sf),
                       _ptr(g), _stream()))
    return q, sf, g


def rotate_quant_act_nvfp4(X, group: int, q=None, sf=None, g=None):
    """NVFP4 activations: (codes uint8 [M, ld] (K4 / 2 bytes defined), tiled block scales,
    row scales float32 [M])."""
    return _rotate_quant_fp4("convrot_rotate_quant_act_nvfp4", X, group, False, q, sf, g)


def prepack_weight_nvfp4(W, group: int, q=None, sf=None, g=None):
    """NVFP4 weights: (codes, tiled block scales for the B operand, row scales [N])."""
    return _rotate_quant_fp4("convrot_prepack_weight_nvfp4", W, group, True, q, sf, g)


def nvfp4_linear(qx, sfx, gx, qw, sfw, gw, K4: int, bias=None, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device)
    _check("convrot_nvfp4_linear",
           lib.convrot_nvfp4_linear(_ptr(qx), qx.stride(0), _ptr(sfx), _ptr(gx), _ptr(qw),
                                    qw.stride(0), _ptr(sfw), _ptr(gw), _ptr(bias), _ptr(out),
                                    out.stride(0), M, N, int(K4), _stream()))
    return out


def nvfp4_gemm_f32(qx, sfx, qw, sfw, K4: int, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32, device=qx.device)
    _check("convrot_nvfp4_gemm_f32",
           lib.convrot_nvfp4_gemm_f32(_ptr(qx), qx.stride(0), _ptr(sfx), _ptr(qw), qw.stride(0),
                                      _ptr(sfw), _ptr(out), out.stride(0), M, N, int(K4),
                                      _stream()))
    return out


def mxfp4_scale_bytes(rows: int, K: int, group: int, weights: bool) -> int:
    v = lib.convrot_mxfp4_scale_bytes(int(rows), int(K), int(group), 1 if weights else 0)
    if v < 0:
        raise ConvRotError("convrot_mxfp4_scale_bytes", 2)
    return int(v)


def _rotate_quant_mx(fn_name, X, group, weights, q=None, sf=None):
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a 2-D bf16 tensor with unit column stride")
    rows, K = X.shape
    K4 = nvfp4_k(K, group)
    if q is None:
        q = torch.empty(rows, packed_stride(K4), dtype=torch.uint8, device=X.device)
    if sf is None:
        sf = torch.empty(max(mxfp4_scale_bytes(rows, K, group, weights), 16), dtype=torch.uint8,
                         device=X.device)
    fn = getattr(lib, fn_name)
    _check(fn_name, fn(_ptr(X), rows, K, X.stride(0), int(group), _ptr(q), q.stride(0), _ptr(sf),
                       _stream()))
    return q, sf


def rotate_quant_act_mxfp4(X, group: int, q=None, sf=None):
    """MXFP4 activations: (codes uint8 [M, ld] (K4 / 2 bytes defined), scale atoms)."""
    return _rotate_quant_mx("convrot_rotate_quant_act_mxfp4", X, group, False, q, sf)


def prepack_weight_mxfp4(W, group: int, q=None, sf=None):
    """MXFP4 weights: (codes, scale images for the B operand)."""
    return _rotate_quant_mx("convrot_prepack_weight_mxfp4", W, group, True, q, sf)


def mxfp4_linear(qx, sfx, qw, sfw, K4: int, bias=None, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device)
    _check("convrot_mxfp4_linear",
           lib.convrot_mxfp4_linear(_ptr(qx), qx.stride(0), _ptr(sfx), _ptr(qw), qw.stride(0),
                                    _ptr(sfw), _ptr(bias), _ptr(out), out.stride(0), M, N,
                                    int(K4), _stream()))
    return out


def mxfp4_gemm_f32(qx, sfx, qw, sfw, K4: int, out=None) -> torch.Tensor:
    M, N = qx.shape[0], qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32, device=qx.device)
    _check("convrot_mxfp4_gemm_f32",
           lib.convrot_mxfp4_gemm_f32(_ptr(qx), qx.stride(0), _ptr(sfx), _ptr(qw), qw.stride(0),
                                      _ptr(sfw), _ptr(out), out.stride(0), M, N, int(K4),
                                      _stream()))
    return out


def conv_linear_mxfp4(X, qw, sfw, group: int, bias=None):
    """The MXFP4 variant's forward on prepacked weights."""
    qx, sfx = rotate_quant_act_mxfp4(X, group)
    return mxfp4_linear(qx, sfx, qw, sfw, nvfp4_k(X.shape[1], group), bias=bias)


def fused_workspace_bytes(M: int, K: int, group: int) -> int:
    """Bytes of device workspace w4a4_linear_fused needs for an [M, K] activation."""
    v = lib.convrot_w4a4_fused_workspace_bytes(int(M), int(K), int(group))
    if v < 0:
        raise ConvRotError("convrot_w4a4_fused_workspace_bytes", 1 if group not in GROUPS else 2)
    return int(v)


def w4a4_linear_fused(X, qw, sw, group: int, bias=None, out=None, workspace=None):
    """The whole ConvLinear4bit layer in one call: bf16 X [M, K] -> bf16 Y [M, N] (the same
    result as rotate_quant_act followed by w4a4_linear). `workspace` (uint8 device tensor of at
    least fused_workspace_bytes(M, K, group) bytes, 256-byte aligned) is allocated here with
    torch when not given."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a 2-D bf16 tensor with unit column stride")
    M, K = X.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
    need = fused_workspace_bytes(M, K, group)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _check("convrot_w4a4_linear_fused",
           lib.convrot_w4a4_linear_fused(_ptr(X), M, K, X.stride(0), int(group), _ptr(qw),
                                         qw.stride(0), _ptr(sw), _ptr(bias), _ptr(out),
                                         out.stride(0), N, _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream()))
    return out


NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


def w4a4_linear_fused_noalloc(X, qw, sw, group: int, bias=None, out=None):
    """The one-call layer with the library's built-in scratch array instead of a workspace
    (for callers that cannot allocate device memory; see convrot_w4a4_linear_fused_noalloc in
    include/convrot.h for the size limit and the rule that overlapping calls race). Allocates
    only `out` (with torch) when it is not given."""
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a 2-D bf16 tensor with unit column stride")
    M, K = X.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
    _check("convrot_w4a4_linear_fused_noalloc",
           lib.convrot_w4a4_linear_fused_noalloc(_ptr(X), M, K, X.stride(0), int(group), _ptr(qw),
                                                 qw.stride(0), _ptr(sw), _ptr(bias), _ptr(out),
                                                 out.stride(0), N, _stream()))
    return out


def selftest_bounded_wait(polls: int = 1 << 16):
    """Make one bounded wait give up on purpose (test of the failure path; no fault)."""
    _check("convrot_selftest_bounded_wait", lib.convrot_selftest_bounded_wait(int(polls), _stream()))


def device_status(clear: bool = False) -> int:
    v = _c_int(0)
    _check("convrot_device_status", lib.convrot_device_status(ctypes.byref(v), int(clear)))
    return int(v.value)


def conv_linear_4bit(X, qw, sw, group: int, K_pad: int, bias=None):
    """The whole ConvLinear4bit forward on prepacked weights: rotate + quantise the
    activations, then the W4A4 GEMM with the fused dequantisation."""
    qx, sx = rotate_quant_act(X, group)
    return w4a4_linear(qx, sx, qw, sw, K_pad, bias=bias)


def conv_linear_nvfp4(X, qw, sfw, gw, group: int, bias=None):
    """The NVFP4 variant's forward on prepacked weights."""
    qx, sfx, gx = rotate_quant_act_nvfp4(X, group)
    return nvfp4_linear(qx, sfx, gx, qw, sfw, gw, nvfp4_k(X.shape[1], group), bias=bias)


def conv_linear_8bit(X, qw, sw, group: int, K_pad: int, bias=None):
    """The W8A8 variant's forward on prepacked int8 weights."""
    qx, sx = rotate_quant_i8(X, group)
    return w8a8_linear(qx, sx, qw, sw, K_pad, bias=bias)
