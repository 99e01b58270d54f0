"""GPU parity of the tcgen05 W4A4 GEMM (+ fused dequantisation) against the CPU oracle.

The int32 accumulators must be bit-exact when the GPU is fed the oracle's codes; the
dequantised bf16 output must agree element by element within the bound of tests/parity.py.
"""

import numpy as np
import pytest
import torch

from oracle import convrot_oracle as O
from synthetic import CONFIGS, make_inputs
from tests.parity import (Y_FROB, bf16_to_f64, check_y_elementwise, gpu_codes, rel_frob)

pytestmark = pytest.mark.gpu


def upload_packed(packed: np.ndarray, K_pad: int, b) -> torch.Tensor:
    ld = b.packed_stride(K_pad)
    buf = torch.zeros(packed.shape[0], ld, dtype=torch.uint8)
    buf[:, : K_pad // 2] = torch.from_numpy(packed)
    return buf.cuda()


def random_packed(rows: int, K_pad: int, seed: int) -> np.ndarray:
    """Seeded random packed bytes: every byte is a valid pair of int4 codes (-8..7)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 256, (rows, K_pad // 2), generator=g, dtype=torch.uint8).numpy()


@pytest.mark.parametrize("M,N,K_pad", [(64, 128, 256), (128, 256, 128), (200, 300, 3008),
                                       (1, 8, 16), (129, 257, 272), (333, 520, 1024),
                                       (256, 512, 4096)])
def test_s32_bit_exact_on_oracle_codes(cuda_lib, M, N, K_pad):
    px = random_packed(M, K_pad, seed=M)
    pw = random_packed(N, K_pad, seed=N + 1)
    acc = cuda_lib.w4a4_gemm_s32(upload_packed(px, K_pad, cuda_lib),
                                 upload_packed(pw, K_pad, cuda_lib), K_pad)
    ref = O.int_gemm(O.unpack_int4(px), O.unpack_int4(pw))
    got = acc.cpu().numpy().astype(np.int64)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} accumulators differ"


def test_s32_extremes(cuda_lib):
    # all codes +7 x -7 (and -8 x -8): the largest magnitudes the accumulator sees
    K_pad = 15360
    px = np.full((130, K_pad // 2), 0x77, dtype=np.uint8)
    pw = np.full((260, K_pad // 2), 0x99, dtype=np.uint8)
    pw[1] = 0x88
    acc = cuda_lib.w4a4_gemm_s32(upload_packed(px, K_pad, cuda_lib),
                                 upload_packed(pw, K_pad, cuda_lib), K_pad).cpu().numpy()
    assert (acc[:, 0] == -49 * K_pad).all() and (acc[:, 1] == -56 * K_pad).all()


def test_s32_maximum_k(cuda_lib):
    """K_pad at the documented maximum (131072) with the largest products of valid codes
    (+-7 x +-7): 256 * 49 * 131072 still fits the int32 accumulator."""
    K_pad = 131072
    px = np.full((130, K_pad // 2), 0x77, dtype=np.uint8)          # +7
    pw = np.full((200, K_pad // 2), 0x99, dtype=np.uint8)          # -7
    pw[1] = 0x77
    pw[2, : K_pad // 4] = 0x11                                     # +1 on the first half of K
    acc = cuda_lib.w4a4_gemm_s32(upload_packed(px, K_pad, cuda_lib),
                                 upload_packed(pw, K_pad, cuda_lib), K_pad).cpu().numpy()
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    assert (acc[:, 0] == -49 * K_pad).all() and (acc[:, 1] == 49 * K_pad).all()
    assert (acc[:, 2] == 7 * (K_pad // 2) - 49 * (K_pad // 2)).all()


@pytest.mark.parametrize("name", ["qkv", "proj_out", "sweep"])
def test_s32_full_size_sampled(cuda_lib, name):
    w = CONFIGS[name]
    K_pad = O.padded_k(w.K, w.group)
    px = random_packed(w.M, K_pad, seed=7)
    pw = random_packed(w.N, K_pad, seed=8)
    acc = cuda_lib.w4a4_gemm_s32(upload_packed(px, K_pad, cuda_lib),
                                 upload_packed(pw, K_pad, cuda_lib), K_pad)
    cx, cw = O.unpack_int4(px), O.unpack_int4(pw)
    rng = np.random.default_rng(1)
    rows = rng.integers(0, w.M, 4096)
    cols = rng.integers(0, w.N, 4096)
    got = acc[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()].cpu().numpy()
    assert np.array_equal(got.astype(np.int64), O.int_gemm_sampled(cx, cw, rows, cols))
    # one full 128-row band (every N tile, every K stage)
    band = slice(w.M - 128, w.M)
    ref = O.int_gemm_fp64(cx[band], cw)
    assert np.array_equal(acc[band].cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("M,N,K_pad", [(64, 128, 256), (200, 300, 3008), (129, 257, 272)])
def test_dequant_epilogue_on_oracle_codes(cuda_lib, M, N, K_pad, with_bias):
    rng = np.random.default_rng(M + N)
    px = random_packed(M, K_pad, seed=M + 3)
    pw = random_packed(N, K_pad, seed=N + 4)
    sx = (rng.uniform(0.01, 3.0, M)).astype(np.float32)
    sw = (rng.uniform(1e-4, 5e-3, N)).astype(np.float32)
    sx[M // 2] = 0.0                                         # an all-zero activation row
    bias = torch.randn(N, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    y = cuda_lib.w4a4_linear(upload_packed(px, K_pad, cuda_lib), torch.from_numpy(sx).cuda(),
                             upload_packed(pw, K_pad, cuda_lib), torch.from_numpy(sw).cuda(),
                             K_pad, bias=bias.cuda() if with_bias else None)
    acc = O.int_gemm(O.unpack_int4(px), O.unpack_int4(pw))
    b64 = bf16_to_f64(bias) if with_bias else None
    check_y_elementwise(bf16_to_f64(y), acc, sx, sw, b64, "dequant")


def test_dequant_tiny_row_scales(cuda_lib):
    """Row scales far below the fp32 normal range against weight scales far above it: the
    epilogue multiplies the exact integer accumulator by the scale as stored ("comfy-kitchen PR
    #65", the fp32 fix of int4_linear: the scales multiply the exact integer product). Row 3's
    scale, 383 * 2^-149, is a subnormal fp32 whose product with any accumulator is exact; a
    1/256 folded into it would round it to 2^-149 (33 % off). Row 4 is a bf16 activation row of
    magnitude ~1e-36 (scale ~1.4e-37)."""
    M, N, K_pad = 64, 96, 512
    rng = np.random.default_rng(11)
    px = random_packed(M, K_pad, seed=21)
    pw = random_packed(N, K_pad, seed=22)
    sx = rng.uniform(0.01, 3.0, M).astype(np.float32)
    sx[3] = np.array([383], dtype=np.uint32).view(np.float32)[0]
    sx[4] = np.float32(1e-36 / 7)
    sw = rng.uniform(1e-4, 5e-3, N).astype(np.float32)
    sw[N // 2:] = np.float32(2.0 ** 100)                       # large-magnitude weight rows
    sw[N // 2:] /= np.float32(1.0) + (np.arange(N - N // 2, dtype=np.float32) % 7)
    qx, qw = upload_packed(px, K_pad, cuda_lib), upload_packed(pw, K_pad, cuda_lib)
    y = cuda_lib.w4a4_linear(qx, torch.from_numpy(sx).cuda(), qw, torch.from_numpy(sw).cuda(),
                             K_pad)
    acc = O.int_gemm(O.unpack_int4(px), O.unpack_int4(pw))
    yg = bf16_to_f64(y)
    check_y_elementwise(yg, acc, sx, sw, None, "tiny row scales")
    big = slice(N // 2, N)
    ref = O.dequant(acc, sx, sw)[3, big]
    assert np.all(np.abs(yg[3, big] - ref) <= 2.0 ** -8 * np.abs(ref)), "row 3 off"
    assert np.count_nonzero(ref) > 0


def test_output_stride_and_zero_sizes(cuda_lib):
    K_pad, M, N = 256, 70, 136
    px, pw = random_packed(M, K_pad, 1), random_packed(N, K_pad, 2)
    qx, qw = upload_packed(px, K_pad, cuda_lib), upload_packed(pw, K_pad, cuda_lib)
    sx = torch.ones(M, device="cuda")
    sw = torch.full((N,), 1.0 / 64, device="cuda")
    big = torch.full((M, N + 24), 7.0, dtype=torch.bfloat16, device="cuda")
    cuda_lib.w4a4_linear(qx, sx, qw, sw, K_pad, out=big[:, :N])
    assert (big[:, N:] == 7.0).all()                         # nothing written past N
    acc = O.int_gemm(O.unpack_int4(px), O.unpack_int4(pw))
    check_y_elementwise(bf16_to_f64(big[:, :N]), acc, np.ones(M), np.full(N, 1 / 64), None, "ld")
    empty = cuda_lib.w4a4_linear(qx[:0], sx[:0], qw, sw, K_pad)
    assert empty.shape == (0, N)


@pytest.mark.parametrize("name", ["tiny", "qkv"])
def test_layer_end_to_end(cuda_lib, name):
    """GPU rotate+quant -> GPU GEMM vs the oracle's whole layer (with bias)."""
    w = CONFIGS[name]
    X, W, bias = make_inputs(w, with_bias=True)
    g = w.group
    K_pad = O.padded_k(w.K, g)
    qw, sw = cuda_lib.prepack_weight(W.cuda(), g)
    y = cuda_lib.conv_linear_4bit(X.cuda(), qw, sw, g, K_pad, bias=bias.cuda())
    torch.cuda.synchronize()
    rows = np.arange(w.M) if w.M <= 256 else np.sort(
        np.random.default_rng(3).choice(w.M, 256, replace=False))
    _, ref_sx, ref_cx = O.rotate_quant(bf16_to_f64(X)[rows], g)
    _, ref_sw, ref_cw = O.rotate_quant(bf16_to_f64(W), g)
    acc = O.int_gemm_fp64(ref_cx, ref_cw)   # exact: integer sums far below 2^53
    y_ref = O.dequant(acc, ref_sx, ref_sw, bf16_to_f64(bias))
    y_gpu = bf16_to_f64(y[torch.from_numpy(rows).cuda()])
    err = rel_frob(y_gpu, y_ref)
    assert err <= Y_FROB, err
    # the quantised layer approximates the unquantised linear (reported, loose bound)
    y_fp = bf16_to_f64(X)[rows] @ bf16_to_f64(W).T + bf16_to_f64(bias)[None, :]
    assert rel_frob(y_gpu, y_fp) < 0.25
    # same codes on both sides -> elementwise bound on a row subset
    codes_x = gpu_codes(cuda_lib.rotate_quant_act(X.cuda(), g)[0], K_pad)[rows]
    assert np.mean(codes_x == ref_cx) >= 0.9999
