"""GPU parity of the NVFP4 variant (rotate + e2m1/e4m3 block quantisation, block-scaled tcgen05
FP4 GEMM + dequantisation) against the CPU oracle, through the C ABI.

Bars (floating point decides the codes, as in the integer path): element codes >= 99.99 %
identical and never more than one code apart; block-scale bytes >= 99.99 % identical and never
more than one code apart; row scales within 1e-6 relative. The GEMM accumulates in fp32 on the
tensor cores: every product is exact, so against the exact fp64 sum each accumulator is within
K4 * 2^-24 of the sum of the magnitudes of its terms (the fp32 summation bound). The bf16 output
meets the dequantisation bound of tests/parity.py; whole layers meet the 1e-2 Frobenius bar.
"""

import numpy as np
import pytest
import torch

from oracle import convrot_oracle as O
from synthetic import CONFIGS, make_inputs
from synthetic.workloads import make_matrix
from tests.parity import (CODE_MATCH, SCALE_RTOL, Y_FROB, bf16_to_f64, check_scales,
                          check_y_elementwise, rel_frob)

pytestmark = pytest.mark.gpu

GROUPS = (16, 64, 256, 1024)
TILE_A, TILE_B = 128, 192


def sf_index(rows, nblk, tile_rows):
    """Byte offsets [rows, nblk, replicas] of block scale (r, b), as stated in
    include/convrot.h: weights (192-row tiles) as 4096-byte images, one per 64-K chunk, in four
    replicas; activations (128-row tiles) as 512-byte atoms, the chunk count per tile rounded
    up to even, one replica."""
    r = np.arange(rows)[:, None, None]
    b = np.arange(nblk)[None, :, None]
    t, rr = r // tile_rows, r % tile_rows
    kc = b // 4
    if tile_rows == TILE_A:
        kc_even = (nblk // 4 + 1) // 2 * 2
        return (t * kc_even + kc) * 512 + 16 * (rr % 32) + 4 * ((rr % 128) // 32) + b % 4
    q = np.arange(4)[None, None, :]
    lane = rr % 32 + 32 * q
    return ((t * (nblk // 4) + kc) * 4096 + 256 * (lane // 8) + 128 * (rr // 128)
            + 16 * (lane % 8) + 4 * ((rr % 128) // 32) + b % 4)


def sf_size(rows, nblk, tile_rows):
    tiles = -(-rows // tile_rows)
    kc = nblk // 4
    return tiles * ((kc + 1) // 2 * 2 * 512 if tile_rows == TILE_A else kc * 4096)


def untile(sf: torch.Tensor, rows, K4, tile_rows):
    """Block-scale bytes [rows, K4 / 16] read back from the images; all replicas agree."""
    v = sf.cpu().numpy()[sf_index(rows, K4 // 16, tile_rows)]
    assert (v == v[:, :, :1]).all(), "replicas of the block scales differ"
    return v[:, :, 0]


def tile(sb_bytes: np.ndarray, tile_rows) -> torch.Tensor:
    rows, nblk = sb_bytes.shape
    flat = np.zeros(sf_size(rows, nblk, tile_rows), dtype=np.uint8)
    idx = sf_index(rows, nblk, tile_rows)
    flat[idx] = np.broadcast_to(sb_bytes[:, :, None], idx.shape)
    return torch.from_numpy(flat)


@pytest.mark.parametrize("tile_rows,rows,nblk", [(TILE_B, 448, 8), (TILE_A, 256, 16),
                                                  (TILE_A, 128, 12)])
def test_scale_layouts_are_injective(tile_rows, rows, nblk):
    """Host check of the test's own index map: no byte is used twice and every index is inside
    the buffer; whole activation tiles with an even chunk count fill it exactly (weights leave
    lanes of rows past 192 unused; an odd chunk count leaves a padding atom per tile)."""
    idx = sf_index(rows, nblk, tile_rows)
    size = sf_size(rows, nblk, tile_rows)
    assert len(np.unique(idx)) == idx.size and idx.max() < size
    if tile_rows == TILE_A and (nblk // 4) % 2 == 0:
        assert idx.size == size


RANK = {v: i for i, v in enumerate(sorted(set(O.e2m1_values().tolist())))}


def code_ranks(values):
    return np.vectorize(lambda v: RANK[0.0 if v == 0 else v])(values)


def unpack_e2m1(q: torch.Tensor, K4):
    p = q[:, : K4 // 2].cpu().numpy().astype(np.int64)
    nib = np.empty((p.shape[0], K4), dtype=np.int64)
    nib[:, 0::2] = p & 15
    nib[:, 1::2] = p >> 4
    return O.e2m1_values()[nib]


def check_fp4(q, sf, g, X, group, tile_rows, what):
    rows, K = X.shape
    K_pad = O.padded_k(K, group)
    K4 = -(-K_pad // 64) * 64
    _, sb_bytes, g_ref, e_ref, _ = O.rotate_quant_nvfp4(bf16_to_f64(X), group)
    # the GPU runs over K4 >= K_pad: whole zero groups past K_pad give zero codes and scales
    e_ref = np.pad(e_ref, ((0, 0), (0, K4 - K_pad)))
    sb_ref_b = np.pad(sb_bytes, ((0, 0), (0, (K4 - K_pad) // 16))).astype(np.int64)
    check_scales(g, g_ref, what)
    sb_gpu = untile(sf, rows, K4, tile_rows).astype(np.int64)
    d = np.abs(sb_gpu - sb_ref_b)
    assert d.max(initial=0) <= 1, f"{what}: block scale off by {d.max()}"
    assert np.mean(d == 0) >= CODE_MATCH, f"{what}: block scales {np.mean(d == 0):.6%} equal"
    same_blk = np.repeat(d == 0, 16, axis=1)
    e_gpu = unpack_e2m1(q, K4)
    de = np.abs(code_ranks(e_gpu) - code_ranks(e_ref))[same_blk]
    assert de.max(initial=0) <= 1, f"{what}: element off by {de.max()} codes"
    assert np.mean(de == 0) >= CODE_MATCH, f"{what}: elements {np.mean(de == 0):.6%} equal"


# ---------------------------------------------------------------------------- quantisation
@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("M,K", [(64, 1024), (37, 3072), (130, 3000), (5, 40), (300, 15360)])
def test_quant_nvfp4_matches_oracle(cuda_lib, g, M, K):
    if K == 15360 and g == 16:
        pytest.skip("covered by the other groups")
    X = make_matrix(M, K, seed=M * 5 + K + g, std=1.0, row_outliers=3, row_scale=40.0)
    q, sf, gs = cuda_lib.rotate_quant_act_nvfp4(X.cuda(), g)
    torch.cuda.synchronize()
    check_fp4(q, sf, gs, X, g, TILE_A, f"act g{g} M{M} K{K}")
    qw, sfw, gw = cuda_lib.prepack_weight_nvfp4(X.cuda(), g)
    torch.cuda.synchronize()
    check_fp4(qw, sfw, gw, X, g, TILE_B, f"wgt g{g} M{M} K{K}")


GUARD = 0xA5


@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("M,K", [(37, 3000), (130, 1088), (225, 1024)])
def test_quant_nvfp4_writes_nothing_outside_its_outputs(cuda_lib, g, M, K):
    """Guard bytes around every output: code rows wider than K4 / 2 and one guard row after the
    last; the block-scale buffer longer than its layout, with the bytes the layout leaves unused
    (an activation tile's padding atom when its chunk count is odd, weight-image lanes of rows
    past the tile) filled too; guard row scales after row M - 1. Each must stay untouched."""
    X = make_matrix(M, K, seed=M + K + g, std=1.0, row_outliers=3, row_scale=40.0)
    K4 = cuda_lib.nvfp4_k(K, g)
    for weights, tile_rows in ((False, TILE_A), (True, TILE_B)):
        ldq = -(-(K4 // 2 + 32) // 16) * 16
        q = torch.full((M + 1, ldq), GUARD, dtype=torch.uint8, device="cuda")
        size = cuda_lib.nvfp4_scale_bytes(M, K, g, weights)
        assert size == sf_size(M, K4 // 16, tile_rows)
        sf = torch.full((size + 256,), GUARD, dtype=torch.uint8, device="cuda")
        gs = torch.full((M + 8,), -123.0, dtype=torch.float32, device="cuda")
        fn = cuda_lib.prepack_weight_nvfp4 if weights else cuda_lib.rotate_quant_act_nvfp4
        fn(padded_rows(X), g, q=q[:M], sf=sf, g=gs[:M])
        torch.cuda.synchronize()
        what = f"{'wgt' if weights else 'act'} g{g} M{M} K{K}"
        assert (q[:M, K4 // 2:] == GUARD).all() and (q[M] == GUARD).all(), what
        assert (gs[M:] == -123.0).all(), what
        used = np.zeros(size + 256, dtype=bool)
        used[sf_index(M, K4 // 16, tile_rows).ravel()] = True
        assert (sf.cpu().numpy()[~used] == GUARD).all(), f"{what}: scale bytes written outside the layout"
        check_fp4(q[:M], sf, gs[:M], X, g, tile_rows, what)


def test_quant_nvfp4_zero_and_onehot_rows(cuda_lib):
    M, K, g = 8, 256, 64
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[1, 70] = 3.0
    X[2] = 1.0                                       # DC row: R 1 = 1 keeps it flat
    q, sf, gs = cuda_lib.rotate_quant_act_nvfp4(X.cuda(), g)
    torch.cuda.synchronize()
    check_fp4(q, sf, gs, X, g, TILE_A, "special rows")
    assert gs[0].item() == 0.0 and not q[0, :128].any()
    e = unpack_e2m1(q, 256)
    assert (np.abs(e[1, 64:128]) == 6.0).all()       # one-hot: +-6 over its group
    assert (e[2] == 6.0).all()                       # flat row: every element the block maximum


def padded_rows(X, extra=8):
    """X with a row stride rounded up to a multiple of 8 elements (the ABI's rule)."""
    ld = -(-X.shape[1] // 8) * 8 + extra
    buf = torch.zeros(X.shape[0], ld, dtype=X.dtype, device="cuda")
    buf[:, : X.shape[1]] = X.cuda()
    return buf[:, : X.shape[1]]


@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("K", [32768, 32763])
def test_quant_nvfp4_maximum_row_length(cuda_lib, g, K):
    """K4 at the documented maximum (32768), whole and ragged rows, both scale layouts."""
    X = make_matrix(37, K, seed=K + 5 * g, std=1.0, row_outliers=3, row_scale=25.0)
    q, sf, gs = cuda_lib.rotate_quant_act_nvfp4(padded_rows(X), g)
    torch.cuda.synchronize()
    check_fp4(q, sf, gs, X, g, TILE_A, f"act K{K} g{g}")
    qw, sfw, gw = cuda_lib.prepack_weight_nvfp4(padded_rows(X), g)
    torch.cuda.synchronize()
    check_fp4(qw, sfw, gw, X, g, TILE_B, f"wgt K{K} g{g}")
    assert cuda_lib.device_status() == 0


# ---------------------------------------------------------------------------- GEMM
def random_operands(rows, K4, seed, tile_rows):
    rng = np.random.default_rng(seed)
    vals = O.e2m1_values()
    e = vals[rng.integers(0, 16, (rows, K4))]
    sb = O.e4m3_values()[rng.integers(0x20, 0x58, (rows, K4 // 16))]
    packed = O.pack_e2m1(e)
    ld = -(-(K4 // 2) // 16) * 16
    buf = torch.zeros(rows, ld, dtype=torch.uint8)
    buf[:, : K4 // 2] = torch.from_numpy(packed)
    sf = tile(O.encode_e4m3(sb), tile_rows)
    return e, sb, buf.cuda(), sf.cuda()


def check_acc(got, ex, sbx, ew, sbw, K4, what):
    ref = O.nvfp4_gemm(ex, sbx, ew, sbw)
    mag = O.nvfp4_gemm(np.abs(ex), sbx, np.abs(ew), sbw)
    bound = K4 * 2.0 ** -24 * mag + 1e-30
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{what}: {bad.sum()} accumulators outside the fp32 bound"


@pytest.mark.parametrize("M,N,K4", [(64, 224, 256), (256, 448, 1024), (200, 300, 3072),
                                    (1, 16, 64), (129, 257, 320), (333, 520, 1024),
                                    (300, 700, 4096)])
def test_gemm_f32_on_oracle_codes(cuda_lib, M, N, K4):
    ex, sbx, qx, sfx = random_operands(M, K4, M + 1, TILE_A)
    ew, sbw, qw, sfw = random_operands(N, K4, N + 2, TILE_B)
    acc = cuda_lib.nvfp4_gemm_f32(qx, sfx, qw, sfw, K4).cpu().numpy().astype(np.float64)
    check_acc(acc, ex, sbx, ew, sbw, K4, f"{M}x{N}x{K4}")


@pytest.mark.parametrize("with_bias", [False, True])
def test_dequant_epilogue_on_oracle_codes(cuda_lib, with_bias):
    M, N, K4 = 200, 300, 1024
    ex, sbx, qx, sfx = random_operands(M, K4, 5, TILE_A)
    ew, sbw, qw, sfw = random_operands(N, K4, 6, TILE_B)
    rng = np.random.default_rng(7)
    gx = rng.uniform(1e-3, 1e-1, M).astype(np.float32)
    gw = rng.uniform(1e-5, 1e-3, N).astype(np.float32)
    gx[M // 3] = 0.0
    bias = torch.randn(N, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    y = cuda_lib.nvfp4_linear(qx, sfx, torch.from_numpy(gx).cuda(), qw, sfw,
                              torch.from_numpy(gw).cuda(), K4,
                              bias=bias.cuda() if with_bias else None)
    acc = O.nvfp4_gemm(ex, sbx, ew, sbw)
    check_y_elementwise(bf16_to_f64(y), acc, gx, gw, bf16_to_f64(bias) if with_bias else None,
                        "nvfp4 dequant")


def test_gemm_maximum_k(cuda_lib):
    """K4 at the documented GEMM maximum (131072): 2048 scale chunks per row."""
    K4 = 131072
    ex, sbx, qx, sfx = random_operands(130, K4, 33, TILE_A)
    ew, sbw, qw, sfw = random_operands(200, K4, 34, TILE_B)
    acc = cuda_lib.nvfp4_gemm_f32(qx, sfx, qw, sfw, K4).cpu().numpy().astype(np.float64)
    assert cuda_lib.device_status() == 0
    check_acc(acc, ex, sbx, ew, sbw, K4, "K4 = 131072")


def test_gemm_full_size_sampled(cuda_lib):
    w = CONFIGS["qkv"]
    K4 = -(-O.padded_k(w.K, w.group) // 64) * 64
    ex, sbx, qx, sfx = random_operands(w.M, K4, 11, TILE_A)
    ew, sbw, qw, sfw = random_operands(w.N, K4, 12, TILE_B)
    acc = cuda_lib.nvfp4_gemm_f32(qx, sfx, qw, sfw, K4)
    rng = np.random.default_rng(1)
    rows, cols = rng.integers(0, w.M, 2048), rng.integers(0, w.N, 2048)
    got = acc[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()].cpu().numpy()
    ax = ex[rows] * np.repeat(sbx[rows], 16, axis=1)
    aw = ew[cols] * np.repeat(sbw[cols], 16, axis=1)
    ref = np.sum(ax * aw, axis=1)
    mag = np.sum(np.abs(ax * aw), axis=1)
    assert (np.abs(got - ref) <= K4 * 2.0 ** -24 * mag + 1e-30).all()
    band = slice(w.M - 128, w.M)
    check_acc(acc[band].cpu().numpy().astype(np.float64), ex[band], sbx[band], ew, sbw, K4, "band")


@pytest.mark.parametrize("name", ["tiny", "qkv"])
def test_layer_end_to_end(cuda_lib, name):
    w = CONFIGS[name]
    X, W, bias = make_inputs(w, with_bias=True)
    g = w.group
    qw, sfw, gw = cuda_lib.prepack_weight_nvfp4(W.cuda(), g)
    y = cuda_lib.conv_linear_nvfp4(X.cuda(), qw, sfw, gw, g, bias=bias.cuda())
    torch.cuda.synchronize()
    rows = np.arange(w.M) if w.M <= 256 else np.sort(
        np.random.default_rng(3).choice(w.M, 256, replace=False))
    X64, W64 = bf16_to_f64(X), bf16_to_f64(W)
    _, _, gx, ex, sbx = O.rotate_quant_nvfp4(X64[rows], g)
    _, _, gw_ref, ew, sbw = O.rotate_quant_nvfp4(W64, g)
    y_ref = O.dequant(O.nvfp4_gemm(ex, sbx, ew, sbw), gx, gw_ref, bf16_to_f64(bias))
    y_gpu = bf16_to_f64(y[torch.from_numpy(rows).cuda()])
    assert rel_frob(y_gpu, y_ref) <= Y_FROB
    y_fp = X64[rows] @ W64.T + bf16_to_f64(bias)[None, :]
    assert rel_frob(y_gpu, y_fp) < 0.25
