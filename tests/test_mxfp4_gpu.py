"""GPU parity of the MXFP4 variant (rotate + e2m1 elements with an e8m0 power-of-two scale per
32 K, block-scaled tcgen05 FP4 GEMM, bias) against the CPU oracle, through the C ABI.

Bars as for NVFP4: scale bytes and element codes >= 99.99 % identical and never more than one
code apart (floating point decides both); fp32 accumulators within K4 * 2^-24 of the sum of the
magnitudes of their terms; the bf16 output within the rounding bound of tests/parity.py; whole
layers within 1e-2 relative Frobenius error of the oracle's layer.
"""

import numpy as np
import pytest
import torch

from oracle import convrot_oracle as O
from synthetic import CONFIGS, make_inputs
from synthetic.workloads import make_matrix
from tests.parity import CODE_MATCH, Y_FROB, bf16_to_f64, rel_frob

pytestmark = pytest.mark.gpu

GROUPS = (16, 64, 256, 1024)
TILE_A, TILE_B = 128, 224


def sf_index(rows, nblk, tile_rows):
    """Byte offsets [rows, nblk, replicas] of scale (r, b) (b = 32-K block), as stated in
    include/convrot.h: chunks of 4 blocks (128 K); activations as 512-byte atoms per 128-row tile
    and chunk (chunk count per tile rounded up to even), weights as 4096-byte images per 224-row
    tile and chunk in four replicas."""
    r = np.arange(rows)[:, None, None]
    b = np.arange(nblk)[None, :, None]
    t, rr = r // tile_rows, r % tile_rows
    kc = b // 4
    chunks = -(-nblk // 4)
    if tile_rows == TILE_A:
        kc_even = (chunks + 1) // 2 * 2
        return (t * kc_even + kc) * 512 + 16 * (rr % 32) + 4 * ((rr % 128) // 32) + b % 4
    q = np.arange(4)[None, None, :]
    lane = rr % 32 + 32 * q
    return ((t * chunks + kc) * 4096 + 256 * (lane // 8) + 128 * (rr // 128) + 16 * (lane % 8)
            + 4 * ((rr % 128) // 32) + b % 4)


def sf_size(rows, nblk, tile_rows):
    tiles = -(-rows // tile_rows)
    chunks = -(-nblk // 4)
    return tiles * ((chunks + 1) // 2 * 2 * 512 if tile_rows == TILE_A else chunks * 4096)


def untile(sf, rows, nblk, tile_rows):
    v = sf.cpu().numpy()[sf_index(rows, nblk, tile_rows)]
    assert (v == v[:, :, :1]).all(), "replicas of the scales differ"
    return v[:, :, 0]


def tile(sbytes, tile_rows):
    rows, nblk = sbytes.shape
    flat = np.zeros(sf_size(rows, nblk, tile_rows), dtype=np.uint8)
    idx = sf_index(rows, nblk, tile_rows)
    flat[idx] = np.broadcast_to(sbytes[:, :, None], idx.shape)
    return torch.from_numpy(flat)


RANK = {v: i for i, v in enumerate(sorted(set(O.e2m1_values().tolist())))}


def code_ranks(values):
    return np.vectorize(lambda v: RANK[0.0 if v == 0 else v])(values)


def unpack_e2m1(q, K4):
    p = q[:, : K4 // 2].cpu().numpy().astype(np.int64)
    nib = np.empty((p.shape[0], K4), dtype=np.int64)
    nib[:, 0::2] = p & 15
    nib[:, 1::2] = p >> 4
    return O.e2m1_values()[nib]


def check_mx(q, sf, X, group, tile_rows, what):
    rows, K = X.shape
    K4 = -(-O.padded_k(K, group) // 64) * 64
    # the GPU runs over K4 >= K_pad (K_pad need not be a multiple of 32 for g = 16): the oracle
    # takes the input zero-padded to K4, whole zero groups that give zero codes, smallest scale
    X4 = np.pad(bf16_to_f64(X), ((0, 0), (0, K4 - K)))
    _, s_bytes, e_ref, _ = O.rotate_quant_mxfp4(X4, group)
    s_ref = s_bytes.astype(np.int64)
    s_gpu = untile(sf, rows, K4 // 32, tile_rows).astype(np.int64)
    d = np.abs(s_gpu - s_ref)
    assert d.max(initial=0) <= 1, f"{what}: scale off by {d.max()}"
    assert np.mean(d == 0) >= CODE_MATCH, f"{what}: scales {np.mean(d == 0):.6%} equal"
    same = np.repeat(d == 0, 32, axis=1)
    de = np.abs(code_ranks(unpack_e2m1(q, K4)) - code_ranks(e_ref))[same]
    assert de.max(initial=0) <= 1, f"{what}: element off by {de.max()} codes"
    assert np.mean(de == 0) >= CODE_MATCH, f"{what}: elements {np.mean(de == 0):.6%} equal"


def test_scale_layouts_are_injective():
    for tile_rows, rows, nblk in ((TILE_B, 448, 8), (TILE_A, 256, 16), (TILE_A, 128, 12),
                                  (TILE_A, 130, 94)):
        idx = sf_index(rows, nblk, tile_rows)
        assert len(np.unique(idx)) == idx.size and idx.max() < sf_size(rows, nblk, tile_rows)


# ---------------------------------------------------------------------------- quantisation
@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("M,K", [(64, 1024), (37, 3072), (130, 3000), (5, 40), (300, 15360)])
def test_quant_mxfp4_matches_oracle(cuda_lib, g, M, K):
    if K == 15360 and g == 16:
        pytest.skip("covered by the other groups")
    X = make_matrix(M, K, seed=M * 7 + K + g, std=1.0, row_outliers=3, row_scale=40.0)
    q, sf = cuda_lib.rotate_quant_act_mxfp4(X.cuda(), g)
    torch.cuda.synchronize()
    check_mx(q, sf, X, g, TILE_A, f"act g{g} M{M} K{K}")
    qw, sfw = cuda_lib.prepack_weight_mxfp4(X.cuda(), g)
    torch.cuda.synchronize()
    check_mx(qw, sfw, X, g, TILE_B, f"wgt g{g} M{M} K{K}")
    assert cuda_lib.device_status() == 0


GUARD = 0xA5


@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("M,K", [(37, 3000), (130, 1088), (225, 1024)])
def test_quant_mxfp4_writes_nothing_outside_its_outputs(cuda_lib, g, M, K):
    """Guard bytes around every output: code rows wider than K4 / 2 and one guard row after the
    last; the scale buffer longer than its layout, with the bytes the layout leaves unused
    (padding atoms, weight-image lanes past the tile) filled too. Each must stay untouched."""
    X = make_matrix(M, K, seed=M + K + 3 * g, std=1.0, row_outliers=3, row_scale=40.0)
    K4 = cuda_lib.nvfp4_k(K, g)
    for weights, tile_rows in ((False, TILE_A), (True, TILE_B)):
        ldq = -(-(K4 // 2 + 32) // 16) * 16
        q = torch.full((M + 1, ldq), GUARD, dtype=torch.uint8, device="cuda")
        size = cuda_lib.mxfp4_scale_bytes(M, K, g, weights)
        assert size == sf_size(M, K4 // 32, tile_rows)
        sf = torch.full((size + 256,), GUARD, dtype=torch.uint8, device="cuda")
        fn = cuda_lib.prepack_weight_mxfp4 if weights else cuda_lib.rotate_quant_act_mxfp4
        fn(padded_rows(X), g, q=q[:M], sf=sf)
        torch.cuda.synchronize()
        what = f"{'wgt' if weights else 'act'} g{g} M{M} K{K}"
        assert (q[:M, K4 // 2:] == GUARD).all() and (q[M] == GUARD).all(), what
        used = np.zeros(size + 256, dtype=bool)
        used[sf_index(M, K4 // 32, tile_rows).ravel()] = True
        assert (sf.cpu().numpy()[~used] == GUARD).all(), f"{what}: scale bytes written outside the layout"
        check_mx(q[:M], sf, X, g, tile_rows, what)


def test_quant_mxfp4_zero_onehot_and_tiny_rows(cuda_lib):
    M, K, g = 8, 256, 64
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[1, 70] = 3.0
    X[2] = 1.0
    X[3] = 2.0 ** -120                               # a block maximum far below 2^-100
    q, sf = cuda_lib.rotate_quant_act_mxfp4(X.cuda(), g)
    torch.cuda.synchronize()
    check_mx(q, sf, X, g, TILE_A, "special rows")
    s = untile(sf, M, 256 // 32, TILE_A)
    assert (s[0] == 0).all() and not q[0, :128].any()   # zero row: smallest scale, zero codes


def padded_rows(X, extra=8):
    """X with a row stride rounded up to a multiple of 8 elements (the ABI's rule)."""
    ld = -(-X.shape[1] // 8) * 8 + extra
    buf = torch.zeros(X.shape[0], ld, dtype=X.dtype, device="cuda")
    buf[:, : X.shape[1]] = X.cuda()
    return buf[:, : X.shape[1]]


@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("K", [32768, 32763])
def test_quant_mxfp4_maximum_row_length(cuda_lib, g, K):
    """K4 at the documented maximum (32768): rows longer than 16384 columns take the
    one-row-per-CTA configuration; a ragged K zero-pads inside the last group."""
    X = make_matrix(37, K, seed=K + 3 * g, std=1.0, row_outliers=3, row_scale=25.0)
    q, sf = cuda_lib.rotate_quant_act_mxfp4(padded_rows(X), g)
    torch.cuda.synchronize()
    check_mx(q, sf, X, g, TILE_A, f"act K{K} g{g}")
    qw, sfw = cuda_lib.prepack_weight_mxfp4(padded_rows(X), g)
    torch.cuda.synchronize()
    check_mx(qw, sfw, X, g, TILE_B, f"wgt K{K} g{g}")
    assert cuda_lib.device_status() == 0


# ---------------------------------------------------------------------------- GEMM
def random_operands(rows, K4, seed, tile_rows):
    rng = np.random.default_rng(seed)
    e = O.e2m1_values()[rng.integers(0, 16, (rows, K4))]
    X = rng.integers(-12, 12, (rows, K4 // 32))
    packed = O.pack_e2m1(e)
    ld = -(-(K4 // 2) // 16) * 16
    buf = torch.zeros(rows, ld, dtype=torch.uint8)
    buf[:, : K4 // 2] = torch.from_numpy(packed)
    return e, X, buf.cuda(), tile(O.encode_e8m0(X), tile_rows).cuda()


def check_acc(got, ex, xx, ew, xw, K4, what):
    ref = O.mxfp4_gemm(ex, xx, ew, xw)
    mag = O.mxfp4_gemm(np.abs(ex), xx, np.abs(ew), xw)
    bad = np.abs(got - ref) > K4 * 2.0 ** -24 * mag + 1e-30
    assert not bad.any(), f"{what}: {bad.sum()} accumulators outside the fp32 bound"


@pytest.mark.parametrize("M,N,K4", [(64, 224, 256), (256, 448, 1024), (200, 300, 3072),
                                    (1, 16, 64), (129, 257, 320), (333, 520, 1088),
                                    (300, 700, 4096)])
def test_gemm_f32_on_oracle_codes(cuda_lib, M, N, K4):
    ex, xx, qx, sfx = random_operands(M, K4, M + 3, TILE_A)
    ew, xw, qw, sfw = random_operands(N, K4, N + 4, TILE_B)
    acc = cuda_lib.mxfp4_gemm_f32(qx, sfx, qw, sfw, K4).cpu().numpy().astype(np.float64)
    assert cuda_lib.device_status() == 0
    check_acc(acc, ex, xx, ew, xw, K4, f"{M}x{N}x{K4}")


def test_gemm_full_size_sampled(cuda_lib):
    """The qkv shape in the launch configuration the bench times: 2048 sampled accumulators
    and one whole 128-row band (the last tile row) against the oracle's block-scaled sums."""
    w = CONFIGS["qkv"]
    K4 = -(-O.padded_k(w.K, w.group) // 64) * 64
    ex, xx, qx, sfx = random_operands(w.M, K4, 21, TILE_A)
    ew, xw, qw, sfw = random_operands(w.N, K4, 22, TILE_B)
    acc = cuda_lib.mxfp4_gemm_f32(qx, sfx, qw, sfw, K4)
    assert cuda_lib.device_status() == 0
    rng = np.random.default_rng(2)
    rows, cols = rng.integers(0, w.M, 2048), rng.integers(0, w.N, 2048)
    got = acc[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()].cpu().numpy()
    ax = ex[rows] * np.repeat(np.exp2(xx[rows].astype(np.float64)), 32, axis=1)
    aw = ew[cols] * np.repeat(np.exp2(xw[cols].astype(np.float64)), 32, axis=1)
    ref = np.sum(ax * aw, axis=1)
    mag = np.sum(np.abs(ax * aw), axis=1)
    assert (np.abs(got - ref) <= K4 * 2.0 ** -24 * mag + 1e-30).all()
    band = slice(w.M - 128, w.M)
    check_acc(acc[band].cpu().numpy().astype(np.float64), ex[band], xx[band], ew, xw, K4, "band")


def test_gemm_maximum_k(cuda_lib):
    """K4 at the documented GEMM maximum (131072): 1024 scale chunks per row."""
    K4 = 131072
    ex, xx, qx, sfx = random_operands(130, K4, 31, TILE_A)
    ew, xw, qw, sfw = random_operands(200, K4, 32, TILE_B)
    acc = cuda_lib.mxfp4_gemm_f32(qx, sfx, qw, sfw, K4).cpu().numpy().astype(np.float64)
    assert cuda_lib.device_status() == 0
    check_acc(acc, ex, xx, ew, xw, K4, "K4 = 131072")


@pytest.mark.parametrize("with_bias", [False, True])
def test_bias_epilogue_on_oracle_codes(cuda_lib, with_bias):
    M, N, K4 = 200, 300, 1024
    ex, xx, qx, sfx = random_operands(M, K4, 15, TILE_A)
    ew, xw, qw, sfw = random_operands(N, K4, 16, TILE_B)
    bias = torch.randn(N, generator=torch.Generator().manual_seed(19)).to(torch.bfloat16)
    y = cuda_lib.mxfp4_linear(qx, sfx, qw, sfw, K4, bias=bias.cuda() if with_bias else None)
    acc = O.mxfp4_gemm(ex, xx, ew, xw)
    b64 = bf16_to_f64(bias)[None, :] if with_bias else np.zeros((1, N))
    y_ref = acc + b64
    # y = bf16(fp32(acc) + bias): the fp32 accumulator's own bound (the block scales spread the
    # terms over 2^+-24, so it is not small against |acc|), then the add and bf16 rounding
    mag = O.mxfp4_gemm(np.abs(ex), xx, np.abs(ew), xw)
    bound = 2.0 ** -8 * np.abs(y_ref) + K4 * 2.0 ** -23 * mag + 2.0 ** -20 * np.abs(b64) + 1e-30
    bad = np.abs(bf16_to_f64(y) - y_ref) > bound
    assert not bad.any(), f"mxfp4 epilogue: {bad.sum()} outputs outside the bound"


@pytest.mark.parametrize("name", ["tiny", "qkv", "proj_out", "sweep"])
def test_layer_end_to_end(cuda_lib, name):
    w = CONFIGS[name]
    X, W, bias = make_inputs(w, with_bias=True)
    g = w.group
    qw, sfw = cuda_lib.prepack_weight_mxfp4(W.cuda(), g)
    y = cuda_lib.conv_linear_mxfp4(X.cuda(), qw, sfw, g, bias=bias.cuda())
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    rows = np.arange(w.M) if w.M <= 256 else np.sort(
        np.random.default_rng(5).choice(w.M, 256, replace=False))
    X64, W64 = bf16_to_f64(X), bf16_to_f64(W)
    ref = O.mxfp4_linear(X64[rows], W64, g, bias=bf16_to_f64(bias))["y"]
    y_gpu = bf16_to_f64(y[torch.from_numpy(rows).cuda()])
    assert rel_frob(y_gpu, ref) <= Y_FROB
    y_fp = X64[rows] @ W64.T + bf16_to_f64(bias)[None, :]
    assert rel_frob(y_gpu, y_fp) < 0.3
