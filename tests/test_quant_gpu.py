"""GPU parity of the fused RHT + int4 quant + pack kernel against the CPU oracle.

Every case calls the C ABI (through the ctypes binding) and compares codes, packed bytes and
scales element by element with oracle/convrot_oracle.py on the same seeded inputs.
"""

import numpy as np
import pytest
import torch

from oracle import convrot_oracle as O
from synthetic import CONFIGS, make_inputs
from synthetic.workloads import make_matrix
from tests.conftest import read_golden
from tests.parity import bf16_to_f64, check_codes, check_scales, gpu_codes

pytestmark = pytest.mark.gpu

GROUPS = (16, 64, 256, 1024)


def strided(X: torch.Tensor, extra: int = 8) -> torch.Tensor:
    """X copied into a wider device buffer (row stride a multiple of 8, > K)."""
    M, K = X.shape
    ld = (K + 7) // 8 * 8 + extra
    buf = torch.full((M, ld), float("nan"), dtype=torch.bfloat16, device="cuda")
    buf[:, :K] = X.cuda()
    return buf[:, :K]


CANARY = 0xA5          # guard byte around every code buffer
SCALE_CANARY = -123.0  # guard value after the last scale


def quant_guarded(fn, X, g, int8=False, extra=32):
    """Run a rotate+quantise entry point into buffers with guard regions: code rows wider than
    their defined K_pad / 2 (or K_pad) bytes, one guard row after the last, and guard scales
    after sx[M - 1]. Asserts that the kernel wrote nothing outside the defined region and returns
    (q, s) views of the defined outputs."""
    M, K = X.shape
    K_pad = O.padded_k(K, g)
    row_bytes = K_pad if int8 else K_pad // 2
    ldq = (row_bytes + extra + 15) // 16 * 16
    qbuf = torch.full((M + 1, ldq), CANARY, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((M + 8,), SCALE_CANARY, dtype=torch.float32, device="cuda")
    fn(X, g, qbuf[:M], sbuf[:M])
    torch.cuda.synchronize()
    assert (qbuf[:M, row_bytes:] == CANARY).all(), "bytes written past the defined code row"
    assert (qbuf[M] == CANARY).all(), "bytes written past the last code row"
    assert (sbuf[M:] == SCALE_CANARY).all(), "scales written past row M - 1"
    return qbuf[:M, :row_bytes], sbuf[:M]


def run_and_check(b, X_cpu, g, what, rows=None, weight=False):
    Xd = X_cpu.cuda()
    fn = b.prepack_weight if weight else b.rotate_quant_act
    q, s = fn(Xd, g)
    torch.cuda.synchronize()
    K_pad = O.padded_k(X_cpu.shape[1], g)
    X64 = bf16_to_f64(X_cpu)
    if rows is not None:
        X64 = X64[rows]
        idx = torch.from_numpy(rows).cuda()
        q, s = q[idx], s[idx]
    ref_q, ref_s, ref_c = O.rotate_quant(X64, g)
    frac = check_codes(gpu_codes(q, K_pad), ref_c, what)
    check_scales(s, ref_s, what)
    return frac


@pytest.mark.parametrize("g", GROUPS)
def test_make_rht_exact(cuda_lib, g):
    R = cuda_lib.make_rht(g).cpu().numpy().astype(np.float64)
    assert np.array_equal(R, O.rht_matrix(g))


def test_onehot_worked_example(cuda_lib):
    golden = {row[0]: row[1:] for row in read_golden("onehot_g16.txt")}
    X = torch.zeros(1, 16, dtype=torch.bfloat16)
    X[0, 0] = 1.0
    q, s = cuda_lib.rotate_quant_act(X.cuda(), 16)
    assert q[0, :8].cpu().tolist() == [int(v, 16) for v in golden["packed"]]
    bits = s.cpu().view(torch.int32).item() & 0xFFFFFFFF
    assert bits == int(golden["scale_fp32_hex"][0], 16)


@pytest.mark.parametrize("g", GROUPS)
def test_quant_ragged_tiles(cuda_lib, g):
    # rows not a multiple of the CTA's rows, K with a ragged 8-element tail, several groups
    M, K = 37, 3 * g + g // 2 + 3
    X = make_matrix(M, K, seed=g, row_outliers=3, row_scale=40.0)
    Xs = strided(X)
    q, s = cuda_lib.rotate_quant_act(Xs, g)
    torch.cuda.synchronize()
    K_pad = O.padded_k(K, g)
    ref_q, ref_s, ref_c = O.rotate_quant(bf16_to_f64(X), g)
    check_codes(gpu_codes(q, K_pad), ref_c, f"ragged g={g}")
    check_scales(s, ref_s, f"ragged g={g}")


@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("int8", [False, True])
@pytest.mark.parametrize("M,K", [(37, None), (300, None), (5, 8), (300, 1088), (300, 9280)])
def test_quant_streamed_rows(cuda_lib, g, int8, M, K):
    """K a multiple of 8 (whole rows stream through the shared ring): ragged K inside the last
    group, row counts that are not a multiple of the rows per round, rows of 2 to 10240 padded
    columns (K = 1088 and 9280 at g = 1024 pad 64 and 960 zero columns into the last group);
    guard bytes around every output."""
    if K is None:
        K = 3 * g + 8
    X = make_matrix(M, K, seed=M + K + g, row_outliers=min(3, M), row_scale=40.0)
    fn = cuda_lib.rotate_quant_i8 if int8 else cuda_lib.rotate_quant_act
    q, s = quant_guarded(fn, strided(X, extra=16), g, int8=int8)
    K_pad = O.padded_k(K, g)
    X64 = bf16_to_f64(X)
    if int8:
        ref_c, ref_s = O.rotate_quant_int8(X64, g)
        got = q.cpu().numpy().view(np.int8)
    else:
        _, ref_s, ref_c = O.rotate_quant(X64, g)
        got = gpu_codes(q, K_pad)
    check_codes(got, ref_c, f"M={M} K={K} g={g} int8={int8}")
    check_scales(s, ref_s, f"M={M} K={K} g={g} int8={int8}")


@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("K", [3 * 64 + 3, 1001])
def test_quant_register_path_guards(cuda_lib, g, K):
    """K not a multiple of 8 (the register-resident kernel): the same guard regions."""
    X = make_matrix(37, K, seed=K + g, row_outliers=3, row_scale=40.0)
    q, s = quant_guarded(cuda_lib.rotate_quant_act, strided(X), g)
    K_pad = O.padded_k(K, g)
    _, ref_s, ref_c = O.rotate_quant(bf16_to_f64(X), g)
    check_codes(gpu_codes(q, K_pad), ref_c, f"K={K} g={g}")
    check_scales(s, ref_s, f"K={K} g={g}")


@pytest.mark.parametrize("g", GROUPS)
def test_quant_edge_rows(cuda_lib, g):
    K = 2 * g
    X = make_matrix(6, K, seed=100 + g)
    X[1] = 0.0                                   # all-zero row -> scale 0, codes 0
    X[2] = 3.0                                   # constant row: R 1 = 1 -> all codes +7
    X[3] = 0.0
    X[3, 5] = -2.5                               # one-hot: codes are +-7 (|R| entries equal)
    X[4] *= 1e4                                  # large magnitudes
    X[5] *= 1e-4                                 # small magnitudes
    q, s = cuda_lib.rotate_quant_act(X.cuda(), g)
    torch.cuda.synchronize()
    codes = gpu_codes(q, K)
    assert s[1].item() == 0.0 and (codes[1] == 0).all()
    assert (codes[2] == 7).all()
    assert (np.abs(codes[3][:g]) == 7).all() and (codes[3][g:] == 0).all()
    ref_q, ref_s, ref_c = O.rotate_quant(bf16_to_f64(X), g)
    check_codes(codes, ref_c, "edge")
    check_scales(s, ref_s, "edge")
    # packed bytes: identical wherever both nibbles agree
    assert (q[:, : K // 2].cpu().numpy() == ref_q).mean() >= 0.999


def test_quant_tiny_k_and_single_row(cuda_lib):
    for g in GROUPS:
        for K in (1, 5, 8, 17):
            X = make_matrix(1, K, seed=K)
            Xs = strided(X)
            q, s = cuda_lib.rotate_quant_act(Xs, g)
            torch.cuda.synchronize()
            ref_q, ref_s, ref_c = O.rotate_quant(bf16_to_f64(X), g)
            check_codes(gpu_codes(q, O.padded_k(K, g)), ref_c, f"K={K} g={g}")
            check_scales(s, ref_s, f"K={K} g={g}")


@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("K", [32768, 32763])
def test_quant_maximum_row_length(cuda_lib, g, K):
    """K_pad at the documented maximum (32768): rows longer than 16384 columns take the
    one-row-per-CTA configuration; a ragged K zero-pads inside the last group."""
    X = make_matrix(37, K, seed=K + g, std=1.0, row_outliers=3, row_scale=25.0)
    ref_q, ref_s, ref_c = O.rotate_quant(bf16_to_f64(X), g)
    K_pad = O.padded_k(K, g)
    for fn in (cuda_lib.rotate_quant_act, cuda_lib.prepack_weight):
        q, s = fn(strided(X), g)            # row stride a multiple of 8 for the ragged K
        torch.cuda.synchronize()
        check_codes(gpu_codes(q, K_pad), ref_c, f"K={K} g={g} {fn.__name__}")
        check_scales(s, ref_s, f"K={K} g={g} {fn.__name__}")


def test_quant_zero_size_is_noop(cuda_lib):
    X = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    q, s = cuda_lib.rotate_quant_act(X, 16)
    assert q.shape[0] == 0
    X = torch.zeros(3, 0, dtype=torch.bfloat16, device="cuda")
    s = torch.full((3,), 5.0, device="cuda")
    q = torch.empty(3, 16, dtype=torch.uint8, device="cuda")
    cuda_lib.rotate_quant_act(X, 16, qx=q, sx=s)
    assert (s.cpu() == 0).all()


def test_quant_tiny_config(cuda_lib):
    w = CONFIGS["tiny"]
    X, W, _ = make_inputs(w)
    run_and_check(cuda_lib, X, w.group, "tiny X")
    run_and_check(cuda_lib, W, w.group, "tiny W", weight=True)


FULL = [("qkv", 256), ("mlp_up", 256), ("proj_out", 1024),
        ("sweep", 16), ("sweep", 64), ("sweep", 256), ("sweep", 1024)]


@pytest.mark.parametrize("name,g", FULL)
def test_quant_full_size(cuda_lib, name, g):
    """Full-size activations (all rows on the GPU and in the oracle) and weights (all rows on the
    GPU, the oracle on a row sample)."""
    w = CONFIGS[name]
    X, W, _ = make_inputs(w)
    rng = np.random.default_rng(5)
    # activations: every row against the oracle (the code-match bar is judged on all M x K_pad)
    q, s = quant_guarded(cuda_lib.rotate_quant_act, X.cuda(), g)
    K_pad = O.padded_k(w.K, g)
    _, ref_s, ref_c = O.rotate_quant(bf16_to_f64(X), g)
    check_codes(gpu_codes(q, K_pad), ref_c, f"{name} X g={g}")
    check_scales(s, ref_s, f"{name} X g={g}")
    wrows = np.sort(rng.choice(w.N, size=min(w.N, 768), replace=False))
    run_and_check(cuda_lib, W, g, f"{name} W g={g}", rows=wrows, weight=True)
