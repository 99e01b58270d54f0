"""GPU parity of the one-call ConvLinear4bit layer (rotation, quantisation, GEMM and
dequantisation in one call; "ConvRot" paper, Abstract) against the CPU oracle.

The call computes the same codes, scales and output formula as rotate_quant_act followed by
w4a4_linear, so its output must equal that path's bit for bit, and the oracle's layer within
the stated bar.
"""

import numpy as np
import pytest
import torch

from oracle import convrot_oracle as O
from synthetic import CONFIGS, make_inputs
from synthetic.workloads import make_matrix
from tests.parity import Y_FROB, bf16_to_f64, rel_frob

pytestmark = pytest.mark.gpu


CASES = [("tiny", 16), ("qkv", 256), ("mlp_up", 256), ("proj_out", 1024), ("sweep", 16),
         ("sweep", 64), ("sweep", 256), ("sweep", 1024)]


@pytest.mark.parametrize("name,g", CASES)
def test_fused_layer_matches_oracle_and_two_calls(cuda_lib, name, g):
    w = CONFIGS[name]
    X, W, bias = make_inputs(w, with_bias=True)
    K_pad = O.padded_k(w.K, g)
    qw, sw = cuda_lib.prepack_weight(W.cuda(), g)
    Xd, bd = X.cuda(), bias.cuda()
    y = cuda_lib.w4a4_linear_fused(Xd, qw, sw, g, bias=bd)
    y2 = cuda_lib.conv_linear_4bit(Xd, qw, sw, g, K_pad, bias=bd)
    torch.cuda.synchronize()
    # the same codes, scales and formula: the two paths agree bit for bit
    assert torch.equal(y, y2), f"{name} g={g}: fused and two-call outputs differ"
    # and the oracle's layer (codes from fp64 rotation) within the stated bar, on a row sample
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(w.M, size=min(w.M, 256), replace=False))
    ref = O.w4a4_linear(bf16_to_f64(X)[rows], bf16_to_f64(W), g, bias=bf16_to_f64(bias))
    err = rel_frob(bf16_to_f64(y)[rows], ref["y"])
    assert err <= Y_FROB, f"{name} g={g}: rel Frobenius {err:.3e}"


def test_fused_edge_rows_stride_and_repeats(cuda_lib):
    """Zero and constant rows, a ragged K (not a multiple of 8), a row stride wider than N, a
    caller workspace reused by consecutive calls with no host synchronisation, and guard bytes
    after the output rows."""
    g, M, K, N = 256, 70, 1001, 136
    X = make_matrix(M, K, seed=5, row_outliers=2, row_scale=30.0)
    Xs = torch.zeros(M, K + 7, dtype=torch.bfloat16)          # row stride a multiple of 8
    X[3] = 0.0
    X[4] = 2.0
    W = make_matrix(N, K, seed=6, std=0.02)
    Ws = torch.zeros(N, K + 7, dtype=torch.bfloat16)
    Ws[:, :K] = W
    qw, sw = cuda_lib.prepack_weight(Ws.cuda()[:, :K], g)
    K_pad = O.padded_k(K, g)
    ws = torch.empty(cuda_lib.fused_workspace_bytes(M, K, g), dtype=torch.uint8, device="cuda")
    big = torch.full((M, N + 24), 7.0, dtype=torch.bfloat16, device="cuda")
    Xs[:, :K] = X
    Xd = Xs.cuda()[:, :K]
    for _ in range(3):
        cuda_lib.w4a4_linear_fused(Xd, qw, sw, g, out=big[:, :N], workspace=ws)
    y2 = cuda_lib.conv_linear_4bit(Xd, qw, sw, g, K_pad)
    torch.cuda.synchronize()
    assert (big[:, N:] == 7.0).all()
    assert torch.equal(big[:, :N], y2)
    assert (big[3, :N] == 0).all()
    ref = O.w4a4_linear(bf16_to_f64(X), bf16_to_f64(W), g)
    assert rel_frob(bf16_to_f64(big[:, :N]), ref["y"]) <= Y_FROB
