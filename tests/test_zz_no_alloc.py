"""The one-call layer for callers that cannot allocate device memory.

convrot_w4a4_linear_fused_noalloc serves callers that are handed streams and tensors but cannot
obtain device memory at call time (code running while a stream is captured into a CUDA graph, a
plugin whose host runtime owns the allocator): instead of a caller workspace it uses a fixed
scratch array the library keeps on the device. Its output must match the workspace entry point
(convrot_w4a4_linear_fused) under the layer's parity bar; this test asks for bit equality, which
is stricter, on two calls in a row through the C ABI, and checks that a shape whose scratch does
not fit the array is rejected before anything runs.

This file is collected last, so that a run stopping at the first failure has run every other
test before it; it also passes on its own in a fresh process.
"""

import ctypes

import pytest
import torch

from synthetic.workloads import make_matrix

pytestmark = pytest.mark.gpu

CONVROT_ERR_SHAPE = 2


def _noalloc(b, X, qw, sw, g, bias, Y):
    M, K = X.shape
    return b.lib.convrot_w4a4_linear_fused_noalloc(
        ctypes.c_void_p(X.data_ptr()), M, K, X.stride(0), g, ctypes.c_void_p(qw.data_ptr()),
        qw.stride(0), ctypes.c_void_p(sw.data_ptr()),
        None if bias is None else ctypes.c_void_p(bias.data_ptr()),
        ctypes.c_void_p(Y.data_ptr()), Y.stride(0), qw.shape[0],
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("g,M,K,N,with_bias", [(256, 300, 3000, 520, True),
                                               (16, 4608, 3072, 256, False)])
def test_noalloc_matches_workspace_call_twice(cuda_lib, g, M, K, N, with_bias):
    b = cuda_lib
    X = make_matrix(M, K, seed=M + K, row_outliers=3, row_scale=30.0).cuda()
    W = make_matrix(N, K, seed=N + K, std=0.02).cuda()
    bias = make_matrix(1, N, seed=9, std=0.02)[0].cuda() if with_bias else None
    qw, sw = b.prepack_weight(W, g)
    ref = b.w4a4_linear_fused(X, qw, sw, g, bias=bias)
    for _ in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(b, X, qw, sw, g, bias, Y) == 0
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)


def test_noalloc_rejects_shapes_beyond_the_scratch_array(cuda_lib):
    b = cuda_lib
    g, M, K, N = 1024, 4608, 15360, 64
    assert b.fused_workspace_bytes(M, K, g) > b.NOALLOC_SCRATCH_BYTES
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    qw = torch.zeros(N, K // 2, dtype=torch.uint8, device="cuda")
    sw = torch.zeros(N, dtype=torch.float32, device="cuda")
    Y = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(b, X, qw, sw, g, None, Y) == CONVROT_ERR_SHAPE
    torch.cuda.synchronize()
    assert (Y == 3.0).all()                       # nothing ran
