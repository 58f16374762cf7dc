"""bq_gemm_decode_noalloc: the decode GEMM for callers that cannot allocate.

Some callers cannot hand libbq a workspace: a plugin inside another engine
that owns every device byte, or a serving loop that plans all memory up front
and may not allocate once it runs.  bq_gemm_decode_noalloc runs the same
split-K decode kernel as bq_gemm, with its scratch in a fixed device array
inside the library.  This test calls it through the C ABI twice in a row
and checks each result against bq_gemm (with a caller workspace) under the
parity tolerance of the other GEMM tests.  It lives in its own file, which
pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_scaled_w8a8_b200 as bq
import bq_synth

pytestmark = pytest.mark.gpu


def _close(out: torch.Tensor, ref: torch.Tensor, what: str):
    g = out.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    d = g - r
    assert np.isfinite(g).all(), what
    assert np.abs(d).max() <= 1e-2 * np.abs(r).max(), what
    assert np.linalg.norm(d) <= 2e-3 * np.linalg.norm(r), what


def _operands(M, N, K, dtype, seed):
    dev = "cuda"
    x = bq_synth.activations(M, K, seed, 41, 30.0, device=dev)
    w = bq_synth.weights(N, K, 0.02, seed, device=dev)
    qa, sa = bq.quant_act(x, 128, dtype)
    qw, sw = bq.quant_weight(w, 128, 128, dtype)
    bias = torch.randn(N, device=dev).to(torch.bfloat16)
    return qa, sa, qw, sw, bias


def _call_c_abi(qa, sa, qw, sw, dtype, bias, out):
    L = bq.lib()
    M, K = qa.shape
    N = qw.shape[0]
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.bq_gemm_decode_noalloc(qa.data_ptr(), K, sa.data_ptr(), qw.data_ptr(), K,
                                    sw.data_ptr(), M, N, K, 128, 128, dtype,
                                    None if bias is None else bias.data_ptr(), out.data_ptr(),
                                    N, st)


@pytest.mark.parametrize("dtype", [bq.INT8, bq.FP8_E4M3])
@pytest.mark.parametrize("M,N,K", [(64, 4096, 4096), (8, 4096, 4096), (1, 640, 1008),
                                   (33, 1000, 2048)])
def test_noalloc_matches_workspace_entry_point_twice(dtype, M, N, K):
    torch.cuda.set_device(0)
    qa, sa, qw, sw, bias = _operands(M, N, K, dtype, 900 + M)
    bq.set_path(bq.PATH_DECODE)
    try:
        ref = bq.gemm(qa, sa, qw, sw, 128, 128, dtype, bias=bias)
    finally:
        bq.set_path(bq.PATH_AUTO)
    outs = []
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_c_abi(qa, sa, qw, sw, dtype, bias, out) == bq.OK, \
            bq.lib().bq_last_error_message()
        outs.append(out)
    torch.cuda.synchronize()
    bq.check_device_status()
    for i, out in enumerate(outs):
        _close(out, ref, f"call {i} dtype={dtype} {M}x{N}x{K}")


def test_noalloc_allocates_nothing_across_shapes_back_to_back():
    """Two shapes with different tile counts, whose partials both go through
    the fixed scratch, called alternately: each call clears the counters it
    uses, and device memory stays exactly as free as before the calls."""
    torch.cuda.set_device(0)
    shapes = [(1, 640, 1008), (33, 1000, 2048)]
    ops = [_operands(M, N, K, bq.INT8, 950 + M) for M, N, K in shapes]
    refs, outs = [], []
    bq.set_path(bq.PATH_DECODE)
    try:
        for (M, N, K), (qa, sa, qw, sw, bias) in zip(shapes, ops):
            refs.append(bq.gemm(qa, sa, qw, sw, 128, 128, bq.INT8, bias=bias))
    finally:
        bq.set_path(bq.PATH_AUTO)
    for (M, N, K) in shapes:
        outs.append([torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
                     for _ in range(2)])
    # the first call looks up the scratch's address; then measure
    qa, sa, qw, sw, bias = ops[0]
    assert _call_c_abi(qa, sa, qw, sw, bq.INT8, bias, outs[0][0]) == bq.OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for rep in range(2):
        for i, (qa, sa, qw, sw, bias) in enumerate(ops):
            assert _call_c_abi(qa, sa, qw, sw, bq.INT8, bias, outs[i][rep]) == bq.OK, \
                bq.lib().bq_last_error_message()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    bq.check_device_status()
    assert free1 == free0, f"device memory changed by {free0 - free1} bytes"
    for i, (M, N, K) in enumerate(shapes):
        for rep in range(2):
            _close(outs[i][rep], refs[i], f"{M}x{N}x{K} call {rep}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    M, N, K = 128, 1920, 4096        # 15 weight tiles x 20 splits: ~19.7 MB of partials
    qa, sa, qw, sw, _ = _operands(M, N, K, bq.INT8, 7)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    st = _call_c_abi(qa, sa, qw, sw, bq.INT8, None, out)
    assert st == bq.ERR_UNSUPPORTED
    assert b"scratch" in bq.lib().bq_last_error_message()
