"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Quantised codes and scales must match bit for bit; GEMM outputs must meet
max|d| <= 1e-2 max|ref| and relative Frobenius <= 2e-3 against the fp64
oracle on the same codes, and lie within one bf16 ulp of the exact value.
"""
import numpy as np
import pytest
import torch

import block_scaled_w8a8_b200 as bq
import bq_synth
import oracle
from gpu_util import (assert_codes_equal, assert_combine_close, assert_gemm_close,
                      assert_scales_equal, bf16_ulp,
                      bf16_values, dev_bf16, dev_f32, dev_i32, dev_u8, host_bits,
                      mx_sf_atoms, mx_sf_rows)

pytestmark = pytest.mark.gpu

INT8, FP8 = bq.INT8, bq.FP8_E4M3
cdiv = bq_synth.cdiv


@pytest.fixture(autouse=True)
def _reset_path():
    bq.set_path(bq.PATH_AUTO)
    yield
    bq.set_path(bq.PATH_AUTO)
    bq.check_device_status()


def act_bits(M, K, seed, n_out=0, scale=1.0):
    return host_bits(bq_synth.activations(M, K, seed, n_out, scale))


# --------------------------------------------------------------------------
# activation quantisation: bit-exact
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M,K,gk,pad", [
    (16, 200, 128, 0),      # tiny workload: partial second group
    (64, 4096, 128, 0),     # decode width
    (37, 1000, 128, 8),     # ragged K, padded row stride
    (5, 300, 32, 0),
    (3, 700, 256, 0),       # group longer than 128 (two-pass)
    (7, 333, 100, 3),       # group not a multiple of 4 (scalar path)
    (1, 1, 128, 0),
    # many rows: the half-warp-per-group path (16-byte loads, K % 8 == 0)
    (300, 1000, 128, 8),    # partial last group (104 elements), padded stride
    (129, 4096, 128, 0),    # odd row count: a half-empty last pair of groups
    (256, 136, 128, 0),     # second group of 8 elements
    (130, 1004, 128, 4),    # K % 8 != 0: the one-warp-per-group path
])
def test_quant_act_bit_exact(dtype, M, K, gk, pad):
    xb = act_bits(M, K + pad, 11 + M, max(1, (K + pad) // 100), 30.0)
    xb[0, :] = 0                                   # an all-zero row
    if M > 2:
        xb[2, :] = 0x0001                          # subnormal amax: scale underflows to 0
    x = dev_bf16(xb)[:, :K]
    q, s = bq.quant_act(x, gk, dtype)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quant_act(np.ascontiguousarray(xb[:, :K]), gk, dtype)
    assert_codes_equal(q, q_ref, "codes")
    assert_scales_equal(s, s_ref, "scales")


@pytest.mark.parametrize("dtype", [INT8, FP8])
def test_quant_act_extremes(dtype):
    # large, tiny and tie-making values in one group
    vals = np.array([3.0e38, -1.0e-38, 2.5, -2.5, 0.5, 1e-40, -0.0, 448.0] * 16, np.float32)
    xb = host_bits(torch.from_numpy(vals).to(torch.bfloat16))[None, :]
    ties = np.concatenate([[127.0], np.arange(-20, 20) + 0.5, np.zeros(87)])
    tb = host_bits(torch.from_numpy(ties.astype(np.float32)).to(torch.bfloat16))[None, :]
    xb = np.concatenate([xb, tb], 0)
    q, s = bq.quant_act(dev_bf16(xb), 128, dtype)
    q_ref, s_ref = oracle.quant_act(xb, 128, dtype)
    assert_codes_equal(q, q_ref, "codes")
    assert_scales_equal(s, s_ref, "scales")


@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("N,K,bn,bk", [(320, 200, 128, 128), (256, 384, 128, 128),
                                       (100, 77, 32, 16)])
def test_quant_weight_bit_exact(dtype, N, K, bn, bk):
    w = bq_synth.weights(N, K, 0.02, 3)
    w[0, :5] = 0.0
    q, s = bq.quant_weight(w.cuda(), bn, bk, dtype)
    q_ref, s_ref = oracle.quant_weight(w.numpy(), bn, bk, dtype)
    assert_codes_equal(q, q_ref, "weight codes")
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# --------------------------------------------------------------------------
# block-scaled GEMM
# --------------------------------------------------------------------------

def make_problem(M, N, K, bn, bk, dtype, seed, bias=False, n_out=3):
    """Operands quantised by the ORACLE (codes and scales are its outputs)."""
    xb = act_bits(M, K, seed, n_out, 20.0)
    w = bq_synth.weights(N, K, 0.02, seed).numpy()
    qa, sa = oracle.quant_act(xb, bk, dtype)
    qw, sw = oracle.quant_weight(w, bn, bk, dtype)
    bb = host_bits(torch.randn(N, generator=torch.Generator().manual_seed(seed)).to(
        torch.bfloat16)) if bias else None
    return xb, qa, sa, qw, sw, bb


GEMM_SHAPES = [
    # M, N, K, bn, bk
    (16, 320, 200, 128, 128),   # the tiny workload: 3x2 scale grid, partial blocks
    (300, 520, 1000, 128, 128), # several tiles, ragged M, N, K
    (1, 256, 512, 128, 128),
    (129, 257, 384, 64, 128),
    (40, 96, 250, 96, 64),      # odd block sizes
]


@pytest.mark.parametrize("path", [bq.PATH_SIMT, bq.PATH_AUTO])
@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M,N,K,bn,bk", GEMM_SHAPES)
def test_gemm_vs_oracle(path, dtype, M, N, K, bn, bk):
    _, qa, sa, qw, sw, bb = make_problem(M, N, K, bn, bk, dtype, 100 + M, bias=(M % 2 == 0))
    bq.set_path(path)
    out = bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), bn, bk, dtype,
                  bias=None if bb is None else dev_bf16(bb))
    torch.cuda.synchronize()
    ref = oracle.gemm(qa, sa, qw, sw, bn, bk, dtype, bias_bf16=bb)
    assert_gemm_close(out, ref, f"gemm path={path} dtype={dtype} {M}x{N}x{K}")


TC_SHAPES = [
    # M, N, K: block 128x128, K a multiple of 16 bytes (TMA row stride)
    (128, 128, 128),
    (300, 520, 1008),     # ragged M and N tiles, partial last K-block (112)
    (1, 256, 512),
    (257, 640, 2048),
    (64, 1280, 384),
    (1000, 384, 4096),
    (513, 768, 640),      # a CTA pair's 256-row tiles: one row past two of them
]


@pytest.mark.parametrize("path", [bq.PATH_TCGEN05_1CTA, bq.PATH_TCGEN05_PAIR])
@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M,N,K", TC_SHAPES)
def test_gemm_tcgen05_vs_oracle(path, dtype, M, N, K):
    _, qa, sa, qw, sw, bb = make_problem(M, N, K, 128, 128, dtype, 300 + M, bias=(N % 256 == 0))
    bq.set_path(path)
    out = bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), 128, 128, dtype,
                  bias=None if bb is None else dev_bf16(bb))
    torch.cuda.synchronize()
    bq.check_device_status()
    ref = oracle.gemm(qa, sa, qw, sw, 128, 128, dtype, bias_bf16=bb)
    assert_gemm_close(out, ref, f"tcgen05 dtype={dtype} {M}x{N}x{K}")


def test_gemm_tcgen05_rejects_ineligible_shapes():
    _, qa, sa, qw, sw, _ = make_problem(16, 320, 200, 128, 128, INT8, 1)
    bq.set_path(bq.PATH_TCGEN05)
    with pytest.raises(bq.BqError) as ei:       # K = 200: row stride not a multiple of 16
        bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), 128, 128, INT8)
    assert ei.value.status == bq.ERR_UNSUPPORTED
    _, qa, sa, qw, sw, _ = make_problem(64, 256, 256, 64, 128, INT8, 2)
    with pytest.raises(bq.BqError) as ei:       # block_n = 64
        bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), 64, 128, INT8)
    assert ei.value.status == bq.ERR_UNSUPPORTED


DECODE_SHAPES = [
    # M, N, K
    (1, 640, 1008),      # 5 weight tiles x 8 splits of one K-block each
    (8, 4096, 4096),     # the decode workload at M = 8
    (16, 256, 512),
    (17, 384, 2048),     # token count not a multiple of 16
    (32, 1000, 1024),    # ragged last weight tile
    (64, 640, 4096),
    (100, 256, 1008),
    (128, 512, 640),
]


@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_gemm_decode_vs_oracle(dtype, M, N, K):
    _, qa, sa, qw, sw, bb = make_problem(M, N, K, 128, 128, dtype, 500 + M, bias=(M % 2 == 1))
    bq.set_path(bq.PATH_DECODE)
    args = (dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), 128, 128, dtype)
    bias = None if bb is None else dev_bf16(bb)
    out1 = bq.gemm(*args, bias=bias)
    out2 = bq.gemm(*args, bias=bias)     # the workspace must have reset itself
    torch.cuda.synchronize()
    bq.check_device_status()
    ref = oracle.gemm(qa, sa, qw, sw, 128, 128, dtype, bias_bf16=bb)
    assert_gemm_close(out1, ref, f"decode dtype={dtype} {M}x{N}x{K}")
    assert torch.equal(out1, out2), "split-K reduction is not deterministic"


@pytest.mark.parametrize("M", [1, 8, 64])
def test_linear_decode_path_with_dependent_launch(M):
    N = K = 4096
    xb = act_bits(M, K, 40 + M, 41, 30.0)
    w = bq_synth.weights(N, K, 0.02, 40 + M).numpy()
    qw, sw = oracle.quant_weight(w, 128, 128, INT8)
    x = dev_bf16(xb)
    qw_d, sw_d = dev_u8(qw), dev_f32(sw)
    outs = [bq.linear(x, qw_d, sw_d, 128, 128, INT8) for _ in range(3)]
    torch.cuda.synchronize()
    bq.check_device_status()
    qa, sa = oracle.quant_act(xb, 128, INT8)
    ref = oracle.gemm(qa, sa, qw, sw, 128, 128, INT8)
    assert_gemm_close(outs[0], ref, f"linear decode M={M}")
    assert all(torch.equal(outs[0], o) for o in outs[1:])


# bq_linear with M <= 128: the activation quantiser, then the cluster decode
# GEMM (split-K reduced over distributed shared memory) as a programmatic
# dependent of it.  The shapes cover clusters of 1 to 8 K-splits (N = 128 up
# to 4096, 3000 ragged), every token tile (16, 32, 64, 128), token counts
# that are not multiples of 16, partial K-blocks, x rows not 16-byte aligned
# (K = 1000), padded row strides and bias.
LINEAR_DECODE_SHAPES = [(1, 2048, 4096, 4096), (5, 4096, 1000, 1000), (16, 2048, 1004, 1008),
                (17, 3000, 4096, 4096), (32, 4096, 8192, 8192), (3, 2100, 300, 304),
                (33, 4096, 4096, 4096), (64, 4096, 4096, 4096), (64, 640, 1008, 1008),
                (100, 1024, 2048, 2056), (128, 4096, 1024, 1024), (1, 128, 128, 128)]


@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M,N,K,ldx", LINEAR_DECODE_SHAPES)
def test_linear_decode_vs_oracle(M, N, K, ldx, dtype):
    xb = act_bits(M, K, 90 + M, 7, 25.0)
    w = bq_synth.weights(N, K, 0.02, 91 + M).numpy()
    qw, sw = oracle.quant_weight(w, 128, 128, dtype)
    bias = oracle.bf16_from_f64(np.random.default_rng(M).normal(0, 0.5, N))
    xpad = np.zeros((M, ldx), dtype=np.uint16)
    xpad[:, :K] = xb
    x = dev_bf16(xpad)[:, :K]
    assert x.stride(0) == ldx
    outs = [bq.linear(x, dev_u8(qw), dev_f32(sw), 128, 128, dtype, bias=dev_bf16(bias))
            for _ in range(2)]
    torch.cuda.synchronize()
    bq.check_device_status()
    qa, sa = oracle.quant_act(xb, 128, dtype)
    ref = oracle.gemm(qa, sa, qw, sw, 128, 128, dtype, bias_bf16=bias)
    assert_gemm_close(outs[0], ref, f"linear decode M={M} N={N} K={K}")
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M", [1, 7, 32, 33, 64, 128])
def test_linear_decode_codes_exact_through_identity_weight(M, dtype):
    """With W = identity (code of 1.0, block scale 1) each output is
    bf16(fl32(q[t, n] * sa[t, n // 128])): one product, rounded to fp32 by the
    kernel's promotion FMA, then to bf16.  Neighbouring INT8 codes (and e4m3
    codes) differ by at least 1/127 (1/8) relatively, more than a bf16 ulp,
    so any wrong code, misplaced activation tile, or partial summed into the
    wrong row by the cluster reduction shows as an exact mismatch against the
    oracle's codes."""
    N = K = 2048
    xb = act_bits(M, K, 300 + M, 11, 40.0)
    one = 1 if dtype == INT8 else int(oracle.e4m3_encode(np.array([1.0]))[0])
    qw = np.zeros((N, K), dtype=np.uint8)
    qw[np.arange(N), np.arange(K)] = one
    sw = np.ones((N // 128, K // 128), dtype=np.float32)
    out = bq.linear(dev_bf16(xb), dev_u8(qw), dev_f32(sw), 128, 128, dtype)
    torch.cuda.synchronize()
    bq.check_device_status()
    qa, sa = oracle.quant_act(xb, 128, dtype)
    vals = oracle.code_values(qa, dtype).astype(np.float32)
    expect = vals * np.repeat(sa, 128, axis=1).astype(np.float32)      # fp32 product
    expect_bits = oracle.bf16_from_f64(expect.astype(np.float64))
    got = host_bits(out)
    # compared as values: the split sum starts from +0, so a -0 product (the
    # e4m3 code 0x80) comes out as +0, as in the oracle's sum
    bad = np.argwhere(oracle.bf16_to_f64(got) != oracle.bf16_to_f64(expect_bits))
    detail = [(int(t), int(n), hex(int(qa[t, n])), float(vals[t, n]),
               float(oracle.bf16_to_f64(got[t, n])), float(oracle.bf16_to_f64(expect_bits[t, n])))
              for t, n in bad[:8]]
    assert len(bad) == 0, \
        f"{len(bad)} outputs differ from bf16(code * scale): (t, n, code, value, got, want) {detail}"


def test_linear_decode_in_cuda_graph():
    M, N, K = 32, 1024, 2048
    xb = act_bits(M, K, 77, 20, 30.0)
    w = bq_synth.weights(N, K, 0.02, 77).numpy()
    qw, sw = oracle.quant_weight(w, 128, 128, INT8)
    x, qw_d, sw_d = dev_bf16(xb), dev_u8(qw), dev_f32(sw)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = bq.workspace(bq.linear_workspace_size(M, N, K), "cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        bq.linear(x, qw_d, sw_d, out=out, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        bq.linear(x, qw_d, sw_d, out=out, ws=ws)
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    bq.check_device_status()
    qa, sa = oracle.quant_act(xb, 128, INT8)
    assert_gemm_close(out, oracle.gemm(qa, sa, qw, sw, 128, 128, INT8), "graph replay")


def test_gemm_strided_operands_and_output():
    M, N, K, bn, bk = 70, 200, 300, 128, 128
    _, qa, sa, qw, sw, _ = make_problem(M, N, K, bn, bk, INT8, 7)
    qa_pad = np.zeros((M, K + 20), np.uint8)
    qa_pad[:, :K] = qa
    qw_pad = np.zeros((N, K + 12), np.uint8)
    qw_pad[:, :K] = qw
    big = torch.full((M, N + 10), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = big[:, 3:3 + N]
    bq.gemm(dev_u8(qa_pad)[:, :K], dev_f32(sa.T), dev_u8(qw_pad)[:, :K], dev_f32(sw), bn, bk,
            INT8, out=out)
    torch.cuda.synchronize()
    assert_gemm_close(out, oracle.gemm(qa, sa, qw, sw, bn, bk, INT8), "strided")
    assert torch.isnan(big[:, :3]).all() and torch.isnan(big[:, 3 + N:]).all()


def test_gemm_k_zero_gives_bias():
    M, N = 3, 5
    bias = torch.randn(N).to(torch.bfloat16).cuda()
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    qa = torch.zeros(M, 0, dtype=torch.uint8, device="cuda")
    qw = torch.zeros(N, 0, dtype=torch.uint8, device="cuda")
    s = torch.zeros(0, M, device="cuda")
    bq.gemm(qa, s, qw, torch.zeros(1, 0, device="cuda"), 128, 128, INT8, bias=bias, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, bias[None, :].expand(M, N))


@pytest.mark.parametrize("dtype", [INT8, FP8])
def test_linear_tiny_workload(dtype):
    cfg = bq_synth.TINY
    a, w = bq_synth.linear_inputs(cfg)
    xb = host_bits(a)
    qw_ref, sw_ref = oracle.quant_weight(w.numpy(), 128, 128, dtype)
    out = bq.linear(dev_bf16(xb), dev_u8(qw_ref), dev_f32(sw_ref), 128, 128, dtype)
    torch.cuda.synchronize()
    qa, sa = oracle.quant_act(xb, 128, dtype)
    assert sw_ref.shape == (3, 2)
    assert_gemm_close(out, oracle.gemm(qa, sa, qw_ref, sw_ref, 128, 128, dtype), "linear")


# --------------------------------------------------------------------------
# MoE steps
# --------------------------------------------------------------------------

def moe_problem(T=200, H=256, I=192, E=8, topk=2, seed=21, dtype=INT8):
    x = act_bits(T, H, seed)
    ids, tw = oracle.moe_route(bq_synth.router_logits(T, E, seed).numpy(), topk)
    w13 = bq_synth.weights(2 * I, H, 0.02, seed, batch=E).numpy()
    w2 = bq_synth.weights(H, I, 0.02, seed + 1, batch=E).numpy()
    q13, s13 = zip(*[oracle.quant_weight_gate_up(w13[e], I, 128, 128, dtype) for e in range(E)])
    q2, s2 = zip(*[oracle.quant_weight(w2[e], 128, 128, dtype) for e in range(E)])
    return dict(x=x, ids=ids, tw=tw, q13=np.stack(q13), s13=np.stack(s13), q2=np.stack(q2),
                s2=np.stack(s2), T=T, H=H, I=I, E=E, topk=topk, dtype=dtype)


def test_moe_permute_bit_exact():
    for T, E, topk in [(200, 8, 2), (1000, 8, 2), (37, 5, 3), (4096, 8, 2)]:
        ids, _ = oracle.moe_route(bq_synth.router_logits(T, E, T).numpy(), topk)
        off, perm, inv = bq.moe_permute(dev_i32(ids), E)
        o_ref, p_ref, i_ref = oracle.moe_permute(ids, E)
        assert np.array_equal(off.cpu().numpy(), o_ref)
        assert np.array_equal(perm.cpu().numpy(), p_ref)
        assert np.array_equal(inv.cpu().numpy(), i_ref)


def test_moe_permute_skewed_and_empty_experts():
    ids = np.zeros((3000, 2), np.int32)
    ids[:, 1] = 7
    ids[::7, 0] = 3
    off, perm, inv = bq.moe_permute(dev_i32(ids), 8)
    o_ref, p_ref, i_ref = oracle.moe_permute(ids, 8)
    assert np.array_equal(off.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy(), p_ref)


def test_moe_layer_stages_vs_oracle():
    p = moe_problem()
    T, H, I, E, topk, dt = p["T"], p["H"], p["I"], p["E"], p["topk"], p["dtype"]
    x = dev_bf16(p["x"])
    off, perm, inv = bq.moe_permute(dev_i32(p["ids"]), E)
    o_ref, p_ref, i_ref = oracle.moe_permute(p["ids"], E)
    # quant + gather: identical to quantising then gathering rows
    qa, sa = bq.moe_quant_gather(x, perm, topk, 128, dt)
    qx_ref, sx_ref = oracle.quant_act(p["x"], 128, dt)
    rows = p_ref // topk
    assert_codes_equal(qa, qx_ref[rows], "gathered codes")
    assert_scales_equal(sa, np.ascontiguousarray(sx_ref[rows]), "gathered scales")
    # w13 grouped GEMM with the gate/up seam (I = 192 is not a multiple of 128)
    y13 = bq.grouped_gemm(qa, sa, off, dev_u8(p["q13"]), dev_f32(p["s13"]), 128, 128,
                          n_seam=I, dtype=dt)
    torch.cuda.synchronize()
    ref13 = oracle.grouped_gemm(qx_ref[rows], sx_ref[rows], o_ref, p["q13"], p["s13"], 128,
                                128, dt, seam=I)
    assert_gemm_close(y13, ref13, "w13")
    # silu * up, requantised: h within one bf16 ulp, codes exact for the GPU's h
    q2a, s2a, h = bq.moe_silu_mul_quant(y13, I, 128, dt, want_h=True)
    torch.cuda.synchronize()
    y13_bits = host_bits(y13)
    h_ref = oracle.bf16_to_f64(oracle.silu_mul(y13_bits, I))
    hv = bf16_values(h)
    assert (np.abs(hv - h_ref) <= bf16_ulp(np.maximum(np.abs(hv), np.abs(h_ref)))).all()
    qh_ref, sh_ref = oracle.quant_act(host_bits(h), 128, dt)
    assert_codes_equal(q2a, qh_ref, "requantised codes")
    assert_scales_equal(s2a, sh_ref, "requantised scales")
    # w2 grouped GEMM
    y2 = bq.grouped_gemm(q2a, s2a, off, dev_u8(p["q2"]), dev_f32(p["s2"]), 128, 128, 0, dt)
    torch.cuda.synchronize()
    ref2 = oracle.grouped_gemm(qh_ref, sh_ref, o_ref, p["q2"], p["s2"], 128, 128, dt)
    assert_gemm_close(y2, ref2, "w2")
    # combine: fp32 accumulate, one rounding
    out = bq.moe_combine(y2, inv, dev_f32(p["tw"]))
    torch.cuda.synchronize()
    yb = host_bits(y2)
    assert_combine_close(out, oracle.moe_combine(yb, i_ref, p["tw"]), yb, i_ref, p["tw"])


@pytest.mark.parametrize("path", [bq.PATH_TCGEN05_1CTA, bq.PATH_TCGEN05_PAIR])
@pytest.mark.parametrize("dtype", [INT8, FP8])
def test_grouped_gemm_tcgen05_vs_oracle(path, dtype):
    p = moe_problem(T=300, H=384, I=256, E=8, dtype=dtype, seed=33)
    T, I, E, topk = p["T"], p["I"], p["E"], p["topk"]
    off, perm, inv = bq.moe_permute(dev_i32(p["ids"]), E)
    o_ref, p_ref, _ = oracle.moe_permute(p["ids"], E)
    qa, sa = bq.moe_quant_gather(dev_bf16(p["x"]), perm, topk, 128, dtype)
    qx, sx = oracle.quant_act(p["x"], 128, dtype)
    rows = p_ref // topk
    bq.set_path(path)
    y13 = bq.grouped_gemm(qa, sa, off, dev_u8(p["q13"]), dev_f32(p["s13"]), 128, 128,
                          n_seam=I, dtype=dtype)
    torch.cuda.synchronize()
    bq.check_device_status()
    ref13 = oracle.grouped_gemm(qx[rows], sx[rows], o_ref, p["q13"], p["s13"], 128, 128, dtype,
                                seam=I)
    assert_gemm_close(y13, ref13, "tcgen05 grouped w13")


@pytest.mark.parametrize("dtype", [INT8, FP8])
def test_cta_pair_and_single_cta_kernels_agree_bit_for_bit(dtype):
    """The CTA-pair kernel (256-row tiles, cta_group::2 MMAs) and the
    single-CTA kernel sum the same K-blocks in the same order and promote
    them identically: every output is the same bits.  Dense with bias (M and
    N ragged against 256, a partial last K-block), one scale block along K,
    the grouped w13 with its gate/up seam, the fused SiLU requantisation and
    the combining w2."""
    def both(fn):
        outs = []
        for path in (bq.PATH_TCGEN05_1CTA, bq.PATH_TCGEN05_PAIR):
            bq.set_path(path)
            outs.append(fn())
        bq.set_path(bq.PATH_AUTO)
        torch.cuda.synchronize()
        bq.check_device_status()
        return outs

    def same(a, b, what):
        a = a if isinstance(a, (tuple, list)) else (a,)
        b = b if isinstance(b, (tuple, list)) else (b,)
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), what

    _, qa, sa, qw, sw, bb = make_problem(600, 640, 1008, 128, 128, dtype, 91, bias=True)
    args = (dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), 128, 128, dtype)
    same(*both(lambda: bq.gemm(*args, bias=dev_bf16(bb))), "dense")
    same(*both(lambda: bq.gemm_partial(*args)), "dense fp32 partial")
    xb = act_bits(520, 512, 92)
    q1, s1 = oracle.quant_act(xb, 512, dtype)
    qw1, sw1 = oracle.quant_weight(bq_synth.weights(768, 512, 0.02, 93).numpy(), 1, 512, dtype)
    same(*both(lambda: bq.gemm(dev_u8(q1), dev_f32(s1.T), dev_u8(qw1), dev_f32(sw1), 1, 512,
                               dtype)), "one scale block along K")
    p = moe_problem(T=700, H=384, I=256, E=8, dtype=dtype, seed=94)
    off, perm, inv = bq.moe_permute(dev_i32(p["ids"]), 8)
    qg, sg = bq.moe_quant_gather(dev_bf16(p["x"]), perm, 2, 128, dtype)
    q13, s13 = dev_u8(p["q13"]), dev_f32(p["s13"])
    same(*both(lambda: bq.grouped_gemm(qg, sg, off, q13, s13, 128, 128, n_seam=256,
                                       dtype=dtype)), "grouped w13")
    (qh, sh), (qh2, sh2) = both(lambda: bq.grouped_gemm_silu_quant(qg, sg, off, q13, s13, dtype))
    same((qh, sh), (qh2, sh2), "fused SiLU requantisation")
    q2, s2, tw = dev_u8(p["q2"]), dev_f32(p["s2"]), dev_f32(p["tw"])

    def comb():
        acc = torch.zeros(700, 384, dtype=torch.float32, device="cuda")
        bq.grouped_gemm_combine(qh, sh, off, q2, s2, perm, tw, acc, dtype)
        return bq.moe_combine_finish(acc)
    same(*both(comb), "combining w2")


# w2 grouped GEMM fused with the weighted top-k combine
# (T, H, I, E, topk, dtype, seed): two 256-wide column tiles, FP8, an output
# width with a ragged last tile (scalar atomics), top-3 (order-dependent fp32
# sums: tolerance only), top-1, and K with a partial last block
COMBINE_CASES = [(300, 384, 256, 8, 2, INT8, 41), (300, 384, 256, 8, 2, FP8, 42),
                 (200, 208, 256, 5, 2, INT8, 43), (100, 256, 128, 4, 3, INT8, 44),
                 (64, 256, 256, 4, 1, FP8, 45), (150, 512, 320, 8, 2, INT8, 46)]


def _combine_exact(y_bits, inv, w):
    """bf16 of the fp32 sum of fp32 products w[t, j] * y[inv[t, j]], summed in
    slot order from zero: what the atomic combine computes for top-k <= 2."""
    T, topk = w.shape
    yv = oracle.bf16_to_f64(y_bits).astype(np.float32)
    acc = np.zeros((T, y_bits.shape[1]), np.float32)
    for j in range(topk):
        acc = acc + w[:, j:j + 1] * yv[inv.reshape(T, topk)[:, j]]
    return oracle.bf16_to_f64(oracle.bf16_from_f64(acc.astype(np.float64)))


@pytest.mark.parametrize("T,H,I,E,topk,dtype,seed", COMBINE_CASES)
def test_grouped_gemm_combine_vs_oracle(T, H, I, E, topk, dtype, seed):
    p = moe_problem(T=T, H=H, I=I, E=E, topk=topk, dtype=dtype, seed=seed)
    off, perm, inv = bq.moe_permute(dev_i32(p["ids"]), E)
    o_ref, p_ref, i_ref = oracle.moe_permute(p["ids"], E)
    qa, sa = bq.moe_quant_gather(dev_bf16(p["x"]), perm, topk, 128, dtype)
    if I % 128 == 0:
        qh, sh = bq.grouped_gemm_silu_quant(qa, sa, off, dev_u8(p["q13"]), dev_f32(p["s13"]),
                                            dtype)
    else:   # the fused SiLU epilogue needs whole 128-column h groups
        y13 = bq.grouped_gemm(qa, sa, off, dev_u8(p["q13"]), dev_f32(p["s13"]), 128, 128,
                              n_seam=I, dtype=dtype)
        qh, sh = bq.moe_silu_mul_quant(y13, I, 128, dtype)
    q2, s2, tw = dev_u8(p["q2"]), dev_f32(p["s2"]), dev_f32(p["tw"])
    # the unfused w2 GEMM on the same tensor-core kernel: its bf16 rows are the
    # y the combining epilogue weights, and they are pinned to the oracle
    bq.set_path(bq.PATH_TCGEN05_1CTA)
    y2 = bq.grouped_gemm(qh, sh, off, q2, s2, 128, 128, 0, dtype)
    acc = torch.zeros(T, H, dtype=torch.float32, device="cuda")
    bq.grouped_gemm_combine(qh, sh, off, q2, s2, perm, tw, acc, dtype)
    out = bq.moe_combine_finish(acc)
    torch.cuda.synchronize()
    bq.check_device_status()
    ref2 = oracle.grouped_gemm(qh.cpu().numpy(), sh.cpu().numpy().T,
                               o_ref, p["q2"], p["s2"], 128, 128, dtype)
    assert_gemm_close(y2, ref2, "w2")
    yb = host_bits(y2)
    assert_combine_close(out, oracle.moe_combine(yb, i_ref, p["tw"]), yb, i_ref, p["tw"],
                         "fused combine")
    if topk <= 2:
        g = bf16_values(out)
        assert np.array_equal(g, _combine_exact(yb, i_ref, p["tw"])), \
            "atomic combine differs from the fp32 slot-order sum"
    assert not acc.any(), "the finish pass must leave the sums zeroed"
    # a second layer call on the zeroed sums gives the same bits
    bq.grouped_gemm_combine(qh, sh, off, q2, s2, perm, tw, acc, dtype)
    out2 = bq.moe_combine_finish(acc)
    torch.cuda.synchronize()
    if topk <= 2:
        assert torch.equal(out2.view(torch.int16), out.view(torch.int16))


def test_grouped_gemm_combine_reports_a_bad_pair_index():
    p = moe_problem(T=64, H=256, I=128, E=4, topk=2, seed=47)
    off, perm, inv = bq.moe_permute(dev_i32(p["ids"]), 4)
    qa, sa = bq.moe_quant_gather(dev_bf16(p["x"]), perm, 2, 128, INT8)
    qh, sh = bq.grouped_gemm_silu_quant(qa, sa, off, dev_u8(p["q13"]), dev_f32(p["s13"]), INT8)
    bad = perm.clone()
    bad[5] = 128                                   # outside [0, R): skipped and recorded
    acc = torch.zeros(64, 256, dtype=torch.float32, device="cuda")
    bq.grouped_gemm_combine(qh, sh, off, dev_u8(p["q2"]), dev_f32(p["s2"]), bad,
                            dev_f32(p["tw"]), acc, INT8)
    torch.cuda.synchronize()
    with pytest.raises(bq.BqError) as ei:
        bq.check_device_status()
    assert ei.value.status == bq.ERR_INVALID_ARG
    bq.check_device_status()                       # read and cleared
    with pytest.raises(bq.BqError) as ei:
        bq.grouped_gemm_combine(qh[:127], sh[:, :127].contiguous(), off, dev_u8(p["q2"]),
                                dev_f32(p["s2"]), perm[:127], dev_f32(p["tw"]), acc, INT8)
    assert ei.value.status == bq.ERR_INVALID_ARG   # R is not T * topk


# w13 grouped GEMM fused with silu(gate) * up and the 1 x 128 requantisation
# (T, H, I, E, dtype, seed): ragged experts, K with a partial last block,
# several 128-column h groups, and an FP8 case
SILU_CASES = [(300, 384, 256, 8, INT8, 33), (300, 384, 256, 8, FP8, 34),
              (1000, 208, 384, 5, INT8, 35), (50, 128, 128, 4, FP8, 36),
              (700, 512, 640, 8, INT8, 37)]


@pytest.mark.parametrize("T,H,I,E,dtype,seed", SILU_CASES)
def test_fused_w13_silu_requant(T, H, I, E, dtype, seed):
    p = moe_problem(T=T, H=H, I=I, E=E, dtype=dtype, seed=seed)
    topk = p["topk"]
    off, perm, inv = bq.moe_permute(dev_i32(p["ids"]), E)
    o_ref, p_ref, _ = oracle.moe_permute(p["ids"], E)
    qa, sa = bq.moe_quant_gather(dev_bf16(p["x"]), perm, topk, 128, dtype)
    q13, s13 = dev_u8(p["q13"]), dev_f32(p["s13"])
    qf, sf = bq.grouped_gemm_silu_quant(qa, sa, off, q13, s13, dtype)
    # the unfused calls: w13 output in bf16, then silu * up and requantisation
    y13 = bq.grouped_gemm(qa, sa, off, q13, s13, 128, 128, n_seam=I, dtype=dtype)
    qu, su, hu = bq.moe_silu_mul_quant(y13, I, 128, dtype, want_h=True)
    torch.cuda.synchronize()
    bq.check_device_status()
    assert torch.equal(qf, qu), "fused codes differ from the unfused calls"
    assert torch.equal(sf.view(torch.int32), su.view(torch.int32)), "fused scales differ"
    # h (fp32 silu * up of the w13 output, one bf16 rounding) is within one
    # bf16 ulp of the oracle's; the codes of that h are the oracle's exactly
    h_or = oracle.bf16_to_f64(oracle.silu_mul(host_bits(y13), I))
    hv = bf16_values(hu)
    assert (np.abs(hv - h_or) <= bf16_ulp(np.maximum(np.abs(hv), np.abs(h_or)))).all()
    qh, sh = oracle.quant_act(host_bits(hu), 128, dtype)
    assert_codes_equal(qf, qh, "fused codes vs oracle quantisation of h")
    assert_scales_equal(sf, sh, "fused scales vs oracle quantisation of h")
    # the whole chain in the oracle (its own w13 GEMM): h agrees to the GEMM's
    # tolerance, so the dequantised codes agree to within one code step
    qx, sx = oracle.quant_act(p["x"], 128, dtype)
    rows = p_ref // topk
    ref13 = oracle.grouped_gemm(qx[rows], sx[rows], o_ref, p["q13"], p["s13"], 128, 128, dtype,
                                seam=I)
    h_ref = oracle.bf16_to_f64(oracle.silu_mul(oracle.bf16_from_f64(ref13), I))
    deq = oracle.code_values(qf.cpu().numpy(), dtype) * np.repeat(sf.cpu().numpy().T, 128,
                                                                    axis=1)[:, :I]
    step = np.repeat(sf.cpu().numpy().T, 128, axis=1)[:, :I]
    hmax = np.repeat(np.abs(h_ref).reshape(-1, I // 128, 128).max(axis=2), 128, axis=1)
    if dtype == INT8:
        tol = 0.5 * step + 2.0 ** -6 * hmax          # half a code + h within the GEMM's error
    else:
        tol = 2.0 ** -4 * np.abs(h_ref) + 2.0 ** -9 * step + 2.0 ** -6 * hmax
    d = np.abs(deq - h_ref)
    assert (d <= tol).all(), f"max excess {(d - tol).max()}"


def test_fused_w13_silu_requant_rows_past_offsets_and_paths():
    p = moe_problem(T=50, H=128, I=256, E=4, seed=38)
    off = np.array([0, 10, 10, 30, 60], np.int32)     # 60 of the 100 rows routed
    R, I = 100, 256
    qa = torch.from_numpy(np.random.default_rng(5).integers(-127, 128, (R, 128)).astype(np.int8)
                          .view(np.uint8)).cuda()
    sa = torch.full((1, R), 0.01, dtype=torch.float32, device="cuda")
    q = torch.full((R, I), 0x5A, dtype=torch.uint8, device="cuda")
    s = torch.full((2, R), -1.0, dtype=torch.float32, device="cuda")
    bq.grouped_gemm_silu_quant(qa, sa, dev_i32(off), dev_u8(p["q13"]), dev_f32(p["s13"]), INT8,
                               q=q, s=s)
    torch.cuda.synchronize()
    assert (q[60:] == 0x5A).all() and (s[:, 60:] == -1.0).all()
    y = bq.grouped_gemm(qa, sa, dev_i32(off), dev_u8(p["q13"]), dev_f32(p["s13"]), 128, 128,
                        n_seam=I, dtype=INT8)
    qu, su = bq.moe_silu_mul_quant(y[:60].contiguous(), I, 128, INT8)
    assert torch.equal(q[:60], qu) and torch.equal(s[:, :60], su)
    # TMA rows must be multiples of 16 bytes (K = 200 is not)
    p2 = moe_problem(T=20, H=200, I=128, E=2, seed=39)
    qa2 = torch.zeros(40, 200, dtype=torch.uint8, device="cuda")
    sa2 = torch.ones(2, 40, dtype=torch.float32, device="cuda")
    with pytest.raises(bq.BqError) as ei:
        bq.grouped_gemm_silu_quant(qa2, sa2, dev_i32(np.array([0, 20, 40], np.int32)),
                                   dev_u8(p2["q13"]), dev_f32(p2["s13"]), INT8)
    assert ei.value.status == bq.ERR_UNSUPPORTED
    # only the tensor-core path has the fused epilogue
    for path in (bq.PATH_SIMT,):
        bq.set_path(path)
        with pytest.raises(bq.BqError) as ei:
            bq.grouped_gemm_silu_quant(qa, sa, dev_i32(off), dev_u8(p["q13"]),
                                       dev_f32(p["s13"]), INT8)
        assert ei.value.status == bq.ERR_UNSUPPORTED
    bq.set_path(bq.PATH_AUTO)


@pytest.mark.parametrize("path", [bq.PATH_SIMT, bq.PATH_TCGEN05_1CTA, bq.PATH_TCGEN05_PAIR])
def test_grouped_gemm_leaves_rows_past_offsets_untouched(path):
    p = moe_problem(T=50, H=128, I=128, E=4)
    bq.set_path(path)
    off = np.array([0, 10, 10, 30, 60], np.int32)     # 60 of the 100 rows routed
    R = 100
    qa = np.random.default_rng(0).integers(-100, 100, (R, 128)).astype(np.int8).view(np.uint8)
    sa = np.full((R, 1), 0.01, np.float32)
    out = torch.full((R, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    bq.grouped_gemm(dev_u8(qa), dev_f32(sa.T), dev_i32(off), dev_u8(p["q2"][:4]),
                    dev_f32(p["s2"][:4]), 128, 128, 0, INT8, out=out)
    torch.cuda.synchronize()
    ref = oracle.grouped_gemm(qa[:60], sa[:60], off, p["q2"][:4], p["s2"][:4], 128, 128, INT8)
    assert_gemm_close(out[:60], ref, "grouped")
    assert (out[60:] == 7.0).all()


# --------------------------------------------------------------------------
# device status word
# --------------------------------------------------------------------------

def test_bounded_wait_reports_timeout_and_context_survives():
    bq.selftest_bounded_wait(2000)
    with pytest.raises(bq.BqError) as ei:
        bq.check_device_status()
    assert ei.value.status == bq.ERR_DEVICE_TIMEOUT
    bq.check_device_status()          # cleared
    q, s = bq.quant_act(torch.ones(2, 128, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert (q.cpu().numpy().view(np.int8) == 127).all()


def test_bad_expert_id_is_reported():
    ids = np.array([[0, 1], [9, 2], [3, -1]], np.int32)
    off, perm, inv = bq.moe_permute(dev_i32(ids), 8)
    with pytest.raises(bq.BqError) as ei:
        bq.check_device_status()
    assert ei.value.status == bq.ERR_INVALID_ARG
    assert off.cpu().numpy()[-1] == 4      # the two bad pairs are placed nowhere


# --------------------------------------------------------------------------
# one scale block along K: per-token activations, per-channel (block_n = 1)
# or per-row-block weights -- the W8A8 degenerate case of the block layout
# --------------------------------------------------------------------------

ONEK_SHAPES = [(300, 512, 512, 1), (1024, 1000, 1000, 1), (260, 768, 4096, 128),
               (513, 2048, 1024, 1)]


@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M,N,K,bn", ONEK_SHAPES)
@pytest.mark.parametrize("path", [bq.PATH_AUTO, bq.PATH_TCGEN05_1CTA, bq.PATH_TCGEN05_PAIR])
def test_one_scale_block_along_k(path, M, N, K, bn, dtype):
    xb = act_bits(M, K, 500 + M, max(1, K // 100), 30.0)
    w = bq_synth.weights(N, K, 0.02, 501 + N).numpy()
    bias = oracle.bf16_from_f64(np.random.default_rng(N).normal(0, 0.5, N))
    qa, sa = oracle.quant_act(xb, K, dtype)                 # one scale per token
    qw, sw = oracle.quant_weight(w, bn, K, dtype)           # one scale per bn rows
    assert sa.shape == (M, 1) and sw.shape == (cdiv(N, bn), 1)
    # the GPU's quantisers give the same codes and scales
    qg, sg = bq.quant_act(dev_bf16(xb), K, dtype)
    qwg, swg = bq.quant_weight(torch.from_numpy(w).cuda(), bn, K, dtype)
    torch.cuda.synchronize()
    assert_codes_equal(qg, qa, "per-token codes")
    assert_scales_equal(sg, sa, "per-token scales")
    assert_codes_equal(qwg, qw, "weight codes")
    assert np.array_equal(swg.cpu().numpy().view(np.uint32), sw.view(np.uint32))
    bq.set_path(path)
    try:
        if path in (bq.PATH_TCGEN05_1CTA, bq.PATH_TCGEN05_PAIR) and K % 16 != 0:
            # TMA rows must be multiples of 16 bytes: the forced path refuses
            with pytest.raises(bq.BqError) as ei:
                bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), bn, K, dtype)
            assert ei.value.status == bq.ERR_UNSUPPORTED
            return
        out = bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qw), dev_f32(sw), bn, K, dtype,
                      bias=dev_bf16(bias))
        lin = bq.linear(dev_bf16(xb), dev_u8(qw), dev_f32(sw), bn, K, dtype, bias=dev_bf16(bias))
        torch.cuda.synchronize()
    finally:
        bq.set_path(bq.PATH_AUTO)
    bq.check_device_status()
    ref = oracle.gemm(qa, sa, qw, sw, bn, K, dtype, bias_bf16=bias)
    assert_gemm_close(out, ref, f"one scale block along K, M={M} N={N} K={K} bn={bn}")
    assert_gemm_close(lin, ref, "bq_linear, one scale block along K")


# --------------------------------------------------------------------------
# MXFP8 dense linear (32-element groups, E8M0 scales, block-scaled MMA)
# --------------------------------------------------------------------------

MX_QUANT_SHAPES = [(1, 128), (7, 256), (130, 384), (300, 1024)]


@pytest.mark.parametrize("M,K", MX_QUANT_SHAPES)
def test_mx_quant_act_and_weight_exact(M, K):
    xb = act_bits(M, K, 700 + M, max(1, K // 100), 30.0)
    xb[0, :32] = 0                                   # an all-zero group
    q, sf = bq.mx_quant_act(dev_bf16(xb))
    w = bq_synth.weights(M, K, 0.02, 701 + K).numpy()
    qw, sfw = bq.mx_quant_weight(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    qr, sr = oracle.mx_quant(oracle.bf16_to_f64(xb))
    assert_codes_equal(q, qr, "MX activation codes")
    assert np.array_equal(mx_sf_rows(sf, M, K), sr), "MX activation scales"
    qwr, swr = oracle.mx_quant(w.astype(np.float64))
    assert_codes_equal(qw, qwr, "MX weight codes")
    assert np.array_equal(mx_sf_rows(sfw, M, K), swr), "MX weight scales"


MX_GEMM_SHAPES = [(1, 256, 128), (16, 320, 256), (200, 300, 512), (513, 1000, 1024),
                  (128, 512, 4096)]


@pytest.mark.parametrize("M,N,K", MX_GEMM_SHAPES)
def test_mx_gemm_vs_oracle(M, N, K):
    # codes and scales from the oracle (independent of the GPU quantiser),
    # with a spread of scale exponents
    rng = np.random.default_rng(M + N + K)
    xa = rng.normal(0, 1, (M, K)) * np.exp2(rng.integers(-6, 7, (M, 1)))
    xw = rng.normal(0, 0.02, (N, K)) * np.exp2(rng.integers(-3, 4, (N, K // 32))).repeat(32, 1)
    qa, sa = oracle.mx_quant(xa)
    qw, sw = oracle.mx_quant(xw)
    bias = oracle.bf16_from_f64(rng.normal(0, 0.5, N))
    out = bq.mx_gemm(dev_u8(qa), dev_u8(mx_sf_atoms(sa, K)), dev_u8(qw),
                     dev_u8(mx_sf_atoms(sw, K)), bias=dev_bf16(bias))
    torch.cuda.synchronize()
    bq.check_device_status()
    assert_gemm_close(out, oracle.mx_gemm(qa, sa, qw, sw, bias), f"MXFP8 {M}x{N}x{K}")


def test_mx_linear_end_to_end_and_errors():
    M, N, K = 96, 384, 640
    xb = act_bits(M, K, 710, 6, 30.0)
    w = bq_synth.weights(N, K, 0.02, 711).numpy()
    qa, sfa = bq.mx_quant_act(dev_bf16(xb))
    qw, sfw = bq.mx_quant_weight(torch.from_numpy(w).cuda())
    out = bq.mx_gemm(qa, sfa, qw, sfw)
    torch.cuda.synchronize()
    qar, sar = oracle.mx_quant(oracle.bf16_to_f64(xb))
    qwr, swr = oracle.mx_quant(w.astype(np.float64))
    assert_gemm_close(out, oracle.mx_gemm(qar, sar, qwr, swr), "MXFP8 linear")
    # the one-call layer runs the same two kernels: identical output
    bias = dev_bf16(oracle.bf16_from_f64(np.linspace(-1, 1, N)))
    lin = bq.mx_linear(dev_bf16(xb), qw, sfw, bias=bias)
    two = bq.mx_gemm(qa, sfa, qw, sfw, bias=bias)
    torch.cuda.synchronize()
    assert torch.equal(lin, two)
    # K must be a multiple of 128; only the tensor-core path has the kernel
    with pytest.raises(bq.BqError) as ei:
        bq.mx_quant_act(dev_bf16(act_bits(4, 96, 712)))
    assert ei.value.status == bq.ERR_UNSUPPORTED
    bq.set_path(bq.PATH_SIMT)
    with pytest.raises(bq.BqError) as ei:
        bq.mx_gemm(qa, sfa, qw, sfw)
    assert ei.value.status == bq.ERR_UNSUPPORTED
    bq.set_path(bq.PATH_AUTO)


def test_shared_workspace_survives_every_entry_point():
    """One workspace buffer serves bq_mx_linear, bq_gemm and bq_linear in any
    order: no call may leave bytes in the region where the decode GEMM keeps
    its split-K arrival counters.  An MXFP8 linear (61 440 code bytes) runs
    first on the binding's cached workspace, then decode GEMMs whose split
    partials are reduced through that workspace, each against the oracle."""
    M, N, K = 96, 384, 640
    xb = act_bits(M, K, 720, 6, 30.0)
    w = bq_synth.weights(N, K, 0.02, 721).numpy()
    qw, sfw = bq.mx_quant_weight(torch.from_numpy(w).cuda())
    x = dev_bf16(xb)
    need = max(bq.mx_linear_workspace_size(M, K), bq.gemm_workspace_size(1, 640, 66560),
               bq.linear_workspace_size(33, 256, 33024))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    bq.mx_linear(x, qw, sfw, ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:65536].count_nonzero()) == 0, "bq_mx_linear wrote into the counter region"
    # split K ranges too long for the cluster kernel's shared memory: these
    # run the split-K kernel that reduces through the workspace
    for (Md, Nd, Kd), seed in (((1, 640, 66560), 722), ((33, 256, 33024), 723)):
        xd, qa, sa, qwd, swd, _ = make_problem(Md, Nd, Kd, 128, 128, INT8, seed)
        ref = oracle.gemm(qa, sa, qwd, swd, 128, 128, INT8)
        assert bq.gemm_workspace_size(Md, Nd, Kd) > 0, "shape must use the workspace"
        out = bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qwd), dev_f32(swd), out=None, ws=ws)
        lin = bq.linear(dev_bf16(xd), dev_u8(qwd), dev_f32(swd), ws=ws)
        bq.mx_linear(x, qw, sfw, ws=ws)
        again = bq.gemm(dev_u8(qa), dev_f32(sa.T), dev_u8(qwd), dev_f32(swd), ws=ws)
        torch.cuda.synchronize()
        bq.check_device_status()
        assert_gemm_close(out, ref, f"decode after mx_linear {Md}x{Nd}x{Kd}")
        assert_gemm_close(lin, ref, f"linear after decode {Md}x{Nd}x{Kd}")
        assert torch.equal(out, again), "decode output depends on the call before it"
        assert int(ws[:65536].count_nonzero()) == 0, "counters not left at zero"


def test_mx_gemm_narrow_n_and_strided_operands():
    # N < 128 (one weight scale atom, half of the 256-wide tile unused) and
    # codes read through row strides wider than K
    rng = np.random.default_rng(77)
    M, N, K = 3, 64, 256
    qa, sa = oracle.mx_quant(rng.normal(0, 1, (M, K)))
    qw, sw = oracle.mx_quant(rng.normal(0, 0.02, (N, K)))
    out = bq.mx_gemm(dev_u8(qa), dev_u8(mx_sf_atoms(sa, K)), dev_u8(qw), dev_u8(mx_sf_atoms(sw, K)))
    torch.cuda.synchronize()
    assert_gemm_close(out, oracle.mx_gemm(qa, sa, qw, sw), "MXFP8 narrow N")
    M, N, K = 150, 400, 384
    qa, sa = oracle.mx_quant(rng.normal(0, 1, (M, K)))
    qw, sw = oracle.mx_quant(rng.normal(0, 0.02, (N, K)))
    wide_a = torch.zeros(M, K + 128, dtype=torch.uint8, device="cuda")
    wide_w = torch.zeros(N, K + 64, dtype=torch.uint8, device="cuda")
    wide_a[:, :K] = dev_u8(qa)
    wide_w[:, :K] = dev_u8(qw)
    out = bq.mx_gemm(wide_a[:, :K], dev_u8(mx_sf_atoms(sa, K)), wide_w[:, :K],
                     dev_u8(mx_sf_atoms(sw, K)))
    torch.cuda.synchronize()
    bq.check_device_status()
    assert_gemm_close(out, oracle.mx_gemm(qa, sa, qw, sw), "MXFP8 strided operands")


# --------------------------------------------------------------------------
# K-sharded (row-parallel) linear: fp32 partials, one rounding at the end
# --------------------------------------------------------------------------

@pytest.mark.parametrize("path", [bq.PATH_AUTO, bq.PATH_SIMT])
@pytest.mark.parametrize("dtype", [INT8, FP8])
@pytest.mark.parametrize("M,N,K,shards", [(1, 4096, 4096, 2),    # cluster decode kernel
                                          (37, 1000, 1536, 3),   # decode, ragged N
                                          (300, 640, 1024, 2),   # tcgen05 kernel
                                          (200, 256, 896, 7)])
def test_gemm_partial_shards_sum_then_round_once(path, dtype, M, N, K, shards):
    _, qa, sa, qw, sw, bb = make_problem(M, N, K, 128, 128, dtype, 800 + M, bias=True)
    bq.set_path(path)
    kb = K // 128 // shards
    edges = [128 * kb * i for i in range(shards)] + [K]
    total = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    for a, b in zip(edges[:-1], edges[1:]):
        part = bq.gemm_partial(dev_u8(np.ascontiguousarray(qa[:, a:b])),
                               dev_f32(np.ascontiguousarray(sa[:, a // 128:b // 128].T)),
                               dev_u8(np.ascontiguousarray(qw[:, a:b])),
                               dev_f32(np.ascontiguousarray(sw[:, a // 128:b // 128])),
                               128, 128, dtype)
        total += part                                  # the all-reduce, on one GPU
    out = bq.finish_bf16(total, dev_bf16(bb))
    torch.cuda.synchronize()
    bq.check_device_status()
    ref = oracle.gemm(qa, sa, qw, sw, 128, 128, dtype, bias_bf16=bb)
    assert_gemm_close(out, ref, f"sharded x{shards} {M}x{N}x{K} dtype={dtype}")


def test_finish_bf16_rounds_the_fp32_sum_once():
    rng = np.random.default_rng(5)
    for M, N in ((3, 7), (64, 4096), (5, 1001)):
        part = torch.from_numpy(rng.normal(0, 3, (M, N)).astype(np.float32))
        bias = torch.from_numpy(rng.normal(0, 1, N).astype(np.float32)).to(torch.bfloat16)
        out = bq.finish_bf16(part.cuda(), bias.cuda())
        torch.cuda.synchronize()
        # the fp32 add, then torch's round-to-nearest-even conversion
        ref = (part + bias.float()[None, :]).to(torch.bfloat16)
        assert torch.equal(out.cpu().view(torch.int16), ref.view(torch.int16))
        out = bq.finish_bf16(part.cuda())
        assert torch.equal(out.cpu().view(torch.int16), part.to(torch.bfloat16).view(torch.int16))


def test_tensor_parallel_layers_on_one_rank_use_the_cuda_kernels():
    """tp.py on a one-rank group (no collective runs): the CUDA backend's
    column- and row-parallel layers equal the unsharded layer."""
    import os
    import socket
    import torch.distributed as dist
    from block_scaled_w8a8_b200 import tp
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        xb, qa, sa, qw, sw, bb = make_problem(24, 512, 768, 128, 128, INT8, 61, bias=True)
        x, qwd, swd, bias = dev_bf16(xb), dev_u8(qw), dev_f32(sw), dev_bf16(bb)
        ycol = tp.column_parallel_linear(x, qwd, swd, bias)
        yrow = tp.row_parallel_linear(x, qwd, swd, bias)
        torch.cuda.synchronize()
        bq.check_device_status()
        ref = oracle.gemm(qa, sa, qw, sw, 128, 128, INT8, bias_bf16=bb)
        assert_gemm_close(ycol, ref, "column parallel, one rank")
        assert_gemm_close(yrow, ref, "row parallel, one rank")
    finally:
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# device-side routing
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,topk", [(4096, 8, 2), (37, 8, 1), (300, 64, 6), (5, 256, 8),
                                      (100, 3, 3), (33, 40, 2)])
def test_moe_route_vs_oracle(T, E, topk):
    lg = bq_synth.router_logits(T, E, 100 + E).numpy()
    lg[: T // 3, E // 2] = lg[: T // 3, 0]            # exact ties: the lower index wins
    ids, w = bq.moe_route(torch.from_numpy(lg).cuda(), topk)
    torch.cuda.synchronize()
    ids_ref, w_ref = oracle.moe_route(lg, topk)
    # the experts come from comparing the same fp32 logits: bit-exact
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    # fp32 expf, sum and division against the fp64 softmax: a few fp32 ulp
    np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=2e-6, atol=1e-7)


def test_moe_route_rejects_out_of_range_shapes():
    lg = torch.zeros(4, 300, device="cuda")
    with pytest.raises(bq.BqError) as ei:
        bq.moe_route(lg, 2)
    assert ei.value.status == bq.ERR_UNSUPPORTED
    with pytest.raises(bq.BqError) as ei:
        bq.moe_route(torch.zeros(4, 4, device="cuda"), 5)
    assert ei.value.status == bq.ERR_INVALID_ARG
