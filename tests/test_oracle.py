"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

Each test ties the oracle to something other than itself: a value printed on
the pages (tests/golden), a closed form, an invariant, a special case that
reduces to a library routine (numpy integer matmul, numpy stable sort, torch's
float8/bf16 casts, BLAS fp64 matmul), or brute force on tiny inputs.  They are
chosen so that a dropped term, a wrong sign or index, or a transposed operand
in the oracle fails at least one of them (see test_oracle_mutants.py).
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from oracle import FP8, INT8, cdiv

import bq_synth


def bits_to_bf16_f64(h):
    return oracle.bf16_to_f64(h)


# --------------------------------------------------------------------------
# scale-grid shapes (pages' worked example + ceil rule)
# --------------------------------------------------------------------------

def test_scale_grid_worked_example(golden):
    ex = golden["scale_grid"][0]
    N, K = ex["weight"]
    bn, bk = ex["block"]
    w = np.zeros((N, K), dtype=np.float32)
    q, s = oracle.quant_weight(w, bn, bk, INT8)
    assert list(s.shape) == ex["scale"] == [32, 32]
    assert q.shape == (N, K)


@pytest.mark.parametrize("N,K,bn,bk,grid", [
    (320, 200, 128, 128, (3, 2)),        # tiny workload: partial blocks both ways
    (14336, 4096, 128, 128, (112, 32)),  # prefill weight
    (4096, 14336, 128, 128, (32, 112)),  # fp8 down-projection
    (129, 257, 128, 128, (2, 3)),
    (1, 1, 128, 128, (1, 1)),
])
def test_scale_grid_ceil(N, K, bn, bk, grid):
    w = np.random.default_rng(0).standard_normal((N, K)).astype(np.float32)
    _, s = oracle.quant_weight(w, bn, bk, INT8)
    assert s.shape == grid == (cdiv(N, bn), cdiv(K, bk))


@pytest.mark.parametrize("I,H,bn,bk", [(14336, 4096, 128, 128), (130, 200, 128, 128),
                                       (64, 128, 128, 128)])
def test_w13_scale_rows(golden, I, H, bn, bk):
    # section 5: 2 * ceil(I/bn) rows, NOT ceil(2I/bn) (they differ for I=130)
    w = np.random.default_rng(1).standard_normal((2 * I, H)).astype(np.float32)
    q, s = oracle.quant_weight_gate_up(w, I, bn, bk, INT8)
    assert s.shape == (2 * cdiv(I, bn), cdiv(H, bk))
    assert q.shape == (2 * I, H)


# --------------------------------------------------------------------------
# INT8 quantisation: invariants and constructed ties
# --------------------------------------------------------------------------

def _random_bf16(shape, seed, scale=1.0):
    t = torch.randn(*shape, generator=torch.Generator().manual_seed(seed)) * scale
    return bq_synth.bf16_bits(t.to(torch.bfloat16))


@pytest.mark.parametrize("K,gk", [(200, 128), (128, 128), (1, 128), (257, 128), (96, 32)])
def test_int8_quant_invariants(golden, K, gk):
    M = 37
    x = _random_bf16((M, K), 3, 5.0)
    # plant an exact-zero group and a group with one huge outlier
    x[0, :] = 0
    x[1, min(5, K - 1)] = bq_synth.bf16_bits(torch.tensor([1e4]).to(torch.bfloat16))[0]
    q, s = oracle.quant_act(x, gk, INT8)
    xv = bits_to_bf16_f64(x)
    qv = q.view(np.int8).astype(np.int64)
    rng = golden["int8_range"]
    assert qv.min() >= rng["min"] and qv.max() <= rng["max"]
    Kb = cdiv(K, gk)
    assert s.shape == (M, Kb)
    for m in range(M):
        for g in range(Kb):
            sl = slice(g * gk, min(K, (g + 1) * gk))
            amax = np.abs(xv[m, sl]).max()
            sc = float(s[m, g])
            if amax == 0:
                assert sc == 0.0 and (qv[m, sl] == 0).all()
                continue
            # scale = amax / 127 to fp32 precision
            assert abs(sc * 127.0 - amax) <= 2 ** -22 * amax
            # dequantisation error within half a step, up to the one fp32
            # rounding of the quotient x/s (|x/s| <= 127, ulp <= 2^-24 * 128)
            err = np.abs(xv[m, sl] - qv[m, sl] * sc)
            assert (err <= sc * (0.5 + 128 * 2 ** -24)).all()
            # the element attaining amax maps to +-127
            i = int(np.argmax(np.abs(xv[m, sl])))
            assert abs(qv[m, sl][i]) == 127
            assert np.sign(qv[m, sl][i]) == np.sign(xv[m, sl][i])


def test_int8_odd_symmetry():
    x = _random_bf16((64, 256), 4, 2.0)
    q, s = oracle.quant_act(x, 128, INT8)
    qn, sn = oracle.quant_act(x ^ np.uint16(0x8000), 128, INT8)
    assert (s == sn).all()
    assert (q.view(np.int8).astype(int) == -qn.view(np.int8).astype(int)).all()


def test_int8_ties_round_half_even():
    # amax = 127 * 2^j gives scale exactly 2^j; x = (k + 1/2) 2^j are ties.
    for j in (-4, 0, 3):
        s = 2.0 ** j
        ks = np.arange(-20, 20)
        vals = np.concatenate([[127 * s], (ks + 0.5) * s])
        x = bq_synth.bf16_bits(torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16))
        assert (bits_to_bf16_f64(x) == vals).all()       # all exact in bf16
        q, sc = oracle.quant_act(x[None, :], 128, INT8)
        assert sc[0, 0] == s
        got = q.view(np.int8)[0, 1:].astype(int)
        want = np.array([k if k % 2 == 0 else k + 1 for k in ks])  # even neighbour
        assert (got == want).all()


def test_partial_group_uses_valid_elements_only():
    # K = 200 with 1x128 groups: the second group has 72 valid elements.
    x = _random_bf16((4, 200), 5)
    q, s = oracle.quant_act(x, 128, INT8)
    xv = bits_to_bf16_f64(x)
    for m in range(4):
        amax = np.float32(np.abs(xv[m, 128:200]).max())
        assert s[m, 1] == np.float32(amax) / np.float32(127.0)


# --------------------------------------------------------------------------
# FP8 e4m3
# --------------------------------------------------------------------------

def test_e4m3_layout_and_roundtrip(golden):
    lay = golden["e4m3_layout"]
    assert (lay["sign_bits"], lay["exponent_bits"], lay["mantissa_bits"]) == (1, 4, 3)
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    nan = np.isnan(vals)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    # library routine: torch's float8_e4m3fn -> float32 decode, all 256 codes
    tv = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    assert np.array_equal(vals[~nan], tv[~nan])
    assert vals[0x7E] == 448.0 and vals[0x08] == 2.0 ** -6 and vals[0x01] == 2.0 ** -9
    # encode(decode(c)) == c for every non-NaN code (incl. -0 -> 0x80)
    enc = oracle.e4m3_encode(vals[~nan].astype(np.float32))
    assert np.array_equal(enc, codes[~nan])
    # non-negative codes are strictly increasing
    assert (np.diff(vals[:0x7F]) > 0).all()


def test_e4m3_midpoints_ties_to_even_and_saturation():
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = 0.5 * (vals[:-1] + vals[1:])
    enc = oracle.e4m3_encode(mids.astype(np.float32))
    lo = np.arange(0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(enc.astype(int), want)
    enc_n = oracle.e4m3_encode(-mids.astype(np.float32))
    assert np.array_equal(enc_n.astype(int), want | 0x80)
    big = np.array([448.0, 449.0, 464.0, 480.0, 1e6, 3.4e38], dtype=np.float32)
    assert (oracle.e4m3_encode(big) == 0x7E).all()
    assert (oracle.e4m3_encode(-big) == 0xFE).all()
    assert oracle.e4m3_encode(np.float32(-1e-30)) == 0x80   # underflow keeps sign


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-12, 6, 20000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    ours = oracle.e4m3_encode(x)
    theirs = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_fp8_quant_error_bound():
    x = _random_bf16((16, 256), 12, 3.0)
    q, s = oracle.quant_act(x, 128, FP8)
    xv = bits_to_bf16_f64(x)
    qv = oracle.code_values(q, FP8)
    for m in range(16):
        for g in range(2):
            sl = slice(128 * g, 128 * (g + 1))
            sc = float(s[m, g])
            assert abs(sc * 448.0 - np.abs(xv[m, sl]).max()) <= 2 ** -22 * 448 * sc
            c = xv[m, sl] / sc
            err = np.abs(c - qv[m, sl])
            normal = np.abs(c) >= 2.0 ** -6
            # e4m3 has 3 mantissa bits: half-ulp relative bound 2^-4 (+fp32 slack)
            assert (err[normal] <= 2.0 ** -4 * np.abs(c[normal]) * (1 + 2 ** -18)).all()
            assert (err[~normal] <= 2.0 ** -10 * (1 + 2 ** -18)).all()
            assert np.abs(qv[m, sl]).max() == 448.0


# --------------------------------------------------------------------------
# bf16 rounding helper
# --------------------------------------------------------------------------

def test_bf16_from_double_matches_torch_on_fp32_values():
    rng = np.random.default_rng(2)
    f = (rng.standard_normal(5000) * np.exp(rng.uniform(-30, 30, 5000))).astype(np.float32)
    ours = oracle.bf16_from_f64(f.astype(np.float64))
    theirs = bq_synth.bf16_bits(torch.from_numpy(f).to(torch.bfloat16))
    assert np.array_equal(ours, theirs)


def test_bf16_from_double_exact_ties_go_to_even():
    # midpoints between adjacent bf16 values (exact in fp32): torch's RNE cast decides
    h = np.arange(0x3F00, 0x3F40, dtype=np.uint16)
    lo, hi = oracle.bf16_to_f64(h[:-1]), oracle.bf16_to_f64(h[1:])
    mids = np.concatenate([(lo + hi) / 2, -(lo + hi) / 2])
    ours = oracle.bf16_from_f64(mids)
    theirs = bq_synth.bf16_bits(torch.from_numpy(mids.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(ours, theirs)
    assert (ours[: len(lo)] % 2 == 0).all()


def test_bf16_from_double_is_nearest():
    rng = np.random.default_rng(3)
    v = rng.standard_normal(3000) * np.exp(rng.uniform(-20, 20, 3000))
    h = oracle.bf16_from_f64(v)
    r = oracle.bf16_to_f64(h)
    # neighbours one bf16 step either side
    up = oracle.bf16_to_f64((h.astype(np.int32) + 1).astype(np.uint16))
    dn = oracle.bf16_to_f64((h.astype(np.int32) - 1).astype(np.uint16))
    assert (np.abs(v - r) <= np.abs(v - up)).all()
    assert (np.abs(v - r) <= np.abs(v - dn)).all()


# --------------------------------------------------------------------------
# GEMM: library special cases, one-hot probes, brute force
# --------------------------------------------------------------------------

def _rand_codes(shape, dtype, rng):
    if dtype == INT8:
        return rng.integers(-128, 128, size=shape).astype(np.int8).view(np.uint8)
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C     # avoid NaN codes
    return c


def test_gemm_unit_scales_is_integer_matmul():
    rng = np.random.default_rng(5)
    M, N, K = 7, 9, 300
    qa = _rand_codes((M, K), INT8, rng)
    qw = _rand_codes((N, K), INT8, rng)
    out = oracle.gemm(qa, np.ones((M, 1), np.float32), qw, np.ones((1, 1), np.float32),
                      bn=N, bk=K, dtype=INT8)
    ref = qa.view(np.int8).astype(np.int64) @ qw.view(np.int8).astype(np.int64).T
    assert np.array_equal(out, ref.astype(np.float64))


def test_gemm_single_block_is_scaled_matmul():
    rng = np.random.default_rng(6)
    M, N, K = 5, 8, 64
    qa = _rand_codes((M, K), INT8, rng)
    qw = _rand_codes((N, K), INT8, rng)
    sa = rng.uniform(0.5, 2, (M, 1)).astype(np.float32)
    sw = np.array([[0.375]], np.float32)
    out = oracle.gemm(qa, sa, qw, sw, bn=128, bk=128, dtype=INT8)
    ref = (qa.view(np.int8).astype(np.int64) @ qw.view(np.int8).astype(np.int64).T)
    assert np.allclose(out, ref * sa.astype(np.float64) * 0.375, rtol=1e-15, atol=0)


@pytest.mark.parametrize("dtype", [INT8, FP8])
def test_gemm_one_hot_probes_pin_scale_indexing(dtype):
    # A single nonzero code pair at (m0,k0)/(n0,k0) isolates one scale product:
    # out[m0,n0] = va*vw*sa[m0,k0//bk]*sw[nb(n0),k0//bk], zero elsewhere.
    rng = np.random.default_rng(7)
    M, N, K, bn, bk = 6, 11, 23, 4, 5
    Kb, Nb = cdiv(K, bk), cdiv(N, bn)
    sa = rng.uniform(1, 2, (M, Kb)).astype(np.float32)
    sw = rng.uniform(3, 4, (Nb, Kb)).astype(np.float32)
    one = np.uint8(1) if dtype == INT8 else np.uint8(0x38)      # e4m3 0x38 = 1.0
    for (m0, n0, k0) in [(0, 0, 0), (5, 10, 22), (2, 7, 9), (3, 4, 15), (1, 9, 4)]:
        qa = np.zeros((M, K), np.uint8)
        qw = np.zeros((N, K), np.uint8)
        qa[m0, k0] = one
        qw[n0, k0] = one
        out = oracle.gemm(qa, sa, qw, sw, bn, bk, dtype)
        want = np.zeros((M, N))
        want[m0, n0] = float(sa[m0, k0 // bk]) * float(sw[n0 // bn, k0 // bk])
        assert np.array_equal(out, want)
    # negative code pins the sign
    qa = np.zeros((M, K), np.uint8)
    qw = np.zeros((N, K), np.uint8)
    qa[1, 3] = np.uint8(0xFF) if dtype == INT8 else np.uint8(0xB8)  # -1
    qw[2, 3] = one
    out = oracle.gemm(qa, sa, qw, sw, bn, bk, dtype)
    assert out[1, 2] == -float(sa[1, 0]) * float(sw[0, 0])


@pytest.mark.parametrize("dtype", [INT8, FP8])
def test_gemm_matches_blas_on_dequantised_operands(dtype):
    rng = np.random.default_rng(8)
    M, N, K, bn, bk = 13, 37, 300, 16, 128
    qa = _rand_codes((M, K), dtype, rng)
    qw = _rand_codes((N, K), dtype, rng)
    sa = rng.uniform(0.01, 1, (M, cdiv(K, bk))).astype(np.float32)
    sw = rng.uniform(0.01, 1, (cdiv(N, bn), cdiv(K, bk))).astype(np.float32)
    bias = bq_synth.bf16_bits(torch.randn(N).to(torch.bfloat16))
    out = oracle.gemm(qa, sa, qw, sw, bn, bk, dtype, bias_bf16=bias)
    ad = oracle.code_values(qa, dtype) * np.repeat(sa.astype(np.float64), bk, 1)[:, :K]
    wd = oracle.code_values(qw, dtype) * np.repeat(
        np.repeat(sw.astype(np.float64), bn, 0), bk, 1)[:N, :K]
    ref = ad @ wd.T + oracle.bf16_to_f64(bias)[None, :]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_gemm_brute_force_tiny_all_blockings():
    rng = np.random.default_rng(9)
    for M, N, K in [(1, 1, 1), (2, 3, 5), (8, 8, 8), (3, 7, 6)]:
        for bn, bk in itertools.product((1, 2, 4), (1, 2, 4)):
            for dtype in (INT8, FP8):
                qa = _rand_codes((M, K), dtype, rng)
                qw = _rand_codes((N, K), dtype, rng)
                sa = rng.uniform(0.1, 1, (M, cdiv(K, bk))).astype(np.float32)
                sw = rng.uniform(0.1, 1, (cdiv(N, bn), cdiv(K, bk))).astype(np.float32)
                out = oracle.gemm(qa, sa, qw, sw, bn, bk, dtype)
                for m in range(M):
                    for n in range(N):
                        d = oracle.dequant_dot(qa, sa, qw, sw, bn, bk, dtype, m, n)
                        assert abs(out[m, n] - d) <= 1e-12 * max(1.0, abs(d))


def test_gemm_seam_blocks_gate_and_up_separately():
    # gate rows [0, I) and up rows [I, 2I) take scale rows from separate grids
    rng = np.random.default_rng(10)
    I, K, bn, bk = 5, 8, 4, 8
    w = rng.standard_normal((2 * I, K)).astype(np.float32)
    qw, sw = oracle.quant_weight_gate_up(w, I, bn, bk, INT8)
    assert sw.shape == (4, 1)
    qa = _rand_codes((3, K), INT8, rng)
    sa = np.ones((3, 1), np.float32)
    out = oracle.gemm(qa, sa, qw, sw, bn, bk, INT8, seam=I)
    gate = oracle.gemm(qa, sa, qw[:I], sw[:2], bn, bk, INT8)
    up = oracle.gemm(qa, sa, qw[I:], sw[2:], bn, bk, INT8)
    assert np.array_equal(out, np.concatenate([gate, up], 1))


def test_weight_quant_block_scale_and_bound():
    rng = np.random.default_rng(12)
    N, K, bn, bk = 200, 300, 128, 128
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    q, s = oracle.quant_weight(w, bn, bk, INT8)
    qv = q.view(np.int8).astype(np.float64)
    for i in range(cdiv(N, bn)):
        for j in range(cdiv(K, bk)):
            blk = np.s_[i * bn:(i + 1) * bn, j * bk:(j + 1) * bk]
            assert s[i, j] == np.float32(np.abs(w[blk]).max()) / np.float32(127)
            err = np.abs(w[blk] - qv[blk] * s[i, j])
            assert (err <= s[i, j] * (0.5 + 128 * 2 ** -24)).all()


def test_quantised_linear_close_to_dense():
    """Sanity (loose): the quantised layer approximates the dense bf16 layer."""
    cfg = bq_synth.TINY
    a, w = bq_synth.linear_inputs(cfg)
    ab = bq_synth.bf16_bits(a)
    qa, sa = oracle.quant_act(ab, 128, INT8)
    qw, sw = oracle.quant_weight(w.numpy(), 128, 128, INT8)
    out = oracle.gemm(qa, sa, qw, sw, 128, 128, INT8)
    dense = oracle.bf16_to_f64(ab) @ w.numpy().astype(np.float64).T
    rel = np.linalg.norm(out - dense) / np.linalg.norm(dense)
    assert rel < 0.05


# --------------------------------------------------------------------------
# MoE pieces
# --------------------------------------------------------------------------

def test_moe_permute_matches_stable_sort():
    ids, _ = oracle.moe_route(bq_synth.router_logits(500, 8, 3).numpy(), 2)
    off, perm, inv = oracle.moe_permute(ids, 8)
    flat = ids.reshape(-1)
    assert off[-1] == flat.size
    assert np.array_equal(np.diff(off), np.bincount(flat, minlength=8))
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(inv[perm], np.arange(flat.size))
    with pytest.raises(ValueError):
        oracle.moe_permute(np.array([[0, 8]], np.int32), 8)


def test_moe_permute_empty_experts():
    ids = np.zeros((10, 2), np.int32)
    ids[:, 1] = 5
    off, perm, inv = oracle.moe_permute(ids, 8)
    assert off.tolist() == [0, 10, 10, 10, 10, 10, 20, 20, 20]


def test_silu_mul_matches_torch():
    y = _random_bf16((9, 2 * 70), 13, 3.0)
    h = oracle.silu_mul(y, 70)
    yv = torch.from_numpy(oracle.bf16_to_f64(y))
    ref = torch.nn.functional.silu(yv[:, :70]) * yv[:, 70:]
    assert np.array_equal(h, oracle.bf16_from_f64(ref.numpy()))


def test_combine_identity_experts():
    # permute, identity experts (y = gathered x), weights 1/topk: combine == x
    T, H, topk = 33, 24, 2
    x = _random_bf16((T, H), 14)
    ids, _ = oracle.moe_route(bq_synth.router_logits(T, 8, 4).numpy(), topk)
    off, perm, inv = oracle.moe_permute(ids, 8)
    y = x[perm // topk]
    w = np.full((T, topk), 1.0 / topk, np.float32)
    assert np.array_equal(oracle.moe_combine(y, inv, w), x)


def test_combine_weighted_sum():
    T, H, topk = 7, 10, 2
    rng = np.random.default_rng(15)
    y = _random_bf16((T * topk, H), 16)
    inv = rng.permutation(T * topk).astype(np.int32)
    w = rng.uniform(0, 1, (T, topk)).astype(np.float32)
    out = oracle.moe_combine(y, inv, w)
    yv = oracle.bf16_to_f64(y)
    ref = sum(w[:, j:j + 1].astype(np.float64) * yv[inv.reshape(T, topk)[:, j]]
              for j in range(topk))
    assert np.array_equal(out, oracle.bf16_from_f64(ref))


def test_weight_bytes_arithmetic(golden):
    g = golden["weight_bytes_70b"]
    # 1 byte per INT8 parameter, 2 per FP16 parameter; block scales add 4/(bn*bk)
    assert g["params"] * 2 / 1e9 == g["fp16_GB"]
    assert g["params"] * 1 / 1e9 == g["int8_GB"]
    overhead = 4.0 / (128 * 128)
    assert overhead < 3e-4


# --------------------------------------------------------------------------
# MXFP8: 32-element groups along K, E8M0 scales 2^(E-127), e4m3 codes
# --------------------------------------------------------------------------

def test_mx_quant_worked_example():
    # amax 3 -> floor(log2 3) = 1 -> exponent 1 - 8 = -7 -> E = 120; the
    # scaled values 384, -192, 32 are e4m3 codes 0 1111 100, 1 1110 100, 0 1100 000
    x = np.zeros((1, 32))
    x[0, :3] = [3.0, -1.5, 0.25]
    q, s = oracle.mx_quant(x)
    assert s.tolist() == [[120]]
    assert [int(v) for v in q[0, :3]] == [0x7C, 0xF4, 0x60]
    assert (q[0, 3:] == 0).all()


def test_mx_quant_saturates_and_zero_group():
    x = np.zeros((1, 96))
    x[0, 32] = 500.0                      # floor(log2 500) = 8 -> E = 127, 500 -> 448
    x[0, 33] = -0.5
    q, s = oracle.mx_quant(x)
    assert s.tolist() == [[0, 127, 0]]    # all-zero groups: E = 0, zero codes
    assert q[0, 32] == 0x7E and oracle.e4m3_decode(np.array([q[0, 33]]))[0] == -0.5
    assert (q[0, :32] == 0).all() and (q[0, 64:] == 0).all()


@pytest.mark.parametrize("p", [-130, -126, -40, 0, 7, 8, 9, 60, 126])
def test_mx_quant_scale_exponent_closed_form(p):
    # a group whose amax is 1.5 * 2^p: E = clamp(p - 8, -127, 127) + 127, and
    # every element that is an e4m3 value times 2^(p-8) comes back exactly
    rng = np.random.default_rng(p + 200)
    codes = rng.integers(0, 0x7F, 32).astype(np.uint8)
    vals = oracle.e4m3_decode(codes) * np.where(rng.random(32) < 0.5, -1.0, 1.0)
    vals[0] = 384.0                        # 1.5 * 2^8: sets the amax
    x = np.ldexp(vals, p - 8)[None, :]
    q, s = oracle.mx_quant(x)
    se = max(-127, min(127, p - 8))
    assert int(s[0, 0]) == se + 127
    if se == p - 8:
        assert np.array_equal(oracle.e4m3_decode(q[0]) * 2.0 ** se, x[0])


def test_mx_quant_partial_last_group():
    x = np.zeros((2, 40))
    x[:, 32:] = [[1, 2, 3, 4, 5, 6, 7, 8], [0.5] * 8]   # 8 valid values
    q, s = oracle.mx_quant(x)
    assert s.shape == (2, 2)
    assert s[0, 1] == 3 - 8 + 127 and s[1, 1] == -1 - 8 + 127     # amax 8 and 0.5
    assert np.array_equal(oracle.e4m3_decode(q[0, 32:]) * 2.0 ** (s[0, 1] - 127.0),
                          x[0, 32:])


def test_mx_quant_matches_torch_float8_cast():
    # the element rule is x / 2^se cast once to e4m3 with saturation; torch's
    # float8_e4m3fn cast is round-to-nearest-even; magnitudes past 448 saturate
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(6, 128, generator=g, dtype=torch.float64) * 3.0)
    q, s = oracle.mx_quant(x.numpy())
    scale = torch.from_numpy(np.ldexp(1.0, s.astype(np.int64) - 127)).repeat_interleave(32, 1)
    scaled = (x / scale).float()
    assert scaled.abs().max() > 448       # the saturation is exercised
    ref = scaled.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_mx_gemm_unit_scales_is_a_matmul():
    # E = 127 everywhere (scale 1): out = decoded A @ decoded W^T (BLAS fp64)
    rng = np.random.default_rng(9)
    qa = rng.integers(0, 256, (5, 96)).astype(np.uint8)
    qw = rng.integers(0, 256, (7, 96)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0          # no NaN codes
    qw[(qw & 0x7F) == 0x7F] = 0
    sa = np.full((5, 3), 127, np.uint8)
    sw = np.full((7, 3), 127, np.uint8)
    ref = oracle.e4m3_decode(qa) @ oracle.e4m3_decode(qw).T
    assert np.array_equal(oracle.mx_gemm(qa, sa, qw, sw), ref)


def test_mx_gemm_scales_are_powers_of_two_per_group():
    # brute force: dequantise every element with its own group's scale and
    # contract in a different order (numpy einsum over dequantised matrices)
    rng = np.random.default_rng(11)
    M, N, K = 4, 6, 100
    qa = rng.integers(0, 0x7E, (M, K)).astype(np.uint8) | (rng.integers(0, 2, (M, K)) << 7).astype(np.uint8)
    qw = rng.integers(0, 0x7E, (N, K)).astype(np.uint8)
    sa = rng.integers(110, 140, (M, 4)).astype(np.uint8)
    sw = rng.integers(110, 140, (N, 4)).astype(np.uint8)
    bias = oracle.bf16_from_f64(rng.normal(0, 1, N))
    ka = np.ldexp(1.0, np.repeat(sa.astype(np.int64) - 127, 32, 1)[:, :K])
    kw = np.ldexp(1.0, np.repeat(sw.astype(np.int64) - 127, 32, 1)[:, :K])
    A = oracle.e4m3_decode(qa) * ka
    W = oracle.e4m3_decode(qw) * kw
    ref = np.einsum("mk,nk->mn", A, W) + oracle.bf16_to_f64(bias)[None, :]
    out = oracle.mx_gemm(qa, sa, qw, sw, bias)
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-300)
    # doubling one row's scale (E + 1) doubles that row's contraction exactly
    sa2 = sa.copy()
    sa2[2, 1] += 1
    d = oracle.mx_gemm(qa, sa2, qw, sw) - oracle.mx_gemm(qa, sa, qw, sw)
    part = (A[2, 32:64][None, :] * W[:, 32:64]).sum(axis=1)
    np.testing.assert_allclose(d[2], part, rtol=1e-12)
    assert (d[[0, 1, 3]] == 0).all()


def test_mx_quant_invariants_over_a_wide_range():
    # whatever the magnitude: E never reaches 255 (NaN), no code is NaN
    # (S.1111.111), and each element dequantises to within half an e4m3 step
    # of its value (relative 2^-4 in the normal range, 2^-10 of the scale in
    # the subnormal range), except where it saturates at 448 * scale
    rng = np.random.default_rng(21)
    R, K = 64, 256
    x = rng.normal(0, 1, (R, K)) * np.exp2(rng.integers(-140, 121, (R, 1)))
    x[5, :] = 0.0
    x[6, 40] = -0.0
    q, s = oracle.mx_quant(x)
    assert s.max() <= 254
    assert not np.any((q & 0x7F) == 0x7F)
    scale = np.exp2(np.repeat(s.astype(np.float64) - 127, 32, axis=1))
    deq = oracle.e4m3_decode(q) * scale
    a = np.abs(x)
    sat = a >= 448 * scale
    err = np.abs(deq - x)
    bound = np.maximum(2.0 ** -4 * a, 2.0 ** -10 * scale)
    ok = (err <= bound) | sat
    # elements below fp32's range after scaling are flushed by the float cast
    tiny = a < 2.0 ** -149 * scale
    assert np.all(ok | tiny)
    assert np.all(np.abs(deq[sat]) == 448 * scale[sat])



# --------------------------------------------------------------------------
# MoE routing (top-k of the softmax of router logits)
# --------------------------------------------------------------------------

def test_route_hand_worked():
    # logits 0 and ln 3: probabilities 1/4 and 3/4
    lg = np.array([[0.0, np.log(3.0)]], np.float32)
    ids, w = oracle.moe_route(lg, 2)
    assert ids.tolist() == [[1, 0]]
    np.testing.assert_allclose(w, [[0.75, 0.25]], rtol=1e-6)
    ids, w = oracle.moe_route(lg, 1)
    assert ids.tolist() == [[1]] and w.tolist() == [[1.0]]
    # equal logits: the lower expert index first
    ids, _ = oracle.moe_route(np.array([[2.0, 5.0, 5.0, 5.0, -1.0]], np.float32), 3)
    assert ids.tolist() == [[1, 2, 3]]


def test_route_matches_a_stable_argsort_of_the_fp64_softmax():
    rng = np.random.default_rng(17)
    lg = rng.normal(0, 1, (300, 8)).astype(np.float32)
    lg[:20, 3] = lg[:20, 5]                          # exact ties
    for topk in (1, 2, 3, 8):
        ids, w = oracle.moe_route(lg, topk)
        z = lg.astype(np.float64)
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        order = np.argsort(-p, axis=1, kind="stable")[:, :topk]
        assert np.array_equal(ids, order)
        top = np.take_along_axis(p, order, axis=1)
        np.testing.assert_allclose(w, top / top.sum(axis=1, keepdims=True), rtol=1e-6)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-6)
        assert np.all(np.diff(w, axis=1) <= 0)       # descending weights
