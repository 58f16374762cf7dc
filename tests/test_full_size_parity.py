"""Parity at the full workload sizes, on the production (AUTO) paths and the
launch configuration that bench.py times:

  decode linear INT8     M in {1, 8, 32, 64}, N = K = 4096        (bq_linear)
  prefill up-proj INT8   M = 4096, N = 14336, K = 4096           (bq_quant_act + bq_gemm)
  blockwise FP8 linear   M = 2048, N = 4096,  K = 14336          (bq_quant_act + bq_gemm)
  MXFP8 linear           M = 2048, N = 4096,  K = 14336          (bq_mx_quant_act + bq_mx_gemm)
  block-INT8 MoE layer   T = 4096, H = 4096, I = 14336, E = 8, top-2 (bench.MoeLayer:
                         device routing, the unfused stages, and the fused w13 and w2
                         epilogues against them)

Activation codes and scales are compared bit-exactly over the whole tensors;
weight codes on whole 128-row block rows; GEMM outputs on sampled rows (every
column of each sampled row, computed by the oracle); the MoE permutation
exactly; the combine over all tokens.  The oracle always receives the GPU's
own input of the stage it checks (bit-exact where the previous stage is
bit-exact), so each comparison isolates one kernel.

Tolerances are those of the block-scaled linear layer (block-wise INT8 page,
section 4; the GEMM rule in gpu_util.assert_gemm_close)."""
import numpy as np
import pytest
import torch

import bq_synth
import oracle
from gpu_util import (assert_codes_equal, assert_combine_close, assert_gemm_close,
                      assert_scales_equal, bf16_values, host_bits, mx_sf_rows)

pytestmark = pytest.mark.gpu

cdiv = bq_synth.cdiv


def _bq():
    import block_scaled_w8a8_b200 as bq
    bq.set_path(bq.PATH_AUTO)
    return bq


def _sample_rows(M, n, seed):
    rng = np.random.default_rng(seed)
    rows = {0, M - 1, M // 2}
    rows.update(int(r) for r in rng.integers(0, M, n))
    return np.array(sorted(rows))


def _check_weight_block_rows(w_dev, q_dev, s_dev, dtype, block_rows, what):
    """Weight codes and scales of whole 128-row block rows against the oracle's
    offline block quantisation of the same fp32 rows."""
    for br in block_rows:
        r0, r1 = 128 * br, min(128 * (br + 1), w_dev.shape[0])
        w = w_dev[r0:r1].float().cpu().numpy()
        qr, sr = oracle.quant_weight(w, 128, 128, dtype)
        assert_codes_equal(q_dev[r0:r1], qr, f"{what} weight block row {br}")
        sg = s_dev[br:br + 1].cpu().numpy()
        assert np.array_equal(sg.view(np.uint32), sr.view(np.uint32)), \
            f"{what} weight scales of block row {br}"


@pytest.mark.parametrize("cfg", bq_synth.DECODE, ids=lambda c: f"M{c.M}")
def test_decode_linear_full_size(cfg):
    bq = _bq()
    M, N, K = cfg.M, cfg.N, cfg.K
    w = bq_synth.weights(N, K, cfg.w_std, 100, device="cuda")
    qw, sw = bq.quant_weight(w, 128, 128, bq.INT8)
    _check_weight_block_rows(w, qw, sw, bq.INT8, [0, 13, N // 128 - 1], "decode")
    x = bq_synth.activations(M, K, cfg.seed, cfg.n_outliers, cfg.outlier_scale, device="cuda")

    # the activation quantiser alone, bit-exact over the whole tensor
    q, s = bq.quant_act(x, 128, bq.INT8)
    qr, sr = oracle.quant_act(host_bits(x), 128, bq.INT8)
    assert_codes_equal(q, qr, "decode act codes")
    assert_scales_equal(s, sr, "decode act scales")

    # the public layer call as the bench makes it (quantiser + split-K GEMM)
    ws = bq.workspace(bq.linear_workspace_size(M, N, K), torch.device("cuda"))
    out = bq.linear(x, qw, sw, 128, 128, bq.INT8, ws=ws)
    out2 = bq.linear(x, qw, sw, 128, 128, bq.INT8, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, out2), "decode split-K reduction is not deterministic"
    ref = oracle.gemm(qr, sr, qw.cpu().numpy(), sw.cpu().numpy(), 128, 128, bq.INT8)
    assert_gemm_close(out, ref, f"decode M={M}")
    bq.check_device_status()


@pytest.mark.parametrize("cfg", [bq_synth.PREFILL, bq_synth.FP8_LINEAR], ids=lambda c: c.name)
def test_big_linear_full_size(cfg):
    bq = _bq()
    M, N, K, dt = cfg.M, cfg.N, cfg.K, cfg.dtype
    w = bq_synth.weights(N, K, cfg.w_std, cfg.seed, device="cuda")
    qw, sw = bq.quant_weight(w, 128, 128, dt)
    _check_weight_block_rows(w, qw, sw, dt, [0, N // 256, cdiv(N, 128) - 1], cfg.name)
    del w
    x = bq_synth.activations(M, K, cfg.seed, cfg.n_outliers, cfg.outlier_scale, device="cuda")

    q, s = bq.quant_act(x, 128, dt)
    qr, sr = oracle.quant_act(host_bits(x), 128, dt)
    assert_codes_equal(q, qr, f"{cfg.name} act codes")
    assert_scales_equal(s, sr, f"{cfg.name} act scales")

    ws = bq.workspace(bq.gemm_workspace_size(M, N, K, 128, 128, dt), torch.device("cuda"))
    out = bq.gemm(q, s, qw, sw, 128, 128, dt, ws=ws)
    torch.cuda.synchronize()
    bq.check_device_status()
    rows = _sample_rows(M, 6, cfg.seed)
    # rows of both 128-row tile halves and the tile edges
    rows = np.unique(np.concatenate([rows, [127, 128, 255, 256]]))
    ref = oracle.gemm(qr[rows], sr[rows], qw.cpu().numpy(), sw.cpu().numpy(), 128, 128, dt)
    assert_gemm_close(out[torch.from_numpy(rows).cuda()], ref, f"{cfg.name} sampled rows")


def test_mx_linear_full_size():
    """The MXFP8 linear on the FP8 shape: activation and weight codes and scales
    bit-exact over the whole tensors, GEMM outputs on sampled rows."""
    bq = _bq()
    cfg = bq_synth.MX_LINEAR
    M, N, K = cfg.M, cfg.N, cfg.K
    w = bq_synth.weights(N, K, cfg.w_std, cfg.seed, device="cuda")
    qw, sfw = bq.mx_quant_weight(w)
    x = bq_synth.activations(M, K, cfg.seed, cfg.n_outliers, cfg.outlier_scale, device="cuda")
    q, sfa = bq.mx_quant_act(x)
    out = bq.mx_gemm(q, sfa, qw, sfw)
    torch.cuda.synchronize()
    bq.check_device_status()
    qwr, swr = oracle.mx_quant(w.cpu().double().numpy())
    del w
    assert_codes_equal(qw, qwr, "MX weight codes")
    assert np.array_equal(mx_sf_rows(sfw, N, K), swr), "MX weight scales"
    qr, sr = oracle.mx_quant(oracle.bf16_to_f64(host_bits(x)))
    assert_codes_equal(q, qr, "MX activation codes")
    assert np.array_equal(mx_sf_rows(sfa, M, K), sr), "MX activation scales"
    rows = np.unique(np.concatenate([_sample_rows(M, 4, cfg.seed), [127, 128]]))
    ref = oracle.mx_gemm(qr[rows], sr[rows], qwr, swr)
    assert_gemm_close(out[torch.from_numpy(rows).cuda()], ref, "MXFP8 sampled rows")


@pytest.fixture(scope="module")
def moe_layer():
    import bench
    bq = _bq()
    layer = bench.MoeLayer(bq, torch.device("cuda"))
    layer.run(bench.MoeLayer.UNFUSED)
    torch.cuda.synchronize()
    bq.check_device_status()
    # the device routing's ids and weights, on the host, for the stages after it
    layer.ids = layer.ids_d.cpu().numpy()
    layer.tw = layer.tw_d.cpu().numpy()
    yield layer
    del layer
    torch.cuda.empty_cache()


def test_moe_route_full_size(moe_layer):
    """Device routing of the T x E logits: expert ids bit-exact, weights to
    the fp32 rounding of the softmax (the oracle's is fp64)."""
    L = moe_layer
    ids, tw = oracle.moe_route(L.logits.cpu().numpy(), L.cfg.topk)
    assert np.array_equal(L.ids, ids), "routed expert ids differ"
    np.testing.assert_allclose(L.tw, tw, rtol=2e-6, atol=1e-7)


def test_moe_permute_full_size(moe_layer):
    L = moe_layer
    off, perm, inv = oracle.moe_permute(L.ids, L.cfg.E)
    assert np.array_equal(L.off.cpu().numpy(), off)
    assert np.array_equal(L.perm.cpu().numpy(), perm)
    assert np.array_equal(L.inv.cpu().numpy(), inv)
    assert off[-1] == L.cfg.T * L.cfg.topk


def test_moe_gather_quant_full_size(moe_layer):
    L = moe_layer
    perm = L.perm.cpu().numpy()
    xb = host_bits(L.x)[perm // L.cfg.topk]
    qr, sr = oracle.quant_act(xb, 128, L.cfg.dtype)
    assert_codes_equal(L.qa, qr, "gathered codes")
    assert_scales_equal(L.sa, sr, "gathered scales")


def _moe_rows(L):
    """First and last row of every non-empty expert, plus random rows."""
    off = L.off.cpu().numpy()
    rows = set()
    for e in range(L.cfg.E):
        if off[e + 1] > off[e]:
            rows.update((int(off[e]), int(off[e + 1]) - 1))
    rows.update(int(r) for r in np.random.default_rng(3).integers(0, off[-1], 4))
    return np.array(sorted(rows))


def _expert_of(off, r):
    return int(np.searchsorted(off, r, side="right") - 1)


def test_moe_w13_sampled_rows(moe_layer):
    L = moe_layer
    c = L.cfg
    off = L.off.cpu().numpy()
    qa = L.qa.cpu().numpy()
    sa = L.sa.cpu().numpy().T
    rows = _moe_rows(L)
    for e in sorted({_expert_of(off, r) for r in rows}):
        rs = np.array([r for r in rows if _expert_of(off, r) == e])
        ref = oracle.gemm(qa[rs], sa[rs], L.q13[e].cpu().numpy(), L.s13[e].cpu().numpy(),
                          128, 128, c.dtype, seam=c.I)
        assert_gemm_close(L.y13[torch.from_numpy(rs).cuda()], ref, f"w13 expert {e}")


def test_moe_w13_weight_quant_block_rows(moe_layer):
    L = moe_layer
    c = L.cfg
    e = c.E - 1
    w13 = L.w13_fp32(e, torch.device("cuda"))
    nb = cdiv(c.I, 128)
    for half in range(2):
        w = w13[half * c.I:(half + 1) * c.I]
        _check_weight_block_rows(w, L.q13[e, half * c.I:(half + 1) * c.I],
                                 L.s13[e, half * nb:(half + 1) * nb], c.dtype,
                                 [0, nb - 1], f"w13 expert {e} half {half}")


def test_moe_silu_requant_sampled_rows(moe_layer):
    L = moe_layer
    c = L.cfg
    rows = _moe_rows(L)
    y = host_bits(L.y13[torch.from_numpy(rows).cuda()])
    h_ref = oracle.silu_mul(y, c.I)
    # the requantised codes of the GPU's h are unique: recompute h on the GPU
    # for these rows through the same kernel and quantise it with the oracle
    yr = L.y13[torch.from_numpy(rows).cuda()].contiguous()
    q, s, h_gpu = L.bq.moe_silu_mul_quant(yr, c.I, 128, c.dtype, want_h=True)
    hg = host_bits(h_gpu)
    d = np.abs(oracle.bf16_to_f64(hg) - oracle.bf16_to_f64(h_ref))
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(oracle.bf16_to_f64(h_ref)), 2.0 ** -126)))
                  - 7)
    assert (d <= ulp).all(), "silu*up beyond one bf16 ulp"
    qr, sr = oracle.quant_act(hg, 128, c.dtype)
    assert_codes_equal(q, qr, "requant codes")
    assert_scales_equal(s, sr, "requant scales")
    # the layer's own codes for these rows are the same bytes
    assert torch.equal(L.qh[torch.from_numpy(rows).cuda()], q)


def test_moe_w2_sampled_rows(moe_layer):
    L = moe_layer
    c = L.cfg
    off = L.off.cpu().numpy()
    qh = L.qh.cpu().numpy()
    sh = L.sh.cpu().numpy().T
    rows = _moe_rows(L)
    for e in sorted({_expert_of(off, r) for r in rows}):
        rs = np.array([r for r in rows if _expert_of(off, r) == e])
        ref = oracle.gemm(qh[rs], sh[rs], L.q2[e].cpu().numpy(), L.s2[e].cpu().numpy(),
                          128, 128, c.dtype)
        assert_gemm_close(L.y2[torch.from_numpy(rs).cuda()], ref, f"w2 expert {e}")


def test_moe_combine_full_size(moe_layer):
    L = moe_layer
    yb = host_bits(L.y2)
    inv = L.inv.cpu().numpy()
    assert_combine_close(L.out, oracle.moe_combine(yb, inv, L.tw), yb, inv, L.tw)
    assert np.isfinite(bf16_values(L.out)).all()


def test_moe_fused_w2_combine_full_size(moe_layer):
    """The w2 GEMM with the combine in its epilogue (atomic fp32 sums, then
    one bf16 rounding), on the full layer: against the oracle's combine of
    the unfused w2 output (which test_moe_w2_sampled_rows pins), and, top-2
    sums being order-free, bit-exact to the fp32 slot-order sum."""
    L = moe_layer
    c = L.cfg
    acc = torch.zeros(c.T, c.H, dtype=torch.float32, device="cuda")
    L.bq.grouped_gemm_combine(L.qh, L.sh, L.off, L.q2, L.s2, L.perm, L.tw_d, acc, c.dtype)
    out = L.bq.moe_combine_finish(acc)
    torch.cuda.synchronize()
    L.bq.check_device_status()
    yb = host_bits(L.y2)
    inv = L.inv.cpu().numpy()
    assert_combine_close(out, oracle.moe_combine(yb, inv, L.tw), yb, inv, L.tw, "fused combine")
    yv = oracle.bf16_to_f64(yb).astype(np.float32)
    s = np.zeros((c.T, c.H), np.float32)
    for j in range(c.topk):
        s = s + L.tw[:, j:j + 1] * yv[inv.reshape(c.T, c.topk)[:, j]]
    exact = oracle.bf16_to_f64(oracle.bf16_from_f64(s.astype(np.float64)))
    assert np.array_equal(bf16_values(out), exact), "atomic combine differs from the fp32 sum"
    assert not acc.any(), "the finish pass must leave the sums zeroed"


def test_moe_fused_w13_silu_requant_full_size(moe_layer):
    """The fused w13 + silu * up + requantisation call gives, on the full
    layer, the same codes and scales as the unfused calls (whose every stage
    the tests above check against the oracle)."""
    L = moe_layer
    c = L.cfg
    q = torch.empty_like(L.qh)
    s = torch.empty_like(L.sh)
    L.bq.grouped_gemm_silu_quant(L.qa, L.sa, L.off, L.q13, L.s13, c.dtype, q=q, s=s)
    torch.cuda.synchronize()
    L.bq.check_device_status()
    assert torch.equal(q, L.qh), "fused codes differ from the unfused calls"
    assert torch.equal(s.view(torch.int32), L.sh.view(torch.int32)), "fused scales differ"
