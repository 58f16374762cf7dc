"""Host-only tests of the C ABI: the library loads without a GPU, exports every
symbol include/bq.h declares, and rejects invalid arguments on the host
before touching the device (the block-wise INT8 page's ValueErrors map to
BQ_ERR_INVALID_ARG)."""
import ctypes
import os
import re

import pytest
import torch

import block_scaled_w8a8_b200 as bq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bq.h")


@pytest.fixture(scope="module")
def L():
    from block_scaled_w8a8_b200 import build
    build.build()
    return bq.lib()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_three_core_calls():
    names = header_functions()
    for core in ("bq_quant_act", "bq_gemm", "bq_grouped_gemm"):
        assert core in names


def test_every_header_symbol_is_exported(L):
    for name in header_functions():
        assert hasattr(L, name), f"libbq.so does not export {name}"


def test_binding_declares_exactly_the_header(L):
    assert sorted(bq.DECLS) == header_functions()


def test_version_and_status_strings(L):
    assert bq.version() >= 100
    for s in range(7):
        assert L.bq_status_string(s)
    assert L.bq_status_string(99) == b"unknown status"


def test_block_config_rejections(L):
    # block-wise INT8 page, section 1: three ValueErrors
    bq.check_block_config(True, True, 2, True)
    bq.check_block_config(False, False, 3, False)      # no block size: accepted
    for args, frag in [((True, False, 2, True), "int8-serialised"),
                       ((True, True, 3, True), "2 dimensions"),
                       ((True, True, 2, False), "dynamic")]:
        with pytest.raises(bq.BqError) as ei:
            bq.check_block_config(*args)
        assert ei.value.status == bq.ERR_INVALID_ARG and frag in ei.value.msg


def test_tp_partition_alignment(L):
    # block-wise INT8 page, section 3
    bq.check_tp_partition(2, 8192, 4096, [4096, 4096], 128, 128)
    with pytest.raises(bq.BqError) as ei:
        bq.check_tp_partition(2, 8000, 4000, [4096], 128, 128)
    assert "block_k" in ei.value.msg
    with pytest.raises(bq.BqError) as ei:
        bq.check_tp_partition(1, 4096, 4096, [4096, 100], 128, 128)
    assert "block_n" in ei.value.msg


def _err(L, status):
    assert status != bq.OK
    return status, L.bq_last_error_message().decode()


def test_gemm_argument_errors_on_host(L):
    P = ctypes.c_void_p
    fake = P(0x1000)
    # bad dtype
    st, msg = _err(L, L.bq_gemm(fake, 128, fake, fake, 128, fake, 4, 4, 128, 128, 128, 7, None,
                                fake, 4, None, 0, None))
    assert st == bq.ERR_INVALID_ARG and "dtype" in msg
    # block_n = 0
    st, msg = _err(L, L.bq_gemm(fake, 128, fake, fake, 128, fake, 4, 4, 128, 0, 128, 0, None,
                                fake, 4, None, 0, None))
    assert st == bq.ERR_INVALID_ARG
    # lda < K
    st, msg = _err(L, L.bq_gemm(fake, 100, fake, fake, 128, fake, 4, 4, 128, 128, 128, 0, None,
                                fake, 4, None, 0, None))
    assert st == bq.ERR_INVALID_ARG and "leading" in msg
    # null output
    st, msg = _err(L, L.bq_gemm(fake, 128, fake, fake, 128, fake, 4, 4, 128, 128, 128, 0, None,
                                None, 4, None, 0, None))
    assert st == bq.ERR_INVALID_ARG
    # int32 partial overflow guard
    st, msg = _err(L, L.bq_gemm(fake, 1 << 20, fake, fake, 1 << 20, fake, 4, 4, 1 << 20, 128,
                                1 << 17, 0, None, fake, 4, None, 0, None))
    assert st == bq.ERR_UNSUPPORTED
    # empty problems are no-ops that touch nothing
    assert L.bq_gemm(None, 128, None, None, 128, None, 0, 4, 128, 128, 128, 0, None, None, 4,
                     None, 0, None) == bq.OK


def test_quant_and_moe_argument_errors_on_host(L):
    P = ctypes.c_void_p
    fake = P(0x1000)
    assert L.bq_quant_act(fake, 4, 128, 128, 0, 0, fake, 128, fake, None) == bq.ERR_INVALID_ARG
    assert L.bq_quant_act(fake, 4, 128, 64, 128, 0, fake, 128, fake, None) == bq.ERR_INVALID_ARG
    assert L.bq_quant_act(None, 0, 128, 128, 128, 0, None, 128, None, None) == bq.OK
    assert L.bq_quant_weight(fake, 4, 4, 4, 0, 128, 0, fake, 4, fake, None) == \
        bq.ERR_INVALID_ARG
    assert L.bq_moe_permute(fake, 4, 0, 8, fake, fake, fake, None, 0, None) == \
        bq.ERR_INVALID_ARG
    assert L.bq_moe_permute(fake, 4, 2, 300, fake, fake, fake, None, 0, None) == \
        bq.ERR_UNSUPPORTED
    assert L.bq_grouped_gemm(fake, 128, fake, 8, fake, 2, fake, fake, 64, 128, 128, 128, 65, 0,
                             fake, 64, None, 0, None) == bq.ERR_INVALID_ARG   # seam > N
    assert L.bq_moe_silu_mul_quant(fake, 100, 4, 64, 128, 0, fake, 64, fake, None, None) == \
        bq.ERR_INVALID_ARG                                                     # ldy < 2I
    # fused w13 + SiLU requantisation: ldq < I, then I not a multiple of 128
    assert L.bq_grouped_gemm_silu_quant(fake, 128, fake, 8, fake, 2, fake, fake, 256, 128, 128,
                                        128, 0, fake, 128, fake, None) == bq.ERR_INVALID_ARG
    st, msg = _err(L, L.bq_grouped_gemm_silu_quant(fake, 128, fake, 8, fake, 2, fake, fake, 192,
                                                   128, 128, 128, 0, fake, 192, fake, None))
    assert st == bq.ERR_UNSUPPORTED and "multiple of 128" in msg
    st, msg = _err(L, L.bq_grouped_gemm_silu_quant(fake, 128, fake, 8, fake, 2, fake, fake, 256,
                                                   128, 64, 128, 0, fake, 256, fake, None))
    assert st == bq.ERR_UNSUPPORTED and "block_n = block_k = 128" in msg
    assert L.bq_grouped_gemm_silu_quant(None, 128, None, 0, fake, 2, None, None, 256, 128, 128,
                                        128, 0, None, 256, None, None) == bq.OK   # R = 0
    assert L.bq_moe_combine(fake, 64, fake, fake, 4, 0, 64, fake, 64, None) == \
        bq.ERR_INVALID_ARG
    # MXFP8: K must be a multiple of 128; ld too small; empty problems
    assert L.bq_mx_quant_act(fake, 4, 96, 96, fake, 96, fake, None) == bq.ERR_UNSUPPORTED
    assert L.bq_mx_quant_act(fake, 4, 128, 64, fake, 128, fake, None) == bq.ERR_INVALID_ARG
    assert L.bq_mx_gemm(fake, 256, fake, fake, 256, fake, 4, 8, 200, None, fake, 8, None) == \
        bq.ERR_UNSUPPORTED
    assert L.bq_mx_gemm(None, 256, None, None, 256, None, 0, 8, 256, None, None, 8, None) == bq.OK
    assert bq.mx_scale_bytes(300, 512) == 3 * 4 * 512
    assert L.bq_set_path(9) == bq.ERR_INVALID_ARG
    assert L.bq_set_path(7) == bq.ERR_INVALID_ARG
    assert L.bq_set_path(6) == bq.ERR_INVALID_ARG
    assert L.bq_set_path(bq.PATH_TCGEN05_PAIR) == bq.OK
    assert L.bq_set_path(bq.PATH_AUTO) == bq.OK
    assert L.bq_selftest_bounded_wait(0, None) == bq.ERR_INVALID_ARG


def test_routing_combine_and_partial_argument_errors_on_host(L):
    P = ctypes.c_void_p
    fake = P(0x1000)
    # routing: topk > E, ld < E, E beyond 256, topk beyond 8; T = 0 is a no-op
    assert L.bq_moe_route(fake, 8, 4, 8, 9, fake, fake, None) == bq.ERR_INVALID_ARG
    assert L.bq_moe_route(fake, 4, 4, 8, 2, fake, fake, None) == bq.ERR_INVALID_ARG
    assert L.bq_moe_route(fake, 300, 4, 300, 2, fake, fake, None) == bq.ERR_UNSUPPORTED
    assert L.bq_moe_route(fake, 16, 4, 16, 9, fake, fake, None) == bq.ERR_UNSUPPORTED
    assert L.bq_moe_route(None, 8, 0, 8, 2, None, None, None) == bq.OK
    # the combining w2 GEMM: topk 0, R not T * topk, ld_acc < N, and a path
    # that is not a tensor-core one; R = 0 is a no-op
    args = (fake, 128, fake, 9, fake, 2, fake, fake, 256, 128, 128, 128, 0, fake, fake)
    assert L.bq_grouped_gemm_combine(*args, 0, fake, 256, None) == bq.ERR_INVALID_ARG
    assert L.bq_grouped_gemm_combine(*args, 2, fake, 256, None) == bq.ERR_INVALID_ARG
    args8 = (fake, 128, fake, 8, fake, 2, fake, fake, 256, 128, 128, 128, 0, fake, fake)
    assert L.bq_grouped_gemm_combine(*args8, 2, fake, 128, None) == bq.ERR_INVALID_ARG
    L.bq_set_path(bq.PATH_SIMT)
    try:
        assert L.bq_grouped_gemm_combine(*args8, 2, fake, 256, None) == bq.ERR_UNSUPPORTED
    finally:
        L.bq_set_path(bq.PATH_AUTO)
    assert L.bq_grouped_gemm_combine(None, 128, None, 0, fake, 2, None, None, 256, 128, 128,
                                     128, 0, None, None, 2, None, 256, None) == bq.OK
    # the finishing passes: leading dimensions below N; empty problems
    assert L.bq_moe_combine_finish(fake, 4, 256, 128, fake, 256, None) == bq.ERR_INVALID_ARG
    assert L.bq_moe_combine_finish(None, 0, 256, 256, None, 256, None) == bq.OK
    assert L.bq_finish_bf16(fake, 128, 4, 256, None, fake, 256, None) == bq.ERR_INVALID_ARG
    assert L.bq_finish_bf16(None, 256, 0, 256, None, None, 256, None) == bq.OK
    # the fp32 partial GEMM: an output stride below N
    assert L.bq_gemm_partial(fake, 128, fake, fake, 128, fake, 4, 256, 128, 128, 128, 0,
                             fake, 128, None, 0, None) == bq.ERR_INVALID_ARG


def test_workspace_queries_are_host_only(L):
    assert bq.gemm_workspace_size(64, 4096, 4096) >= 0
    assert bq.linear_workspace_size(64, 4096, 4096) >= 64 * 4096 + 32 * 64 * 4
    assert bq.grouped_gemm_workspace_size(8192, 28672, 4096, 8) >= 0
    with pytest.raises(bq.BqError):
        bq.gemm_workspace_size(-1, 4, 4)


def test_path_override_is_thread_local(L):
    import threading
    bq.set_path(bq.PATH_SIMT)
    seen = []
    t = threading.Thread(target=lambda: seen.append(bq.get_path()))
    t.start()
    t.join()
    assert seen == [bq.PATH_AUTO] and bq.get_path() == bq.PATH_SIMT
    bq.set_path(bq.PATH_AUTO)


def test_binding_refuses_cpu_tensors(L):
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        bq.quant_act(x, 128, bq.INT8, q=torch.zeros(4, 128, dtype=torch.uint8),
                     s=torch.zeros(1, 4))


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "block_scaled_w8a8_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src
                assert "bq_oracle" not in src and "bq_ref_" not in src
