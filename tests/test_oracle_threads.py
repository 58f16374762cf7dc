"""The oracle's OpenMP build (used only to time the CPU baseline on all host
cores) against its plain build: same arithmetic, rows split over threads.

Kept apart from test_oracle.py, whose tests are the pins that every planted
mutant of the oracle must fail (this one compares two builds of one source)."""
import numpy as np

import oracle


def test_threaded_build_computes_the_same_results():
    # the OpenMP build only splits rows over threads (used to time the CPU
    # baseline on all host cores): every output is bit-identical to the
    # single-threaded build's
    rng = np.random.default_rng(31)
    M, N, K = 37, 300, 520
    xb = oracle.bf16_from_f64(rng.normal(0, 1, (M, K)))
    w = rng.normal(0, 0.02, (N, K))
    y = oracle.bf16_from_f64(rng.normal(0, 1, (24, 2 * 96)))
    inv = rng.permutation(24).astype(np.int32)
    tw = rng.random(24).astype(np.float32)
    results = []
    for threads in (1, 4):
        oracle.use_threads(threads)
        try:
            qa, sa = oracle.quant_act(xb, 128, oracle.INT8)
            qw, sw = oracle.quant_weight(w, 128, 128, oracle.INT8)
            o64 = oracle.gemm(qa, sa, qw, sw, 128, 128, oracle.INT8)
            h = oracle.silu_mul(y, 96)
            c = oracle.moe_combine(y, inv, tw.reshape(12, 2))
            mq, ms = oracle.mx_quant(w[:5, :512])
            mo = oracle.mx_gemm(mq, ms, mq, ms)
            results.append((qa, sa, qw, sw, o64, h, c, mo))
        finally:
            oracle.use_threads(1)
    for a, b in zip(*results):
        assert np.array_equal(a, b)
