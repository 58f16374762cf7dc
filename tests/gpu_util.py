"""Helpers shared by the GPU parity tests (comparison rules, transfers)."""
import numpy as np
import torch

import bq_synth


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return bq_synth.from_bf16_bits(bits).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return bq_synth.bf16_bits(t)


def bf16_values(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_ulp(a: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at magnitude a (8 significant bits)."""
    a = np.maximum(np.abs(a), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def assert_gemm_close(out: torch.Tensor, ref64: np.ndarray, what: str = ""):
    """The tolerance of the block-scaled linear layer:
      max|d| <= 1e-2 * max|ref| and ||d||_F <= 2e-3 * ||ref||_F  (fp64 reference);
    plus a stronger element-wise rule: every output lies within one bf16 ulp
    of the exact value (the kernel's fp32 sum differs from the exact sum by
    far less than a bf16 ulp, so only the final rounding may differ)."""
    g = bf16_values(out)
    assert g.shape == ref64.shape, (g.shape, ref64.shape)
    d = g - ref64
    amax = np.abs(ref64).max() if ref64.size else 0.0
    if ref64.size == 0:
        return
    assert np.isfinite(g).all(), f"{what}: non-finite outputs"
    assert np.abs(d).max() <= 1e-2 * amax + 1e-30, f"{what}: max|d| {np.abs(d).max()} vs {amax}"
    fro = np.linalg.norm(d) / max(np.linalg.norm(ref64), 1e-30)
    assert fro <= 2e-3, f"{what}: relative Frobenius error {fro:.3e}"
    tol = bf16_ulp(np.maximum(np.abs(g), np.abs(ref64))) + 1e-6 * amax
    bad = np.abs(d) > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} outputs off by more than one bf16 ulp; first at "
            f"{tuple(i)}: gpu {g[tuple(i)]!r} ref {ref64[tuple(i)]!r}")


def assert_codes_equal(q_gpu: torch.Tensor, q_ref: np.ndarray, what: str = ""):
    qg = q_gpu.cpu().numpy()
    if not np.array_equal(qg, q_ref):
        idx = np.argwhere(qg != q_ref)
        i = tuple(idx[0])
        raise AssertionError(f"{what}: {len(idx)} codes differ; first at {i}: "
                             f"gpu {qg[i]:#04x} oracle {q_ref[i]:#04x}")


def assert_scales_equal(s_gpu_kbmajor: torch.Tensor, s_ref_rowmajor: np.ndarray, what=""):
    sg = s_gpu_kbmajor.cpu().numpy().T
    if not np.array_equal(sg.view(np.uint32), s_ref_rowmajor.view(np.uint32)):
        idx = np.argwhere(sg.view(np.uint32) != s_ref_rowmajor.view(np.uint32))
        i = tuple(idx[0])
        raise AssertionError(f"{what}: {len(idx)} scales differ; first at {i}: "
                             f"gpu {sg[i]!r} oracle {s_ref_rowmajor[i]!r}")


def assert_combine_close(out: torch.Tensor, ref_bits: np.ndarray, y_bits: np.ndarray,
                         inv_perm: np.ndarray, w: np.ndarray, what: str = "combine"):
    """The weighted top-k combine is an fp32 sum of fp32 products rounded once
    to bf16; the oracle's is exact before its one rounding.  Where the terms
    nearly cancel, the kernel's fp32 product roundings (each within 2^-24 of
    its term) exceed one bf16 ulp of the small result, so the bound is one
    bf16 ulp plus 2^-22 * sum_j |w_j * y_j| (a factor-4 margin over the two
    fp32 roundings)."""
    import oracle
    g = bf16_values(out)
    r = oracle.bf16_to_f64(ref_bits)
    T, topk = w.shape
    yv = oracle.bf16_to_f64(y_bits)
    mag = np.zeros_like(r)
    for j in range(topk):
        mag += np.abs(w[:, j:j + 1].astype(np.float64) * yv[inv_perm.reshape(T, topk)[:, j]])
    tol = bf16_ulp(np.maximum(np.abs(g), np.abs(r))) + 2.0 ** -22 * mag
    bad = np.abs(g - r) > tol
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} outputs beyond the fp32-sum bound; "
                             f"first at {i}: gpu {g[i]!r} oracle {r[i]!r} tol {tol[i]!r}")


# MXFP8 scale arrays: the library's tensor-core layout <-> the oracle's rows
def _mx_sf_index(R, K):
    r = np.arange(R)[:, None]
    g = np.arange(K // 32)[None, :]
    return (((r // 128) * (K // 128) + g // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32)
            + g % 4)


def mx_sf_rows(sf: torch.Tensor, R: int, K: int) -> np.ndarray:
    """Scale atoms (flat uint8 tensor) -> per-row exponents [R, K/32]."""
    return sf.cpu().numpy().reshape(-1)[_mx_sf_index(R, K)]


def mx_sf_atoms(s_rows: np.ndarray, K: int) -> np.ndarray:
    """Per-row exponents [R, K/32] -> the library's scale atoms (pad rows 127)."""
    R = s_rows.shape[0]
    out = np.full(((R + 127) // 128) * (K // 128) * 512, 127, np.uint8)
    out[_mx_sf_index(R, K)] = s_rows
    return out
