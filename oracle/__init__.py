"""CPU oracle for the block-scaled W8A8 linear layer and its MoE variant.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are its only users.  The product path (the
CUDA library and its Python binding) never imports this package, and this
package imports nothing from the product path.

The arithmetic lives in ``bq_oracle.c`` (plain C, fp64, compiled with gcc
without fast-math).  This module compiles it on first use and wraps each
function for numpy arrays.  Layout conventions here are the natural ones:
activation scales are ``[M, Kb]`` and weight scales ``[Nb, Kb]``, row-major.

Sources are cited in ``bq_oracle.c``; in short:
  * block-wise INT8 page ("[SGLang] Block-wise INT8"): weight layout and scale
    grid (structure diagram, section 2), dynamic activation quantisation
    (section 4), MoE gate+up fused weights (section 5), int8 range (design
    rationale item 3);
  * SGLang quantization doc, "GEMM backends for FP4/FP8": blockwise FP8;
  * "LLM quantization overview" page, FP8 section: e4m3 bit layout;
  * MXFP8 (the doc's "MXFP8 dense linear"): the pages name it without
    defining it; the reading is the microscaling format the name refers to
    (32-element groups along K, power-of-two E8M0 scales, e4m3 elements).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

INT8 = 0
FP8 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_bq_oracle.so")
_LIB_OMP_PATH = os.path.join(_HERE, "_bq_oracle_omp.so")
_lock = threading.Lock()
_lib = None
_lib_omp = None
_use_omp = False

# gcc flags: IEEE semantics, no fast-math, no FTZ.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off"]


def _build_one(path: str, extra, force: bool) -> str:
    stale = (not os.path.exists(path)) or os.path.getmtime(path) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = path + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, *extra, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, path)
    return path


def build(force: bool = False) -> str:
    """Compile bq_oracle.c into _bq_oracle.so next to it (if stale), and the
    same source with -fopenmp into _bq_oracle_omp.so: its row loops then run
    on several threads (same arithmetic per element; used only to time the
    CPU baseline on all host cores)."""
    _build_one(_LIB_OMP_PATH, ["-fopenmp"], force)
    return _build_one(_LIB_PATH, [], force)


def use_threads(n: int) -> int:
    """Run the oracle's row loops on n threads (the OpenMP build) when n > 1,
    or on one thread (the plain build) when n <= 1.  Returns the thread count
    now in use.  Results are identical either way: every output element is
    computed by the same code, only rows are split over threads."""
    global _use_omp
    with _lock:
        _use_omp = n > 1
    lib = _load()
    return int(lib.bq_ref_threads(n if n > 1 else 1))


def configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    P, L, I, D = ctypes.c_void_p, ctypes.c_long, ctypes.c_int, ctypes.c_double
    lib.bq_ref_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.bq_ref_bf16_to_double.restype = D
    lib.bq_ref_bf16_from_double.argtypes = [D]
    lib.bq_ref_bf16_from_double.restype = ctypes.c_uint16
    lib.bq_ref_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.bq_ref_e4m3_decode.restype = D
    lib.bq_ref_e4m3_encode.argtypes = [ctypes.c_float]
    lib.bq_ref_e4m3_encode.restype = ctypes.c_uint8
    lib.bq_ref_quant_act.argtypes = [P, L, L, L, L, I, P, L, P]
    lib.bq_ref_quant_act.restype = None
    lib.bq_ref_quant_weight.argtypes = [P, L, L, L, L, L, I, P, L, P]
    lib.bq_ref_quant_weight.restype = None
    lib.bq_ref_gemm_entry.argtypes = [P, L, P, P, L, P, L, L, L, L, L, I, P, L, L]
    lib.bq_ref_gemm_entry.restype = D
    lib.bq_ref_gemm.argtypes = [P, L, P, P, L, P, L, L, L, L, L, L, I, P, P]
    lib.bq_ref_gemm.restype = None
    lib.bq_ref_dequant_dot.argtypes = [P, L, P, P, L, P, L, L, L, L, L, I, L, L]
    lib.bq_ref_dequant_dot.restype = D
    lib.bq_ref_moe_permute.argtypes = [P, L, L, L, P, P, P]
    lib.bq_ref_moe_permute.restype = I
    lib.bq_ref_silu_mul.argtypes = [P, L, L, L, P]
    lib.bq_ref_silu_mul.restype = None
    lib.bq_ref_moe_combine.argtypes = [P, L, P, P, L, L, L, P]
    lib.bq_ref_moe_combine.restype = None
    lib.bq_ref_mx_quant.argtypes = [P, L, L, L, P, L, P]
    lib.bq_ref_mx_quant.restype = None
    lib.bq_ref_mx_gemm.argtypes = [P, L, P, P, L, P, L, L, L, P, P]
    lib.bq_ref_mx_gemm.restype = None
    lib.bq_ref_moe_route.argtypes = [P, L, L, L, L, P, P]
    lib.bq_ref_moe_route.restype = None
    lib.bq_ref_threads.argtypes = [I]
    lib.bq_ref_threads.restype = I
    return lib


def _load():
    global _lib, _lib_omp
    with _lock:
        if _lib is None or _lib_omp is None:
            build()
            _lib = configure(ctypes.CDLL(_LIB_PATH))
            _lib_omp = configure(ctypes.CDLL(_LIB_OMP_PATH))
        return _lib_omp if _use_omp else _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def cdiv(a: int, b: int) -> int:
    """Ceil division, the scale-grid rule of the block-wise INT8 page, section 2."""
    return (a + b - 1) // b


# --------------------------------------------------------------------------
# scalar helpers
# --------------------------------------------------------------------------

def bf16_to_f64(h) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values."""
    h = np.asarray(h, dtype=np.uint16)
    u = h.astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_from_f64(v) -> np.ndarray:
    """Round float64 values once to bf16 (RNE); returns uint16 bit patterns."""
    lib = _load()
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    flat_in, flat_out = v.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = lib.bq_ref_bf16_from_double(float(flat_in[i]))
    return out


def e4m3_decode(c) -> np.ndarray:
    lib = _load()
    c = np.asarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    fi, fo = c.reshape(-1), out.reshape(-1)
    for i in range(fi.size):
        fo[i] = lib.bq_ref_e4m3_decode(int(fi[i]))
    return out


def e4m3_encode(x) -> np.ndarray:
    lib = _load()
    x = np.asarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    fi, fo = x.reshape(-1), out.reshape(-1)
    for i in range(fi.size):
        fo[i] = lib.bq_ref_e4m3_encode(float(fi[i]))
    return out


def code_values(q: np.ndarray, dtype: int) -> np.ndarray:
    """Exact values of stored codes (raw bytes)."""
    q = np.asarray(q, dtype=np.uint8)
    if dtype == INT8:
        return q.view(np.int8).astype(np.float64)
    table = e4m3_decode(np.arange(256, dtype=np.uint8))
    return table[q]


# --------------------------------------------------------------------------
# quantisation
# --------------------------------------------------------------------------

def quant_act(x_bf16: np.ndarray, group_k: int, dtype: int):
    """Dynamic 1 x group_k activation quantisation.

    x_bf16: uint16 [M, K] bf16 bit patterns.  Returns (q uint8 [M, K],
    s float32 [M, Kb])."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    Kb = cdiv(K, group_k)
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, Kb), dtype=np.float32)
    lib.bq_ref_quant_act(_ptr(x), M, K, K, group_k, dtype, _ptr(q), K, _ptr(s))
    return q, s


def quant_weight(w: np.ndarray, bn: int, bk: int, dtype: int):
    """Offline [bn, bk] block quantisation of fp32 W [N, K].

    Returns (q uint8 [N, K], s float32 [ceil(N/bn), ceil(K/bk)])."""
    lib = _load()
    w = _c(w, np.float32)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((cdiv(N, bn), cdiv(K, bk)), dtype=np.float32)
    lib.bq_ref_quant_weight(_ptr(w), N, K, K, bn, bk, dtype, _ptr(q), K, _ptr(s))
    return q, s


def quant_weight_gate_up(w13: np.ndarray, I: int, bn: int, bk: int, dtype: int):
    """Fused gate+up weight [2I, K]: the gate half [0, I) and the up half
    [I, 2I) are blocked separately, so the scale grid has 2*ceil(I/bn) rows
    (block-wise INT8 page, section 5)."""
    q1, s1 = quant_weight(w13[:I], bn, bk, dtype)
    q2, s2 = quant_weight(w13[I:], bn, bk, dtype)
    return np.concatenate([q1, q2], 0), np.concatenate([s1, s2], 0)


# --------------------------------------------------------------------------
# GEMM
# --------------------------------------------------------------------------

def gemm(qa, sa, qw, sw, bn: int, bk: int, dtype: int, bias_bf16=None, seam: int = 0):
    """out64 [M, N] = sum_kb P_kb * sa[m,kb] * sw[nb(n),kb] (+ bias), fp64."""
    lib = _load()
    qa, qw = _c(qa, np.uint8), _c(qw, np.uint8)
    sa, sw = _c(sa, np.float32), _c(sw, np.float32)
    M, K = qa.shape
    N = qw.shape[0]
    bias = None if bias_bf16 is None else _c(bias_bf16, np.uint16)
    out = np.empty((M, N), dtype=np.float64)
    lib.bq_ref_gemm(_ptr(qa), K, _ptr(sa), _ptr(qw), K, _ptr(sw), M, N, K, bn, bk, seam,
                    dtype, _ptr(bias), _ptr(out))
    return out


def gemm_entries(qa, sa, qw, sw, bn: int, bk: int, dtype: int, rows, cols,
                 bias_bf16=None, seam: int = 0):
    """Selected outputs out64[rows[i], cols[i]], computed one by one."""
    lib = _load()
    qa, qw = _c(qa, np.uint8), _c(qw, np.uint8)
    sa, sw = _c(sa, np.float32), _c(sw, np.float32)
    K = qa.shape[1]
    N = qw.shape[0]
    bias = None if bias_bf16 is None else _c(bias_bf16, np.uint16)
    res = np.empty(len(rows), dtype=np.float64)
    for i, (m, n) in enumerate(zip(rows, cols)):
        res[i] = lib.bq_ref_gemm_entry(_ptr(qa), K, _ptr(sa), _ptr(qw), K, _ptr(sw), N, K,
                                       bn, bk, seam, dtype, _ptr(bias), int(m), int(n))
    return res


def dequant_dot(qa, sa, qw, sw, bn: int, bk: int, dtype: int, m: int, n: int,
                seam: int = 0) -> float:
    lib = _load()
    qa, qw = _c(qa, np.uint8), _c(qw, np.uint8)
    sa, sw = _c(sa, np.float32), _c(sw, np.float32)
    K = qa.shape[1]
    N = qw.shape[0]
    return lib.bq_ref_dequant_dot(_ptr(qa), K, _ptr(sa), _ptr(qw), K, _ptr(sw), N, K, bn, bk,
                                  seam, dtype, m, n)


# --------------------------------------------------------------------------
# MoE
# --------------------------------------------------------------------------

def moe_route(logits: np.ndarray, topk: int):
    """Top-k routing of each row of fp32 logits [T, E]: softmax in fp64,
    experts by descending probability (ties to the lower index), the top-k
    probabilities renormalised to sum to one.  Returns (ids int32 [T, topk],
    weights float32 [T, topk])."""
    lib = _load()
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, topk), dtype=np.int32)
    w = np.empty((T, topk), dtype=np.float32)
    lib.bq_ref_moe_route(_ptr(lg), E, T, E, topk, _ptr(ids), _ptr(w))
    return ids, w


def moe_permute(ids: np.ndarray, E: int):
    """Stable expert-major order of the (token, slot) pairs.

    Returns (offsets int32 [E+1], perm int32 [T*topk], inv_perm int32 [T*topk])."""
    lib = _load()
    ids = _c(ids, np.int32)
    T, topk = ids.shape
    R = T * topk
    off = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(R, dtype=np.int32)
    inv = np.empty(R, dtype=np.int32)
    rc = lib.bq_ref_moe_permute(_ptr(ids), T, topk, E, _ptr(off), _ptr(perm), _ptr(inv))
    if rc != 0:
        raise ValueError("expert id out of range")
    return off, perm, inv


def silu_mul(y_bf16: np.ndarray, I: int):
    """h = bf16(silu(gate) * up) with gate = y[:, :I], up = y[:, I:2I]."""
    lib = _load()
    y = _c(y_bf16, np.uint16)
    R = y.shape[0]
    h = np.empty((R, I), dtype=np.uint16)
    lib.bq_ref_silu_mul(_ptr(y), R, I, y.shape[1], _ptr(h))
    return h


def moe_combine(y_bf16: np.ndarray, inv_perm: np.ndarray, w: np.ndarray):
    """out[t] = bf16(sum_j w[t,j] * y[inv_perm[t*topk+j]]), fp64."""
    lib = _load()
    y = _c(y_bf16, np.uint16)
    w = _c(w, np.float32)
    inv = _c(inv_perm, np.int32)
    T, topk = w.shape
    H = y.shape[1]
    out = np.empty((T, H), dtype=np.uint16)
    lib.bq_ref_moe_combine(_ptr(y), H, _ptr(inv), _ptr(w), T, topk, H, _ptr(out))
    return out


def grouped_gemm(qa, sa, offsets, qw_e, sw_e, bn: int, bk: int, dtype: int, seam: int = 0):
    """Per expert e, rows [offsets[e], offsets[e+1]) of qa against qw_e[e]."""
    R = qa.shape[0]
    N = qw_e.shape[1]
    out = np.empty((R, N), dtype=np.float64)
    for e in range(len(offsets) - 1):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            out[r0:r1] = gemm(qa[r0:r1], sa[r0:r1], qw_e[e], sw_e[e], bn, bk, dtype,
                              seam=seam)
    return out


# --------------------------------------------------------------------------
# MXFP8 (32-element groups along K, E8M0 scales, e4m3 codes)
# --------------------------------------------------------------------------

MX_GROUP = 32


def mx_quant(x: np.ndarray):
    """MX quantisation of the rows of x, float values given as a float array
    (bf16 or fp32 inputs converted exactly).  Returns (q uint8 [R, K] e4m3
    codes, s uint8 [R, ceil(K/32)] E8M0 exponents, scale = 2^(s - 127))."""
    lib = _load()
    x = _c(x, np.float64)
    R, K = x.shape
    G = cdiv(K, MX_GROUP)
    q = np.empty((R, K), dtype=np.uint8)
    s = np.empty((R, G), dtype=np.uint8)
    lib.bq_ref_mx_quant(_ptr(x), R, K, K, _ptr(q), K, _ptr(s))
    return q, s


def mx_gemm(qa, sa, qw, sw, bias_bf16=None):
    """out64[m, n] = sum_g 2^(sa-127) 2^(sw-127) sum_{k in g} qa qw (+ bias), fp64."""
    lib = _load()
    qa = _c(qa, np.uint8)
    qw = _c(qw, np.uint8)
    sa = _c(sa, np.uint8)
    sw = _c(sw, np.uint8)
    M, K = qa.shape
    N = qw.shape[0]
    assert sa.shape == (M, cdiv(K, MX_GROUP)) and sw.shape == (N, cdiv(K, MX_GROUP))
    b = None if bias_bf16 is None else _c(bias_bf16, np.uint16)
    out = np.empty((M, N), dtype=np.float64)
    lib.bq_ref_mx_gemm(_ptr(qa), K, _ptr(sa), _ptr(qw), K, _ptr(sw), M, N, K, _ptr(b),
                       _ptr(out))
    return out
