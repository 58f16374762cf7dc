"""Python binding of libbq (block-scaled W8A8 linear layers for B200).

Argument marshalling only: every step runs in the CUDA kernels of libbq.so,
called through its C ABI (include/bq.h).  PyTorch provides device memory and
the current CUDA stream.  There is no CPU fallback: if libbq.so is missing,
or a tensor is not on a CUDA device, the call raises.

Layouts (see include/bq.h):
  activation codes  uint8 [M, K] (int8 two's complement or e4m3 bits)
  activation scales float32 [ceil(K/group_k), M]   (K-block-major)
  weight codes      uint8 [N, K];  weight scales float32 [ceil(N/bn), ceil(K/bk)]
  outputs           bfloat16 [M, N]
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

INT8 = 0
FP8_E4M3 = 1

PATH_AUTO, PATH_SIMT, PATH_TCGEN05, PATH_DECODE, PATH_TCGEN05_1CTA, PATH_TCGEN05_PAIR = \
    0, 1, 2, 3, 4, 5

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, \
    ERR_DEVICE_TIMEOUT = range(7)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbq.so")

_P, _I64, _INT, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SZP = ctypes.POINTER(ctypes.c_size_t)

# name -> (restype, argtypes); mirrors include/bq.h one to one.
DECLS = {
    "bq_version": (_INT, []),
    "bq_status_string": (ctypes.c_char_p, [_INT]),
    "bq_last_error_message": (ctypes.c_char_p, []),
    "bq_set_path": (_INT, [_INT]),
    "bq_get_path": (_INT, []),
    "bq_check_device_status": (_INT, [_P]),
    "bq_selftest_bounded_wait": (_INT, [_I64, _P]),
    "bq_check_block_config": (_INT, [_INT, _INT, _I64, _INT]),
    "bq_check_tp_partition": (_INT, [_I64, _I64, _I64, ctypes.POINTER(ctypes.c_int64), _I64,
                                     _I64, _I64]),
    "bq_quant_act": (_INT, [_P, _I64, _I64, _I64, _I64, _INT, _P, _I64, _P, _P]),
    "bq_quant_weight": (_INT, [_P, _I64, _I64, _I64, _I64, _I64, _INT, _P, _I64, _P, _P]),
    "bq_gemm_workspace_size": (_INT, [_I64, _I64, _I64, _I64, _I64, _INT, _SZP]),
    "bq_gemm": (_INT, [_P, _I64, _P, _P, _I64, _P, _I64, _I64, _I64, _I64, _I64, _INT, _P, _P,
                       _I64, _P, _SZ, _P]),
    "bq_gemm_partial": (_INT, [_P, _I64, _P, _P, _I64, _P, _I64, _I64, _I64, _I64, _I64, _INT,
                               _P, _I64, _P, _SZ, _P]),
    "bq_finish_bf16": (_INT, [_P, _I64, _I64, _I64, _P, _P, _I64, _P]),
    "bq_gemm_decode_noalloc": (_INT, [_P, _I64, _P, _P, _I64, _P, _I64, _I64, _I64, _I64, _I64,
                                      _INT, _P, _P, _I64, _P]),
    "bq_linear_workspace_size": (_INT, [_I64, _I64, _I64, _I64, _I64, _INT, _SZP]),
    "bq_linear": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _P, _I64, _I64, _I64, _INT, _P, _P,
                         _I64, _P, _SZ, _P]),
    "bq_moe_route": (_INT, [_P, _I64, _I64, _I64, _I64, _P, _P, _P]),
    "bq_moe_permute_workspace_size": (_INT, [_I64, _I64, _I64, _SZP]),
    "bq_moe_permute": (_INT, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    "bq_moe_quant_gather": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _I64, _INT, _P, _I64, _P,
                                   _P]),
    "bq_grouped_gemm_workspace_size": (_INT, [_I64, _I64, _I64, _I64, _I64, _I64, _INT, _SZP]),
    "bq_grouped_gemm": (_INT, [_P, _I64, _P, _I64, _P, _I64, _P, _P, _I64, _I64, _I64, _I64,
                               _I64, _INT, _P, _I64, _P, _SZ, _P]),
    "bq_grouped_gemm_silu_quant": (_INT, [_P, _I64, _P, _I64, _P, _I64, _P, _P, _I64, _I64,
                                          _I64, _I64, _INT, _P, _I64, _P, _P]),
    "bq_grouped_gemm_combine": (_INT, [_P, _I64, _P, _I64, _P, _I64, _P, _P, _I64, _I64, _I64,
                                       _I64, _INT, _P, _P, _I64, _P, _I64, _P]),
    "bq_moe_combine_finish": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _P]),
    "bq_moe_silu_mul_quant": (_INT, [_P, _I64, _I64, _I64, _I64, _INT, _P, _I64, _P, _P, _P]),
    "bq_mx_scale_bytes": (_INT, [_I64, _I64, _SZP]),
    "bq_mx_quant_act": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "bq_mx_quant_weight": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "bq_mx_gemm": (_INT, [_P, _I64, _P, _P, _I64, _P, _I64, _I64, _I64, _P, _P, _I64, _P]),
    "bq_mx_linear_workspace_size": (_INT, [_I64, _I64, _SZP]),
    "bq_mx_linear": (_INT, [_P, _I64, _I64, _I64, _P, _I64, _P, _I64, _P, _P, _I64, _P, _SZ,
                            _P]),
    "bq_moe_combine": (_INT, [_P, _I64, _P, _P, _I64, _I64, _I64, _P, _I64, _P]),
}

_lib = None
_lock = threading.Lock()


class BqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libbq status {status}: {msg}")
        self.status = status
        self.msg = msg


def lib() -> ctypes.CDLL:
    """The loaded libbq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m block_scaled_w8a8_b200.build` (nvcc, sm_100a)")
                L = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in DECLS.items():
                    fn = getattr(L, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = L
    return _lib


def _check(status: int):
    if status != OK:
        msg = lib().bq_last_error_message().decode(errors="replace")
        raise BqError(status, msg)


def _cuda(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (libbq has no CPU path)")
    return t.data_ptr()


def _opt(t, name):
    return None if t is None else _cuda(t, name)


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0)


def _stream(dev=None) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


# ---- workspaces (zero-filled device buffers, cached per device) -----------

_ws_cache: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor | None:
    """A zero-filled device buffer of at least nbytes, reused across calls.
    libbq leaves a workspace zero-filled after every successful call."""
    if nbytes == 0:
        return None
    dev = torch.device(device)
    key = (dev.type, dev.index)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
        _ws_cache[key] = buf
    return buf


# ---- thin wrappers ---------------------------------------------------------

def version() -> int:
    return lib().bq_version()


def set_path(path: int):
    _check(lib().bq_set_path(path))


def get_path() -> int:
    return lib().bq_get_path()


def check_device_status(device=None):
    _check(lib().bq_check_device_status(_P(_stream(device))))


def selftest_bounded_wait(spin_limit: int, device=None):
    _check(lib().bq_selftest_bounded_wait(spin_limit, _P(_stream(device))))


def check_block_config(has_block_size: bool, checkpoint_int8_serialized: bool,
                       n_block_dims: int, dynamic_activation: bool):
    _check(lib().bq_check_block_config(int(has_block_size), int(checkpoint_int8_serialized),
                                       n_block_dims, int(dynamic_activation)))


def check_tp_partition(tp_size, input_size, input_size_per_partition, output_partition_sizes,
                       block_n, block_k):
    arr = (ctypes.c_int64 * len(output_partition_sizes))(*output_partition_sizes)
    _check(lib().bq_check_tp_partition(tp_size, input_size, input_size_per_partition, arr,
                                       len(output_partition_sizes), block_n, block_k))


def quant_act(x: torch.Tensor, group_k: int = 128, dtype: int = INT8, q=None, s=None):
    """Dynamic 1 x group_k quantisation of bf16 x [M, K] -> (q [M,K], s [Kb, M])."""
    assert x.dtype == torch.bfloat16
    M, K = x.shape
    if q is None:
        q = torch.empty(M, K, dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.empty(cdiv(K, group_k), M, dtype=torch.float32, device=x.device)
    _check(lib().bq_quant_act(_cuda(x, "x"), M, K, _ld(x), group_k, dtype, _cuda(q, "q"),
                              _ld(q), _cuda(s, "s"), _P(_stream(x.device))))
    return q, s


def quant_weight(w: torch.Tensor, block_n: int = 128, block_k: int = 128, dtype: int = INT8):
    """Offline block quantisation of fp32 W [N, K] -> (q [N, K], s [Nb, Kb])."""
    assert w.dtype == torch.float32
    N, K = w.shape
    q = torch.empty(N, K, dtype=torch.uint8, device=w.device)
    s = torch.empty(cdiv(N, block_n), cdiv(K, block_k), dtype=torch.float32, device=w.device)
    _check(lib().bq_quant_weight(_cuda(w, "w"), N, K, _ld(w), block_n, block_k, dtype,
                                 _cuda(q, "q"), _ld(q), _cuda(s, "s"), _P(_stream(w.device))))
    return q, s


def gemm_workspace_size(M, N, K, block_n=128, block_k=128, dtype=INT8) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().bq_gemm_workspace_size(M, N, K, block_n, block_k, dtype, ctypes.byref(n)))
    return n.value


def gemm(qa, sa, qw, sw, block_n=128, block_k=128, dtype=INT8, bias=None, out=None, ws=None):
    """Block-scaled GEMM of quantised operands -> bf16 [M, N]."""
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qa.device)
    nbytes = gemm_workspace_size(M, N, K, block_n, block_k, dtype)
    if ws is None:
        ws = workspace(nbytes, qa.device)
    _check(lib().bq_gemm(_cuda(qa, "qa"), _ld(qa), _cuda(sa, "sa"), _cuda(qw, "qw"), _ld(qw),
                         _cuda(sw, "sw"), M, N, K, block_n, block_k, dtype,
                         _opt(bias, "bias"), _cuda(out, "out"), _ld(out), _opt(ws, "ws"),
                         0 if ws is None else ws.numel(), _P(_stream(qa.device))))
    return out


def gemm_partial(qa, sa, qw, sw, block_n=128, block_k=128, dtype=INT8, out=None, ws=None):
    """Unrounded fp32 sum over the K-blocks of qa/qw (no bias): the per-GPU
    part of a K-sharded linear layer, finished by finish_bf16."""
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32, device=qa.device)
    nbytes = gemm_workspace_size(M, N, K, block_n, block_k, dtype)
    if ws is None:
        ws = workspace(nbytes, qa.device)
    _check(lib().bq_gemm_partial(_cuda(qa, "qa"), _ld(qa), _cuda(sa, "sa"), _cuda(qw, "qw"),
                                 _ld(qw), _cuda(sw, "sw"), M, N, K, block_n, block_k, dtype,
                                 _cuda(out, "out"), _ld(out), _opt(ws, "ws"),
                                 0 if ws is None else ws.numel(), _P(_stream(qa.device))))
    return out


def finish_bf16(part, bias=None, out=None):
    """bf16(part + bias), one rounding."""
    M, N = part.shape
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=part.device)
    _check(lib().bq_finish_bf16(_cuda(part, "part"), _ld(part), M, N, _opt(bias, "bias"),
                                _cuda(out, "out"), _ld(out), _P(_stream(part.device))))
    return out


def gemm_decode_noalloc(qa, sa, qw, sw, block_n=128, block_k=128, dtype=INT8, bias=None,
                        out=None):
    """bq_gemm on the decode kernel with the library's fixed scratch: no
    workspace, no device allocation inside the call (for callers that cannot
    allocate).  Overlapping calls race on the shared scratch."""
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qa.device)
    _check(lib().bq_gemm_decode_noalloc(_cuda(qa, "qa"), _ld(qa), _cuda(sa, "sa"),
                                        _cuda(qw, "qw"), _ld(qw), _cuda(sw, "sw"), M, N, K,
                                        block_n, block_k, dtype, _opt(bias, "bias"),
                                        _cuda(out, "out"), _ld(out), _P(_stream(qa.device))))
    return out


def linear_workspace_size(M, N, K, block_n=128, block_k=128, dtype=INT8) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().bq_linear_workspace_size(M, N, K, block_n, block_k, dtype, ctypes.byref(n)))
    return n.value


def linear(x, qw, sw, block_n=128, block_k=128, dtype=INT8, bias=None, out=None, ws=None):
    """apply_w8a8_block_int8_linear(x, W, [bn, bk], sw, input_scale=None, bias)."""
    M, K = x.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    nbytes = linear_workspace_size(M, N, K, block_n, block_k, dtype)
    if ws is None:
        ws = workspace(nbytes, x.device)
    _check(lib().bq_linear(_cuda(x, "x"), _ld(x), M, K, _cuda(qw, "qw"), _ld(qw),
                           _cuda(sw, "sw"), N, block_n, block_k, dtype, _opt(bias, "bias"),
                           _cuda(out, "out"), _ld(out), _opt(ws, "ws"),
                           0 if ws is None else ws.numel(), _P(_stream(x.device))))
    return out


def moe_route(logits: torch.Tensor, topk: int, ids=None, weights=None):
    """Top-k experts of fp32 router logits [T, E] and their renormalised
    softmax weights -> (ids int32 [T, topk], weights float32 [T, topk])."""
    assert logits.dtype == torch.float32
    T, E = logits.shape
    if ids is None:
        ids = torch.empty(T, topk, dtype=torch.int32, device=logits.device)
    if weights is None:
        weights = torch.empty(T, topk, dtype=torch.float32, device=logits.device)
    _check(lib().bq_moe_route(_cuda(logits, "logits"), _ld(logits), T, E, topk,
                              _cuda(ids, "ids"), _cuda(weights, "weights"),
                              _P(_stream(logits.device))))
    return ids, weights


def moe_permute(topk_ids: torch.Tensor, E: int):
    """(expert_offsets [E+1], perm [T*topk], inv_perm [T*topk]), all int32."""
    T, topk = topk_ids.shape
    dev = topk_ids.device
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * topk, dtype=torch.int32, device=dev)
    inv = torch.empty(T * topk, dtype=torch.int32, device=dev)
    _check(lib().bq_moe_permute(_cuda(topk_ids, "topk_ids"), T, topk, E, _cuda(off, "off"),
                                _cuda(perm, "perm"), _cuda(inv, "inv"), None, 0,
                                _P(_stream(dev))))
    return off, perm, inv


def moe_quant_gather(x, perm, topk, group_k=128, dtype=INT8, q=None, s=None):
    T, H = x.shape
    R = T * topk
    if q is None:
        q = torch.empty(R, H, dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.empty(cdiv(H, group_k), R, dtype=torch.float32, device=x.device)
    _check(lib().bq_moe_quant_gather(_cuda(x, "x"), T, H, _ld(x), _cuda(perm, "perm"), topk,
                                     group_k, dtype, _cuda(q, "q"), _ld(q), _cuda(s, "s"),
                                     _P(_stream(x.device))))
    return q, s


def grouped_gemm_workspace_size(R, N, K, E, block_n=128, block_k=128, dtype=INT8) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().bq_grouped_gemm_workspace_size(R, N, K, E, block_n, block_k, dtype,
                                                ctypes.byref(n)))
    return n.value


def grouped_gemm(qa, sa, offsets, qw, sw, block_n=128, block_k=128, n_seam=0, dtype=INT8,
                 out=None, ws=None):
    """Per-expert block-scaled GEMM; qw [E, N, K] codes, sw [E, Nbs, Kb]."""
    R, K = qa.shape
    E, N, _ = qw.shape
    if out is None:
        out = torch.empty(R, N, dtype=torch.bfloat16, device=qa.device)
    nbytes = grouped_gemm_workspace_size(R, N, K, E, block_n, block_k, dtype)
    if ws is None:
        ws = workspace(nbytes, qa.device)
    assert qw.is_contiguous() and sw.is_contiguous()
    _check(lib().bq_grouped_gemm(_cuda(qa, "qa"), _ld(qa), _cuda(sa, "sa"), R,
                                 _cuda(offsets, "offsets"), E, _cuda(qw, "qw"), _cuda(sw, "sw"),
                                 N, K, block_n, block_k, n_seam, dtype, _cuda(out, "out"),
                                 _ld(out), _opt(ws, "ws"), 0 if ws is None else ws.numel(),
                                 _P(_stream(qa.device))))
    return out


def grouped_gemm_silu_quant(qa, sa, offsets, qw13, sw13, dtype=INT8, q=None, s=None):
    """w13 grouped GEMM fused with silu(gate) * up and its 1 x 128 requantisation.

    qw13 [E, 2I, K] codes (gate rows then up rows), sw13 [E, 2I/128, Kb].
    Returns the codes q [R, I] and scales s [I/128, R] of h; raises BqError
    (ERR_UNSUPPORTED) where only the unfused calls apply.
    """
    R, K = qa.shape
    E, N2, _ = qw13.shape
    I = N2 // 2
    if q is None:
        q = torch.empty(R, I, dtype=torch.uint8, device=qa.device)
    if s is None:
        s = torch.empty(cdiv(I, 128), R, dtype=torch.float32, device=qa.device)
    assert qw13.is_contiguous() and sw13.is_contiguous()
    _check(lib().bq_grouped_gemm_silu_quant(_cuda(qa, "qa"), _ld(qa), _cuda(sa, "sa"), R,
                                            _cuda(offsets, "offsets"), E, _cuda(qw13, "qw13"),
                                            _cuda(sw13, "sw13"), I, K, 128, 128, dtype,
                                            _cuda(q, "q"), _ld(q), _cuda(s, "s"),
                                            _P(_stream(qa.device))))
    return q, s


def grouped_gemm_combine(qh, sh, offsets, qw2, sw2, perm, topk_w, acc, dtype=INT8):
    """w2 grouped GEMM fused with the weighted top-k combine: adds
    topk_w[perm[r]] * bf16(row r of the GEMM) into fp32 acc [T, N] row
    perm[r] // topk.  acc must hold zeros on entry; moe_combine_finish rounds
    it to bf16 and zeroes it."""
    R, K = qh.shape
    E, N, _ = qw2.shape
    T, topk = topk_w.shape
    assert acc.dtype == torch.float32 and acc.shape[0] == T and acc.shape[1] >= N
    assert qw2.is_contiguous() and sw2.is_contiguous() and topk_w.is_contiguous()
    _check(lib().bq_grouped_gemm_combine(_cuda(qh, "qh"), _ld(qh), _cuda(sh, "sh"), R,
                                         _cuda(offsets, "offsets"), E, _cuda(qw2, "qw2"),
                                         _cuda(sw2, "sw2"), N, K, 128, 128, dtype,
                                         _cuda(perm, "perm"), _cuda(topk_w, "topk_w"), topk,
                                         _cuda(acc, "acc"), _ld(acc), _P(_stream(qh.device))))
    return acc


def moe_combine_finish(acc, out=None):
    """bf16(acc) into out [T, N]; acc is zeroed."""
    T, N = acc.shape
    if out is None:
        out = torch.empty(T, N, dtype=torch.bfloat16, device=acc.device)
    _check(lib().bq_moe_combine_finish(_cuda(acc, "acc"), T, N, _ld(acc), _cuda(out, "out"),
                                       _ld(out), _P(_stream(acc.device))))
    return out


def mx_scale_bytes(R, K):
    n = ctypes.c_size_t(0)
    _check(lib().bq_mx_scale_bytes(R, K, ctypes.byref(n)))
    return n.value


def _mx_quant(fn, x, q=None, sf=None):
    R, K = x.shape
    if q is None:
        q = torch.empty(R, K, dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(mx_scale_bytes(R, K), dtype=torch.uint8, device=x.device)
    _check(fn(_cuda(x, "x"), R, K, _ld(x), _cuda(q, "q"), _ld(q), _cuda(sf, "sf"),
              _P(_stream(x.device))))
    return q, sf


def mx_quant_act(x, q=None, sf=None):
    """MXFP8 quantisation of bf16 activations [M, K]: (e4m3 codes, scale atoms)."""
    assert x.dtype == torch.bfloat16
    return _mx_quant(lib().bq_mx_quant_act, x, q, sf)


def mx_quant_weight(w, q=None, sf=None):
    """MXFP8 quantisation of fp32 weights [N, K]: (e4m3 codes, scale atoms)."""
    assert w.dtype == torch.float32
    return _mx_quant(lib().bq_mx_quant_weight, w, q, sf)


def mx_gemm(qa, sfa, qw, sfw, bias=None, out=None):
    """MXFP8 linear: bf16 out [M, N] from e4m3 codes and their scale atoms."""
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qa.device)
    _check(lib().bq_mx_gemm(_cuda(qa, "qa"), _ld(qa), _cuda(sfa, "sfa"), _cuda(qw, "qw"),
                            _ld(qw), _cuda(sfw, "sfw"), M, N, K, _opt(bias, "bias"),
                            _cuda(out, "out"), _ld(out), _P(_stream(qa.device))))
    return out


def mx_linear_workspace_size(M, K):
    n = ctypes.c_size_t(0)
    _check(lib().bq_mx_linear_workspace_size(M, K, ctypes.byref(n)))
    return n.value


def mx_linear(x, qw, sfw, bias=None, out=None, ws=None):
    """MXFP8 dense linear: bf16 x [M, K] -> bf16 [M, N] (activation MX
    quantisation into the workspace, then the block-scaled MMA GEMM)."""
    assert x.dtype == torch.bfloat16
    M, K = x.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    nbytes = mx_linear_workspace_size(M, K)
    if ws is None:
        ws = workspace(nbytes, x.device)
    _check(lib().bq_mx_linear(_cuda(x, "x"), _ld(x), M, K, _cuda(qw, "qw"), _ld(qw),
                              _cuda(sfw, "sfw"), N, _opt(bias, "bias"), _cuda(out, "out"),
                              _ld(out), _opt(ws, "ws"), 0 if ws is None else ws.numel(),
                              _P(_stream(x.device))))
    return out


def moe_silu_mul_quant(y, I, group_k=128, dtype=INT8, want_h=False, q=None, s=None):
    R = y.shape[0]
    if q is None:
        q = torch.empty(R, I, dtype=torch.uint8, device=y.device)
    if s is None:
        s = torch.empty(cdiv(I, group_k), R, dtype=torch.float32, device=y.device)
    h = torch.empty(R, I, dtype=torch.bfloat16, device=y.device) if want_h else None
    _check(lib().bq_moe_silu_mul_quant(_cuda(y, "y"), _ld(y), R, I, group_k, dtype,
                                       _cuda(q, "q"), _ld(q), _cuda(s, "s"), _opt(h, "h"),
                                       _P(_stream(y.device))))
    return (q, s, h) if want_h else (q, s)


def moe_combine(y, inv_perm, topk_w, out=None):
    T, topk = topk_w.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y.device)
    _check(lib().bq_moe_combine(_cuda(y, "y"), _ld(y), _cuda(inv_perm, "inv_perm"),
                                _cuda(topk_w, "topk_w"), T, topk, H, _cuda(out, "out"),
                                _ld(out), _P(_stream(y.device))))
    return out
