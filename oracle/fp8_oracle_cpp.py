"""ctypes wrapper of the C++ oracle (``fp8_oracle.cpp``; test infrastructure).

Argument marshalling only: arrays are converted to contiguous numpy buffers
and handed to the C++ functions, which do all of the arithmetic. The API is
the same as the numpy statement in ``fp8_oracle.py`` (same names, arguments
and results), so the two can be checked against each other and against the
same pins.

Inputs may be torch tensors (bf16 widens exactly to fp32) or arrays of
bf16-exact floats.
"""

import ctypes

import numpy as np

from . import build_oracle
from .fp8_oracle import E4M3_MAX, GROUP, bf16_ulp  # noqa: F401  (constants, tolerance ulp)

_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64

_SIGS = {
    "orc_set_threads": (None, [ctypes.c_int]),
    "orc_threads": (ctypes.c_int, []),
    "orc_e4m3_encode": (None, [_P, _I64, _P]),
    "orc_e4m3_decode": (None, [_P, _I64, _P]),
    "orc_quant_act_group128": (None, [_P, _I64, _I64, _P, _P]),
    "orc_quant_weight_block128": (None, [_P, _I64, _I64, _P, _P]),
    "orc_prune24_compress": (None, [_P, _I64, _I64, _P, _P, _P, _P]),
    "orc_decompress24": (None, [_P, _P, _I64, _I64, _P]),
    "orc_block_gemm": (None, [_P, _P, _I64, _P, _P, _I64, _I64, _P, _I64, _P]),
    "orc_sparse24_gemm": (None, [_P, _P, _I64, _P, _P, _P, _I64, _I64, _P, _I64, _P]),
    "orc_gemm_abs_sum": (None, [_P, _P, _I64, _P, _P, _I64, _I64, _P, _I64, _P]),
    "orc_grouped_gemm": (None, [_P, _P, _I64, _P, _P, _P, _I64, _I64, _I64, _P]),
    "orc_swiglu": (None, [_P, _P, _I64, _P]),
    "orc_swiglu_bound": (None, [_P, _P, _P, _P, _I64, _P]),
    "orc_ue8m0_decode": (None, [_P, _I64, _P]),
    "orc_ue8m0_of_amax": (None, [_P, _I64, _P]),
    "orc_quant_act_group128_ue8m0": (None, [_P, _I64, _I64, _P, _P]),
    "orc_quant_weight_block128_ue8m0": (None, [_P, _I64, _I64, _P, _P]),
}


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        h = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def set_threads(n):
    """Worker threads of the C++ oracle (0 = every hardware thread)."""
    lib().orc_set_threads(int(n))


def threads():
    return int(lib().orc_threads())


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _u8(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.uint8))


def _cols(cols, N):
    if cols is None:
        return None, N
    c = np.ascontiguousarray(np.asarray(cols, dtype=np.int64).reshape(-1))
    if c.size and (c.min() < 0 or c.max() >= N):
        raise IndexError("column index out of range")
    return c, c.size


def _check_k(K):
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")


def e4m3_encode(v):
    v = _f32(v)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode(_p(v), v.size, _p(out))
    return out


def e4m3_decode(code):
    c = _u8(code)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode(_p(c), c.size, _p(out))
    return out


def quant_act_group128(x):
    """(qA uint8 [M, K], sA float32 [M, K/128]) of activations x [M, K]."""
    x = _f32(x)
    M, K = x.shape
    _check_k(K)
    qa = np.empty((M, K), np.uint8)
    sa = np.empty((M, K // GROUP), np.float32)
    lib().orc_quant_act_group128(_p(x), M, K, _p(qa), _p(sa))
    return qa, sa


def quant_weight_block128(w):
    """(qW uint8 [N, K], sW float32 [ceil(N/128), K/128]) of weights w [N, K]."""
    w = _f32(w)
    N, K = w.shape
    _check_k(K)
    qw = np.empty((N, K), np.uint8)
    sw = np.empty((-(-N // GROUP), K // GROUP), np.float32)
    lib().orc_quant_weight_block128(_p(w), N, K, _p(qw), _p(sw))
    return qw, sw


def prune24_compress(w):
    """(vals [N, K/2], meta [N, K/8], sW [NB, KB], w_pruned float32 [N, K])."""
    w = _f32(w)
    N, K = w.shape
    _check_k(K)
    vals = np.empty((N, K // 2), np.uint8)
    meta = np.empty((N, K // 8), np.uint8)
    sw = np.empty((-(-N // GROUP), K // GROUP), np.float32)
    wp = np.empty((N, K), np.float32)
    lib().orc_prune24_compress(_p(w), N, K, _p(vals), _p(meta), _p(sw), _p(wp))
    return vals, meta, sw, wp


def decompress24(vals, meta):
    vals, meta = _u8(vals), _u8(meta)
    N, K2 = vals.shape
    q = np.empty((N, 2 * K2), np.uint8)
    lib().orc_decompress24(_p(vals), _p(meta), N, 2 * K2, _p(q))
    return q


def block_gemm(qA, sA, qW, sW, cols=None):
    """Y float64 [M, N or len(cols)] = sum_kb sA sW (qA_kb . qW_kb^T)."""
    qa, qw = _u8(qA), _u8(qW)
    sa = np.ascontiguousarray(np.asarray(sA, np.float32))
    sw = np.ascontiguousarray(np.asarray(sW, np.float32))
    M, K = qa.shape
    N = qw.shape[0]
    c, nc = _cols(cols, N)
    y = np.empty((M, nc), np.float64)
    lib().orc_block_gemm(_p(qa), _p(sa), M, _p(qw), _p(sw), N, K, _p(c), nc, _p(y))
    return y


def sparse24_gemm(qA, sA, vals, meta, sW, cols=None):
    qa, vals, meta = _u8(qA), _u8(vals), _u8(meta)
    sa = np.ascontiguousarray(np.asarray(sA, np.float32))
    sw = np.ascontiguousarray(np.asarray(sW, np.float32))
    M, K = qa.shape
    N = vals.shape[0]
    c, nc = _cols(cols, N)
    y = np.empty((M, nc), np.float64)
    lib().orc_sparse24_gemm(_p(qa), _p(sa), M, _p(vals), _p(meta), _p(sw), N, K, _p(c), nc,
                            _p(y))
    return y


def grouped_gemm(qA, sA, qW, sW, m_indices):
    """Mixture-of-experts GEMM: Y[m] = the block-scaled product of token row m
    with the weights of its expert e = m_indices[m] (qW [E, N, K], sW
    [E, ceil(N/128), K/128]); rows with e outside [0, E) are NaN."""
    qa, qw = _u8(qA), _u8(qW)
    sa = np.ascontiguousarray(np.asarray(sA, np.float32))
    sw = np.ascontiguousarray(np.asarray(sW, np.float32))
    mi = np.ascontiguousarray(np.asarray(m_indices, np.int32))
    M, K = qa.shape
    E, N, _ = qw.shape
    if mi.shape != (M,) or sw.shape != (E, -(-N // GROUP), K // GROUP):
        raise ValueError("grouped_gemm: shape mismatch")
    y = np.empty((M, N), np.float64)
    lib().orc_grouped_gemm(_p(qa), _p(sa), M, _p(qw), _p(sw), _p(mi), E, N, K, _p(y))
    return y


def grouped_gemm_ue8m0(qA, sA8, qW, sW8, m_indices):
    """The grouped GEMM with UE8M0 scale codes."""
    return grouped_gemm(qA, ue8m0_decode(sA8), qW, ue8m0_decode(sW8), m_indices)


def gemm_abs_sum(qA, sA, qW, sW, cols=None):
    """sum_k |a_k * w_k| of the dequantized operands, per output."""
    qa, qw = _u8(qA), _u8(qW)
    sa = np.ascontiguousarray(np.asarray(sA, np.float32))
    sw = np.ascontiguousarray(np.asarray(sW, np.float32))
    M, K = qa.shape
    N = qw.shape[0]
    c, nc = _cols(cols, N)
    out = np.empty((M, nc), np.float64)
    lib().orc_gemm_abs_sum(_p(qa), _p(sa), M, _p(qw), _p(sw), N, K, _p(c), nc, _p(out))
    return out


def gemm_error_bound(qA, sA, qW, sW, cols=None, rel=1e-2):
    """Per-output tolerance rel * sum_k |a_k * w_k| (the test adds one bf16
    ulp of the reference on top)."""
    return rel * gemm_abs_sum(qA, sA, qW, sW, cols=cols)


# ----------------------------------------------------------- UE8M0 scales --

def ue8m0_decode(code):
    """fp32 value 2^(c - 127) of each UE8M0 scale code (NaN for 0xFF)."""
    c = _u8(code)
    out = np.empty(c.shape, np.float32)
    lib().orc_ue8m0_decode(_p(c), c.size, _p(out))
    return out


def ue8m0_of_amax(amax):
    """UE8M0 code of the smallest power of two s with 448 * s >= amax."""
    a = _f32(amax)
    out = np.empty(a.shape, np.uint8)
    lib().orc_ue8m0_of_amax(_p(a), a.size, _p(out))
    return out


def quant_act_group128_ue8m0(x):
    """(qA uint8 [M, K], sA8 uint8 [M, K/128] UE8M0 codes)."""
    x = _f32(x)
    M, K = x.shape
    _check_k(K)
    qa = np.empty((M, K), np.uint8)
    sa8 = np.empty((M, K // GROUP), np.uint8)
    lib().orc_quant_act_group128_ue8m0(_p(x), M, K, _p(qa), _p(sa8))
    return qa, sa8


def quant_weight_block128_ue8m0(w):
    """(qW uint8 [N, K], sW8 uint8 [ceil(N/128), K/128] UE8M0 codes)."""
    w = _f32(w)
    N, K = w.shape
    _check_k(K)
    qw = np.empty((N, K), np.uint8)
    sw8 = np.empty((-(-N // GROUP), K // GROUP), np.uint8)
    lib().orc_quant_weight_block128_ue8m0(_p(w), N, K, _p(qw), _p(sw8))
    return qw, sw8


def block_gemm_ue8m0(qA, sA8, qW, sW8, cols=None):
    """The block-scaled GEMM with UE8M0 scales: the same formula, each scale
    being the power of two its code stands for."""
    return block_gemm(qA, ue8m0_decode(sA8), qW, ue8m0_decode(sW8), cols=cols)


def gemm_error_bound_ue8m0(qA, sA8, qW, sW8, cols=None, rel=1e-2):
    return gemm_error_bound(qA, ue8m0_decode(sA8), qW, ue8m0_decode(sW8), cols=cols, rel=rel)


# ------------------------------------------------------- gated MLP / SwiGLU --

def _f64(a):
    return np.ascontiguousarray(np.asarray(a, np.float64))


def swiglu(g, u):
    """h = silu(g) * u, silu(g) = g / (1 + e^-g), in double."""
    g, u = _f64(g), _f64(u)
    h = np.empty(g.shape, np.float64)
    lib().orc_swiglu(_p(g), _p(u), g.size, _p(h))
    return h


def swiglu_error_bound(g, u, tg, tu):
    """Tolerance of h from the tolerances tg, tu of g and u (|silu'| < 1.1)."""
    g, u, tg, tu = _f64(g), _f64(u), _f64(tg), _f64(tu)
    out = np.empty(g.shape, np.float64)
    lib().orc_swiglu_bound(_p(g), _p(u), _p(tg), _p(tu), g.size, _p(out))
    return out


def gemm_swiglu(qA, sA, qW_gate_up, sW_gate_up, rel=1e-2):
    """The gated MLP's gate+up GEMM followed by SwiGLU: the weights are
    [W_gate; W_up] ([2I, K], scales [2I/128, K/128]); returns (h float64
    [M, I], its tolerance): g, u the block-scaled GEMMs with the gate and up
    rows, h = swiglu(g, u), tolerance swiglu_error_bound with the GEMM bound
    rel * sum |a w| of g and of u."""
    qW = np.asarray(qW_gate_up, np.uint8)
    sW = np.asarray(sW_gate_up, np.float32)
    I = qW.shape[0] // 2
    g = block_gemm(qA, sA, qW[:I], sW[:I // GROUP])
    u = block_gemm(qA, sA, qW[I:], sW[I // GROUP:])
    tg = gemm_error_bound(qA, sA, qW[:I], sW[:I // GROUP], rel=rel)
    tu = gemm_error_bound(qA, sA, qW[I:], sW[I // GROUP:], rel=rel)
    return swiglu(g, u), swiglu_error_bound(g, u, tg, tu)
