"""Thin ctypes binding of libfp8bs (the C ABI declared in include/fp8bs.h).

Argument marshalling only: torch tensors supply device pointers and the
current CUDA stream; every step of the computation runs in the library's
kernels. The library is loaded from this package directory and there is no
fallback: if it is missing, or the device is not a B200, calls raise.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8bs.so")

FP8BS_OK = 0
STATUS = {
    0: "FP8BS_OK", 1: "FP8BS_ERR_NULL", 2: "FP8BS_ERR_SHAPE", 3: "FP8BS_ERR_ALIGN",
    4: "FP8BS_ERR_WORKSPACE", 5: "FP8BS_ERR_CUDA", 6: "FP8BS_ERR_DEVICE_TIMEOUT",
    7: "FP8BS_ERR_ARCH", 8: "FP8BS_ERR_SCRATCH_LIMIT",
}

# name -> (restype, argtypes), mirroring include/fp8bs.h
_P, _I64, _SZ, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "fp8_quant_act_group128": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_quant_weight_block128": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "prune24_compress": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "fp8_block_gemm": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "fp8_block_gemm_quant": (_I, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "fp8_sparse24_gemm": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "fp8_quant_act_group128_ue8m0": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_quant_weight_block128_ue8m0": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "fp8_block_gemm_ue8m0": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "fp8_grouped_gemm": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "fp8_grouped_gemm_ue8m0": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "fp8_gemm_swiglu_quant": (_I, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "fp8_gemm_swiglu_quant_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "fp8bs_swiglu_workspace_bytes": (_SZ, [_I64, _I64]),
    "fp8_gather_columns": (_I, [_P, _I64, _I64, _I64, _P, _P]),
    "fp8bs_gemm_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I]),
    "fp8bs_get_device_error": (_I, [_P]),
    "fp8bs_set_wait_limit": (None, [ctypes.c_longlong]),
    "fp8bs_status_string": (ctypes.c_char_p, [_I]),
    "fp8bs_version": (_I, []),
}

_lib = None


class Fp8bsError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = lib().fp8bs_status_string(status).decode()
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({msg})")


def lib():
    """Load libfp8bs.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m fp8_block_scaled_group128_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, ref):
    if stream is None:
        stream = torch.cuda.current_stream(ref.device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, st):
    if st != FP8BS_OK:
        raise Fp8bsError(fn, st)


def _dev(t, dtype, shape, name):
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def fp8_quant_act_group128(x, qa=None, sa=None, stream=None):
    """x bf16 [M, K] -> (qa uint8 [M, K] E4M3 codes, sa fp32 [M, K/128])."""
    M, K = x.shape
    _dev(x, torch.bfloat16, (M, K), "x")
    qa = _empty((M, K), torch.uint8, x.device) if qa is None else qa
    sa = _empty((M, K // 128), torch.float32, x.device) if sa is None else sa
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa, torch.float32, (M, K // 128), "sa")
    _check("fp8_quant_act_group128",
           lib().fp8_quant_act_group128(_ptr(x), M, K, _ptr(qa), _ptr(sa), _stream(stream, x)))
    return qa, sa


def fp8_quant_weight_block128(w, qw=None, sw=None, stream=None):
    """w bf16 [N, K] -> (qw uint8 [N, K], sw fp32 [ceil(N/128), K/128])."""
    N, K = w.shape
    _dev(w, torch.bfloat16, (N, K), "w")
    NB = -(-N // 128)
    qw = _empty((N, K), torch.uint8, w.device) if qw is None else qw
    sw = _empty((NB, K // 128), torch.float32, w.device) if sw is None else sw
    _dev(qw, torch.uint8, (N, K), "qw")
    _dev(sw, torch.float32, (NB, K // 128), "sw")
    _check("fp8_quant_weight_block128",
           lib().fp8_quant_weight_block128(_ptr(w), N, K, _ptr(qw), _ptr(sw), _stream(stream, w)))
    return qw, sw


def prune24_compress(w, vals=None, meta=None, sw=None, w_pruned=None, want_pruned=False,
                     stream=None):
    """w bf16 [N, K] -> (vals uint8 [N, K/2], meta uint8 [N, K/8], sw fp32 [NB, KB],
    w_pruned bf16 [N, K] or None)."""
    N, K = w.shape
    _dev(w, torch.bfloat16, (N, K), "w")
    NB = -(-N // 128)
    vals = _empty((N, K // 2), torch.uint8, w.device) if vals is None else vals
    meta = _empty((N, K // 8), torch.uint8, w.device) if meta is None else meta
    sw = _empty((NB, K // 128), torch.float32, w.device) if sw is None else sw
    if w_pruned is None and want_pruned:
        w_pruned = _empty((N, K), torch.bfloat16, w.device)
    _dev(vals, torch.uint8, (N, K // 2), "vals")
    _dev(meta, torch.uint8, (N, K // 8), "meta")
    _dev(sw, torch.float32, (NB, K // 128), "sw")
    if w_pruned is not None:
        _dev(w_pruned, torch.bfloat16, (N, K), "w_pruned")
    _check("prune24_compress",
           lib().prune24_compress(_ptr(w), N, K, _ptr(vals), _ptr(meta), _ptr(sw),
                                  _ptr(w_pruned), _stream(stream, w)))
    return vals, meta, sw, w_pruned


def gemm_workspace_bytes(M, N, K, sparse=False):
    return int(lib().fp8bs_gemm_workspace_bytes(M, N, K, 1 if sparse else 0))


def _workspace(M, N, K, sparse, device, workspace):
    need = gemm_workspace_bytes(M, N, K, sparse)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    size = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return workspace, size


def fp8_block_gemm(qa, sa, qw, sw, y=None, workspace=None, stream=None):
    """Block-scaled FP8 GEMM: y bf16 [M, N] = dequant(qa) . dequant(qw)^T."""
    M, K = qa.shape
    N = qw.shape[0]
    NB, KB = -(-N // 128), K // 128
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa, torch.float32, (M, KB), "sa")
    _dev(qw, torch.uint8, (N, K), "qw")
    _dev(sw, torch.float32, (NB, KB), "sw")
    y = _empty((M, N), torch.bfloat16, qa.device) if y is None else y
    _dev(y, torch.bfloat16, (M, N), "y")
    ws, ws_bytes = _workspace(M, N, K, False, qa.device, workspace)
    _check("fp8_block_gemm",
           lib().fp8_block_gemm(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), _ptr(y), M, N, K,
                                _ptr(ws), ws_bytes, _stream(stream, qa)))
    return y


def fp8_block_gemm_quant(qa, sa, qw, sw, y=None, qy=None, sy=None, want_y=True, workspace=None,
                         stream=None):
    """fp8_block_gemm plus the next layer's input quantization of its bf16 output:
    returns (y, qy, sy) with qy, sy = fp8_quant_act_group128(y). With want_y=False
    and M > 256, y is not written (returned as None)."""
    M, K = qa.shape
    N = qw.shape[0]
    NB, KB = -(-N // 128), K // 128
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa, torch.float32, (M, KB), "sa")
    _dev(qw, torch.uint8, (N, K), "qw")
    _dev(sw, torch.float32, (NB, KB), "sw")
    if y is None and (want_y or M <= 256):
        y = _empty((M, N), torch.bfloat16, qa.device)
    if y is not None:
        _dev(y, torch.bfloat16, (M, N), "y")
    qy = _empty((M, N), torch.uint8, qa.device) if qy is None else qy
    sy = _empty((M, N // 128), torch.float32, qa.device) if sy is None else sy
    _dev(qy, torch.uint8, (M, N), "qy")
    _dev(sy, torch.float32, (M, N // 128), "sy")
    ws, ws_bytes = _workspace(M, N, K, False, qa.device, workspace)
    _check("fp8_block_gemm_quant",
           lib().fp8_block_gemm_quant(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), _ptr(y), _ptr(qy),
                                      _ptr(sy), M, N, K, _ptr(ws), ws_bytes, _stream(stream, qa)))
    return y, qy, sy


def fp8_sparse24_gemm(qa, sa, vals, meta, sw, y=None, workspace=None, stream=None):
    """2:4 sparse block-scaled FP8 GEMM on (vals, meta, sw) from prune24_compress."""
    M, K = qa.shape
    N = vals.shape[0]
    NB, KB = -(-N // 128), K // 128
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa, torch.float32, (M, KB), "sa")
    _dev(vals, torch.uint8, (N, K // 2), "vals")
    _dev(meta, torch.uint8, (N, K // 8), "meta")
    _dev(sw, torch.float32, (NB, KB), "sw")
    y = _empty((M, N), torch.bfloat16, qa.device) if y is None else y
    _dev(y, torch.bfloat16, (M, N), "y")
    ws, ws_bytes = _workspace(M, N, K, True, qa.device, workspace)
    _check("fp8_sparse24_gemm",
           lib().fp8_sparse24_gemm(_ptr(qa), _ptr(sa), _ptr(vals), _ptr(meta), _ptr(sw), _ptr(y),
                                   M, N, K, _ptr(ws), ws_bytes, _stream(stream, qa)))
    return y


def fp8_quant_act_group128_ue8m0(x, qa=None, sa8=None, stream=None):
    """x bf16 [M, K] -> (qa uint8 [M, K] E4M3 codes, sa8 uint8 [M, K/128] UE8M0 codes)."""
    M, K = x.shape
    _dev(x, torch.bfloat16, (M, K), "x")
    qa = _empty((M, K), torch.uint8, x.device) if qa is None else qa
    sa8 = _empty((M, K // 128), torch.uint8, x.device) if sa8 is None else sa8
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa8, torch.uint8, (M, K // 128), "sa8")
    _check("fp8_quant_act_group128_ue8m0",
           lib().fp8_quant_act_group128_ue8m0(_ptr(x), M, K, _ptr(qa), _ptr(sa8), _stream(stream, x)))
    return qa, sa8


def fp8_quant_weight_block128_ue8m0(w, qw=None, sw8=None, stream=None):
    """w bf16 [N, K] -> (qw uint8 [N, K], sw8 uint8 [ceil(N/128), K/128] UE8M0 codes)."""
    N, K = w.shape
    _dev(w, torch.bfloat16, (N, K), "w")
    NB = -(-N // 128)
    qw = _empty((N, K), torch.uint8, w.device) if qw is None else qw
    sw8 = _empty((NB, K // 128), torch.uint8, w.device) if sw8 is None else sw8
    _dev(qw, torch.uint8, (N, K), "qw")
    _dev(sw8, torch.uint8, (NB, K // 128), "sw8")
    _check("fp8_quant_weight_block128_ue8m0",
           lib().fp8_quant_weight_block128_ue8m0(_ptr(w), N, K, _ptr(qw), _ptr(sw8),
                                                 _stream(stream, w)))
    return qw, sw8


def fp8_block_gemm_ue8m0(qa, sa8, qw, sw8, y=None, workspace=None, stream=None):
    """Block-scaled FP8 GEMM with UE8M0 scales (the tensor cores' block scaling)."""
    M, K = qa.shape
    N = qw.shape[0]
    NB, KB = -(-N // 128), K // 128
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa8, torch.uint8, (M, KB), "sa8")
    _dev(qw, torch.uint8, (N, K), "qw")
    _dev(sw8, torch.uint8, (NB, KB), "sw8")
    y = _empty((M, N), torch.bfloat16, qa.device) if y is None else y
    _dev(y, torch.bfloat16, (M, N), "y")
    ws, ws_bytes = _workspace(M, N, K, False, qa.device, workspace)
    _check("fp8_block_gemm_ue8m0",
           lib().fp8_block_gemm_ue8m0(_ptr(qa), _ptr(sa8), _ptr(qw), _ptr(sw8), _ptr(y), M, N, K,
                                      _ptr(ws), ws_bytes, _stream(stream, qa)))
    return y


def _grouped(name, qa, sa, qw, sw, m_indices, y, scale_dtype, stream):
    M, K = qa.shape
    E, N, _ = qw.shape
    NB, KB = -(-N // 128), K // 128
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa, scale_dtype, (M, KB), "sa")
    _dev(qw, torch.uint8, (E, N, K), "qw")
    _dev(sw, scale_dtype, (E, NB, KB), "sw")
    _dev(m_indices, torch.int32, (M,), "m_indices")
    y = _empty((M, N), torch.bfloat16, qa.device) if y is None else y
    _dev(y, torch.bfloat16, (M, N), "y")
    _check(name, getattr(lib(), name)(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), _ptr(m_indices),
                                      _ptr(y), M, N, K, E, None, 0, _stream(stream, qa)))
    return y


def fp8_grouped_gemm(qa, sa, qw, sw, m_indices, y=None, stream=None):
    """Mixture-of-experts block-scaled GEMM (fp32 scales): row m of qa uses the
    weights qw[m_indices[m]] ([E, N, K]); each 128-row tile holds one expert."""
    return _grouped("fp8_grouped_gemm", qa, sa, qw, sw, m_indices, y, torch.float32, stream)


def fp8_grouped_gemm_ue8m0(qa, sa8, qw, sw8, m_indices, y=None, stream=None):
    """The grouped GEMM with UE8M0 scale codes."""
    return _grouped("fp8_grouped_gemm_ue8m0", qa, sa8, qw, sw8, m_indices, y, torch.uint8, stream)


def fp8_gemm_swiglu_quant(qa, sa, qw_gate_up, sw_gate_up, h=None, qh=None, sh=None, want_h=True,
                          workspace=None, stream=None):
    """Gate+up GEMM with SwiGLU and the down projection's 1x128 quantization
    fused: returns (h bf16 [M, I] or None, qh uint8 [M, I], sh fp32 [M, I/128])
    for weights [W_gate; W_up] ([2I, K])."""
    M, K = qa.shape
    N2 = qw_gate_up.shape[0]
    I = N2 // 2
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa, torch.float32, (M, K // 128), "sa")
    _dev(qw_gate_up, torch.uint8, (N2, K), "qw_gate_up")
    _dev(sw_gate_up, torch.float32, (-(-N2 // 128), K // 128), "sw_gate_up")
    if h is None and want_h:
        h = _empty((M, I), torch.bfloat16, qa.device)
    if h is not None:
        _dev(h, torch.bfloat16, (M, I), "h")
    qh = _empty((M, I), torch.uint8, qa.device) if qh is None else qh
    sh = _empty((M, I // 128), torch.float32, qa.device) if sh is None else sh
    _dev(qh, torch.uint8, (M, I), "qh")
    _dev(sh, torch.float32, (M, I // 128), "sh")
    need = int(lib().fp8bs_swiglu_workspace_bytes(M, I))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=qa.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("fp8_gemm_swiglu_quant",
           lib().fp8_gemm_swiglu_quant(_ptr(qa), _ptr(sa), _ptr(qw_gate_up), _ptr(sw_gate_up),
                                       _ptr(h), _ptr(qh), _ptr(sh), M, I, K, _ptr(workspace),
                                       ws_bytes, _stream(stream, qa)))
    return h, qh, sh


def fp8_gemm_swiglu_quant_noalloc(qa, sa, qw_gate_up, sw_gate_up, h, qh, sh, stream=None):
    """fp8_gemm_swiglu_quant into caller-given outputs, with the library's
    fixed device scratch in place of a workspace: this call allocates
    nothing. h may be None; qh uint8 [M, I] and sh fp32 [M, I/128] are
    required."""
    M, K = qa.shape
    N2 = qw_gate_up.shape[0]
    I = N2 // 2
    _dev(qa, torch.uint8, (M, K), "qa")
    _dev(sa, torch.float32, (M, K // 128), "sa")
    _dev(qw_gate_up, torch.uint8, (N2, K), "qw_gate_up")
    _dev(sw_gate_up, torch.float32, (-(-N2 // 128), K // 128), "sw_gate_up")
    if h is not None:
        _dev(h, torch.bfloat16, (M, I), "h")
    _dev(qh, torch.uint8, (M, I), "qh")
    _dev(sh, torch.float32, (M, I // 128), "sh")
    _check("fp8_gemm_swiglu_quant_noalloc",
           lib().fp8_gemm_swiglu_quant_noalloc(_ptr(qa), _ptr(sa), _ptr(qw_gate_up),
                                               _ptr(sw_gate_up), _ptr(h), _ptr(qh), _ptr(sh),
                                               M, I, K, _stream(stream, qa)))
    return h, qh, sh


def fp8_gather_columns(src, dst=None, stream=None):
    """Rank-major column shards src bf16 [P, M, Np] -> full rows dst [M, P * Np]."""
    P, M, Np = src.shape
    _dev(src, torch.bfloat16, (P, M, Np), "src")
    dst = _empty((M, P * Np), torch.bfloat16, src.device) if dst is None else dst
    _dev(dst, torch.bfloat16, (M, P * Np), "dst")
    _check("fp8_gather_columns",
           lib().fp8_gather_columns(_ptr(src), P, M, Np, _ptr(dst), _stream(stream, src)))
    return dst


def get_device_error(stream=None, device=None):
    """Synchronise the stream and return (and clear) the device error word."""
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return int(lib().fp8bs_get_device_error(ctypes.c_void_p(s.cuda_stream)))


def set_wait_limit(cycles):
    lib().fp8bs_set_wait_limit(int(cycles))


def fp8_linear(x, qw, sw, y=None, stream=None):
    """The fine-grained FP8 linear layer: quantise x per 1x128 group, then the
    block-scaled GEMM against pre-quantised weights."""
    qa, sa = fp8_quant_act_group128(x, stream=stream)
    return fp8_block_gemm(qa, sa, qw, sw, y=y, stream=stream)
