"""Plain CPU oracle of the fine-grained FP8 linear layer (test infrastructure).

This module is the slow, obviously-correct statement of what the layer
computes, written in numpy. The same definitions are written a second time in
plain C++ (``fp8_oracle.cpp``), which is the oracle the GPU tests use; the CPU
tests hold both to the same pins and to each other. Used only by the tests,
the smoke check and the CPU baseline of the benchmark; the CUDA library never
imports it and the two share no code.

Sources (by page title and section):

* "FP8 à granularité fine" (Hugging Face transformers docs,
  quantization/finegrained_fp8), opening bullets: weights are quantised to 8
  bits per 2-D block, ``weight_block_size=(128, 128)``; activations are
  quantised to 8 bits per group per token, the group being 128 input channels.
  Section "Chemin rapide de DeepGEMM": ``activation_scheme="dynamic"``, i.e.
  activation scales are computed at run time from the activations themselves.
  Section "Format d'échelle UE8M0": scales stay plain float32
  (``scale_fmt="float"``), not power-of-two UE8M0.
* "Déployer la parcimonie 2:4 avec FP8 sur Hopper: un guide de production",
  pipeline steps 2 and 4 and "Exemples pratiques, 1) Application de masque
  2:4": 2:4 groups are 4 contiguous values along K, scored by magnitude, the
  top two kept; step 6: prune first, then recompute the FP8 scales.
* "Combiner élagage et quantification pour maximiser la vitesse des modèles
  linguistiques", section "La clé : la sparsité structurée 2:4": of every 4
  weights the two largest are kept.

What the pages leave open is fixed as follows (each is a reading, listed with
its justification in the design notes):

* the 8-bit format is OCP FP8 E4M3 ("fn": bias 7, no infinities, largest
  finite 448); conversion is round-to-nearest-even with saturation to +-448;
* a group's / block's scale is ``amax / 448`` computed in fp32 (IEEE division);
* an element is encoded as ``e4m3(fl32(x / s))``: one fp32 IEEE division,
  then one rounding to E4M3; a group with amax == 0 has s == 0 and encodes
  every element as a signed zero;
* the GEMM is ``Y[m,n] = sum_kb sA[m,kb] * sW[n//128,kb] * sum_{k in kb}
  qA[m,k] * qW[n,k]``; here it is evaluated in fp64 (the library accumulates
  in fp32 and rounds the result to bf16);
* 2:4 ties go to the lower index; pruned positions become +0.

Layouts (row-major throughout): X, qA [M, K]; sA [M, K/128]; W, qW [N, K];
sW [ceil(N/128), K/128]; vals [N, K/2]; meta [N, K/8] (byte j holds group 2j
in bits 0-3 and group 2j+1 in bits 4-7, each nibble = i0 | i1 << 2 with
i0 < i1 the kept positions); Y [M, N].
"""

import numpy as np

E4M3_MAX = 448.0
GROUP = 128

_MIN_NORMAL = 2.0 ** -6   # smallest normal E4M3 magnitude (exponent field 1)
_SUB_STEP = 2.0 ** -9     # spacing of E4M3 subnormals (exponent field 0)


# ----------------------------------------------------------------------------
# E4M3 codec, from the OCP 8-bit floating point definition (E4M3, "fn")
# ----------------------------------------------------------------------------

def _e4m3_value(code):
    """Value of each E4M3 byte, as float64 (NaN for 0x7F / 0xFF).

    Field layout S.EEEE.MMM, exponent bias 7. Exponent field 0 is subnormal,
    value (M/8) * 2^-6; otherwise (1 + M/8) * 2^(E-7). S.1111.111 is NaN and
    there are no infinities, so the largest finite magnitude is
    1.75 * 2^8 = 448.
    """
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * _SUB_STEP, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


# The definition above evaluated once for each of the 256 codes.
_DECODE_TABLE = _e4m3_value(np.arange(256, dtype=np.uint8))


def e4m3_decode(code):
    """Value of each E4M3 byte as float64 (``_e4m3_value``, by table lookup)."""
    return _DECODE_TABLE[np.asarray(code, dtype=np.uint8)]


def e4m3_encode(v):
    """Encode float32 values as E4M3 bytes: round to nearest, ties to even,
    saturating to +-448 (so no value ever becomes NaN); the sign of zero is
    kept. NaN input (outside the contract) maps to 0x7F.

    The rounding is done on the exact value of each fp32 input: in fp64 the
    magnitude is divided by the spacing of E4M3 values in its binade (a power
    of two, so exact), rounded half-to-even to an integer, and multiplied back.
    """
    v = np.asarray(v, dtype=np.float32)
    neg = np.signbit(v)
    a = np.abs(v.astype(np.float64))
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    # Saturation: E4M3 has no value above 448 and no infinity.
    a = np.minimum(a, E4M3_MAX)
    # Spacing of representable values around a: 2^(floor(log2 a) - 3) for
    # normals, 2^-9 for subnormals. frexp gives floor(log2 a) exactly.
    _, ex = np.frexp(a)
    step = np.where(a >= _MIN_NORMAL, np.ldexp(1.0, ex - 1 - 3), _SUB_STEP)
    q = np.rint(a / step) * step          # np.rint: round half to even
    q = np.minimum(q, E4M3_MAX)           # cannot exceed 448 after the clamp
    # Bit pattern of the rounded magnitude.
    _, qe = np.frexp(q)
    qexp = qe - 1                         # floor(log2 q) for q > 0
    normal = q >= _MIN_NORMAL
    e_field = np.where(normal, qexp + 7, 0)
    m_field = np.where(normal,
                       np.rint(np.ldexp(q, -qexp) * 8.0 - 8.0),
                       np.rint(q / _SUB_STEP))
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = np.where(q == 0.0, 0, code)
    code = code | np.where(neg, 0x80, 0)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


# ----------------------------------------------------------------------------
# Quantizers
# ----------------------------------------------------------------------------

def _as_f32(x):
    """bf16 (torch) or float arrays -> float32 numpy (bf16 widens exactly)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float32)


def _quantize_with_scale(x32, s32):
    """q = e4m3(fl32(x / s)) with s broadcast over x; s == 0 (an all-zero
    group or block) encodes each element as a zero of the element's sign."""
    s_b = np.broadcast_to(s32, x32.shape).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (x32 / s_b).astype(np.float32)   # fp32 IEEE division
    q = e4m3_encode(ratio)
    zero_scale = s_b == 0.0
    q = np.where(zero_scale, np.where(np.signbit(x32), 0x80, 0x00), q)
    return q.astype(np.uint8)


def quant_act_group128(x):
    """Dynamic per-token activation quantization in 1x128 groups along K.

    "FP8 à granularité fine", opening bullets (activations: one scale per
    group of 128 input channels per token) and "Chemin rapide de DeepGEMM"
    (dynamic activation scheme). For token m and group g:
    sA[m,g] = fl32(amax_{k in g} |x[m,k]| / 448), qA[m,k] = e4m3(fl32(x / sA)).

    x: [M, K] (bf16 tensor or float array), K % 128 == 0.
    Returns (qA uint8 [M, K], sA float32 [M, K/128]).
    """
    x32 = _as_f32(x)
    M, K = x32.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    KB = K // GROUP
    g = x32.reshape(M, KB, GROUP)
    amax = np.abs(g).max(axis=2) if M * KB else np.zeros((M, KB), np.float32)
    sA = (amax.astype(np.float32) / np.float32(E4M3_MAX)).astype(np.float32)
    qA = _quantize_with_scale(g, sA[:, :, None]).reshape(M, K)
    return qA, sA


def quant_weight_block128(w):
    """Weight quantization in 128x128 blocks ("FP8 à granularité fine",
    opening bullets, ``weight_block_size=(128, 128)``).

    For block (nb, kb): sW = fl32(amax |w| / 448) over the block's valid rows
    (the last row-block is ragged when N % 128 != 0), qW = e4m3(fl32(w / sW)).

    w: [N, K], K % 128 == 0.
    Returns (qW uint8 [N, K], sW float32 [ceil(N/128), K/128]).
    """
    w32 = _as_f32(w)
    N, K = w32.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    NB, KB = -(-N // GROUP), K // GROUP
    sW = np.zeros((NB, KB), np.float32)
    qW = np.zeros((N, K), np.uint8)
    for nb in range(NB):
        r0, r1 = nb * GROUP, min(N, (nb + 1) * GROUP)
        for kb in range(KB):
            c0, c1 = kb * GROUP, (kb + 1) * GROUP
            blk = w32[r0:r1, c0:c1]
            s = np.float32(np.abs(blk).max()) / np.float32(E4M3_MAX)
            sW[nb, kb] = s
            qW[r0:r1, c0:c1] = _quantize_with_scale(blk, np.float32(s))
    return qW, sW


# ----------------------------------------------------------------------------
# 2:4 pruning and compression
# ----------------------------------------------------------------------------

def _bf16_magnitude_key(w32):
    """|w| as an orderable integer: the fp32 bit pattern with the sign cleared
    (bf16 values widen exactly to fp32, and for non-negative IEEE floats the
    bit pattern orders like the value; +0 and -0 get the same key)."""
    return w32.view(np.uint32) & np.uint32(0x7FFFFFFF)


def prune24_select(w):
    """Kept positions of every group of 4 contiguous values along K.

    "Déployer la parcimonie 2:4 avec FP8 sur Hopper", step 4 and the 2:4 mask
    example (top two magnitudes of each group of 4 along K); "Combiner élagage
    et quantification...", section on 2:4 (keep the two largest). Ties in
    magnitude go to the lower index.

    Returns int arrays (i0, i1) of shape [N, K/4] with i0 < i1.
    """
    w32 = _as_f32(w)
    N, K = w32.shape
    key = _bf16_magnitude_key(np.ascontiguousarray(w32)).reshape(N, K // 4, 4)
    key = key.astype(np.int64)
    # Rank each member: how many others beat it (larger key, or equal key at
    # a lower index). The two with rank 0 and 1 are kept.
    rank = np.zeros(key.shape, np.int64)
    for i in range(4):
        for j in range(4):
            if i == j:
                continue
            beats = (key[..., j] > key[..., i]) | ((key[..., j] == key[..., i]) & (j < i))
            rank[..., i] += beats
    kept = rank < 2
    idx = np.arange(4)
    # i0 = smaller kept position, i1 = larger.
    i0 = np.where(kept, idx, 4).min(axis=-1)
    i1 = np.where(kept, idx, -1).max(axis=-1)
    return i0, i1


def prune24_compress(w):
    """2:4 magnitude pruning along K, then block quantization and compression.

    Follows "Déployer la parcimonie 2:4 avec FP8 sur Hopper", step 6 (prune,
    then compute the FP8 scales on the pruned weights). Pruned positions are
    set to +0; the pruned matrix is quantized in 128x128 blocks exactly as
    ``quant_weight_block128``; the two kept codes of each group are stored in
    order of position with a 4-bit index nibble.

    w: [N, K] bf16 / float, K % 128 == 0.
    Returns (vals uint8 [N, K/2], meta uint8 [N, K/8], sW float32 [NB, KB],
    w_pruned float32 [N, K] holding bf16-exact values).
    """
    w32 = _as_f32(w)
    N, K = w32.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    i0, i1 = prune24_select(w32)
    g = w32.reshape(N, K // 4, 4)
    idx = np.arange(4)[None, None, :]
    keep = (idx == i0[..., None]) | (idx == i1[..., None])
    w_pruned = np.where(keep, g, np.float32(0.0)).astype(np.float32).reshape(N, K)
    qW, sW = quant_weight_block128(w_pruned)
    qg = qW.reshape(N, K // 4, 4)
    vals = np.empty((N, K // 4, 2), np.uint8)
    vals[..., 0] = np.take_along_axis(qg, i0[..., None], axis=-1)[..., 0]
    vals[..., 1] = np.take_along_axis(qg, i1[..., None], axis=-1)[..., 0]
    nib = (i0 | (i1 << 2)).astype(np.uint8)            # [N, K/4]
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return vals.reshape(N, K // 2), meta, sW, w_pruned


def decompress24(vals, meta):
    """Dense E4M3 codes [N, K] from (vals [N, K/2], meta [N, K/8]); the two
    pruned positions of every group hold code 0x00 (+0)."""
    vals = np.asarray(vals, np.uint8)
    meta = np.asarray(meta, np.uint8)
    N, K2 = vals.shape
    K = 2 * K2
    nib = np.empty((N, K // 4), np.uint8)
    nib[:, 0::2] = meta & 0xF
    nib[:, 1::2] = meta >> 4
    i0 = (nib & 0x3).astype(np.int64)
    i1 = (nib >> 2).astype(np.int64)
    q = np.zeros((N, K // 4, 4), np.uint8)
    v = vals.reshape(N, K // 4, 2)
    np.put_along_axis(q, i0[..., None], v[..., 0:1], axis=-1)
    np.put_along_axis(q, i1[..., None], v[..., 1:2], axis=-1)
    return q.reshape(N, K)


# ----------------------------------------------------------------------------
# Block-scaled GEMMs
# ----------------------------------------------------------------------------

def _weight_rows(qW, sW, cols):
    """Codes and per-row scales of the weight rows n in ``cols`` (all rows
    when None); row n uses the scale row n // 128."""
    qW = np.asarray(qW, np.uint8)
    n = np.arange(qW.shape[0]) if cols is None else np.asarray(cols, np.int64)
    return qW[n], np.asarray(sW, np.float64)[n // GROUP]            # [n, K], [n, KB]


def _gemm_rows(qA, sA, q_w, s_w):
    """sum_kb sA[:,kb] * s_w[:,kb] * (qA_kb . q_w_kb^T) for weight rows q_w
    with their own scale rows s_w [n, KB]; fp64."""
    qA = np.asarray(qA, np.uint8)
    M, K = qA.shape
    a = e4m3_decode(qA)
    w = e4m3_decode(q_w)
    s_a = np.asarray(sA, np.float64)                               # [M, KB]
    y = np.zeros((M, q_w.shape[0]), np.float64)
    for kb in range(K // GROUP):
        ks = slice(kb * GROUP, (kb + 1) * GROUP)
        partial = a[:, ks] @ w[:, ks].T                            # exact
        y += (s_a[:, kb:kb + 1] * s_w[None, :, kb]) * partial
    return y


def block_gemm(qA, sA, qW, sW, cols=None):
    """Y = sum over K-blocks of sA[m,kb] * sW[n//128,kb] * (qA_kb . qW_kb^T).

    The formula of the block-scaled FP8 linear ("FP8 à granularité fine":
    1x128 activation groups against 128x128 weight blocks), written out one
    128-deep K-block at a time as the method states it, in fp64. Each K-block
    partial is a sum of 128 products of E4M3 values and is exact in fp64.

    ``cols`` optionally restricts the output to the columns n listed (for
    sampled checks of large shapes). Returns Y float64 [M, N or len(cols)]
    (the unrounded reference).
    """
    q_w, s_w = _weight_rows(qW, sW, cols)
    return _gemm_rows(qA, sA, q_w, s_w)


def sparse24_gemm(qA, sA, vals, meta, sW, cols=None):
    """The same GEMM with the weight given in 2:4 compressed form: the
    weight codes are rebuilt by ``decompress24`` and multiplied densely."""
    vals = np.asarray(vals, np.uint8)
    meta = np.asarray(meta, np.uint8)
    n = np.arange(vals.shape[0]) if cols is None else np.asarray(cols, np.int64)
    q_w = decompress24(vals[n], meta[n])
    return _gemm_rows(qA, sA, q_w, np.asarray(sW, np.float64)[n // GROUP])


def gemm_abs_sum(qA, sA, qW, sW, cols=None):
    """sum_k |a_k * w_k| per output, on the dequantized operands (fp64)."""
    qA = np.asarray(qA, np.uint8)
    q_w, s_w = _weight_rows(qW, sW, cols)
    a = np.abs(e4m3_decode(qA)) * np.repeat(np.abs(np.asarray(sA, np.float64)), GROUP, axis=1)
    w = np.abs(e4m3_decode(q_w)) * np.repeat(np.abs(s_w), GROUP, axis=1)
    return a @ w.T


def gemm_error_bound(qA, sA, qW, sW, cols=None, rel=1e-2):
    """Per-output tolerance rel * sum_k |a_k * w_k| on the dequantized
    operands (the test adds one bf16 ulp of the reference on top)."""
    return rel * gemm_abs_sum(qA, sA, qW, sW, cols=cols)


def bf16_ulp(y):
    """Spacing of bf16 values at |y| (8 significant bits; subnormal spacing
    2^-133 below 2^-126)."""
    y = np.abs(np.asarray(y, np.float64))
    _, ex = np.frexp(np.where(y == 0, 1.0, y))
    e = np.maximum(ex - 1, -126)
    ulp = np.ldexp(1.0, e - 7)
    return np.where(y == 0, 2.0 ** -133, ulp)


# ----------------------------------------------------------------------------
# UE8M0 scale variant ("Format d'échelle UE8M0": scales stored as
# float8_e8m0fnu, a bare power of two)
# ----------------------------------------------------------------------------

def ue8m0_decode(code):
    """fp32 value 2^(c - 127) of each UE8M0 code (8 exponent bits, no sign,
    no mantissa; 0xFF is NaN)."""
    c = np.asarray(code, np.uint8).astype(np.int64)
    v = np.ldexp(np.float64(1.0), c - 127).astype(np.float32)
    return np.where(c == 255, np.float32(np.nan), v)


def ue8m0_of_amax(amax):
    """Code of the smallest power of two s with 448 * s >= amax (no element
    of the group saturates), clamped to the codes 0..254; amax == 0 -> 0."""
    a = np.asarray(amax, np.float32).astype(np.float64)
    # candidate e from the binade of amax / 448, then settled exactly with
    # the comparisons 448 * 2^e >= amax > 448 * 2^(e - 1)
    _, e = np.frexp(np.where(a > 0, a / E4M3_MAX, 1.0))
    e = e.astype(np.int64)
    for _ in range(2):
        e = np.where(np.ldexp(E4M3_MAX, e - 1) >= a, e - 1, e)
    for _ in range(2):
        e = np.where(np.ldexp(E4M3_MAX, e) < a, e + 1, e)
    e = np.clip(e, -127, 127)
    return np.where(a > 0, e + 127, 0).astype(np.uint8)


def quant_act_group128_ue8m0(x):
    """Per 1x128 group: code c = ue8m0_of_amax(amax), s = 2^(c - 127),
    qA = e4m3(fl32(x / s)). Returns (qA [M, K], sA8 uint8 [M, K/128])."""
    x32 = _as_f32(x)
    M, K = x32.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    g = x32.reshape(M, K // GROUP, GROUP)
    amax = np.abs(g).max(axis=2) if M * K else np.zeros((M, K // GROUP), np.float32)
    sa8 = ue8m0_of_amax(amax)
    qa = _quantize_with_scale(g, ue8m0_decode(sa8)[:, :, None]).reshape(M, K)
    return qa, sa8


def quant_weight_block128_ue8m0(w):
    """Per 128x128 block (ragged last row block over its valid rows): the
    same with the block amax. Returns (qW [N, K], sW8 uint8 [NB, KB])."""
    w32 = _as_f32(w)
    N, K = w32.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    NB, KB = -(-N // GROUP), K // GROUP
    sw8 = np.zeros((NB, KB), np.uint8)
    qw = np.zeros((N, K), np.uint8)
    for nb in range(NB):
        r0, r1 = nb * GROUP, min(N, (nb + 1) * GROUP)
        for kb in range(KB):
            blk = w32[r0:r1, kb * GROUP:(kb + 1) * GROUP]
            c = ue8m0_of_amax(np.float32(np.abs(blk).max()))
            sw8[nb, kb] = c
            qw[r0:r1, kb * GROUP:(kb + 1) * GROUP] = _quantize_with_scale(blk, ue8m0_decode(c))
    return qw, sw8


def block_gemm_ue8m0(qA, sA8, qW, sW8, cols=None):
    """The block-scaled GEMM with each scale the power of two of its code."""
    return block_gemm(qA, ue8m0_decode(sA8), qW, ue8m0_decode(sW8), cols=cols)


def gemm_error_bound_ue8m0(qA, sA8, qW, sW8, cols=None, rel=1e-2):
    return gemm_error_bound(qA, ue8m0_decode(sA8), qW, ue8m0_decode(sW8), cols=cols, rel=rel)


# ----------------------------------------------------------------------------
# Grouped (mixture-of-experts) GEMM ("FP8 à granularité fine", section
# "Chemin rapide de DeepGEMM": the experts' products go through grouped
# kernels)
# ----------------------------------------------------------------------------

def grouped_gemm(qA, sA, qW, sW, m_indices):
    """Y[m] = the block-scaled product of token row m with the weights of its
    expert e = m_indices[m] (qW [E, N, K], sW [E, ceil(N/128), K/128]); rows
    with e outside [0, E) are NaN."""
    qA = np.asarray(qA, np.uint8)
    qW = np.asarray(qW, np.uint8)
    sW = np.asarray(sW, np.float32)
    mi = np.asarray(m_indices, np.int64)
    M, K = qA.shape
    E, N, _ = qW.shape
    y = np.full((M, N), np.nan)
    for e in range(E):
        rows = np.nonzero(mi == e)[0]
        if rows.size:
            y[rows] = block_gemm(qA[rows], np.asarray(sA)[rows], qW[e], sW[e])
    return y


def grouped_gemm_ue8m0(qA, sA8, qW, sW8, m_indices):
    return grouped_gemm(qA, ue8m0_decode(sA8), qW, ue8m0_decode(sW8), m_indices)


# ----------------------------------------------------------------------------
# Gated MLP: SwiGLU of the gate and up outputs (TensorRT-LLM docs,
# performance/fp8-quantization, section "GEMM + SwiGLU Fusion in Gated-MLP")
# ----------------------------------------------------------------------------

def swiglu(g, u):
    """h = silu(g) * u with silu(g) = g / (1 + e^-g), float64."""
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g)) * np.asarray(u, np.float64)


def swiglu_error_bound(g, u, tg, tu):
    """1.1 tg (|u| + tu) + |silu(g)| tu + 1e-5 |h|: |silu'| < 1.1 everywhere."""
    g = np.asarray(g, np.float64)
    u = np.asarray(u, np.float64)
    sg = g / (1.0 + np.exp(-g))
    return 1.1 * np.asarray(tg) * (np.abs(u) + tu) + np.abs(sg) * tu + 1e-5 * np.abs(sg * u)


def gemm_swiglu(qA, sA, qW_gate_up, sW_gate_up, rel=1e-2):
    qW = np.asarray(qW_gate_up, np.uint8)
    sW = np.asarray(sW_gate_up, np.float32)
    I = qW.shape[0] // 2
    g = block_gemm(qA, sA, qW[:I], sW[:I // GROUP])
    u = block_gemm(qA, sA, qW[I:], sW[I // GROUP:])
    tg = gemm_error_bound(qA, sA, qW[:I], sW[:I // GROUP], rel=rel)
    tu = gemm_error_bound(qA, sA, qW[I:], sW[I // GROUP:], rel=rel)
    return swiglu(g, u), swiglu_error_bound(g, u, tg, tu)
