"""Plain, slow CPU restatement of the online W4A4 rotated linear layer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may import or run this module.  It shares
no code with the CUDA library (``w4a4_rotation_quantized_b200``) and imports
nothing from it; both sides draw their inputs from ``workloads`` only.

Everything here is numpy in float64, written for a reader to check against the
pages by eye: rotations are dense matrix products (never a fast transform),
quantization is division then round-half-to-even, and the integer GEMM is an
exact dot product.  The pages cited, by title:

* [QS]  "QuaRot & SpinQuant" reading notes (chenghuawang.github.io, papers/
        quant_quarot_spinquant): §1 Computational Invariance, §2 Quarot,
        §3 SpinQuant.
* [FQ]  "LLM量化新篇章：4-bit权重激活量化几乎无损！FlatQuant的平坦之道":
        §2.3 方法概述 (affine transform, Kronecker decomposition, per-channel
        scaling, clipping), 模型架构, §3 实验结果 (量化设置).
* [GSR] "Grouped Sequency-arranged Rotation: Optimizing Rotation
        Transformation for Quantization for Free": 方法详解, 摘要（原文）.
* [QK]  "QUIK：LLM上的一种4-bit推理方法": QUIK量化 §1 (workflow), §3
        (outlier selection), §4 (efficient inference).
* [SR]  "SpinQuant: LLM Quantization with Learned Rotations" (review
        discussion): Q1/A1 (min-max quantizer), reviewer Jf43 W1/A1 (QuIP#
        incoherence bound), W2/A2 (R1/R2 absorbed into the weights).

Readings taken where the pages are silent or garbled:

R1  Codes are symmetric in [-(2^(b-1)-1), 2^(b-1)-1] = [-7, 7] for 4 bits;
    the range printed in [SR] Q1/A1 is garbled, -8 is never produced.
R2  Scale s = alpha * absmax / 7 (min-max, [SR] Q1/A1), alpha the clip ratio
    ([FQ] §2.3 clipping, applied to both sides); codes are clamped to +-7.
R3  Rounding is round-half-to-even.  The pages fix neither the rounding rule
    nor the precision of x/s; the scale is a float32 number (one per row,
    the type the layer hands from one step to the next), so the quotient is
    formed in float32 from the float32 rotated value and scale.  Forming it
    in another precision moves a code only where x/s lies within a few
    float32 ulps of a half-integer, inside the 1e-4 tie window that the
    parity rule leaves open.
R4  An all-zero row gets s = 0 and all-zero codes.
R5  Hadamard matrices are Sylvester-ordered, scaled by 1/sqrt(n).
R6  X' = X R and W' = W R^{-T} with W stored [N out x K in], so that
    X' W'^T = X W^T ([QS] §1; [QK] §1 writes the linear layer as X W^T).
R7  A GSR block is the sequency-ordered Walsh matrix: the rows of the
    Sylvester Hadamard matrix sorted by their number of sign changes,
    scaled by 1/sqrt(b); blocks are contiguous along K ([GSR]).
R8  The Kronecker transform acts on a row x as x (P1 (x) P2), i.e.
    vec(P1^T mat(x) P2) with mat(x)[a, b] = x[a*n2 + b]; the per-channel
    scale divides X and multiplies W before the transform ([FQ] §2.3).
R9  QUIK: the outlier columns stay fp16 and unrotated; the remaining columns,
    in ascending order, are zero-padded to a multiple of the block size and
    rotated; activations are quantized symmetrically (not asymmetrically as
    [QK] §1 says of the original), weights by RTN instead of GPTQ.
R10 Outlier columns are the top-k columns by infinity-norm over a calibration
    batch, ties to the lower index, returned in ascending order ([QK] §3).
R11 A "random Hadamard rotation" ([SR] reviewer brBn W2/A2) is R = D B with
    D a diagonal of random signs +-1 and B the block-diagonal Hadamard: a
    row becomes (x .* d) B.  The signs act on the rotated-domain columns
    (after the outlier split and zero padding).  D B is orthogonal, so the
    weight side uses the same R.
R12 QUIK's activations are asymmetric per token, dynamic ([QK] §1).  Read
    as min-max over the unsigned range [0, 15]: lo = alpha*min, hi =
    alpha*max, s = (hi - lo)/15, zero point z = round(-lo/s), q =
    clamp(round(x/s) + z, 0, 15), dequantized s*(q - z); both decisions in
    float32, half to even.  The codes are stored as the signed nibble
    q - 8 (two's complement, [-8, 7]) with the zero point z - 8, so that
    s*(q - z) = s*((q - 8) - (z - 8)) and the same integer GEMM applies.
R13 The KV-cache path.  R3 ([SR] reviewer brBn Q2/A2; [QS] §3, Fig 5) is
    the same orthogonal matrix applied to the query and key rows of every
    head after RoPE, so that (q R3)(k R3)^T = q k^T; the pages do not say
    which matrix it is, and it is read as the normalized Hadamard of the
    head dimension, H_d / sqrt(d) (QuaRot's online rotation, [QS] §2).
    [QS] §3 remarks that the query branch should carry R3^{-1}; for the
    symmetric Hadamard R3^{-1} = R3^T = R3, so both readings agree.  The
    KV cache is quantized group-wise asymmetrically with groups of 128
    ([FQ] §3 量化设置), read as 4 bits with the R12 quantizer applied to
    each group of consecutive values of a token's (heads x head_dim) row:
    keys after R3, values as they are; queries stay fp16.
R14 QUIK's 8-bit layers ([QK] QUIK量化, results: the LLaMA-2 down_proj in
    INT8 with the outlier count raised in proportion to its input width;
    QUIK-8B: every layer INT8).  Read as the R1/R2 quantizer with b = 8:
    codes in [-127, 127], s = alpha * absmax / 127, round half to even in
    float32, stored one int8 per value; the outlier count of a layer of K
    inputs is round(256 * K / 4096) (688 for K = 11008).
R15 FP4 on Blackwell ([SR] reviewer brBn W3/A3 names a W-fp4/A-fp4 benchmark
    on Blackwell's fp4 tensor cores as planned work, with no format).  Read as the e2m1 element type with a per-row
    fp32 scale, the direct analogue of R2: s = alpha * absmax / 6, each
    x/s (float32) rounded to the nearest e2m1 value {0, 0.5, 1, 1.5, 2, 3,
    4, 6} (with sign), ties to the even mantissa, saturating at 6.  The
    e2m1 nibble is sign (bit 3), exponent (bits 2-1, bias 1), mantissa
    (bit 0); +-0 both decode to 0.  The integers 5 and 7 of the INT4 grid
    are not representable, so FP4 is a different quantizer, not a
    re-encoding of the INT4 codes.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

QMAX = 7                      # R1: 4-bit symmetric range [-7, 7]
NONE, HADAMARD, GSR, KRON = "none", "hadamard", "gsr", "kron"


# --------------------------------------------------------------------------
# Rotation matrices
# --------------------------------------------------------------------------

def hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_n (entries +-1, unscaled), n a power of 2.

    [QS] §2: QuaRot rotates with Hadamard matrices; the pages do not name a
    construction, so the Sylvester doubling H_2n = [[H, H], [H, -H]] (R5).
    """
    if n < 1 or n & (n - 1):
        raise ValueError(f"Hadamard size must be a power of two, got {n}")
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def sign_changes(row: np.ndarray) -> int:
    """Number of sign changes along a +-1 row (its sequency)."""
    return int(np.count_nonzero(row[1:] != row[:-1]))


def walsh_sequency(n: int) -> np.ndarray:
    """Sequency-ordered Walsh matrix: Hadamard rows sorted by sign changes.

    [GSR] 摘要（原文）/方法详解: the Walsh-Hadamard transform with sequency
    ordering, which clusters similar frequency components (R7).
    """
    h = hadamard(n)
    seq = np.array([sign_changes(r) for r in h])
    return h[np.argsort(seq, kind="stable")]


@dataclass
class Rotation:
    """What the layer does to a row before quantizing it."""
    kind: str = NONE
    block: int = 1                       # HADAMARD / GSR block size
    P1: Optional[np.ndarray] = None      # KRON factors, [n1 x n1], [n2 x n2]
    P2: Optional[np.ndarray] = None
    chan_scale: Optional[np.ndarray] = None   # KRON per-channel scale c [K]
    clip_ratio: float = 1.0
    signs: Optional[np.ndarray] = None   # HADAMARD / GSR: random +-1 diagonal d [K_p] (R11)


def packed_width(rot: Rotation, K: int, n_out: int = 0) -> int:
    """Width K_p of the rotated, quantized part of a row.

    The K - n_out non-outlier columns are zero-padded to a multiple of the
    block size and of 128 (R9; 128 keeps every row a whole number of the
    GEMM's K steps).  A Kronecker transform needs exactly n1*n2 columns.
    """
    kr = K - n_out
    if rot.kind == KRON:
        n = rot.P1.shape[0] * rot.P2.shape[0]
        if kr != n:
            raise ValueError("Kronecker transform needs K - n_out == n1*n2")
        return n
    unit = 128
    if rot.kind in (HADAMARD, GSR):
        unit = max(unit, rot.block)
    return -(-kr // unit) * unit


def block_rotation(kind: str, block: int) -> np.ndarray:
    """One diagonal block of R: H_b/sqrt(b) (HADAMARD) or Wal_b/sqrt(b) (GSR)."""
    base = hadamard(block) if kind == HADAMARD else walsh_sequency(block)
    return base / np.sqrt(block)


def dense_rotation(rot: Rotation, k_p: int) -> np.ndarray:
    """The full K_p x K_p rotation R as a dense matrix (small sizes only)."""
    if rot.kind == NONE:
        return np.eye(k_p)
    if rot.kind == KRON:
        return np.kron(rot.P1.astype(np.float64), rot.P2.astype(np.float64))
    blk = block_rotation(rot.kind, rot.block)
    r = np.kron(np.eye(k_p // rot.block), blk)
    if rot.signs is not None:
        r = np.diag(np.asarray(rot.signs, np.float64)) @ r
    return r


def _apply_blocks(x: np.ndarray, blk: np.ndarray) -> np.ndarray:
    b = blk.shape[0]
    rows, k = x.shape
    return (x.reshape(rows, k // b, b) @ blk).reshape(rows, k)


def _apply_kron(x: np.ndarray, p1: np.ndarray, p2: np.ndarray) -> np.ndarray:
    """x (P1 (x) P2) row by row, as the two small products P1^T mat(x) P2.

    [FQ] §2.3 Kronecker Decomposition / 模型架构: the transform is stored as
    two small matrices and applied as two small matmuls per token (R8).
    """
    n1, n2 = p1.shape[0], p2.shape[0]
    xm = x.reshape(x.shape[0], n1, n2)
    return np.einsum("ac,mab,bd->mcd", p1, xm, p2, optimize=True).reshape(x.shape[0], n1 * n2)


def rotate_activations(x: np.ndarray, rot: Rotation) -> np.ndarray:
    """X' = X R (fp64).  [QS] §2 (online Hadamard on activations), [GSR],
    [FQ] §2.3 (per-channel scale divides X, then the affine transform)."""
    x = np.asarray(x, dtype=np.float64)
    if rot.kind == NONE:
        return x.copy()
    if rot.kind in (HADAMARD, GSR):
        if rot.signs is not None:                    # R11: (x .* d) B
            x = x * np.asarray(rot.signs, np.float64)[None, :]
        return _apply_blocks(x, block_rotation(rot.kind, rot.block))
    if rot.chan_scale is not None:
        x = x / rot.chan_scale.astype(np.float64)[None, :]
    return _apply_kron(x, rot.P1.astype(np.float64), rot.P2.astype(np.float64))


def rotate_weights(w: np.ndarray, rot: Rotation) -> np.ndarray:
    """W' = W R^{-T} (fp64), so that X' W'^T = X W^T (R6).

    For the orthogonal rotations R^{-T} = R ([QS] §1, §2; [SR] W2/A2: R1/R2
    are merged into the weights offline).  For the Kronecker transform
    (P1 (x) P2)^{-T} = P1^{-T} (x) P2^{-T}, and the per-channel scale
    multiplies W ([FQ] §2.3).
    """
    w = np.asarray(w, dtype=np.float64)
    if rot.kind == NONE:
        return w.copy()
    if rot.kind in (HADAMARD, GSR):
        if rot.signs is not None:                    # R11: D B is orthogonal
            w = w * np.asarray(rot.signs, np.float64)[None, :]
        return _apply_blocks(w, block_rotation(rot.kind, rot.block))
    if rot.chan_scale is not None:
        w = w * rot.chan_scale.astype(np.float64)[None, :]
    q1 = np.linalg.inv(rot.P1.astype(np.float64)).T
    q2 = np.linalg.inv(rot.P2.astype(np.float64)).T
    return _apply_kron(w, q1, q2)


# --------------------------------------------------------------------------
# Quantization, packing, GEMM, epilogue
# --------------------------------------------------------------------------

@dataclass
class Quantized:
    codes: np.ndarray        # int8 [rows x K_p], values in [-7, 7]
    scales: np.ndarray       # float32 [rows]
    quotient: np.ndarray     # float32 x/s before rounding (for the tie window)


def quantize_rows(xr: np.ndarray, clip_ratio: float = 1.0, bits: int = 4) -> Quantized:
    """Symmetric per-row min-max quantization to `bits`-bit codes (4, or 8
    for QUIK's INT8 layers, R14).

    [SR] Q1/A1: min-max quantization scales each row into the symmetric
    range (R1, R2); [FQ] §3 量化设置: activations per token, weights per
    output channel, both symmetric.  The decision q = round(x/s) is taken in
    float32 with round-half-to-even (R3); zero rows give s = 0 (R4).
    """
    x32 = np.asarray(xr, dtype=np.float64).astype(np.float32)
    absmax = np.max(np.abs(x32), axis=1) if x32.shape[1] else np.zeros(x32.shape[0], np.float32)
    qmax = QMAX if bits == 4 else 2 ** (bits - 1) - 1
    s = (np.float32(clip_ratio) * absmax) / np.float32(qmax)
    s = s.astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    v = (x32 / safe[:, None]).astype(np.float32)
    v[s == 0] = 0.0
    q = np.clip(np.rint(v), -qmax, qmax).astype(np.int8)
    return Quantized(codes=q, scales=s, quotient=v)


def quik_outlier_count(K: int) -> int:
    """Outlier columns of a QUIK layer of K inputs (R14): 256 per 4096."""
    return int(np.rint(256 * K / 4096))


# e2m1 magnitudes by 3-bit code (exponent, mantissa); R15
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@dataclass
class Fp4Quantized:
    codes: np.ndarray        # uint8 [rows x K_p]: e2m1 nibbles (sign bit 3)
    scales: np.ndarray       # float32 [rows]
    quotient: np.ndarray     # float32 x/s before rounding (tie window)


def e2m1_round(v: np.ndarray) -> np.ndarray:
    """Nearest e2m1 value of each v (float), ties to the even mantissa,
    saturating at +-6 (R15); returns the 4-bit codes."""
    v = np.asarray(v, np.float64)
    mag = np.minimum(np.abs(v), 6.0)
    d = np.abs(mag[..., None] - E2M1)                   # distance to every grid value
    best = np.min(d, axis=-1, keepdims=True)
    cand = d == best                                    # one, or two at a tie
    even = (np.arange(8) % 2 == 0)                      # mantissa bit 0 clear
    pick = np.where(cand.sum(-1, keepdims=True) > 1, cand & even, cand)
    code = np.argmax(pick, axis=-1).astype(np.uint8)
    return code | np.where((v < 0) & (code > 0), 8, 0).astype(np.uint8)


def e2m1_value(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, np.int64)
    return np.where(code & 8, -1.0, 1.0) * E2M1[code & 7]


def quantize_rows_fp4(xr: np.ndarray, clip_ratio: float = 1.0) -> Fp4Quantized:
    """Per-row e2m1 quantization with an fp32 scale (R15)."""
    x32 = np.asarray(xr, dtype=np.float64).astype(np.float32)
    absmax = np.max(np.abs(x32), axis=1) if x32.shape[1] else np.zeros(x32.shape[0], np.float32)
    s = ((np.float32(clip_ratio) * absmax) / np.float32(6)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    v = (x32 / safe[:, None]).astype(np.float32)
    v[s == 0] = 0.0
    return Fp4Quantized(codes=e2m1_round(v), scales=s, quotient=v)


def dequant_fp4_rows(q: Fp4Quantized) -> np.ndarray:
    return np.asarray(q.scales, np.float64)[:, None] * e2m1_value(q.codes)


def pack_fp4(codes: np.ndarray) -> np.ndarray:
    """e2m1 nibbles two per byte, element 2j in the low nibble (R15)."""
    c = np.asarray(codes, dtype=np.int64)
    if c.shape[-1] % 2:
        raise ValueError("packed rows need an even width")
    return ((c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)).astype(np.uint8)


def unpack_fp4(b: np.ndarray) -> np.ndarray:
    """Inverse of pack_fp4: uint8 nibble codes."""
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def fp4_gemm(ca: np.ndarray, cw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k e2m1(ca[m, k]) e2m1(cw[n, k]) as float64, exact.

    Every e2m1 value is a multiple of 1/2 of magnitude <= 6, so each product
    is a multiple of 1/4 below 36 and every partial sum is an exact float64
    (and float32, below 2^22 quarters) whatever the order (R15).
    """
    a = e2m1_value(ca)
    w = e2m1_value(cw)
    if a.shape[1] * 36 * 4 >= 2 ** 53:
        raise ValueError("K too large for an exact float64 dot product")
    return a @ w.T


@dataclass
class AsymQuantized:
    codes: np.ndarray        # int8 [rows x K_p]: q - 8, in [-8, 7]
    scales: np.ndarray       # float32 [rows]
    zeros: np.ndarray        # int32 [rows]: z - 8
    quotient: np.ndarray     # float32 x/s before rounding (tie window)
    zero_quotient: np.ndarray  # float32 -lo/s before rounding (tie window of z)


def quantize_rows_asym(xr: np.ndarray, clip_ratio: float = 1.0) -> AsymQuantized:
    """Asymmetric per-row min-max quantization to 4-bit codes (R12).

    [QK] QUIK量化 §1: activations are quantized asymmetrically per token,
    dynamically; weights stay symmetric (quantize_rows).
    """
    x32 = np.asarray(xr, dtype=np.float64).astype(np.float32)
    rows = x32.shape[0]
    if x32.shape[1]:
        lo = (np.float32(clip_ratio) * np.min(x32, axis=1)).astype(np.float32)
        hi = (np.float32(clip_ratio) * np.max(x32, axis=1)).astype(np.float32)
    else:
        lo = hi = np.zeros(rows, np.float32)
    s = ((hi - lo) / np.float32(15)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    zq = (-lo / safe).astype(np.float32)
    zq[s == 0] = 0.0
    z = np.rint(zq).astype(np.int64)
    v = (x32 / safe[:, None]).astype(np.float32)
    v[s == 0] = 0.0
    q = np.clip(np.rint(v).astype(np.int64) + z[:, None], 0, 15)
    return AsymQuantized(codes=(q - 8).astype(np.int8), scales=s, zeros=(z - 8).astype(np.int32),
                         quotient=v, zero_quotient=zq)


def dequant_asym_rows(q: AsymQuantized) -> np.ndarray:
    """X_hat = s * (codes - zeros) in float64 (R12)."""
    return np.asarray(q.scales, np.float64)[:, None] * (
        q.codes.astype(np.float64) - q.zeros.astype(np.float64)[:, None])


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Two's-complement nibbles, two per byte, element 2j in the low nibble."""
    q = np.asarray(q, dtype=np.int64)
    if q.shape[-1] % 2:
        raise ValueError("packed rows need an even width")
    lo = q[..., 0::2] & 0xF
    hi = q[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(b: np.ndarray) -> np.ndarray:
    """Inverse of pack_int4."""
    b = np.asarray(b, dtype=np.int64)
    lo = b & 0xF
    hi = (b >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def int_gemm(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k qa[m, k] qw[n, k], exact, as int64.

    [QK] §4: the INT4 x INT4 product accumulates in INT32.  The products are
    formed in float64: every product and partial sum is an integer below
    49 * K < 2^53, so each float64 operation is exact whatever the order.
    """
    a = np.asarray(qa, dtype=np.float64)
    w = np.asarray(qw, dtype=np.float64)
    big = max(1.0, float(np.abs(a).max(initial=0.0)), float(np.abs(w).max(initial=0.0)))
    if a.shape[1] * big * big >= 2 ** 53:
        raise ValueError("K too large for an exact float64 dot product")
    return np.rint(a @ w.T).astype(np.int64)


def dequant_epilogue(acc: np.ndarray, sa: np.ndarray, sw: np.ndarray,
                     x_out: Optional[np.ndarray] = None,
                     w_out: Optional[np.ndarray] = None) -> np.ndarray:
    """Y = fp16( acc * s_a[m] * s_w[n] + X_out W_out^T ).

    [QK] §1: the INT4 product is dequantized to FP16 and added to the FP16
    product of the outlier columns.  The sum is formed in float64 and rounded
    once to fp16 (round-to-nearest-even).
    """
    y = acc.astype(np.float64) * np.asarray(sa, np.float64)[:, None] \
        * np.asarray(sw, np.float64)[None, :]
    if x_out is not None and w_out is not None and x_out.shape[1]:
        y = y + np.asarray(x_out, np.float64) @ np.asarray(w_out, np.float64).T
    return y.astype(np.float16)


# --------------------------------------------------------------------------
# QUIK outlier columns
# --------------------------------------------------------------------------

def select_outliers(x_calib: np.ndarray, k: int) -> np.ndarray:
    """Top-k columns by infinity-norm over the calibration batch (R10).

    [QK] §3: outliers are chosen by the column infinity-norm (the largest
    absolute entry) and kept in FP16; §1: they are found from calibration
    activations.
    """
    norms = np.max(np.abs(np.asarray(x_calib, np.float64)), axis=0)
    order = np.lexsort((np.arange(norms.size), -norms))   # by -norm, then index
    return np.sort(order[:k]).astype(np.int32)


def split_outliers(x: np.ndarray, idx: Optional[np.ndarray]):
    """(X_in, X_out): the kept columns in ascending order, and X[:, idx].

    [QK] §1: outlier columns are moved to the end; the permutation has no
    numerical effect, so the kept columns simply keep their order (R9).
    """
    x = np.asarray(x)
    if idx is None or len(idx) == 0:
        return x, x[:, :0]
    keep = np.ones(x.shape[1], dtype=bool)
    keep[np.asarray(idx)] = False
    return x[:, keep], x[:, np.asarray(idx)]


def pad_columns(x: np.ndarray, k_p: int) -> np.ndarray:
    out = np.zeros((x.shape[0], k_p), dtype=np.float64)
    out[:, : x.shape[1]] = x
    return out


# --------------------------------------------------------------------------
# The layer, end to end
# --------------------------------------------------------------------------

@dataclass
class Side:
    """One operand after rotation and quantization."""
    rotated: np.ndarray      # fp64 [rows x K_p]
    q: Quantized
    packed: np.ndarray       # uint8 [rows x K_p/2]
    fp16_part: np.ndarray    # the outlier columns, fp16 [rows x n_out]


def _stored(q: Quantized, bits: int) -> np.ndarray:
    """Codes as stored: two nibbles per byte (4 bits), one int8 each (8 bits, R14)."""
    return pack_int4(q.codes) if bits == 4 else q.codes.astype(np.int8)


def quantize_activations(x: np.ndarray, rot: Rotation,
                         outlier_idx: Optional[np.ndarray] = None, bits: int = 4) -> Side:
    """Online activation path: outlier split, rotation, per-token quantization
    (4-bit codes, or 8-bit for QUIK's INT8 layers, R14)."""
    x_in, x_out = split_outliers(x, outlier_idx)
    n_out = 0 if outlier_idx is None else len(outlier_idx)
    k_p = packed_width(rot, np.asarray(x).shape[1], n_out)
    xr = rotate_activations(pad_columns(np.asarray(x_in, np.float64), k_p), rot)
    q = quantize_rows(xr, rot.clip_ratio, bits)
    return Side(xr, q, _stored(q, bits), np.asarray(x_out, np.float16))


def quantize_weights(w: np.ndarray, rot: Rotation,
                     outlier_idx: Optional[np.ndarray] = None, bits: int = 4) -> Side:
    """Offline weight path: the same split, W R^{-T}, per-channel RTN ([QS] §2)."""
    w_in, w_out = split_outliers(w, outlier_idx)
    n_out = 0 if outlier_idx is None else len(outlier_idx)
    k_p = packed_width(rot, np.asarray(w).shape[1], n_out)
    wr = rotate_weights(pad_columns(np.asarray(w_in, np.float64), k_p), rot)
    q = quantize_rows(wr, rot.clip_ratio, bits)
    return Side(wr, q, _stored(q, bits), np.asarray(w_out, np.float16))


def linear(a: Side, w: Side):
    """(acc, Y) of the quantized layer for prepared operands."""
    acc = int_gemm(a.q.codes, w.q.codes)
    y = dequant_epilogue(acc, a.q.scales, w.q.scales, a.fp16_part, w.fp16_part)
    return acc, y


def quantize_activations_asym(x: np.ndarray, rot: Rotation,
                              outlier_idx: Optional[np.ndarray] = None) -> Side:
    """The online activation path with QUIK's asymmetric quantizer (R12)."""
    x_in, x_out = split_outliers(x, outlier_idx)
    n_out = 0 if outlier_idx is None else len(outlier_idx)
    k_p = packed_width(rot, np.asarray(x).shape[1], n_out)
    xr = rotate_activations(pad_columns(np.asarray(x_in, np.float64), k_p), rot)
    q = quantize_rows_asym(xr, rot.clip_ratio)
    return Side(xr, q, pack_int4(q.codes), np.asarray(x_out, np.float16))


def linear_asym(a: Side, w: Side):
    """(acc, Y) for asymmetric activation codes: acc = sum (q_a - 8) q_w
    (what the integer GEMM accumulates), Y = fp16(X_hat W_hat^T + X_out
    W_out^T) with X_hat = s_a (codes - zeros), W_hat = s_w q_w, formed in
    float64 from the dequantized operands ([QK] §1, §4; R12)."""
    acc = int_gemm(a.q.codes, w.q.codes)
    x_hat = dequant_asym_rows(a.q)
    w_hat = np.asarray(w.q.scales, np.float64)[:, None] * w.q.codes.astype(np.float64)
    y = x_hat @ w_hat.T
    if a.fp16_part.shape[1]:
        y = y + np.asarray(a.fp16_part, np.float64) @ np.asarray(w.fp16_part, np.float64).T
    return acc, y.astype(np.float16)


def linear_forward_asym(x, w, rot: Rotation, outlier_idx=None):
    """The whole layer with asymmetric activations and symmetric weights."""
    a = quantize_activations_asym(x, rot, outlier_idx)
    ws = quantize_weights(w, rot, outlier_idx)
    acc, y = linear_asym(a, ws)
    return a, ws, acc, y


def linear_forward(x, w, rot: Rotation, outlier_idx=None, bits: int = 4):
    """The whole layer: Y ~= X W^T through rotated 4-bit (or 8-bit, R14) codes."""
    a = quantize_activations(x, rot, outlier_idx, bits)
    ws = quantize_weights(w, rot, outlier_idx, bits)
    acc, y = linear(a, ws)
    return a, ws, acc, y


def quantize_activations_fp4(x: np.ndarray, rot: Rotation,
                             outlier_idx: Optional[np.ndarray] = None) -> Side:
    """The online activation path with e2m1 codes and a per-token scale (R15)."""
    x_in, x_out = split_outliers(x, outlier_idx)
    n_out = 0 if outlier_idx is None else len(outlier_idx)
    k_p = packed_width(rot, np.asarray(x).shape[1], n_out)
    xr = rotate_activations(pad_columns(np.asarray(x_in, np.float64), k_p), rot)
    q = quantize_rows_fp4(xr, rot.clip_ratio)
    return Side(xr, q, pack_fp4(q.codes), np.asarray(x_out, np.float16))


def quantize_weights_fp4(w: np.ndarray, rot: Rotation,
                         outlier_idx: Optional[np.ndarray] = None) -> Side:
    """The offline weight path with e2m1 codes and a per-channel scale (R15)."""
    w_in, w_out = split_outliers(w, outlier_idx)
    n_out = 0 if outlier_idx is None else len(outlier_idx)
    k_p = packed_width(rot, np.asarray(w).shape[1], n_out)
    wr = rotate_weights(pad_columns(np.asarray(w_in, np.float64), k_p), rot)
    q = quantize_rows_fp4(wr, rot.clip_ratio)
    return Side(wr, q, pack_fp4(q.codes), np.asarray(w_out, np.float16))


def linear_fp4(a: Side, w: Side):
    """(acc, Y) of the FP4 layer: acc = sum e2m1(q_a) e2m1(q_w) (exact),
    Y = fp16(acc s_a s_w + X_out W_out^T) as for the integer codes (R15)."""
    acc = fp4_gemm(a.q.codes, w.q.codes)
    y = dequant_epilogue(acc, a.q.scales, w.q.scales, a.fp16_part, w.fp16_part)
    return acc, y


def linear_forward_fp4(x, w, rot: Rotation, outlier_idx=None):
    """The whole layer through rotated e2m1 codes (R15)."""
    a = quantize_activations_fp4(x, rot, outlier_idx)
    ws = quantize_weights_fp4(w, rot, outlier_idx)
    acc, y = linear_fp4(a, ws)
    return a, ws, acc, y


# --------------------------------------------------------------------------
# KV cache: R3 on queries and keys, group-wise asymmetric KV quantization
# --------------------------------------------------------------------------

def rotate_heads(x: np.ndarray, head_dim: int) -> np.ndarray:
    """Each head's slice of a token row times H_d / sqrt(d) (R13)."""
    x = np.asarray(x, np.float64)
    t, w = x.shape
    if w % head_dim:
        raise ValueError("row width must be a multiple of head_dim")
    h = hadamard(head_dim) / np.sqrt(head_dim)
    return (x.reshape(t, w // head_dim, head_dim) @ h).reshape(t, w)


@dataclass
class GroupQuantized:
    codes: np.ndarray        # int8 [tokens x width]: q - 8, in [-8, 7]
    scales: np.ndarray       # float32 [tokens x width/group]
    zeros: np.ndarray        # int32 [tokens x width/group]: z - 8
    quotient: np.ndarray     # float32 [tokens x width] x/s before rounding
    zero_quotient: np.ndarray  # float32 [tokens x width/group]


def quantize_groups_asym(x: np.ndarray, group: int) -> GroupQuantized:
    """Group-wise asymmetric 4-bit quantization (R13): every `group`
    consecutive values of a row are one row of the R12 quantizer."""
    x = np.asarray(x, np.float64)
    t, w = x.shape
    if w % group:
        raise ValueError("row width must be a multiple of the group size")
    q = quantize_rows_asym(x.reshape(t * (w // group), group))
    return GroupQuantized(codes=q.codes.reshape(t, w), scales=q.scales.reshape(t, w // group),
                          zeros=q.zeros.reshape(t, w // group),
                          quotient=q.quotient.reshape(t, w),
                          zero_quotient=q.zero_quotient.reshape(t, w // group))


def dequant_groups_asym(q: GroupQuantized, group: int) -> np.ndarray:
    """s * (codes - zeros) per group, float64."""
    t, w = q.codes.shape
    s = np.repeat(np.asarray(q.scales, np.float64), group, axis=1)
    z = np.repeat(q.zeros.astype(np.float64), group, axis=1)
    return s * (q.codes.astype(np.float64) - z)


def kv_quantize(q: np.ndarray, k: np.ndarray, v: np.ndarray, head_dim: int, group: int = 128):
    """The online KV-cache step (R13): (q R3, Q_g(k R3), Q_g(v)); q, k, v
    are [tokens x heads*head_dim] after RoPE."""
    return (rotate_heads(q, head_dim), quantize_groups_asym(rotate_heads(k, head_dim), group),
            quantize_groups_asym(v, group))


# --------------------------------------------------------------------------
# Diagnostics used by the pins
# --------------------------------------------------------------------------

def rmsnorm(x: np.ndarray) -> np.ndarray:
    """x_i <- x_i / ||x_i|| per row, the no-rescale RMSNorm of [QS] §1."""
    x = np.asarray(x, np.float64)
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def incoherence_bound(w: np.ndarray, delta: float) -> float:
    """mu ||W||_F / sqrt(mn) with mu = 2 log(4mn/delta) ([SR] Jf43 W1/A1)."""
    m, n = w.shape
    mu = 2.0 * np.log(4.0 * m * n / delta)
    return mu * np.linalg.norm(w) / np.sqrt(m * n)
