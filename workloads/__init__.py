"""Seeded synthetic inputs for the online W4A4 rotated linear layer.

This module only draws inputs: activations X, weights W, the outlier-channel
injection that makes them hard to quantize, the calibration batch of the
QUIK-style workload, and the transform parameters (P1, P2, per-channel
scales c) that the FlatQuant-style layer takes as inputs.  It holds none of
the method's arithmetic -- no rotation, quantization, GEMM or outlier
selection -- so that both the CPU oracle and the CUDA path can draw from it
without sharing any of the computation they are compared on.

Shapes follow LLaMA-2-7B and LLaMA-3-70B linear layers.  The models and
their calibration datasets are not available, so seeded synthetic tensors
with the stated distributions stand in for them.  Values are drawn in
fp32/fp64 and rounded once to fp16; those fp16 tensors are the inputs of
record for both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

# rotation kinds, by name (the C ABI has its own integer enum)
HADAMARD = "hadamard"
GSR = "gsr"
KRON = "kron"
NONE = "none"


@dataclass(frozen=True)
class Spec:
    """Shape and distribution recipe of one synthetic linear-layer workload."""
    name: str
    M: int                      # tokens
    K: int                      # input features
    N: int                      # output features
    seed: int
    rotation: str               # HADAMARD / GSR / KRON / NONE
    block: int = 0              # Hadamard / Walsh block size (0 = whole row)
    clip_ratio: float = 1.0
    n_outlier_channels: int = 0
    outlier_scale: float = 1.0
    massive_token_scale: float = 0.0
    x_dist: str = "normal"      # normal / silu_gated / student_t3
    w_std: float = 0.02
    n1: int = 0                 # Kronecker factor sizes (KRON only)
    n2: int = 0
    n_keep_fp16: int = 0        # QUIK fp16 outlier columns selected by calibration
    calib_tokens: int = 0
    bits: int = 4               # code width of the layer (8: QUIK's INT8 layers)
    fp4: bool = False           # 4-bit codes are e2m1 values (FP4) instead of integers
    description: str = ""


SPECS = {
    "tiny_256": Spec(
        "tiny_256", M=16, K=256, N=256, seed=20261203, rotation=HADAMARD,
        block=256, n_outlier_channels=4, outlier_scale=50.0,
        description="single tiny linear: X[16x256] N(0,1) with 4 outlier "
                    "channels x50, W[256x256] N(0,0.02^2), full 256-point "
                    "Hadamard"),
    "qkv_prefill_4096": Spec(
        "qkv_prefill_4096", M=2048, K=4096, N=12288, seed=20261204,
        rotation=HADAMARD, block=4096, n_outlier_channels=16,
        outlier_scale=30.0, massive_token_scale=300.0,
        description="LLaMA-2-7B-shaped fused QKV prefill: X[2048x4096] "
                    "N(0,1), 16 outlier channels x30, one massive token x300;"
                    " W[12288x4096] N(0,0.02^2); full 4096-point Hadamard"),
    "down_proj_gsr_11008": Spec(
        "down_proj_gsr_11008", M=2048, K=11008, N=4096, seed=20261205,
        rotation=GSR, block=128, n_outlier_channels=32, outlier_scale=40.0,
        x_dist="silu_gated",
        description="LLaMA-2-7B-shaped down_proj: X[2048x11008] = "
                    "SiLU(A)*B, A,B N(0,1), 32 outlier channels x40; "
                    "W[4096x11008] N(0,0.02^2); 86 sequency-ordered "
                    "128x128 Walsh blocks"),
    "flatquant_gate_up_8192": Spec(
        "flatquant_gate_up_8192", M=4096, K=8192, N=57344, seed=20261206,
        rotation=KRON, n1=128, n2=64, clip_ratio=0.9,
        n_outlier_channels=64, outlier_scale=20.0, x_dist="student_t3",
        w_std=0.015,
        description="LLaMA-3-70B-shaped gate+up prefill: X[4096x8192] "
                    "Student-t(3), 64 outlier channels x20; W[57344x8192] "
                    "N(0,0.015^2); P1 128x128, P2 64x64 (random orthogonal "
                    "+ 0.05 N(0,1)), c ~ U(0.5,2), clip ratio 0.9"),
    "quik_decode_8192": Spec(
        "quik_decode_8192", M=64, K=8192, N=8192, seed=20261207,
        rotation=HADAMARD, block=4096, n_outlier_channels=256,
        outlier_scale=50.0, n_keep_fp16=256, calib_tokens=512,
        description="QUIK-style decode: tokens in {1,4,16,64}, K=N=8192, "
                    "256 outlier columns x50 kept fp16 (chosen on a 512-token "
                    "calibration batch), the other 7936 columns rotated by "
                    "4096-point Hadamard blocks"),
    "qkv_prefill_fp4_4096": Spec(
        "qkv_prefill_fp4_4096", M=2048, K=4096, N=12288, seed=20261204,
        rotation=HADAMARD, block=4096, n_outlier_channels=16,
        outlier_scale=30.0, massive_token_scale=300.0, fp4=True,
        description="the fused QKV prefill layer (same inputs as qkv_prefill_4096) "
                    "with e2m1 (FP4) codes for activations and weights, per-token "
                    "and per-channel fp32 scales, on the fp4 tensor-core operands"),
    "down_proj_int8_11008": Spec(
        "down_proj_int8_11008", M=2048, K=11008, N=4096, seed=20261209,
        rotation=GSR, block=128, n_outlier_channels=32, outlier_scale=40.0,
        x_dist="silu_gated", n_keep_fp16=688, calib_tokens=512, bits=8,
        description="QUIK's INT8 LLaMA-2-7B down_proj: X[2048x11008] = "
                    "SiLU(A)*B, 32 outlier channels x40; 688 fp16 outlier "
                    "columns (256 per 4096 inputs) chosen on a 512-token "
                    "calibration batch; the other 10320 columns GSR-rotated "
                    "in 128-blocks; 8-bit activations and weights; "
                    "W[4096x11008] N(0,0.02^2)"),
}

DECODE_TOKENS = (1, 4, 16, 64)


@dataclass
class Workload:
    spec: Spec
    X: np.ndarray                         # fp16 [M x K]
    W: Optional[np.ndarray]               # fp16 [N x K] (None if not drawn)
    P1: Optional[np.ndarray] = None       # fp32 [n1 x n1]
    P2: Optional[np.ndarray] = None       # fp32 [n2 x n2]
    chan_scale: Optional[np.ndarray] = None   # fp32 [K]
    X_calib: Optional[np.ndarray] = None  # fp16 [calib_tokens x K]
    outlier_channels: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    massive_token: int = -1


def _random_orthogonal(rng: np.random.Generator, n: int) -> np.ndarray:
    """Haar-like random orthogonal matrix (QR of a Gaussian, signs fixed)."""
    g = rng.standard_normal((n, n))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def make_workload(name: str, *, M: Optional[int] = None, with_weights: bool = True,
                  N: Optional[int] = None) -> Workload:
    """Draw the seeded inputs of workload `name`.

    M overrides the token count (rows are a prefix of the full draw only for
    the decode workload, whose eval batch is drawn at its maximum of 64
    tokens); N overrides the output width (a prefix of the weight rows).
    """
    s = SPECS[name]
    rng = np.random.default_rng(s.seed)
    K = s.K
    # Outlier channels and the massive-activation token come first so that
    # they do not depend on the sizes drawn afterwards.
    ch = np.sort(rng.choice(K, size=s.n_outlier_channels, replace=False)) \
        if s.n_outlier_channels else np.zeros(0, np.int64)
    m_full = s.M
    massive = int(rng.integers(m_full)) if s.massive_token_scale else -1

    def draw_x(rows: int, gen: np.random.Generator) -> np.ndarray:
        if s.x_dist == "normal":
            x = gen.standard_normal((rows, K), dtype=np.float32)
        elif s.x_dist == "silu_gated":
            a = gen.standard_normal((rows, K), dtype=np.float32)
            b = gen.standard_normal((rows, K), dtype=np.float32)
            x = (a / (1.0 + np.exp(-a))) * b
        elif s.x_dist == "student_t3":
            x = gen.standard_t(3.0, size=(rows, K)).astype(np.float32)
        else:
            raise ValueError(s.x_dist)
        if len(ch):
            x[:, ch] *= np.float32(s.outlier_scale)
        return x

    x = draw_x(m_full, np.random.default_rng([s.seed, 1]))
    if massive >= 0:
        x[massive, :] *= np.float32(s.massive_token_scale)
    X = x.astype(np.float16)
    if M is not None:
        if M > m_full:
            raise ValueError(f"{name}: M={M} exceeds the drawn {m_full} tokens")
        X = np.ascontiguousarray(X[:M])

    X_calib = None
    if s.calib_tokens:
        X_calib = draw_x(s.calib_tokens, np.random.default_rng([s.seed, 2])).astype(np.float16)

    W = None
    if with_weights:
        n_rows = s.N if N is None else N
        wr = np.random.default_rng([s.seed, 3])
        W = (wr.standard_normal((n_rows, K), dtype=np.float32) * np.float32(s.w_std)).astype(np.float16)

    P1 = P2 = c = None
    if s.rotation == KRON:
        pr = np.random.default_rng([s.seed, 4])
        P1 = (_random_orthogonal(pr, s.n1) + 0.05 * pr.standard_normal((s.n1, s.n1))).astype(np.float32)
        P2 = (_random_orthogonal(pr, s.n2) + 0.05 * pr.standard_normal((s.n2, s.n2))).astype(np.float32)
        c = pr.uniform(0.5, 2.0, size=K).astype(np.float32)

    return Workload(spec=s, X=X, W=W, P1=P1, P2=P2, chan_scale=c, X_calib=X_calib,
                    outlier_channels=ch, massive_token=massive)


def random_codes_rows(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """Integer codes in [-7, 7] with a +-7 in every row (for exactness pins)."""
    q = rng.integers(-7, 8, size=(rows, cols)).astype(np.int64)
    pos = rng.integers(cols, size=rows)
    q[np.arange(rows), pos] = np.where(rng.random(rows) < 0.5, 7, -7)
    return q


def random_signs(seed: int, k_p: int) -> np.ndarray:
    """A seeded random +-1 diagonal of length k_p (int8), the input of a
    randomized Hadamard rotation.  Drawn here so that both the oracle and the
    CUDA path receive the same signs."""
    rng = np.random.default_rng([seed, 99])
    return np.where(rng.random(k_p) < 0.5, -1, 1).astype(np.int8)


# --------------------------------------------------------------------------
# KV cache (the R3 rotation of queries and keys, group-wise KV quantization)
# --------------------------------------------------------------------------

@dataclass
class KVSpec:
    name: str
    tokens: int
    heads: int
    head_dim: int
    group: int
    seed: int
    n_outlier_channels: int      # key channels scaled by outlier_scale
    outlier_scale: float


KV_SPECS = {
    # LLaMA-2-7B attention: 32 heads of 128, a 2048-token prefill
    "kv_cache_llama2_7b": KVSpec("kv_cache_llama2_7b", tokens=2048, heads=32, head_dim=128,
                                 group=128, seed=20261208, n_outlier_channels=32,
                                 outlier_scale=20.0),
}


def make_kv(name: str, tokens: Optional[int] = None):
    """Seeded post-RoPE q, k, v (fp16 [tokens x heads*head_dim]): N(0,1), with
    a few key channels scaled up (the outlier channels rotation spreads)."""
    s = KV_SPECS[name]
    t = s.tokens if tokens is None else tokens
    w = s.heads * s.head_dim
    rng = np.random.default_rng(s.seed)
    ch = np.sort(rng.choice(w, size=s.n_outlier_channels, replace=False))
    g = np.random.default_rng([s.seed, 1])
    q = g.standard_normal((t, w), dtype=np.float32)
    k = g.standard_normal((t, w), dtype=np.float32)
    v = g.standard_normal((t, w), dtype=np.float32)
    k[:, ch] *= np.float32(s.outlier_scale)
    return s, q.astype(np.float16), k.astype(np.float16), v.astype(np.float16)
