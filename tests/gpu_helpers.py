"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the C ABI, and compare with the oracle under the
parity rules:

* int32 accumulators bit-exact given identical codes;
* rotated rows within 1e-5 of the row L2 norm;
* codes identical except where |x/s - round(x/s)| is within 1e-4 of 0.5;
* fp16 outputs within 2e-3 relative Frobenius error.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q

ROT_TOL = 1e-5
TIE_WINDOW = 1e-4
Y_TOL = 2e-3
SCALE_TOL = 2e-6

KIND = {O.NONE: Q.NONE, O.HADAMARD: Q.HADAMARD, O.GSR: Q.GSR, O.KRON: Q.KRON}


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def gpu_rotation(r: O.Rotation) -> Q.Rotation:
    """The CUDA-side descriptor of the same rotation (activation side)."""
    return Q.Rotation(KIND[r.kind], block=r.block if r.kind in (O.HADAMARD, O.GSR) else 1,
                      p1=None if r.P1 is None else dev(np.asarray(r.P1, np.float32)),
                      p2=None if r.P2 is None else dev(np.asarray(r.P2, np.float32)),
                      chan_scale=None if r.chan_scale is None else dev(np.asarray(r.chan_scale,
                                                                                 np.float32)),
                      clip_ratio=r.clip_ratio,
                      signs=None if r.signs is None else dev(np.asarray(r.signs, np.int8)))


def unpack(codes: torch.Tensor) -> np.ndarray:
    return O.unpack_int4(host(codes))


def check_side(gpu, ref: O.Side, what: str, clip: float = 1.0, check_rot: bool = True):
    """Compares (codes, scales, fp16 part, rotated) from the GPU with an oracle Side."""
    codes, scales, out16, rot = gpu
    scales = host(scales)
    if check_rot and rot is not None and ref.rotated.shape[1]:
        r = host(rot).astype(np.float64)
        norm = np.linalg.norm(ref.rotated, axis=1)
        err = np.abs(r - ref.rotated).max(axis=1)
        bad = err > ROT_TOL * np.maximum(norm, 1e-30)
        assert not bad.any(), (f"{what}: rotated rows off by up to "
                               f"{(err / np.maximum(norm, 1e-30)).max():.3g} of the row norm")
    # |max_gpu - max_ref| <= max_i |x_gpu,i - x_ref,i| <= ROT_TOL * ||x||, so the
    # scale alpha*max/7 may move by alpha*ROT_TOL*||x||/7 (plus fp32 rounding).
    ref_s = ref.q.scales.astype(np.float64)
    norm = np.linalg.norm(ref.rotated, axis=1)
    allowed = clip * ROT_TOL * norm / 7.0 + SCALE_TOL * ref_s
    off = np.abs(scales.astype(np.float64) - ref_s)
    assert np.all(off <= allowed), f"{what}: scales off by up to {(off / np.maximum(ref_s, 1e-30)).max():.3g}"
    got = unpack(codes)
    want = ref.q.codes
    assert got.shape == want.shape, (got.shape, want.shape)
    v = ref.q.quotient.astype(np.float64)
    frac = np.abs(v - np.rint(v))
    tie = np.abs(frac - 0.5) < TIE_WINDOW
    diff = got != want
    assert not (diff & ~tie).any(), (
        f"{what}: {int((diff & ~tie).sum())} codes differ outside the tie window")
    assert np.all(np.abs(got[diff] - want[diff]) <= 1)
    if out16 is not None:
        np.testing.assert_array_equal(host(out16).view(np.uint16),
                                      np.asarray(ref.fp16_part, np.float16).view(np.uint16))
    return int(diff.sum())


# Rotate + quantize calls with at most this many rows run one CTA per row;
# more rows run the row-group kernels.  Tests tile their rows past it to
# cover both.
FEW_ROWS = 148


def tile_rows(x: np.ndarray, min_rows: int = FEW_ROWS + 52) -> tuple[np.ndarray, int]:
    """x repeated row-wise to at least `min_rows` rows, and the repeat count."""
    reps = -(-min_rows // max(1, x.shape[0]))
    return np.tile(x, (reps, 1)), reps


def tile_side(ref: O.Side, reps: int) -> O.Side:
    """The oracle Side of rows repeated `reps` times."""
    t = lambda a: np.tile(a, (reps, 1)) if a.ndim == 2 else np.tile(a, reps)
    q = O.Quantized(codes=t(ref.q.codes), scales=t(ref.q.scales), quotient=t(ref.q.quotient))
    return O.Side(rotated=t(ref.rotated), q=q, packed=t(ref.packed), fp16_part=t(ref.fp16_part))


def check_side_asym(gpu, ref: O.Side, what: str, clip: float = 1.0):
    """Compares (codes, scales, zeros, fp16 part, rotated) from the GPU with an
    oracle Side of asymmetric activation codes (zero points exact except
    where -lo/s lies within the tie window of a half; such rows' codes are
    not compared)."""
    codes, scales, zeros, out16, rot = gpu
    q = ref.q
    if rot is not None and ref.rotated.shape[1]:
        r = host(rot).astype(np.float64)
        norm = np.linalg.norm(ref.rotated, axis=1)
        err = np.abs(r - ref.rotated).max(axis=1)
        assert not (err > ROT_TOL * np.maximum(norm, 1e-30)).any(), f"{what}: rotated rows off"
    norm = np.linalg.norm(ref.rotated, axis=1)
    ref_s = q.scales.astype(np.float64)
    allowed = clip * 2 * ROT_TOL * norm / 15.0 + SCALE_TOL * ref_s
    off = np.abs(host(scales).astype(np.float64) - ref_s)
    assert np.all(off <= allowed), f"{what}: scales off by up to {(off / np.maximum(ref_s, 1e-30)).max():.3g}"
    zq = q.zero_quotient.astype(np.float64)
    ztie = np.abs(np.abs(zq - np.rint(zq)) - 0.5) < TIE_WINDOW
    gz = host(zeros).astype(np.int64)
    assert np.array_equal(gz[~ztie], q.zeros.astype(np.int64)[~ztie]), f"{what}: zero points differ"
    got = unpack(codes)
    want = q.codes
    v = q.quotient.astype(np.float64)
    tie = (np.abs(np.abs(v - np.rint(v)) - 0.5) < TIE_WINDOW) | ztie[:, None]
    diff = got != want
    assert not (diff & ~tie).any(), f"{what}: {int((diff & ~tie).sum())} codes differ outside ties"
    if out16 is not None:
        np.testing.assert_array_equal(host(out16).view(np.uint16),
                                      np.asarray(ref.fp16_part, np.float16).view(np.uint16))
    return int(diff.sum())


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def oracle_rows_from_gpu_codes(a_codes, a_scales, w_codes, w_scales, x_out=None, w_out=None):
    """(acc, Y) the oracle computes from the GPU's codes and scales."""
    qa = unpack(a_codes)
    qw = unpack(w_codes)
    acc = O.int_gemm(qa, qw)
    y = O.dequant_epilogue(acc, host(a_scales), host(w_scales),
                           None if x_out is None else host(x_out),
                           None if w_out is None else host(w_out))
    return acc, y
