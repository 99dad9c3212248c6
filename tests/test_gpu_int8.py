"""GPU parity of the 8-bit layers (QUIK's INT8 down_proj and W8A8, oracle
reading R14) against the oracle, through the C ABI: 8-bit rotate + quantize
of activations and weights, the W8A8 linear with and without fp16 outlier
columns, and a whole INT8 down_proj-shaped layer."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q
import workloads
from tests.gpu_helpers import (ROT_TOL, SCALE_TOL, TIE_WINDOW, dev, gpu_rotation, host, rel_fro,
                               require_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    assert Q._lib.qr_device_status() == 0


def check_side8(gpu, ref: O.Side, what: str, clip: float = 1.0):
    """(codes int8, scales, fp16 part, rotated) from the GPU against an
    oracle Side with 8-bit codes, under the parity rules."""
    codes, scales, out16, rot = gpu
    r = host(rot).astype(np.float64)
    norm = np.linalg.norm(ref.rotated, axis=1)
    err = np.abs(r - ref.rotated).max(axis=1) if r.shape[1] else np.zeros(len(norm))
    assert not (err > ROT_TOL * np.maximum(norm, 1e-30)).any(), f"{what}: rotated rows off"
    ref_s = ref.q.scales.astype(np.float64)
    allowed = clip * ROT_TOL * norm / 127.0 + SCALE_TOL * ref_s
    off = np.abs(host(scales).astype(np.float64) - ref_s)
    assert np.all(off <= allowed), f"{what}: scales off"
    got = host(codes).astype(np.int64)
    want = ref.q.codes.astype(np.int64)
    assert got.shape == want.shape
    v = ref.q.quotient.astype(np.float64)
    tie = np.abs(np.abs(v - np.rint(v)) - 0.5) < TIE_WINDOW
    diff = got != want
    assert not (diff & ~tie).any(), f"{what}: {int((diff & ~tie).sum())} codes differ outside ties"
    assert np.all(np.abs(got[diff] - want[diff]) <= 1)
    assert got.min() >= -127 and got.max() <= 127
    if out16 is not None:
        np.testing.assert_array_equal(host(out16).view(np.uint16),
                                      np.asarray(ref.fp16_part, np.float16).view(np.uint16))


def _rows(rng, m, k, outl=(), scale=1.0):
    x = rng.standard_normal((m, k)).astype(np.float32) * scale
    for c in outl:
        x[:, c] *= 40
    return x.astype(np.float16)


ROW_CASES = [
    # (name, K, rotation, n_out, clip)
    ("none", 384, O.Rotation(O.NONE), 0, 1.0),
    ("had8", 256, O.Rotation(O.HADAMARD, block=8), 0, 1.0),
    ("gsr64", 640, O.Rotation(O.GSR, block=64), 0, 1.0),
    ("had256", 512, O.Rotation(O.HADAMARD, block=256), 0, 1.0),
    ("had4096", 4096, O.Rotation(O.HADAMARD, block=4096), 0, 1.0),
    ("gsr128_11008", 11008, O.Rotation(O.GSR, block=128), 0, 1.0),
    ("had128_outliers", 1000, O.Rotation(O.HADAMARD, block=128), 24, 1.0),
    ("gsr128_clip", 2048, O.Rotation(O.GSR, block=128, clip_ratio=0.9), 0, 0.9),
]


@pytest.mark.parametrize("name,K,rot,n_out,clip", ROW_CASES)
@pytest.mark.parametrize("rows", [5, 300])     # the few-rows kernel, then the row-group kernels
def test_rotate_quant8_matches_oracle(name, K, rot, n_out, clip, rows):
    rng = np.random.default_rng(K + rows)
    idx = np.sort(rng.choice(K, n_out, replace=False)).astype(np.int32) if n_out else None
    x = _rows(rng, rows, K, outl=tuple(rng.choice(K, 3, replace=False)))
    x[1] = 0                                               # an all-zero row: s = 0, codes 0
    grot = gpu_rotation(rot)
    gi = None if idx is None else dev(idx)
    for weights in (False, True):
        if weights:
            gpu = Q.pack_weights8(dev(x), Q.weight_rotation(grot), gi, debug=True)
            ref = O.quantize_weights(x.astype(np.float64), rot, idx, bits=8)
        else:
            gpu = Q.rotate_quant8(dev(x), grot, gi, debug=True)
            ref = O.quantize_activations(x.astype(np.float64), rot, idx, bits=8)
        torch.cuda.synchronize()
        check_side8(gpu, ref, f"{name} rows={rows} weights={weights}", clip)
        assert host(gpu[1])[1] == 0 and np.all(host(gpu[0])[1] == 0)


def test_rotate_quant8_random_signs():
    rng = np.random.default_rng(77)
    K = 4096
    signs = workloads.random_signs(5, K)
    rot = O.Rotation(O.HADAMARD, block=1024, signs=signs)
    x = _rows(rng, 40, K)
    gpu = Q.rotate_quant8(dev(x), gpu_rotation(rot), None, debug=True)
    torch.cuda.synchronize()
    check_side8(gpu, O.quantize_activations(x.astype(np.float64), rot, None, bits=8), "signs")


LINEAR8_CASES = [
    # (M, N, K, n_out)
    (1, 16, 128, 0), (7, 100, 256, 0), (128, 256, 512, 0), (129, 300, 384, 0),
    (200, 520, 384, 0), (300, 1000, 1024, 0), (257, 600, 11008, 0), (1000, 700, 256, 0),
    (4, 64, 256, 8), (100, 300, 384, 64), (256, 384, 256, 200), (130, 70, 0, 24),
    (2048, 640, 10368, 688), (65, 33, 0, 0),
]


@pytest.mark.parametrize("M,N,K,n_out", LINEAR8_CASES)
def test_linear8_matches_oracle(M, N, K, n_out):
    rng = np.random.default_rng(M * 1000 + N + K + 7)
    qa = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sa = rng.uniform(0.001, 0.02, M).astype(np.float32)
    sw = rng.uniform(0.0001, 0.001, N).astype(np.float32)
    xo = (rng.standard_normal((M, n_out)) * 3).astype(np.float16) if n_out else None
    wo = (rng.standard_normal((N, n_out)) * 0.02).astype(np.float16) if n_out else None
    y, acc = Q.w8a8_linear(dev(qa), dev(sa), dev(qw), dev(sw),
                           None if xo is None else dev(xo), None if wo is None else dev(wo),
                           acc_debug=True)
    torch.cuda.synchronize()
    want_acc = O.int_gemm(qa, qw)
    assert np.array_equal(host(acc).astype(np.int64), want_acc)
    want_y = O.dequant_epilogue(want_acc, sa, sw, xo, wo).astype(np.float64)
    got_y = host(y).astype(np.float64)
    ulp = np.maximum(np.abs(want_y), 2.0 ** -14) * 2.0 ** -10
    assert np.all(np.abs(got_y - want_y) <= ulp + 1e-3 * np.abs(want_y).max() * (n_out > 0))
    assert rel_fro(got_y, want_y) < 1e-3


def test_linear8_extreme_codes_are_exact():
    # all +-127 at the largest K: |acc| = 127^2 K = 1.06e9, inside int32
    K, M = 65536, 3
    a = np.full((M, K), 127, np.int8); a[1] = -127
    w = np.full((40, K), 127, np.int8); w[1::2, ::2] = -127
    y, acc = Q.w8a8_linear(dev(a), dev(np.ones(M, np.float32)), dev(w),
                           dev(np.ones(40, np.float32)), acc_debug=True)
    assert np.array_equal(host(acc).astype(np.int64), O.int_gemm(a, w))


def test_int8_down_proj_layer_end_to_end():
    # QUIK's INT8 down_proj: 688 fp16 outlier columns chosen on calibration
    # tokens, the other 10320 columns GSR-rotated in 128-blocks (padded to
    # 10368), 8-bit activations and weights
    wl = workloads.make_workload("down_proj_int8_11008", M=64, N=320)
    s = wl.spec
    idx = O.select_outliers(wl.X_calib, s.n_keep_fp16)
    rot = O.Rotation(O.GSR, block=s.block)
    a, ws, acc, y = O.linear_forward(wl.X.astype(np.float64), wl.W.astype(np.float64), rot, idx,
                                     bits=8)
    grot = gpu_rotation(rot)
    gidx = Q.select_outliers(dev(wl.X_calib), s.n_keep_fp16)
    assert np.array_equal(host(gidx), idx)
    wc, wsc, wo, _ = Q.pack_weights8(dev(wl.W), Q.weight_rotation(grot), gidx)
    ac, asc, xo, _ = Q.rotate_quant8(dev(wl.X), grot, gidx)
    gy, _ = Q.w8a8_linear(ac, asc, wc, wsc, xo, wo)
    torch.cuda.synchronize()
    assert rel_fro(host(gy), y) < 2e-3
    exact = wl.X.astype(np.float64) @ wl.W.astype(np.float64).T
    # 8 bits with the outliers kept: well inside the 4-bit error
    assert rel_fro(host(gy), exact) < 0.02
