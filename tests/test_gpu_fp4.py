"""GPU parity of the FP4 layers (e2m1 codes with a per-row scale, oracle
reading R15) against the oracle, through the C ABI: e2m1 rotate + quantize
of activations and weights, the FP4 linear on the tensor core's e2m1
operands with and without fp16 outlier columns, and a whole layer."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q
import workloads
from tests.gpu_helpers import (ROT_TOL, SCALE_TOL, TIE_WINDOW, dev, gpu_rotation, host, rel_fro,
                               require_gpu)

pytestmark = pytest.mark.gpu

# e2m1 rounding ties: midpoints of the grid {0, .5, 1, 1.5, 2, 3, 4, 6}
E2M1_TIES = (O.E2M1[1:] + O.E2M1[:-1]) / 2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    assert Q._lib.qr_device_status() == 0


def check_side_fp4(gpu, ref: O.Side, what: str, clip: float = 1.0):
    """(packed codes, scales, fp16 part, rotated) from the GPU against an
    oracle Side with e2m1 codes: code values equal except within the tie
    window of a grid midpoint, where they may be the two neighbours."""
    codes, scales, out16, rot = gpu
    r = host(rot).astype(np.float64)
    norm = np.linalg.norm(ref.rotated, axis=1)
    err = np.abs(r - ref.rotated).max(axis=1) if r.shape[1] else np.zeros(len(norm))
    assert not (err > ROT_TOL * np.maximum(norm, 1e-30)).any(), f"{what}: rotated rows off"
    ref_s = ref.q.scales.astype(np.float64)
    allowed = clip * ROT_TOL * norm / 6.0 + SCALE_TOL * ref_s
    assert np.all(np.abs(host(scales).astype(np.float64) - ref_s) <= allowed), f"{what}: scales off"
    got = O.e2m1_value(O.unpack_fp4(host(codes)))
    want = O.e2m1_value(ref.q.codes)
    assert got.shape == want.shape
    v = np.abs(ref.q.quotient.astype(np.float64))
    tie = (np.abs(v[..., None] - E2M1_TIES) < TIE_WINDOW).any(-1)
    diff = got != want
    assert not (diff & ~tie).any(), f"{what}: {int((diff & ~tie).sum())} codes differ outside ties"
    if diff.any():                                    # at a tie: one of the two neighbours
        grid = np.concatenate([-O.E2M1[::-1], O.E2M1])
        gi = np.searchsorted(grid, got[diff])
        wi = np.searchsorted(grid, want[diff])
        assert np.all(np.abs(gi - wi) <= 1)
    if out16 is not None:
        np.testing.assert_array_equal(host(out16).view(np.uint16),
                                      np.asarray(ref.fp16_part, np.float16).view(np.uint16))


def _rows(rng, m, k, outl=()):
    x = rng.standard_normal((m, k)).astype(np.float32)
    for c in outl:
        x[:, c] *= 40
    return x.astype(np.float16)


ROW_CASES = [
    # (name, K, rotation, n_out, clip)
    ("had4096", 4096, O.Rotation(O.HADAMARD, block=4096), 0, 1.0),
    ("had4096x2", 8192, O.Rotation(O.HADAMARD, block=4096), 0, 1.0),
    ("gsr128_11008", 11008, O.Rotation(O.GSR, block=128), 0, 1.0),
    ("gsr64", 640, O.Rotation(O.GSR, block=64), 0, 1.0),
    ("had256_clip", 512, O.Rotation(O.HADAMARD, block=256, clip_ratio=0.9), 0, 0.9),
    ("had128_outliers", 1000, O.Rotation(O.HADAMARD, block=128), 24, 1.0),
    ("gsr128_outliers", 11008, O.Rotation(O.GSR, block=128), 688, 1.0),
]


@pytest.mark.parametrize("name,K,rot,n_out,clip", ROW_CASES)
@pytest.mark.parametrize("rows", [5, 300])
def test_rotate_quant_fp4_matches_oracle(name, K, rot, n_out, clip, rows):
    rng = np.random.default_rng(K + rows + 1)
    idx = np.sort(rng.choice(K, n_out, replace=False)).astype(np.int32) if n_out else None
    x = _rows(rng, rows, K, outl=tuple(rng.choice(K, 3, replace=False)))
    x[1] = 0                                               # an all-zero row: s = 0, codes 0
    grot = gpu_rotation(rot)
    gi = None if idx is None else dev(idx)
    for weights in (False, True):
        if weights:
            gpu = Q.pack_weights_fp4(dev(x), Q.weight_rotation(grot), gi, debug=True)
            ref = O.quantize_weights_fp4(x.astype(np.float64), rot, idx)
        else:
            gpu = Q.rotate_quant_fp4(dev(x), grot, gi, debug=True)
            ref = O.quantize_activations_fp4(x.astype(np.float64), rot, idx)
        torch.cuda.synchronize()
        check_side_fp4(gpu, ref, f"{name} rows={rows} weights={weights}", clip)
        assert host(gpu[1])[1] == 0 and np.all(O.e2m1_value(O.unpack_fp4(host(gpu[0])[1])) == 0)


def test_rotate_quant_fp4_random_signs():
    rng = np.random.default_rng(78)
    K = 4096
    rot = O.Rotation(O.HADAMARD, block=4096, signs=workloads.random_signs(6, K))
    x = _rows(rng, 40, K)
    gpu = Q.rotate_quant_fp4(dev(x), gpu_rotation(rot), None, debug=True)
    torch.cuda.synchronize()
    check_side_fp4(gpu, O.quantize_activations_fp4(x.astype(np.float64), rot, None), "signs")


def test_rotate_quant_fp4_unsupported_blocks():
    x = dev(np.zeros((4, 1024), np.float16))
    with pytest.raises(Q._lib.QrError):
        Q.rotate_quant_fp4(x, gpu_rotation(O.Rotation(O.HADAMARD, block=1024)))


LINEAR_CASES = [
    # (M, N, K, n_out)
    (1, 16, 128, 0), (7, 100, 256, 0), (128, 256, 512, 0), (129, 300, 384, 0),
    (300, 1000, 1024, 0), (257, 600, 4096, 0), (1000, 700, 256, 0), (600, 520, 11008, 0),
    (4, 64, 256, 8), (100, 300, 384, 64), (256, 384, 256, 200), (130, 70, 0, 24),
]


@pytest.mark.parametrize("M,N,K,n_out", LINEAR_CASES)
def test_fp4_linear_matches_oracle(M, N, K, n_out):
    rng = np.random.default_rng(M * 1000 + N + K + 11)
    ca = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    sa = rng.uniform(0.001, 0.02, M).astype(np.float32)
    sw = rng.uniform(0.0001, 0.001, N).astype(np.float32)
    xo = (rng.standard_normal((M, n_out)) * 3).astype(np.float16) if n_out else None
    wo = (rng.standard_normal((N, n_out)) * 0.02).astype(np.float16) if n_out else None
    y, acc = Q.fp4_linear(dev(O.pack_fp4(ca)), dev(sa), dev(O.pack_fp4(cw)), dev(sw),
                          None if xo is None else dev(xo), None if wo is None else dev(wo),
                          acc_debug=True)
    torch.cuda.synchronize()
    want_acc = O.fp4_gemm(ca, cw)
    assert np.array_equal(host(acc).astype(np.float64), want_acc)
    want_y = O.dequant_epilogue(want_acc, sa, sw, xo, wo).astype(np.float64)
    got_y = host(y).astype(np.float64)
    ulp = np.maximum(np.abs(want_y), 2.0 ** -14) * 2.0 ** -10
    assert np.all(np.abs(got_y - want_y) <= ulp + 1e-3 * np.abs(want_y).max() * (n_out > 0))
    assert rel_fro(got_y, want_y) < 1e-3


def test_fp4_linear_extreme_codes_are_exact():
    # all +-6 at K = 65536: |acc| = 36 K = 2359296, exact in fp32
    K, M = 65536, 3
    a = np.full((M, K), 7, np.uint8); a[1] = 15
    w = np.full((40, K), 7, np.uint8); w[1::2, ::2] = 15
    y, acc = Q.fp4_linear(dev(O.pack_fp4(a)), dev(np.ones(M, np.float32)), dev(O.pack_fp4(w)),
                          dev(np.ones(40, np.float32)), acc_debug=True)
    assert np.array_equal(host(acc).astype(np.float64), O.fp4_gemm(a, w))


def test_fp4_layer_end_to_end():
    # the QKV layer shape (full 4096-point Hadamard), 64 tokens x 320 outputs
    wl = workloads.make_workload("qkv_prefill_4096", M=64, N=320)
    rot = O.Rotation(O.HADAMARD, block=4096)
    a, ws, acc, y = O.linear_forward_fp4(wl.X.astype(np.float64), wl.W.astype(np.float64), rot)
    grot = gpu_rotation(rot)
    wc, wsc, _, _ = Q.pack_weights_fp4(dev(wl.W), Q.weight_rotation(grot))
    ac, asc, _, _ = Q.rotate_quant_fp4(dev(wl.X), grot)
    gy, _ = Q.fp4_linear(ac, asc, wc, wsc)
    torch.cuda.synchronize()
    assert rel_fro(host(gy), y) < 2e-3
    exact = wl.X.astype(np.float64) @ wl.W.astype(np.float64).T
    assert rel_fro(host(gy), exact) < 0.2         # the oracle's own error here is 0.165
