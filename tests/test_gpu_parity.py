"""GPU parity of the CUDA path against the oracle on small seeded cases that
span several tiles and ragged tails, plus edge cases.  All calls go through
the C ABI (libqr.so)."""
import zlib

import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q
import workloads
from tests.gpu_helpers import (Y_TOL, check_side, check_side_asym, dev, gpu_rotation, host,
                               oracle_rows_from_gpu_codes, rel_fro, require_gpu, tile_rows,
                               tile_side, unpack)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    assert Q._lib.qr_device_status() == 0


def _rows(rng, m, k, scale=1.0, outl=()):
    x = rng.standard_normal((m, k)).astype(np.float32) * scale
    for c in outl:
        x[:, c] *= 40
    return x.astype(np.float16)


def _run_rows(x16, orot, idx=None, weights=False, many=False):
    """GPU and oracle results for the rows of x16; with `many`, the GPU call
    gets the rows repeated past the few-rows kernel's limit."""
    reps = 1
    x_run = x16
    if many:
        x_run, reps = tile_rows(x16)
    xg = dev(x_run)
    ig = None if idx is None else dev(np.asarray(idx, np.int32))
    grot = gpu_rotation(orot)
    if weights:
        gpu = Q.pack_weights(xg, Q.weight_rotation(grot), ig, debug=True)
        ref = O.quantize_weights(x16.astype(np.float64), orot, idx)
    else:
        gpu = Q.rotate_quant(xg, grot, ig, debug=True)
        ref = O.quantize_activations(x16.astype(np.float64), orot, idx)
    torch.cuda.synchronize()
    return gpu, (tile_side(ref, reps) if reps > 1 else ref)


# ---------------------------------------------------------------- rotate + quantize

ROW_CASES = [
    # (name, K, rows, rotation)
    ("had256", 256, 16, O.Rotation(O.HADAMARD, block=256)),
    ("had4096", 4096, 19, O.Rotation(O.HADAMARD, block=4096)),
    ("had8192_cross_warp", 8192, 5, O.Rotation(O.HADAMARD, block=8192)),
    ("had16384_cross_warp", 16384, 3, O.Rotation(O.HADAMARD, block=16384)),
    ("had_blocks2", 384, 9, O.Rotation(O.HADAMARD, block=2)),
    ("had_blocks8", 640, 9, O.Rotation(O.HADAMARD, block=8)),
    ("had_blocks64", 640, 9, O.Rotation(O.HADAMARD, block=64)),
    ("had_blocks512", 1536, 9, O.Rotation(O.HADAMARD, block=512)),
    ("had_blocks4096_two", 8192, 4, O.Rotation(O.HADAMARD, block=4096)),
    ("gsr128", 11008, 7, O.Rotation(O.GSR, block=128)),
    ("gsr2", 256, 5, O.Rotation(O.GSR, block=2)),
    ("gsr16", 384, 5, O.Rotation(O.GSR, block=16)),
    ("gsr256", 768, 5, O.Rotation(O.GSR, block=256)),
    ("none_ragged", 200, 11, O.Rotation(O.NONE)),
    ("none_long", 8192, 3, O.Rotation(O.NONE)),
    ("had_clip", 1024, 9, O.Rotation(O.HADAMARD, block=1024, clip_ratio=0.5)),
    ("had4096_clip", 4096, 5, O.Rotation(O.HADAMARD, block=4096, clip_ratio=0.8)),
    ("gsr_clip", 1024, 9, O.Rotation(O.GSR, block=128, clip_ratio=0.9)),
]


@pytest.mark.parametrize("name,K,rows,rot", ROW_CASES, ids=[c[0] for c in ROW_CASES])
@pytest.mark.parametrize("weights", [False, True], ids=["act", "wgt"])
@pytest.mark.parametrize("many", [False, True], ids=["few", "many"])
def test_rotate_quant_matches_oracle(name, K, rows, rot, weights, many):
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    x = _rows(rng, rows, K, outl=(3, K // 2))
    x[rows // 2] = 0                                 # an all-zero row
    gpu, ref = _run_rows(x, rot, weights=weights, many=many)
    check_side(gpu, ref, name, clip=rot.clip_ratio)
    assert host(gpu[1])[rows // 2] == 0 and not host(gpu[0])[rows // 2].any()


@pytest.mark.parametrize("many", [False, True], ids=["few", "many"])
def test_rotate_quant_unaligned_leading_dimension(many):
    rng = np.random.default_rng(1)
    full = _rows(rng, 6, 203)
    reps = 1
    if many:
        full, reps = tile_rows(full)
    x = dev(full)[:, :200]                           # ldx = 203: scalar loads
    rot = O.Rotation(O.HADAMARD, block=128)
    gpu = Q.rotate_quant(x, gpu_rotation(rot), debug=True)
    ref = O.quantize_activations(full[:6, :200].astype(np.float64), rot)
    check_side(gpu, tile_side(ref, reps) if reps > 1 else ref, "ldx203")


@pytest.mark.parametrize("K,n_out,block", [(300, 5, 64), (8192, 256, 4096), (1000, 40, 128),
                                           (256, 256, 128)])
def test_rotate_quant_with_outlier_columns(K, n_out, block):
    rng = np.random.default_rng(K + n_out)
    idx = np.sort(rng.choice(K, size=n_out, replace=False)).astype(np.int32)
    x = _rows(rng, 7, K, outl=idx[:3])
    rot = O.Rotation(O.HADAMARD, block=block)
    for weights in (False, True):
        for many in (False, True):
            gpu, ref = _run_rows(x, rot, idx, weights=weights, many=many)
            check_side(gpu, ref, f"outliers K={K} n_out={n_out} many={many}")


def test_kron_rotate_quant_small_factors():
    rng = np.random.default_rng(3)
    n1, n2 = 16, 8
    p1 = (np.eye(n1) + 0.3 * rng.standard_normal((n1, n1))).astype(np.float32)
    p2 = (np.eye(n2) + 0.3 * rng.standard_normal((n2, n2))).astype(np.float32)
    c = rng.uniform(0.5, 2.0, n1 * n2).astype(np.float32)
    rot = O.Rotation(O.KRON, P1=p1, P2=p2, chan_scale=c, clip_ratio=0.9)
    x = _rows(rng, 9, n1 * n2, outl=(5,))
    for weights in (False, True):
        gpu, ref = _run_rows(x, rot, weights=weights)
        check_side(gpu, ref, "kron16x8", clip=0.9)


def test_kron_flatquant_factors_with_outliers():
    wl = workloads.make_workload("flatquant_gate_up_8192", M=8, N=8)
    rot = O.Rotation(O.KRON, P1=wl.P1, P2=wl.P2, chan_scale=wl.chan_scale, clip_ratio=0.9)
    for x in (wl.X, wl.W):
        gpu, ref = _run_rows(x, rot, weights=x is wl.W)
        check_side(gpu, ref, "flatquant", clip=0.9)
    # Kronecker transform together with an outlier split: 8 fp16 columns + 8192 rotated
    rng = np.random.default_rng(4)
    idx = np.sort(rng.choice(8200, 8, replace=False)).astype(np.int32)
    x = _rows(rng, 5, 8200)
    gpu, ref = _run_rows(x, rot, idx)
    check_side(gpu, ref, "flatquant+outliers", clip=0.9)


def _kron_rows_any_magnitude(wl, m, rng):
    """Rows of every magnitude for the tensor-core Kronecker kernel: norms
    from ~1e-2 to ~1e5, a zero row, a constant row, and a row whose x/c
    exceeds the fp16 range (60000 on a channel with c < 0.9)."""
    x = rng.standard_normal((m, 8192)).astype(np.float32)
    x *= (10.0 ** rng.uniform(-4.0, 3.3, size=m)).astype(np.float32)[:, None]
    x[1] = 0.0
    x[2] = 0.75
    ch = int(np.argmin(wl.chan_scale))
    x[3, ch] = 60000.0
    return x.astype(np.float16)


@pytest.mark.parametrize("m", [1, 2, 3, 16, 2 * 148 * 3 + 1])
def test_kron_tc_rows_of_any_magnitude(m):
    # one token, one pair, a short pair, and three pairs on most CTAs with a
    # short last pair; per-token power-of-two normalization keeps every fp16
    # operand in range
    wl = workloads.make_workload("flatquant_gate_up_8192", M=8, N=8)
    rng = np.random.default_rng(1000 + m)
    x = _kron_rows_any_magnitude(wl, max(m, 4), rng)[:m]
    rot = O.Rotation(O.KRON, P1=wl.P1, P2=wl.P2, chan_scale=wl.chan_scale, clip_ratio=0.9)
    gpu, ref = _run_rows(x, rot)
    check_side(gpu, ref, f"kron tc m={m}", clip=0.9)
    gpu, ref = _run_rows(x, rot, weights=True)
    check_side(gpu, ref, f"kron tc weights m={m}", clip=0.9)


def test_kron_tc_factor_scales_and_no_channel_scale():
    # P1 and P2 far from unit scale (normalized by powers of two inside the
    # kernel), no per-channel scale, no clipping
    wl = workloads.make_workload("flatquant_gate_up_8192", M=40, N=8)
    p1 = (wl.P1 * np.float32(3e-3)).astype(np.float32)
    p2 = (wl.P2 * np.float32(250.0)).astype(np.float32)
    rot = O.Rotation(O.KRON, P1=p1, P2=p2, chan_scale=None, clip_ratio=1.0)
    gpu, ref = _run_rows(wl.X, rot)
    check_side(gpu, ref, "kron tc scaled factors")


def test_invert_transpose_matches_numpy():
    wl = workloads.make_workload("flatquant_gate_up_8192", M=1, N=1)
    for p in (wl.P1, wl.P2):
        q = host(Q.invert_transpose(dev(p)))
        want = np.linalg.inv(p.astype(np.float64)).T
        np.testing.assert_allclose(q, want, rtol=0, atol=1e-6 * np.abs(want).max())
    with pytest.raises(ValueError):
        Q.invert_transpose(dev(np.zeros((4, 4), np.float32)))


def test_select_outliers_matches_oracle():
    wl = workloads.make_workload("quik_decode_8192", with_weights=False)
    idx = host(Q.select_outliers(dev(wl.X_calib), 256))
    assert np.array_equal(idx, O.select_outliers(wl.X_calib, 256))
    rng = np.random.default_rng(5)
    x = rng.integers(-3, 4, size=(16, 1000)).astype(np.float16)   # many exact ties
    for k in (1, 7, 100, 1000):
        assert np.array_equal(host(Q.select_outliers(dev(x), k)), O.select_outliers(x, k))


# ---------------------------------------------------------------- W4A4 linear

LINEAR_CASES = [
    # (M, N, K, n_out)
    (1, 16, 128, 0), (7, 100, 256, 0), (16, 256, 640, 0), (33, 300, 384, 0), (64, 512, 256, 0),
    (65, 129, 128, 0), (128, 256, 512, 0), (200, 520, 384, 0), (300, 1000, 1024, 0),
    (4, 64, 256, 8), (16, 200, 512, 40), (64, 256, 256, 256), (100, 300, 384, 64),
    (256, 384, 256, 32), (3, 40, 0, 16), (130, 70, 0, 24),
    # two-SM tiles: 256-row pairs, widths 128 and 160, ragged edges, long K
    (257, 225, 384, 0), (512, 448, 1280, 0), (300, 1000, 11008, 0), (1000, 700, 256, 0),
    (100, 4096, 128, 0), (65, 33, 0, 0),
    # several tiles per CTA pair with an odd number of ring slots per tile,
    # with and without outliers (the outlier tile leaves two A stages)
    (2048, 7104, 640, 0), (1024, 4096, 640, 64),
    # decode: K split over 1, 2 or 4 CTAs; outlier steps only on the first
    (5, 12288, 256, 0), (33, 8192, 512, 0), (64, 384, 128, 256), (2, 1000, 2048, 32),
    (17, 130, 8192, 0), (16, 256, 128, 256),
]


@pytest.mark.parametrize("M,N,K,n_out", LINEAR_CASES)
def test_linear_matches_oracle(M, N, K, n_out):
    rng = np.random.default_rng(M * 1000 + N + K)
    qa = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
    qw = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    sa = rng.uniform(0.01, 0.2, M).astype(np.float32)
    sw = rng.uniform(0.001, 0.01, N).astype(np.float32)
    xo = (rng.standard_normal((M, n_out)) * 3).astype(np.float16) if n_out else None
    wo = (rng.standard_normal((N, n_out)) * 0.02).astype(np.float16) if n_out else None
    a_codes = dev(O.pack_int4(qa) if K else np.zeros((M, 0), np.uint8))
    w_codes = dev(O.pack_int4(qw) if K else np.zeros((N, 0), np.uint8))
    y, acc = Q.w4a4_linear(a_codes, dev(sa), w_codes, dev(sw),
                           None if xo is None else dev(xo), None if wo is None else dev(wo),
                           acc_debug=True)
    torch.cuda.synchronize()
    want_acc = O.int_gemm(qa, qw)
    assert np.array_equal(host(acc).astype(np.int64), want_acc)
    want_y = O.dequant_epilogue(want_acc, sa, sw, xo, wo).astype(np.float64)
    got_y = host(y).astype(np.float64)
    # fp32 epilogue vs float64: at most one fp16 rounding step apart
    ulp = np.maximum(np.abs(want_y), 2.0 ** -14) * 2.0 ** -10
    assert np.all(np.abs(got_y - want_y) <= ulp + 1e-3 * np.abs(want_y).max() * (n_out > 0))
    assert rel_fro(got_y, want_y) < 1e-3


@pytest.mark.parametrize("M", [2, 100])
def test_linear_extreme_codes_are_exact(M):
    # all +-7 at the largest K: |acc| = 49*K, the int32 headroom case
    K = 65536
    a = np.full((M, K), 7, np.int8); a[1::2] = -7
    w = np.full((32, K), 7, np.int8); w[1::2, ::2] = -7
    y, acc = Q.w4a4_linear(dev(O.pack_int4(a)), dev(np.ones(M, np.float32)),
                           dev(O.pack_int4(w)), dev(np.ones(32, np.float32)), acc_debug=True)
    assert np.array_equal(host(acc).astype(np.int64), O.int_gemm(a, w))


@pytest.mark.parametrize("M", [40, 100])
def test_linear_writes_into_strided_output(M):
    rng = np.random.default_rng(9)
    N, K = 96, 256
    qa = rng.integers(-7, 8, size=(M, K)); qw = rng.integers(-7, 8, size=(N, K))
    big = torch.full((M, N + 13), 7.0, dtype=torch.float16, device="cuda")
    out = big[:, 5:5 + N]                                   # ldy = N + 13, unaligned base
    Q.w4a4_linear(dev(O.pack_int4(qa)), dev(np.ones(M, np.float32)),
                  dev(O.pack_int4(qw)), dev(np.full(N, 0.5, np.float32)), out=out)
    torch.cuda.synchronize()
    want = O.dequant_epilogue(O.int_gemm(qa, qw), np.ones(M), np.full(N, 0.5))
    np.testing.assert_array_equal(host(out), want)
    assert np.all(host(big[:, :5]) == 7) and np.all(host(big[:, 5 + N:]) == 7)


# ---------------------------------------------------------------- end to end

E2E_CASES = [
    ("tiny_256", None, None),
    ("qkv_prefill_4096", 96, 512),
    ("down_proj_gsr_11008", 40, 384),
    ("flatquant_gate_up_8192", 24, 256),
]


def _oracle_rotation(wl):
    s = wl.spec
    if s.rotation == workloads.KRON:
        return O.Rotation(O.KRON, P1=wl.P1, P2=wl.P2, chan_scale=wl.chan_scale,
                          clip_ratio=s.clip_ratio)
    kind = {workloads.HADAMARD: O.HADAMARD, workloads.GSR: O.GSR, workloads.NONE: O.NONE}
    return O.Rotation(kind[s.rotation], block=s.block, clip_ratio=s.clip_ratio)


@pytest.mark.parametrize("name,M,N", E2E_CASES, ids=[c[0] for c in E2E_CASES])
def test_layer_end_to_end(name, M, N):
    wl = workloads.make_workload(name, M=M, N=N)
    rot = _oracle_rotation(wl)
    layer = Q.QuantizedLinear(dev(wl.W), gpu_rotation(rot))
    y = layer(dev(wl.X))
    torch.cuda.synchronize()
    a, ws, acc, y_ref = O.linear_forward(wl.X.astype(np.float64), wl.W.astype(np.float64), rot)
    assert rel_fro(host(y), y_ref) < Y_TOL
    # and the accumulators from the GPU's own codes are exact
    codes, scales, _, _ = Q.rotate_quant(dev(wl.X), gpu_rotation(rot))
    y2, acc2 = Q.w4a4_linear(codes, scales, layer.w_codes, layer.w_scales, acc_debug=True)
    acc_ref, y2_ref = oracle_rows_from_gpu_codes(codes, scales, layer.w_codes, layer.w_scales)
    assert np.array_equal(host(acc2).astype(np.int64), acc_ref)
    assert rel_fro(host(y2), y2_ref) < 1e-3


@pytest.mark.parametrize("M", workloads.DECODE_TOKENS)
def test_quik_decode_end_to_end(M):
    wl = workloads.make_workload("quik_decode_8192", M=M, N=1024)
    rot = _oracle_rotation(wl)
    idx = O.select_outliers(wl.X_calib, wl.spec.n_keep_fp16)
    idx_g = Q.select_outliers(dev(wl.X_calib), wl.spec.n_keep_fp16)
    layer = Q.QuantizedLinear(dev(wl.W), gpu_rotation(rot), idx_g)
    y = layer(dev(wl.X))
    torch.cuda.synchronize()
    _, _, _, y_ref = O.linear_forward(wl.X.astype(np.float64), wl.W.astype(np.float64), rot, idx)
    assert rel_fro(host(y), y_ref) < Y_TOL


@pytest.mark.parametrize("M", [1, 64])
def test_graphed_layer_matches_eager(M):
    # the CUDA-graph replay computes what the eager calls compute, bit for bit,
    # on fresh inputs copied in from pinned host memory
    wl = workloads.make_workload("quik_decode_8192", M=M, N=512)
    rot = _oracle_rotation(wl)
    idx_g = Q.select_outliers(dev(wl.X_calib), wl.spec.n_keep_fp16)
    layer = Q.QuantizedLinear(dev(wl.W), gpu_rotation(rot), idx_g)
    glin = Q.GraphedLinear(layer, M)
    rng = np.random.default_rng(M)
    for _ in range(2):
        x = (rng.standard_normal(wl.X.shape) * 0.5).astype(np.float16)
        y_graph = host(glin(torch.from_numpy(x).pin_memory())).copy()
        y_eager = host(layer(dev(x)))
        assert np.array_equal(y_graph.view(np.uint16), y_eager.view(np.uint16))
    with pytest.raises(ValueError):
        glin(dev(np.zeros((M + 1, wl.spec.K), np.float16)))


# ---------------------------------------------------------------- randomized Hadamard

SIGN_CASES = [
    # (name, K, rows, kind, block, n_out, clip)
    ("had4096", 4096, 9, O.HADAMARD, 4096, 0, 1.0),
    ("had64_clip", 640, 7, O.HADAMARD, 64, 0, 0.7),
    ("gsr128", 11008, 5, O.GSR, 128, 0, 1.0),
    ("had4096_outliers", 8192, 6, O.HADAMARD, 4096, 256, 1.0),
    ("had8", 256, 5, O.HADAMARD, 8, 0, 1.0),
]


@pytest.mark.parametrize("name,K,rows,kind,block,n_out,clip", SIGN_CASES,
                         ids=[c[0] for c in SIGN_CASES])
@pytest.mark.parametrize("many", [False, True], ids=["few", "many"])
def test_rotate_quant_random_signs(name, K, rows, kind, block, n_out, clip, many):
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    idx = np.sort(rng.choice(K, size=n_out, replace=False)).astype(np.int32) if n_out else None
    x = _rows(rng, rows, K, outl=(1,) if not n_out else idx[:2])
    probe = O.Rotation(kind, block=block, clip_ratio=clip)
    kp = O.packed_width(probe, K, n_out)
    rot = O.Rotation(kind, block=block, clip_ratio=clip, signs=workloads.random_signs(7, kp))
    for weights in (False, True):
        gpu, ref = _run_rows(x, rot, idx, weights=weights, many=many)
        check_side(gpu, ref, f"{name} signs", clip=clip)


def test_layer_random_signs_end_to_end():
    wl = workloads.make_workload("qkv_prefill_4096", M=96, N=512)
    kp = O.packed_width(O.Rotation(O.HADAMARD, block=4096), wl.spec.K)
    rot = O.Rotation(O.HADAMARD, block=4096, signs=workloads.random_signs(1, kp))
    layer = Q.QuantizedLinear(dev(wl.W), gpu_rotation(rot))
    y = layer(dev(wl.X))
    torch.cuda.synchronize()
    _, _, _, y_ref = O.linear_forward(wl.X.astype(np.float64), wl.W.astype(np.float64), rot)
    assert rel_fro(host(y), y_ref) < Y_TOL


# ---------------------------------------------------------------- asymmetric activations

ASYM_CASES = [
    # (name, K, rows, kind, block, n_out, clip)
    ("had4096", 4096, 9, O.HADAMARD, 4096, 0, 1.0),
    ("gsr128", 11008, 5, O.GSR, 128, 0, 1.0),
    ("had64_clip", 640, 7, O.HADAMARD, 64, 0, 0.8),
    ("none_ragged", 200, 6, O.NONE, 1, 0, 1.0),
    ("had4096_outliers", 8192, 6, O.HADAMARD, 4096, 256, 1.0),
    ("had8", 256, 5, O.HADAMARD, 8, 0, 1.0),
]


@pytest.mark.parametrize("name,K,rows,kind,block,n_out,clip", ASYM_CASES,
                         ids=[c[0] for c in ASYM_CASES])
@pytest.mark.parametrize("many", [False, True], ids=["few", "many"])
def test_rotate_quant_asym(name, K, rows, kind, block, n_out, clip, many):
    rng = np.random.default_rng(zlib.crc32(name.encode()) + 5)
    idx = np.sort(rng.choice(K, size=n_out, replace=False)).astype(np.int32) if n_out else None
    x = _rows(rng, rows, K, outl=(1,) if not n_out else idx[:2])
    x[0] = 0                                         # a zero row
    x[1] = np.abs(x[1]) + np.float16(1.0)            # a row far from zero
    rot = O.Rotation(kind, block=block, clip_ratio=clip)
    reps = 1
    x_run = x
    if many:
        x_run, reps = tile_rows(x)
    ig = None if idx is None else dev(idx)
    gpu = Q.rotate_quant_asym(dev(x_run), gpu_rotation(rot), ig, debug=True)
    torch.cuda.synchronize()
    ref = O.quantize_activations_asym(x.astype(np.float64), rot, idx)
    if reps > 1:
        codes, scales, zeros, out16, dbg = gpu
        rows0 = x.shape[0]
        for r in range(reps):
            sl = slice(r * rows0, (r + 1) * rows0)
            check_side_asym((codes[sl], scales[sl], zeros[sl], None if out16 is None else out16[sl],
                             dbg[sl]), ref, f"{name} asym copy {r}", clip=clip)
    else:
        check_side_asym(gpu, ref, f"{name} asym", clip=clip)
    assert host(gpu[1])[0] == 0


def test_weight_code_sums():
    rng = np.random.default_rng(4)
    q = rng.integers(-7, 8, size=(300, 1280)).astype(np.int8)
    got = host(Q.weight_code_sums(dev(O.pack_int4(q))))
    assert np.array_equal(got, q.astype(np.int64).sum(axis=1))


ASYM_LINEAR_CASES = [(1, 512, 1024, 0), (16, 8192, 512, 0), (64, 384, 256, 64), (40, 1000, 2048, 32),
                     (300, 1000, 1024, 0), (257, 225, 384, 32)]


@pytest.mark.parametrize("M,N,K,n_out", ASYM_LINEAR_CASES)
def test_linear_asym_matches_oracle(M, N, K, n_out):
    rng = np.random.default_rng(M * 7 + N + K)
    qa = rng.integers(-8, 8, size=(M, K)).astype(np.int8)
    qw = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    za = rng.integers(-20, 20, size=M).astype(np.int32)
    sa = rng.uniform(0.01, 0.2, M).astype(np.float32)
    sw = rng.uniform(0.001, 0.01, N).astype(np.float32)
    xo = (rng.standard_normal((M, n_out)) * 3).astype(np.float16) if n_out else None
    wo = (rng.standard_normal((N, n_out)) * 0.02).astype(np.float16) if n_out else None
    w_codes = dev(O.pack_int4(qw))
    sums = Q.weight_code_sums(w_codes)
    y, acc = Q.w4a4_linear_asym(dev(O.pack_int4(qa)), dev(sa), dev(za), w_codes, dev(sw), sums,
                                None if xo is None else dev(xo), None if wo is None else dev(wo),
                                acc_debug=True)
    torch.cuda.synchronize()
    assert np.array_equal(host(acc).astype(np.int64), O.int_gemm(qa, qw))
    aq = O.AsymQuantized(codes=qa, scales=sa, zeros=za, quotient=None, zero_quotient=None)
    a_side = O.Side(rotated=None, q=aq, packed=None,
                    fp16_part=xo if xo is not None else np.zeros((M, 0), np.float16))
    w_side = O.Side(rotated=None, q=O.Quantized(codes=qw, scales=sw, quotient=None), packed=None,
                    fp16_part=wo if wo is not None else np.zeros((N, 0), np.float16))
    _, want = O.linear_asym(a_side, w_side)
    assert rel_fro(host(y), want) < 1e-3


@pytest.mark.parametrize("name,M,N", [("quik_decode_8192", 1, 1024), ("quik_decode_8192", 64, 1024),
                                      ("qkv_prefill_4096", 96, 512)])
def test_layer_asym_end_to_end(name, M, N):
    wl = workloads.make_workload(name, M=M, N=N)
    rot = _oracle_rotation(wl)
    idx = idx_g = None
    if wl.spec.n_keep_fp16:
        idx = O.select_outliers(wl.X_calib, wl.spec.n_keep_fp16)
        idx_g = Q.select_outliers(dev(wl.X_calib), wl.spec.n_keep_fp16)
    layer = Q.QuantizedLinear(dev(wl.W), gpu_rotation(rot), idx_g, asym_activations=True)
    y = layer(dev(wl.X))
    torch.cuda.synchronize()
    _, _, _, y_ref = O.linear_forward_asym(wl.X.astype(np.float64), wl.W.astype(np.float64), rot,
                                           idx)
    assert rel_fro(host(y), y_ref) < Y_TOL
    g = Q.GraphedLinear(layer, M)
    y2 = host(g(torch.from_numpy(wl.X).pin_memory())).copy()
    assert np.array_equal(y2.view(np.uint16), host(y).view(np.uint16))

