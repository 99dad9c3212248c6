"""GPU parity of the fused decode step (qr_w4a4_linear_fused: rotate +
quantize of the M <= 64 token rows and the W4A4 GEMM in one kernel).

The fused kernel computes exactly what the two calls compute, so its codes,
scales, zero points, outlier copy and Y must equal theirs bit for bit; the
codes are also checked against the oracle under the usual parity rules, and
Y end to end against the oracle's layer.  Cases cover every rotation kind
the call takes, outlier columns, random signs, clipping, asymmetric
activations, ragged K and N, 1..64 tokens, and the full QUIK decode shape."""
import zlib

import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q
import workloads
from tests.gpu_helpers import (Y_TOL, check_side, check_side_asym, dev, gpu_rotation, host,
                               rel_fro, require_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    assert Q._lib.qr_device_status() == 0


def _inputs(name, M, K, N, n_out):
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, size=n_out, replace=False)).astype(np.int32) if n_out else None
    hot = idx[: max(1, n_out // 4)] if n_out else rng.choice(K, size=2, replace=False)
    x[:, hot] *= 30.0
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    return x.astype(np.float16), w, idx


def _same(a, b):
    a, b = host(a), host(b)
    return a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def _check_case(name, M, K, N, rot, n_out=0, asym=False):
    x, w, idx = _inputs(name, M, K, N, n_out)
    grot = gpu_rotation(rot)
    ig = None if idx is None else dev(idx)
    layer = Q.QuantizedLinear(dev(w), grot, ig, asym_activations=asym, fused_decode=False)
    xg = dev(x)
    sync = torch.zeros(2, dtype=torch.int32, device="cuda")
    y, codes, scales, zeros, x_out = Q.w4a4_linear_fused(
        xg, grot, ig, layer.w_codes, layer.w_scales, layer.w_out, layer.w_sums, asym, sync)
    # the two-call path on the same inputs
    if asym:
        c2, s2, z2, o2, _ = Q.rotate_quant_asym(xg, grot, ig)
        y2, _ = Q.w4a4_linear_asym(c2, s2, z2, layer.w_codes, layer.w_scales, layer.w_sums, o2,
                                   layer.w_out)
    else:
        c2, s2, o2, _ = Q.rotate_quant(xg, grot, ig)
        y2, _ = Q.w4a4_linear(c2, s2, layer.w_codes, layer.w_scales, o2, layer.w_out)
    torch.cuda.synchronize()
    assert _same(codes, c2), f"{name}: codes differ from the two-call path"
    assert _same(scales, s2), f"{name}: scales differ from the two-call path"
    if asym:
        assert _same(zeros, z2), f"{name}: zero points differ from the two-call path"
    if n_out:
        assert _same(x_out, o2), f"{name}: outlier copy differs from the two-call path"
    assert _same(y, y2), f"{name}: Y differs from the two-call path"
    # the grid barrier left its count at zero and counted one call
    assert host(sync).tolist() == [0, 1]
    # against the oracle: codes under the parity rules; Y from the GPU's own
    # codes through the oracle's integer product and epilogue; Y end to end
    x64, w64 = x.astype(np.float64), w.astype(np.float64)
    acc = O.int_gemm(O.unpack_int4(host(codes)), O.unpack_int4(host(layer.w_codes)))
    if asym:
        ref_a = O.quantize_activations_asym(x64, rot, idx)
        check_side_asym((codes, scales, zeros, x_out, None), ref_a, f"{name} fused", clip=rot.clip_ratio)
        acc = acc - (host(zeros).astype(np.int64)[:, None] *
                     host(layer.w_sums).astype(np.int64)[None, :])
        _, _, _, y_ref = O.linear_forward_asym(x64, w64, rot, idx)
    else:
        ref_a = O.quantize_activations(x64, rot, idx)
        check_side((codes, scales, x_out, None), ref_a, f"{name} fused", clip=rot.clip_ratio)
        _, _, _, y_ref = O.linear_forward(x64, w64, rot, idx)
    y_codes = O.dequant_epilogue(acc, host(scales), host(layer.w_scales),
                                 None if x_out is None else host(x_out),
                                 None if layer.w_out is None else host(layer.w_out))
    assert rel_fro(host(y), y_codes) < 1e-3, name
    if rot.kind != O.NONE:
        # (without a rotation the two x30 columns set every row's scale, and
        # one round-half tie, which the parity rules let either side take,
        # moves Y by a whole code step: the comparison would measure the tie)
        err = rel_fro(host(y), y_ref)
        assert err < Y_TOL, (name, err)


CASES = [
    # (name, M, K, N, rotation, n_out, asym)
    ("had4096_out256", 16, 8192, 384, O.Rotation(O.HADAMARD, block=4096), 256, False),
    ("had4096_one_token", 1, 4096, 256, O.Rotation(O.HADAMARD, block=4096), 0, False),
    ("had4096_64_tokens", 64, 4096, 512, O.Rotation(O.HADAMARD, block=4096), 0, False),
    ("had256_ragged_n", 33, 1024, 200, O.Rotation(O.HADAMARD, block=256), 0, False),
    ("had64_out_pad", 7, 1000, 640, O.Rotation(O.HADAMARD, block=64), 40, False),
    ("had1024_clip", 5, 2048, 256, O.Rotation(O.HADAMARD, block=1024, clip_ratio=0.8), 0, False),
    ("gsr128", 9, 11008, 256, O.Rotation(O.GSR, block=128), 0, False),
    ("gsr64_out", 3, 4096, 256, O.Rotation(O.GSR, block=64), 64, False),
    ("none_ragged_k", 4, 1030, 136, O.Rotation(O.NONE), 0, False),
    ("had4096_asym_out", 16, 8192, 384, O.Rotation(O.HADAMARD, block=4096), 256, True),
    ("gsr128_asym", 40, 4096, 256, O.Rotation(O.GSR, block=128), 0, True),
    ("had8192_row", 2, 8192, 128, O.Rotation(O.HADAMARD, block=8192), 0, False),
]


@pytest.mark.parametrize("name,M,K,N,rot,n_out,asym", CASES, ids=[c[0] for c in CASES])
def test_fused_matches_two_calls_and_oracle(name, M, K, N, rot, n_out, asym):
    _check_case(name, M, K, N, rot, n_out, asym)


def test_fused_random_signs():
    K = 4096
    probe = O.Rotation(O.HADAMARD, block=4096)
    kp = O.packed_width(probe, K, 0)
    rot = O.Rotation(O.HADAMARD, block=4096, signs=workloads.random_signs(3, kp))
    _check_case("had4096_signs", 12, K, 256, rot)


def test_fused_sync_words_are_reused():
    # consecutive calls on one pair of words: the count returns to zero and
    # the generation counts the calls; results repeat bit for bit
    x, w, _ = _inputs("reuse", 8, 4096, 256, 0)
    grot = gpu_rotation(O.Rotation(O.HADAMARD, block=4096))
    layer = Q.QuantizedLinear(dev(w), grot, fused_decode=False)
    sync = torch.zeros(2, dtype=torch.int32, device="cuda")
    xg = dev(x)
    ys = [host(Q.w4a4_linear_fused(xg, grot, None, layer.w_codes, layer.w_scales, sync=sync)[0])
          for _ in range(5)]
    torch.cuda.synchronize()
    assert host(sync).tolist() == [0, 5]
    for y in ys[1:]:
        assert np.array_equal(y.view(np.uint16), ys[0].view(np.uint16))


@pytest.mark.parametrize("M", workloads.DECODE_TOKENS)
def test_fused_quik_decode_full_size(M):
    # the benchmark's decode layer (K = N = 8192, 256 fp16 outlier columns)
    wl = workloads.make_workload("quik_decode_8192", M=M)
    s = wl.spec
    rot = O.Rotation(O.HADAMARD, block=s.block, clip_ratio=s.clip_ratio)
    grot = gpu_rotation(rot)
    idx_g = Q.select_outliers(dev(wl.X_calib), s.n_keep_fp16)
    idx = O.select_outliers(wl.X_calib, s.n_keep_fp16)
    layer = Q.QuantizedLinear(dev(wl.W), grot, idx_g, fused_decode=False)
    xg = dev(wl.X)
    y, codes, scales, _, x_out = Q.w4a4_linear_fused(xg, grot, idx_g, layer.w_codes,
                                                     layer.w_scales, layer.w_out)
    c2, s2, o2, _ = Q.rotate_quant(xg, grot, idx_g)
    y2, _ = Q.w4a4_linear(c2, s2, layer.w_codes, layer.w_scales, o2, layer.w_out)
    torch.cuda.synchronize()
    assert _same(codes, c2) and _same(scales, s2) and _same(x_out, o2)
    assert _same(y, y2)
    ref_a = O.quantize_activations(wl.X.astype(np.float64), rot, idx)
    check_side((codes, scales, x_out, None), ref_a, "quik decode fused", clip=rot.clip_ratio)
    cols = np.linspace(0, s.N - 1, 512).astype(int)
    ref_w = O.quantize_weights(wl.W[cols].astype(np.float64), rot, idx)
    _, y_ref = O.linear(ref_a, ref_w)
    assert rel_fro(host(y)[:, cols], y_ref) < Y_TOL


def test_layer_decode_runs_fused_and_graphs():
    # QuantizedLinear(fused_decode=True) takes the fused kernel for a decode
    # batch; eager and CUDA-graph replays agree with the two-call layer bit
    # for bit
    wl = workloads.make_workload("quik_decode_8192", M=16, N=512)
    s = wl.spec
    grot = gpu_rotation(O.Rotation(O.HADAMARD, block=s.block))
    idx_g = Q.select_outliers(dev(wl.X_calib), s.n_keep_fp16)
    w = dev(wl.W)
    fused = Q.QuantizedLinear(w, grot, idx_g, fused_decode=True)
    plain = Q.QuantizedLinear(w, grot, idx_g)
    xg = dev(wl.X)
    y_f = host(fused(xg)).copy()
    y_p = host(plain(xg)).copy()
    assert host(fused._sync).tolist()[1] >= 1        # the fused kernel ran
    assert np.array_equal(y_f.view(np.uint16), y_p.view(np.uint16))
    g = Q.GraphedLinear(fused, 16)
    y_g = host(g(torch.from_numpy(wl.X).pin_memory())).copy()
    assert np.array_equal(y_g.view(np.uint16), y_p.view(np.uint16))


def test_fused_unsupported_shapes_fall_back():
    # more than 64 tokens, or a Kronecker rotation: UNSUPPORTED, no launch
    x, w, _ = _inputs("fallback", 65, 1024, 128, 0)
    grot = gpu_rotation(O.Rotation(O.HADAMARD, block=1024))
    layer = Q.QuantizedLinear(dev(w), grot, fused_decode=False)
    assert Q.w4a4_linear_fused(dev(x), grot, None, layer.w_codes, layer.w_scales,
                               check=False) is None
    with pytest.raises(Q._lib.QrError):
        Q.w4a4_linear_fused(dev(x), grot, None, layer.w_codes, layer.w_scales)
