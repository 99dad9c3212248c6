"""GPU check of qr_w4a4_linear_fused_noalloc, the fused decode step with its
intermediate arrays and grid-barrier words in the library's own per-device
scratch.  Two calls in a row must give the Y that qr_w4a4_linear_fused gives
with caller-owned buffers, bit for bit: the second call shows that the first
left the scratch's barrier ready for reuse.  (This file is collected last,
so the scratch has seen no other call before its first use here.)"""
import zlib

import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q
from tests.gpu_helpers import dev, gpu_rotation, host, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    assert Q._lib.qr_device_status() == 0


CASES = [
    # (name, M, K, N, rotation, n_out, asym)
    ("had4096_out256", 16, 8192, 384, O.Rotation(O.HADAMARD, block=4096), 256, False),
    ("gsr128", 9, 11008, 256, O.Rotation(O.GSR, block=128), 0, False),
    ("had1024_asym", 64, 2048, 512, O.Rotation(O.HADAMARD, block=1024, clip_ratio=0.9), 0, True),
]


@pytest.mark.parametrize("name,M,K,N,rot,n_out,asym", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_fused_twice(name, M, K, N, rot, n_out, asym):
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, size=n_out, replace=False)).astype(np.int32) if n_out else None
    if n_out:
        x[:, idx[:8]] *= 30.0
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    grot = gpu_rotation(rot)
    ig = None if idx is None else dev(idx)
    layer = Q.QuantizedLinear(dev(w), grot, ig, asym_activations=asym)
    xg = dev(x.astype(np.float16))
    y_ref = Q.w4a4_linear_fused(xg, grot, ig, layer.w_codes, layer.w_scales, layer.w_out,
                                layer.w_sums, asym)[0]
    ys = [Q.w4a4_linear_fused_noalloc(xg, grot, ig, layer.w_codes, layer.w_scales, layer.w_out,
                                      layer.w_sums, asym) for _ in range(2)]
    torch.cuda.synchronize()
    want = host(y_ref).view(np.uint16)
    for i, y in enumerate(ys):
        assert np.array_equal(host(y).view(np.uint16), want), f"{name}: call {i + 1} differs"
