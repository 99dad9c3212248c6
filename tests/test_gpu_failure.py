"""Failure detection on the GPU without a fault: a kernel's bounded wait on an
mbarrier that nothing arrives on runs out after a short limit, records its
code in the device status word and returns; the context stays usable.  The
wait is the routine every kernel of the library waits with."""
import time

import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q
from tests.gpu_helpers import check_side, dev, gpu_rotation, require_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_reports_and_recovers():
    require_gpu()
    L = Q._lib
    assert L.qr_device_status() == 0
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    L.qr_check_wait_timeout(2_000_000, stream)            # 2 ms
    code = L.qr_device_status()                            # synchronizes
    elapsed = time.perf_counter() - t0
    assert code == L.QR_DEV_TIMEOUT_SELFCHECK
    assert elapsed < 5.0
    assert L.qr_device_status() == 0                       # read once, then cleared
    # the first recorded code wins until it is read
    L.qr_check_wait_timeout(1000, stream)
    L.qr_check_wait_timeout(1000, stream)
    assert L.qr_device_status() == L.QR_DEV_TIMEOUT_SELFCHECK
    assert L.qr_device_status() == 0
    # the context still computes: a small rotate + quantize matches the oracle
    rng = np.random.default_rng(17)
    x = rng.standard_normal((5, 256)).astype(np.float16)
    rot = O.Rotation(O.HADAMARD, block=256)
    gpu = Q.rotate_quant(dev(x), gpu_rotation(rot), None, debug=True)
    torch.cuda.synchronize()
    check_side(gpu, O.quantize_activations(x.astype(np.float64), rot, None), "after the timeout")
    assert L.qr_device_status() == 0
