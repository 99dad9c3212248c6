"""GPU parity at the full layer sizes, in the launch configurations bench.py
times.  The whole layer runs on the GPU; the oracle checks sampled outputs
it can afford: sampled token rows covering every 256-row tile (and the
massive-activation token), sampled weight rows, the int32 accumulators of
the sampled token rows against ALL output columns (bit-exact, from the
GPU's own codes), and end-to-end outputs on the sampled rows x columns."""
import numpy as np
import pytest
import torch

import oracle as O
import w4a4_rotation_quantized_b200 as Q
import workloads
from tests.gpu_helpers import (Y_TOL, check_side, dev, gpu_rotation, host, rel_fro,
                               require_gpu, unpack)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    assert Q._lib.qr_device_status() == 0


def _rotation(wl):
    s = wl.spec
    if s.rotation == workloads.KRON:
        return O.Rotation(O.KRON, P1=wl.P1, P2=wl.P2, chan_scale=wl.chan_scale,
                          clip_ratio=s.clip_ratio)
    kind = {workloads.HADAMARD: O.HADAMARD, workloads.GSR: O.GSR, workloads.NONE: O.NONE}
    return O.Rotation(kind[s.rotation], block=s.block, clip_ratio=s.clip_ratio)


def _sample_rows(n, count, extra=()):
    rows = set(np.linspace(0, n - 1, count).astype(int).tolist()) | {n - 1} | set(extra)
    return np.array(sorted(r for r in rows if 0 <= r < n))


def _acc_rows(a_codes_rows, w_codes, chunk=4096):
    """Exact int32 accumulators of some token rows against all weight rows."""
    qa = O.unpack_int4(a_codes_rows)
    out = []
    for n0 in range(0, w_codes.shape[0], chunk):
        out.append(O.int_gemm(qa, O.unpack_int4(w_codes[n0:n0 + chunk])))
    return np.concatenate(out, axis=1)


def _run_full(name, M=None, row_samples=128, col_samples=512, outliers=False):
    wl = workloads.make_workload(name, M=M)
    s = wl.spec
    rot = _rotation(wl)
    grot = gpu_rotation(rot)
    idx = idx_g = None
    if outliers:
        idx = O.select_outliers(wl.X_calib, s.n_keep_fp16)
        idx_g = Q.select_outliers(dev(wl.X_calib), s.n_keep_fp16)
    xg = dev(wl.X)
    layer = Q.QuantizedLinear(dev(wl.W), grot, idx_g)
    a_codes, a_scales, x_out, x_rot = Q.rotate_quant(xg, grot, idx_g, debug=True)
    y, acc = Q.w4a4_linear(a_codes, a_scales, layer.w_codes, layer.w_scales, x_out, layer.w_out,
                           acc_debug=True)
    torch.cuda.synchronize()
    Mx = wl.X.shape[0]
    rows = _sample_rows(Mx, row_samples, [wl.massive_token])
    cols = _sample_rows(s.N, col_samples)
    rt = torch.as_tensor(rows, device="cuda")
    ct = torch.as_tensor(cols, device="cuda")

    # rotate + quantize of the sampled token rows
    ref_a = O.quantize_activations(wl.X[rows].astype(np.float64), rot, idx)
    check_side((a_codes[rt], a_scales[rt], None if x_out is None else x_out[rt],
                x_rot[rt]), ref_a, f"{name} activations", clip=rot.clip_ratio)
    # offline weight pack of the sampled weight rows
    ref_w = O.quantize_weights(wl.W[cols].astype(np.float64), rot, idx)
    check_side((layer.w_codes[ct], layer.w_scales[ct],
                None if layer.w_out is None else layer.w_out[ct], None), ref_w,
               f"{name} weights", clip=rot.clip_ratio)

    # bit-exact accumulators of the sampled rows against every column
    w_all = host(layer.w_codes)
    acc_ref = _acc_rows(host(a_codes[rt]), w_all)
    assert np.array_equal(host(acc[rt]).astype(np.int64), acc_ref)
    del acc
    # the dequantized outputs of those rows from the GPU's codes
    y_rows = host(y[rt])
    y_from_codes = O.dequant_epilogue(acc_ref, host(a_scales[rt]), host(layer.w_scales),
                                      None if x_out is None else host(x_out[rt]),
                                      None if layer.w_out is None else host(layer.w_out))
    assert rel_fro(y_rows, y_from_codes) < 1e-3
    # end to end on rows x columns, every step from the oracle
    _, y_ref = O.linear(ref_a, ref_w)
    err = rel_fro(y_rows[:, cols], y_ref)
    assert err < Y_TOL, err
    return err


def test_qkv_prefill_full_size():
    _run_full("qkv_prefill_4096")


def test_down_proj_gsr_full_size():
    _run_full("down_proj_gsr_11008")


def test_flatquant_gate_up_full_size():
    _run_full("flatquant_gate_up_8192", row_samples=64, col_samples=256)


@pytest.mark.parametrize("M", workloads.DECODE_TOKENS)
def test_quik_decode_full_size(M):
    _run_full("quik_decode_8192", M=M, row_samples=64, col_samples=512, outliers=True)
