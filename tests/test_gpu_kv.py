"""GPU parity of the KV-cache step (R3 on queries and keys, group-wise
asymmetric 4-bit keys and values) against the oracle, through the C ABI."""
import numpy as np
import pytest

import oracle as O
import w4a4_rotation_quantized_b200 as Q
from tests.gpu_helpers import ROT_TOL, check_side_asym, dev, host, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    assert Q._lib.qr_device_status() == 0


def _kv_inputs(seed, tokens, width, outl=()):
    """Seeded post-RoPE rows: N(0,1), a few large channels (keys carry them)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((tokens, width)).astype(np.float32)
    k = rng.standard_normal((tokens, width)).astype(np.float32)
    v = rng.standard_normal((tokens, width)).astype(np.float32)
    for c in outl:
        k[:, c] *= 20.0
        q[:, c] *= 3.0
    return q.astype(np.float16), k.astype(np.float16), v.astype(np.float16)


class _RowSide:
    """The oracle's group quantization seen as rows of one group each."""

    def __init__(self, g: O.GroupQuantized, rotated: np.ndarray, group: int):
        t, w = g.codes.shape
        rows = t * (w // group)
        self.q = O.AsymQuantized(codes=g.codes.reshape(rows, group),
                                 scales=g.scales.reshape(rows), zeros=g.zeros.reshape(rows),
                                 quotient=g.quotient.reshape(rows, group),
                                 zero_quotient=g.zero_quotient.reshape(rows))
        self.rotated = np.asarray(rotated, np.float64).reshape(rows, group)
        self.fp16_part = None


def _check_group_side(gpu, g, rotated, group, what):
    codes, scales, zeros = gpu
    rows = codes.shape[0] * codes.shape[1] * 2 // group
    check_side_asym((codes.view(rows, group // 2), scales.view(rows), zeros.view(rows), None, None),
                    _RowSide(g, rotated, group), what)


KV_CASES = [
    # tokens, heads, head_dim, group
    (5, 4, 128, 128),
    (37, 8, 64, 128),
    (3, 2, 128, 256),
    (1, 32, 128, 128),
    (129, 4, 256, 256),
    (64, 8, 32, 128),
    (1000, 2, 128, 128),          # 2000 groups: one pass of the warps
    # 40000 groups, more than the grid's warps x groups per warp (at most
    # sm_count * 8 blocks * 8 warps * 4 groups, 37888 on 148 SMs): the
    # grid-stride loop runs a second iteration with a ragged batch tail
    (20000, 2, 128, 128),
]


@pytest.mark.parametrize("tokens,heads,head_dim,group", KV_CASES)
def test_kv_quantize_matches_oracle(tokens, heads, head_dim, group):
    width = heads * head_dim
    q, k, v = _kv_inputs(tokens * 131 + width, tokens, width, outl=(1, width // 2 + 3))
    q_rot, ks, vs = Q.kv_quantize(dev(q), dev(k), dev(v), head_dim, group)
    ref_q, ref_k, ref_v = O.kv_quantize(q.astype(np.float64), k.astype(np.float64),
                                        v.astype(np.float64), head_dim, group)
    # q: fp16 of the rotated row (half an ulp) plus the fp32 rotation error
    got = host(q_rot).astype(np.float64)
    hn = np.repeat(np.linalg.norm(ref_q.reshape(tokens, heads, head_dim), axis=2), head_dim, axis=1)
    assert np.all(np.abs(got - ref_q) <= 2.0 ** -11 * np.abs(ref_q) + ROT_TOL * hn + 1e-7)
    _check_group_side(ks, ref_k, O.rotate_heads(k.astype(np.float64), head_dim), group, "keys")
    _check_group_side(vs, ref_v, v.astype(np.float64), group, "values")


def test_kv_quantize_parts_and_scores():
    tokens, heads, d = 48, 4, 128
    q, k, v = _kv_inputs(7, tokens, heads * d, outl=(5, 300))
    # keys only
    q_rot, ks, vs = Q.kv_quantize(None, dev(k), None, d)
    assert q_rot is None and vs is None
    ref_k = O.quantize_groups_asym(O.rotate_heads(k.astype(np.float64), d), 128)
    _check_group_side(ks, ref_k, O.rotate_heads(k.astype(np.float64), d), 128, "keys only")
    # scores from the GPU's rotated queries and dequantized keys track q k^T
    q_rot, ks, _ = Q.kv_quantize(dev(q), dev(k), None, d)
    gk = O.GroupQuantized(codes=O.unpack_int4(host(ks[0])), scales=host(ks[1]),
                          zeros=host(ks[2]), quotient=None, zero_quotient=None)
    k_hat = O.dequant_groups_asym(gk, 128)
    qr = host(q_rot).astype(np.float64)
    q64, k64 = q.astype(np.float64), k.astype(np.float64)
    for h in range(heads):
        sl = slice(h * d, (h + 1) * d)
        exact = q64[:, sl] @ k64[:, sl].T
        assert np.linalg.norm(qr[:, sl] @ k_hat[:, sl].T - exact) < 0.15 * np.linalg.norm(exact)


def test_kv_quantize_constant_and_zero_groups():
    tokens, heads, d = 4, 2, 128
    k = np.zeros((tokens, heads * d), np.float16)
    k[1, :128] = 1.5                     # constant group -> rotated: one spike
    v = np.zeros_like(k)
    v[2, 128:] = -2.0                    # constant group: s = 0, codes -8
    _, ks, vs = Q.kv_quantize(None, dev(k), dev(v), d)
    ref_k = O.quantize_groups_asym(O.rotate_heads(k.astype(np.float64), d), 128)
    _check_group_side(ks, ref_k, O.rotate_heads(k.astype(np.float64), d), 128, "keys")
    ref_v = O.quantize_groups_asym(v.astype(np.float64), 128)
    _check_group_side(vs, ref_v, v.astype(np.float64), 128, "values")
    assert host(vs[1])[2, 1] == 0 and np.all(O.unpack_int4(host(vs[0]))[2, 128:] == -8)
