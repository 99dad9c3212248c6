"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test fixes one part of the oracle against a hand-worked fixture
(tests/golden), a closed form, an invariant from the pages, or an
independent algorithm (a butterfly transform, brute-force loops), chosen so
that a dropped term, a wrong sign or index, or a transposed operand fails.
"""
import numpy as np
import pytest

import oracle as O
import workloads
from tests.conftest import read_golden_rows


def _golden_matrix(name):
    return np.array([[float(v) for v in r] for r in read_golden_rows(name)])


# ---------------------------------------------------------------- Hadamard

def test_hadamard_matches_textbook_h4():
    assert np.array_equal(O.hadamard(4), _golden_matrix("hadamard4.txt"))


@pytest.mark.parametrize("n", [1, 2, 8, 64, 1024])
def test_hadamard_closed_form_entries(n):
    # Sylvester order has H[i, j] = (-1)^popcount(i & j).
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    assert np.array_equal(O.hadamard(n), np.where(pc % 2 == 0, 1.0, -1.0))


@pytest.mark.parametrize("n", [1, 2, 4, 16, 128, 2048])
def test_hadamard_orthogonal(n):
    h = O.hadamard(n)
    assert np.array_equal(h @ h.T, n * np.eye(n))


def _fwht(x):
    """Independent radix-2 butterfly transform along the last axis (unscaled)."""
    x = np.array(x, dtype=np.float64)
    n = x.shape[-1]
    hlen = 1
    while hlen < n:
        y = x.reshape(x.shape[:-1] + (n // (2 * hlen), 2, hlen))
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :], y[..., 1, :] = a + b, a - b
        x = y.reshape(x.shape)
        hlen *= 2
    return x


@pytest.mark.parametrize("n", [2, 8, 32, 64, 4096])
def test_dense_hadamard_rotation_equals_butterfly(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((3, n))
    rot = O.Rotation(O.HADAMARD, block=n)
    np.testing.assert_allclose(O.rotate_activations(x, rot), _fwht(x) / np.sqrt(n),
                               rtol=0, atol=1e-12 * np.sqrt(n))


def test_block_diagonal_hadamard_acts_per_block():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 8192))
    rot = O.Rotation(O.HADAMARD, block=4096)
    y = O.rotate_activations(x, rot)
    np.testing.assert_allclose(y[:, :4096], _fwht(x[:, :4096]) / 64, atol=1e-11)
    np.testing.assert_allclose(y[:, 4096:], _fwht(x[:, 4096:]) / 64, atol=1e-11)


# ---------------------------------------------------------------- Walsh / GSR

def test_walsh_matches_textbook_order8():
    assert np.array_equal(O.walsh_sequency(8), _golden_matrix("walsh8_sequency.txt"))


@pytest.mark.parametrize("n", [2, 4, 16, 128, 1024])
def test_walsh_row_i_has_i_sign_changes(n):
    w = O.walsh_sequency(n)
    assert [O.sign_changes(r) for r in w] == list(range(n))


def _bitrev(v, bits):
    return int(format(v, f"0{bits}b")[::-1], 2) if bits else 0


@pytest.mark.parametrize("n", [2, 8, 128, 512])
def test_walsh_is_gray_bitreversed_hadamard_and_symmetric(n):
    # Textbook: sequency index i corresponds to natural index bitrev(gray(i)).
    bits = n.bit_length() - 1
    h = O.hadamard(n)
    w = O.walsh_sequency(n)
    perm = [_bitrev(i ^ (i >> 1), bits) for i in range(n)]
    assert np.array_equal(w, h[perm])
    assert np.array_equal(w, w.T)
    assert np.array_equal(w @ w.T, n * np.eye(n))


def test_gsr_rotation_is_blockwise_permuted_fwht():
    rng = np.random.default_rng(2)
    b, nb = 128, 86
    x = rng.standard_normal((2, b * nb))
    y = O.rotate_activations(x, O.Rotation(O.GSR, block=b))
    perm = [_bitrev(i ^ (i >> 1), 7) for i in range(b)]
    for blk in (0, 41, 85):
        z = _fwht(x[:, blk * b:(blk + 1) * b]) / np.sqrt(b)
        np.testing.assert_allclose(y[:, blk * b:(blk + 1) * b], z[:, perm], atol=1e-12)


# ---------------------------------------------------------------- Kronecker

def test_kron_of_hadamards_is_the_8192_hadamard():
    # H_128 (x) H_64 = H_8192 in Sylvester order: pins the x (P1 (x) P2)
    # index convention mat(x)[a, b] = x[a*n2 + b].
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 8192))
    kron = O.Rotation(O.KRON, P1=O.hadamard(128) / np.sqrt(128), P2=O.hadamard(64) / 8.0)
    had = O.Rotation(O.HADAMARD, block=8192)
    np.testing.assert_allclose(O.rotate_activations(x, kron), O.rotate_activations(x, had),
                               atol=1e-11)


def test_kron_factored_form_equals_dense_kron_product():
    rng = np.random.default_rng(4)
    p1, p2 = rng.standard_normal((4, 4)), rng.standard_normal((8, 8))
    x = rng.standard_normal((5, 32))
    rot = O.Rotation(O.KRON, P1=p1, P2=p2)
    np.testing.assert_allclose(O.rotate_activations(x, rot), x @ np.kron(p1, p2), rtol=1e-12,
                               atol=1e-12)


def test_kron_identity_factors_are_no_rotation():
    x = np.random.default_rng(5).standard_normal((3, 64))
    rot = O.Rotation(O.KRON, P1=np.eye(8), P2=np.eye(8))
    np.testing.assert_array_equal(O.rotate_activations(x, rot), x)


def test_kron_affine_pair_preserves_the_product():
    # X' = (X / c)(P1 (x) P2), W' = (W c)(P1 (x) P2)^{-T}  =>  X' W'^T = X W^T.
    wl = workloads.make_workload("flatquant_gate_up_8192", M=4, N=6)
    rot = O.Rotation(O.KRON, P1=wl.P1, P2=wl.P2, chan_scale=wl.chan_scale, clip_ratio=0.9)
    x, w = wl.X.astype(np.float64), wl.W.astype(np.float64)
    xr, wr = O.rotate_activations(x, rot), O.rotate_weights(w, rot)
    ref = x @ w.T
    np.testing.assert_allclose(xr @ wr.T, ref, rtol=0, atol=1e-9 * np.abs(ref).max())


# ---------------------------------------------------------------- invariance

@pytest.mark.parametrize("kind,block,k", [(O.HADAMARD, 256, 256), (O.HADAMARD, 64, 512),
                                          (O.GSR, 128, 1024)])
def test_computational_invariance(kind, block, k):
    rng = np.random.default_rng(6)
    x, w = rng.standard_normal((8, k)), rng.standard_normal((16, k))
    rot = O.Rotation(kind, block=block)
    xr, wr = O.rotate_activations(x, rot), O.rotate_weights(w, rot)
    np.testing.assert_allclose(xr @ wr.T, x @ w.T, rtol=1e-12, atol=1e-12 * np.abs(x @ w.T).max())
    np.testing.assert_allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


def test_rmsnorm_hand_worked_rows():
    # x_i <- x_i / ||x_i|| per row (the QuaRot/SpinQuant notes, §1): fixes the
    # value, which the commutation identity below cannot (any row-wise
    # normalisation, the identity map included, commutes with Q).
    from fractions import Fraction
    for r in read_golden_rows("rmsnorm_3x3.txt"):
        x = np.array([[float(v) for v in r[:3]]])
        want = np.array([[float(Fraction(v)) for v in r[3:]]])
        np.testing.assert_allclose(O.rmsnorm(x), want, rtol=0, atol=1e-15)


def test_rmsnorm_commutes_with_rotation():
    # RMSNorm(X) = RMSNorm(X Q^T) Q for orthogonal Q (the QuaRot/SpinQuant notes, §1).
    rng = np.random.default_rng(7)
    x = rng.standard_normal((4, 128))
    q = O.dense_rotation(O.Rotation(O.GSR, block=64), 128)
    np.testing.assert_allclose(O.rmsnorm(x @ q.T) @ q, O.rmsnorm(x), atol=1e-13)


def test_zero_padding_is_exact():
    rng = np.random.default_rng(8)
    x, w = rng.standard_normal((3, 7936)), rng.standard_normal((5, 7936))
    rot = O.Rotation(O.HADAMARD, block=4096)
    xp, wp = O.pad_columns(x, 8192), O.pad_columns(w, 8192)
    got = O.rotate_activations(xp, rot) @ O.rotate_weights(wp, rot).T
    np.testing.assert_allclose(got, x @ w.T, rtol=1e-12, atol=1e-10)


# ---------------------------------------------------------------- quantizer

def test_quantizer_hand_example():
    rows = read_golden_rows("quantizer_1x8.txt")
    x = np.array([[float(v) for v in rows[0][1:]]])
    for r in rows[1:]:
        alpha, scale = float(r[1]), float(r[3])
        codes = [int(v) for v in r[5:]]
        q = O.quantize_rows(x, alpha)
        assert q.scales[0] == np.float32(scale)
        assert q.codes[0].tolist() == codes


def test_quantizer_properties():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((64, 256)) * rng.uniform(0.01, 100, size=(64, 1))
    x[3] = 0.0
    q = O.quantize_rows(x, 1.0)
    assert q.codes.min() >= -7 and q.codes.max() <= 7
    assert q.scales[3] == 0 and not q.codes[3].any()
    nz = np.arange(64) != 3
    assert np.all(np.abs(q.codes[nz]).max(axis=1) == 7)
    err = np.abs(x[nz] - q.scales[nz, None].astype(np.float64) * q.codes[nz])
    assert np.all(err <= 0.5 * q.scales[nz, None] * (1 + 1e-6))


def test_quantizer_clips_beyond_alpha():
    x = np.array([[10.0, -10.0, 1.0, 0.0]])
    q = O.quantize_rows(x, 0.5)        # s = 0.5 * 10 / 7
    assert q.codes[0].tolist() == [7, -7, 1, 0]
    assert np.isclose(q.scales[0], 5.0 / 7.0)


def test_pack_hand_example_and_roundtrip():
    rows = read_golden_rows("pack_int4.txt")
    codes = np.array([[int(v) for v in rows[0][1:]]])
    expect = np.array([[int(v, 16) for v in rows[1][1:]]], dtype=np.uint8)
    assert np.array_equal(O.pack_int4(codes), expect)
    assert np.array_equal(O.unpack_int4(expect), codes)
    q = np.random.default_rng(10).integers(-7, 8, size=(5, 64))
    assert np.array_equal(O.unpack_int4(O.pack_int4(q)), q)


# ---------------------------------------------------------------- GEMM, epilogue

def test_int_gemm_equals_brute_force():
    rng = np.random.default_rng(11)
    for m, n, k in [(1, 1, 2), (3, 5, 7), (7, 4, 33)]:
        a = rng.integers(-7, 8, size=(m, k))
        w = rng.integers(-7, 8, size=(n, k))
        brute = [[sum(int(a[i, t]) * int(w[j, t]) for t in range(k)) for j in range(n)]
                 for i in range(m)]
        assert O.int_gemm(a, w).tolist() == brute


def test_int_gemm_extremes_exact():
    k = 11008
    a = np.full((2, k), 7)
    a[1] = -7
    w = np.full((3, k), -7)
    w[2, ::2] = 7
    acc = O.int_gemm(a, w)
    assert acc[0, 0] == -49 * k and acc[1, 0] == 49 * k and acc[0, 2] == 0


def test_epilogue_hand_example():
    acc = np.array([[10, -3], [0, 2048]])
    sa = np.array([0.5, 2.0 ** -11], np.float32)
    sw = np.array([0.25, 1.0], np.float32)
    y = O.dequant_epilogue(acc, sa, sw)
    # 10*.5*.25 = 1.25 ; -3*.5 = -1.5 ; 0 ; 2048*2^-11 = 1
    assert y.tolist() == [[1.25, -1.5], [0.0, 1.0]]
    # fp16 round-half-even: 1 + 2^-11 is a tie between 1 and 1 + 2^-10
    y = O.dequant_epilogue(np.array([[2049]]), np.array([2.0 ** -11]), np.array([1.0]))
    assert y[0, 0] == np.float16(1.0)
    # outlier product is added: 1*2 + 3*4 = 14
    y = O.dequant_epilogue(np.array([[4]]), np.array([1.0]), np.array([1.0]),
                           np.array([[1.0, 3.0]]), np.array([[2.0, 4.0]]))
    assert y[0, 0] == 18.0


# ---------------------------------------------------------------- QUIK outliers

def test_select_outliers_hand_example_ties_to_lower_index():
    x = np.array([[3.0, -5.0, 5.0, 1.0], [0.0, 1.0, -2.0, 0.5]])
    assert O.select_outliers(x, 2).tolist() == [1, 2]
    assert O.select_outliers(x, 1).tolist() == [1]
    assert O.select_outliers(x, 3).tolist() == [0, 1, 2]


def test_select_outliers_recovers_injected_columns():
    wl = workloads.make_workload("quik_decode_8192", with_weights=False)
    idx = O.select_outliers(wl.X_calib, 256)
    assert np.array_equal(idx, np.sort(wl.outlier_channels))


def test_outlier_split_partitions_the_product():
    rng = np.random.default_rng(12)
    x, w = rng.standard_normal((4, 40)), rng.standard_normal((6, 40))
    idx = np.array([3, 17, 18, 39])
    xi, xo = O.split_outliers(x, idx)
    wi, wo = O.split_outliers(w, idx)
    assert xi.shape == (4, 36) and xo.shape == (4, 4)
    np.testing.assert_allclose(xi @ wi.T + xo @ wo.T, x @ w.T, atol=1e-12)
    assert np.array_equal(xo, x[:, idx])


# ---------------------------------------------------------------- end to end

def _exact_case(kind, k, rng, clip=1.0, n_out=0):
    """X, W built so that the rotated rows are integer codes with absmax 7."""
    m, n = 6, 10
    qa = workloads.random_codes_rows(rng, m, k)
    qw = workloads.random_codes_rows(rng, n, k)
    if kind == O.KRON:
        n1, n2 = 8, k // 8
        p1 = rng.standard_normal((n1, n1)) + 3 * np.eye(n1)
        p2 = rng.standard_normal((n2, n2)) + 3 * np.eye(n2)
        c = rng.uniform(0.5, 2.0, size=k)
        rot = O.Rotation(O.KRON, P1=p1, P2=p2, chan_scale=c, clip_ratio=clip)
        p = np.kron(p1, p2)
        x = (qa @ np.linalg.inv(p)) * c[None, :]          # (x / c) P = qa
        w = (qw @ p.T) / c[None, :]                        # (w c) P^{-T} = qw
    else:
        rot = O.Rotation(kind, block=32 if kind == O.GSR else 64, clip_ratio=clip)
        r = O.dense_rotation(rot, k)
        x, w = qa @ r.T, qw @ r.T                          # x R = qa, w R = qw
    xo = wo = None
    idx = None
    if n_out:
        idx = np.sort(rng.choice(k + n_out, size=n_out, replace=False))
        keep = np.setdiff1d(np.arange(k + n_out), idx)
        xf = np.zeros((m, k + n_out)); xf[:, keep] = x
        wf = np.zeros((n, k + n_out)); wf[:, keep] = w
        xo = rng.integers(-4, 5, size=(m, n_out)).astype(np.float64)
        wo = rng.integers(-4, 5, size=(n, n_out)).astype(np.float64)
        xf[:, idx] = xo; wf[:, idx] = wo
        x, w = xf, wf
    return rot, x, w, qa, qw, idx, xo, wo


@pytest.mark.parametrize("kind", [O.NONE, O.HADAMARD, O.GSR, O.KRON])
def test_end_to_end_on_exactly_representable_rows(kind):
    rng = np.random.default_rng(13)
    rot, x, w, qa, qw, _, _, _ = _exact_case(kind, 128, rng)
    a, ws, acc, y = O.linear_forward(x, w, rot)
    assert np.array_equal(a.q.codes, qa) and np.array_equal(ws.q.codes, qw)
    np.testing.assert_allclose(a.q.scales, 1.0, rtol=1e-6)
    assert np.array_equal(acc, qa @ qw.T)
    np.testing.assert_array_equal(y, (qa @ qw.T).astype(np.float16))


def test_end_to_end_with_outliers_and_padding():
    rng = np.random.default_rng(14)
    # 128 rotated columns + 8 fp16 outlier columns; hadamard blocks of 64
    rot, x, w, qa, qw, idx, xo, wo = _exact_case(O.HADAMARD, 128, rng, n_out=8)
    a, ws, acc, y = O.linear_forward(x, w, rot, idx)
    assert np.array_equal(a.q.codes, qa) and np.array_equal(ws.q.codes, qw)
    np.testing.assert_array_equal(y, (qa @ qw.T + xo @ wo.T).astype(np.float16))


def test_end_to_end_clip_ratio_maps_codes():
    # alpha = 0.9: s = 0.9, codes = clamp(rne(q / 0.9), -7, 7) -> 0..7 map to 0,1,2,3,4,6,7,7
    rng = np.random.default_rng(15)
    rot, x, w, qa, qw, _, _, _ = _exact_case(O.KRON, 128, rng, clip=0.9)
    a, ws, acc, y = O.linear_forward(x, w, rot)
    lut = np.array([0, 1, 2, 3, 4, 6, 7, 7])
    expect_a = np.sign(qa) * lut[np.abs(qa)]
    expect_w = np.sign(qw) * lut[np.abs(qw)]
    assert np.array_equal(a.q.codes, expect_a) and np.array_equal(ws.q.codes, expect_w)
    np.testing.assert_allclose(a.q.scales, 0.9, rtol=1e-6)


def test_rotation_reduces_error_on_outlier_inputs():
    # The pages' claim (QuaRot §2, FlatQuant §2, GSR): rotating spreads the
    # outlier channels, so the 4-bit layer is closer to X W^T than without.
    wl = workloads.make_workload("tiny_256")
    x, w = wl.X.astype(np.float64), wl.W.astype(np.float64)
    exact = x @ w.T
    errs, act = {}, {}
    for name, rot in [("none", O.Rotation(O.NONE)), ("had", O.Rotation(O.HADAMARD, block=256))]:
        a, _, _, y = O.linear_forward(x, w, rot)
        errs[name] = np.linalg.norm(y.astype(np.float64) - exact) / np.linalg.norm(exact)
        deq = a.q.codes * a.q.scales[:, None].astype(np.float64)
        act[name] = np.linalg.norm(deq - a.rotated) / np.linalg.norm(a.rotated)
    assert errs["had"] < errs["none"], errs
    assert act["had"] < 0.6 * act["none"], act


def test_incoherence_bound_hand_worked():
    # mu ||W||_F / sqrt(mn), mu = 2 ln(4mn/delta) (SpinQuant review, reviewer
    # Jf43 W1/A1): values worked by hand; a log2, a dropped factor 2 or a
    # missing sqrt(mn) each changes them.
    for r in read_golden_rows("incoherence_bound.txt"):
        m, n, delta = int(r[0]), int(r[1]), float(r[2])
        w = np.array([float(v) for v in r[3:3 + m * n]]).reshape(m, n)
        want = float(r[3 + m * n]) * np.log(2.0)
        assert abs(O.incoherence_bound(w, delta) - want) <= 1e-12 * want


def test_hadamard_bounds_weight_entries_incoherence():
    wl = workloads.make_workload("tiny_256")
    wr = O.rotate_weights(wl.W.astype(np.float64), O.Rotation(O.HADAMARD, block=256))
    assert np.abs(wr).max() <= O.incoherence_bound(wr, 0.01)


# ---------------------------------------------------------------- randomized Hadamard (R11)

def test_random_sign_hadamard_hand_example():
    x, d, want = _golden_matrix("random_sign_hadamard4.txt")
    rot = O.Rotation(O.HADAMARD, block=4, signs=d.astype(np.int8))
    np.testing.assert_allclose(O.rotate_activations(x[None, :], rot)[0], want, atol=1e-12)
    # signs applied after the rotation would give H(x) .* d instead
    wrong = (x @ O.hadamard(4) / 2) * d
    assert not np.allclose(wrong, want)


@pytest.mark.parametrize("kind,block,k", [(O.HADAMARD, 64, 256), (O.GSR, 16, 128),
                                          (O.HADAMARD, 4096, 4096)])
def test_random_sign_rotation_is_diag_times_blocks(kind, block, k):
    rng = np.random.default_rng(block)
    d = workloads.random_signs(block, k)
    x = rng.standard_normal((5, k))
    rot = O.Rotation(kind, block=block, signs=d)
    plain = O.Rotation(kind, block=block)
    # an independent construction: the explicit matrix diag(d) kron(I, B)
    r = np.diag(d.astype(np.float64)) @ np.kron(np.eye(k // block), O.block_rotation(kind, block))
    np.testing.assert_allclose(O.rotate_activations(x, rot), x @ r, atol=1e-10)
    np.testing.assert_allclose(O.rotate_weights(x, rot), x @ r, atol=1e-10)
    np.testing.assert_allclose(r @ r.T, np.eye(k), atol=1e-12)          # orthogonal
    # all-plus signs reduce to the plain rotation
    ones = O.Rotation(kind, block=block, signs=np.ones(k, np.int8))
    np.testing.assert_allclose(O.rotate_activations(x, ones), O.rotate_activations(x, plain),
                               atol=0)


def test_random_sign_rotation_keeps_invariance():
    rng = np.random.default_rng(11)
    K = 256
    x = rng.standard_normal((6, K))
    w = rng.standard_normal((5, K))
    rot = O.Rotation(O.HADAMARD, block=128, signs=workloads.random_signs(3, K))
    np.testing.assert_allclose(O.rotate_activations(x, rot) @ O.rotate_weights(w, rot).T,
                               x @ w.T, atol=1e-10)


def test_random_signs_are_seeded_and_balanced():
    a = workloads.random_signs(5, 4096)
    assert a.dtype == np.int8 and set(np.unique(a)) == {-1, 1}
    assert np.array_equal(a, workloads.random_signs(5, 4096))
    assert not np.array_equal(a, workloads.random_signs(6, 4096))
    assert abs(int(a.sum())) < 300


# ---------------------------------------------------------------- asymmetric activations (R12)

def test_asym_quantizer_hand_example():
    for r in read_golden_rows("quantizer_asym_1x4.txt"):
        v = [float(t) for t in r]
        x, codes, scale, zero = np.array(v[:4]), np.array(v[4:8]), v[8], v[9]
        q = O.quantize_rows_asym(x[None, :])
        assert np.array_equal(q.codes[0], codes.astype(np.int8))
        assert q.scales[0] == np.float32(scale) and q.zeros[0] == zero


def test_asym_quantizer_properties():
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal((6, 300)),
                        np.abs(rng.standard_normal((3, 300))) + 2.0,     # all positive
                        np.zeros((1, 300))])
    q = O.quantize_rows_asym(x)
    assert q.codes.min() >= -8 and q.codes.max() <= 7
    xhat = O.dequant_asym_rows(q)
    s = q.scales.astype(np.float64)[:, None]
    assert np.all(np.abs(xhat - x) <= s / 2 * (1 + 1e-5) + 1e-12)    # half a step, unclipped
    assert not xhat[-1].any() and q.scales[-1] == 0
    # each row's minimum lands on the bottom code (q = 0)
    assert np.array_equal(q.codes[np.arange(10), np.argmin(x, axis=1)][:-1], np.full(9, -8))
    # clipping shrinks the range and clamps into [0, 15]
    qc = O.quantize_rows_asym(x, clip_ratio=0.5)
    assert qc.codes.min() >= -8 and qc.codes.max() <= 7
    assert np.all(qc.scales[:-1] < q.scales[:-1])


def test_asym_beats_symmetric_on_one_sided_rows():
    # QUIK's reason for asymmetric activations: rows far from symmetric
    rng = np.random.default_rng(9)
    a = rng.standard_normal((64, 512))
    x = a / (1 + np.exp(-a))                       # SiLU: bounded below, long upper tail
    e_asym = np.abs(O.dequant_asym_rows(O.quantize_rows_asym(x)) - x).mean()
    qs = O.quantize_rows(x)
    e_sym = np.abs(qs.scales.astype(np.float64)[:, None] * qs.codes - x).mean()
    assert e_asym < 0.75 * e_sym


def test_asym_linear_matches_the_dequantized_product():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((5, 256)).astype(np.float16)
    w = (rng.standard_normal((7, 256)) * 0.05).astype(np.float16)
    rot = O.Rotation(O.HADAMARD, block=128)
    a, ws, acc, y = O.linear_forward_asym(x.astype(np.float64), w.astype(np.float64), rot)
    # acc is the integer product of the stored codes; the zero point enters
    # only through X_hat: Y = s_a s_w (acc - z' sum_k q_w)
    zsum = a.q.zeros.astype(np.int64)[:, None] * ws.q.codes.astype(np.int64).sum(axis=1)[None, :]
    alt = (acc - zsum) * a.q.scales.astype(np.float64)[:, None] * ws.q.scales.astype(np.float64)[None, :]
    np.testing.assert_allclose(y.astype(np.float64), alt, rtol=2e-3, atol=1e-3)
    # and the layer tracks X W^T
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.2


# ---------------------------------------------------------------- KV cache (R13)

def _sylvester(n):
    """H[i, j] = (-1)^popcount(i & j), written out independently."""
    return np.array([[(-1) ** bin(i & j).count("1") for j in range(n)] for i in range(n)], float)


def test_rotate_heads_hand_example():
    row = _golden_matrix("rotate_heads_2x4.txt")[0]
    np.testing.assert_allclose(O.rotate_heads(row[None, :8], 4)[0], row[8:], atol=1e-12)


@pytest.mark.parametrize("head_dim,heads", [(4, 3), (64, 2), (128, 3)])
def test_rotate_heads_is_block_diagonal_hadamard(head_dim, heads):
    rng = np.random.default_rng(head_dim + heads)
    x = rng.standard_normal((5, heads * head_dim))
    r = np.kron(np.eye(heads), _sylvester(head_dim) / np.sqrt(head_dim))
    np.testing.assert_allclose(O.rotate_heads(x, head_dim), x @ r, atol=1e-10)


def test_r3_keeps_every_heads_attention_scores():
    # (q R3)(k R3)^T = q k^T head by head, the identity the review answer gives
    rng = np.random.default_rng(31)
    d, heads = 128, 4
    q = rng.standard_normal((6, heads * d))
    k = rng.standard_normal((9, heads * d))
    qr, kr = O.rotate_heads(q, d), O.rotate_heads(k, d)
    for h in range(heads):
        sl = slice(h * d, (h + 1) * d)
        np.testing.assert_allclose(qr[:, sl] @ kr[:, sl].T, q[:, sl] @ k[:, sl].T, atol=1e-9)


def test_r3_inverse_reading_coincides_for_hadamard():
    # the notes' R3^{-1} on the query branch equals R3 for the symmetric Hadamard
    h = _sylvester(128) / np.sqrt(128)
    np.testing.assert_allclose(np.linalg.inv(h), h, atol=1e-12)


def test_group_quantizer_is_rows_of_the_asym_quantizer():
    # the two hand-worked 1x4 rows side by side form one 8-wide row of two groups
    rows = [[float(t) for t in r] for r in read_golden_rows("quantizer_asym_1x4.txt")]
    x = np.array([rows[0][:4] + rows[1][:4]])
    g = O.quantize_groups_asym(x, 4)
    assert np.array_equal(g.codes[0], np.array(rows[0][4:8] + rows[1][4:8], np.int8))
    assert list(g.scales[0]) == [rows[0][8], rows[1][8]]
    assert list(g.zeros[0]) == [rows[0][9], rows[1][9]]


def test_group_quantizer_properties():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((7, 512)) * np.linspace(0.1, 5.0, 512)
    x[3, 128:256] = 2.5                                   # a constant group
    g = O.quantize_groups_asym(x, 128)
    assert g.codes.shape == x.shape and g.scales.shape == (7, 4) and g.zeros.shape == (7, 4)
    assert g.codes.min() >= -8 and g.codes.max() <= 7
    xh = O.dequant_groups_asym(g, 128)
    s = np.repeat(g.scales.astype(np.float64), 128, axis=1)
    assert np.all(np.abs(xh - x)[s > 0] <= (s / 2 * (1 + 1e-5) + 1e-12)[s > 0])
    assert g.scales[3, 1] == 0 and not xh[3, 128:256].any()


def test_kv_quantize_keeps_scores_close_and_rotation_helps_keys():
    # keys with a few large channels: R3 spreads them over the head, so the
    # g128 4-bit keys give attention scores closer to the exact ones
    rng = np.random.default_rng(33)
    d, heads = 128, 4
    q = rng.standard_normal((16, heads * d))
    k = rng.standard_normal((64, heads * d))
    k[:, [5, 140, 300, 420]] *= 25.0
    v = rng.standard_normal((64, heads * d))
    qr, kq, vq = O.kv_quantize(q, k, v, d, 128)
    kr_hat = O.dequant_groups_asym(kq, 128)
    plain = O.dequant_groups_asym(O.quantize_groups_asym(k, 128), 128)
    exact = [q[:, h * d:(h + 1) * d] @ k[:, h * d:(h + 1) * d].T for h in range(heads)]
    rot = [qr[:, h * d:(h + 1) * d] @ kr_hat[:, h * d:(h + 1) * d].T for h in range(heads)]
    unrot = [q[:, h * d:(h + 1) * d] @ plain[:, h * d:(h + 1) * d].T for h in range(heads)]
    err_rot = sum(np.linalg.norm(a - b) for a, b in zip(rot, exact)) / sum(map(np.linalg.norm, exact))
    err_unrot = sum(np.linalg.norm(a - b) for a, b in zip(unrot, exact)) / sum(map(np.linalg.norm, exact))
    assert err_rot < 0.1 and err_rot < err_unrot
    v_hat = O.dequant_groups_asym(vq, 128)
    assert np.linalg.norm(v_hat - v) / np.linalg.norm(v) < 0.1


# ---------------------------------------------------------------- 8-bit layers (R14)

def test_int8_quantizer_hand_example():
    v = [float(t) for t in read_golden_rows("quantizer_int8_1x8.txt")[0]]
    q = O.quantize_rows(np.array([v[:8]]), bits=8)
    assert np.array_equal(q.codes[0], np.array(v[8:16], np.int8))
    assert q.scales[0] == np.float32(v[16])


def test_int8_quantizer_properties_and_exact_products():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((9, 700)) * np.exp(rng.standard_normal((9, 1)))
    q = O.quantize_rows(x, bits=8)
    assert q.codes.min() >= -127 and q.codes.max() <= 127
    assert np.all(np.abs(q.codes).max(axis=1) == 127)
    s = q.scales.astype(np.float64)[:, None]
    assert np.all(np.abs(s * q.codes - x) <= s / 2 * (1 + 1e-5) + 1e-12)
    # the exact integer GEMM at the 8-bit extremes (brute force)
    a = np.full((2, 11008), 127, np.int8)
    a[1, ::2] = -127
    w = np.full((3, 11008), -127, np.int8)
    acc = O.int_gemm(a, w)
    brute = [[sum(int(p) * int(r) for p, r in zip(a[i], w[j])) for j in range(3)] for i in range(2)]
    assert acc.tolist() == brute and abs(acc).max() < 2 ** 31


@pytest.mark.parametrize("kind", [O.NONE, O.HADAMARD, O.GSR])
def test_int8_layer_on_exactly_representable_rows(kind):
    # 8-bit codes through the whole activation / weight / linear path (R14):
    # rows built so that x R = qa and w R = qw, integer codes with absmax 127,
    # give those codes, unit scales and the exact integer product
    rng = np.random.default_rng(43)
    k, m, n = 256, 5, 7
    def codes(rows):
        q = rng.integers(-127, 128, size=(rows, k)).astype(np.int64)
        q[np.arange(rows), rng.integers(k, size=rows)] = np.where(rng.random(rows) < 0.5, 127, -127)
        return q
    qa, qw = codes(m), codes(n)
    rot = O.Rotation(kind, block=32 if kind == O.GSR else 64)
    r = O.dense_rotation(rot, k)
    a, ws, acc, y = O.linear_forward(qa @ r.T, qw @ r.T, rot, bits=8)
    assert np.array_equal(a.q.codes, qa) and np.array_equal(ws.q.codes, qw)
    assert a.packed.dtype == np.int8 and a.packed.shape == (m, k)
    np.testing.assert_allclose(a.q.scales, 1.0, rtol=1e-6)
    np.testing.assert_allclose(ws.q.scales, 1.0, rtol=1e-6)
    assert np.array_equal(acc, qa @ qw.T)


def test_quik_outlier_count_scales_with_width():
    assert O.quik_outlier_count(4096) == 256
    assert O.quik_outlier_count(11008) == 688          # the INT8 down_proj
    assert O.quik_outlier_count(8192) == 512


# ---------------------------------------------------------------- FP4 (R15)

def test_fp4_quantizer_hand_example():
    v = [float(t) for t in read_golden_rows("fp4_e2m1_1x12.txt")[0]]
    q = O.quantize_rows_fp4(np.array([v[:12]]))
    assert np.array_equal(q.codes[0], np.array(v[12:24], np.uint8))
    assert q.scales[0] == np.float32(v[24])


def test_e2m1_grid_and_rounding():
    # every code decodes to the grid, and rounding a grid value returns it
    vals = O.e2m1_value(np.arange(16))
    assert sorted(set(np.abs(vals))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        if c != 8:                                   # -0 rounds to +0
            assert O.e2m1_round(np.array([vals[c]]))[0] == c
    # nearest value: brute force over a fine sweep (ties excluded)
    xs = np.linspace(-7, 7, 2801)
    got = O.e2m1_value(O.e2m1_round(xs))
    grid = np.concatenate([-O.E2M1[::-1], O.E2M1])
    near = grid[np.argmin(np.abs(np.clip(xs, -6, 6)[:, None] - grid[None, :]), axis=1)]
    mids = (O.E2M1[1:] + O.E2M1[:-1]) / 2
    tie = np.isin(np.round(np.abs(xs), 9), np.round(mids, 9))
    assert np.array_equal(got[~tie], near[~tie])


def test_fp4_quantizer_error_bound():
    rng = np.random.default_rng(43)
    x = rng.standard_normal((6, 256))
    q = O.quantize_rows_fp4(x)
    xh = O.dequant_fp4_rows(q)
    s = q.scales.astype(np.float64)[:, None]
    v = np.abs(x) / s
    # half the grid gap at each magnitude: 0.25 below 2, 0.5 below 4, 1 up to 6
    gap = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
    assert np.all(np.abs(xh - x) <= gap * s * (1 + 1e-5) + 1e-12)
    # each row's largest value lands on the top of the grid (6 s = absmax)
    np.testing.assert_allclose(np.abs(xh).max(axis=1), np.abs(x).max(axis=1), rtol=1e-6)


def _e2m1_decode_bits(c: int) -> float:
    """e2m1 decoded from its fields, independently of the oracle's table:
    sign bit 3, exponent bits 2-1 (bias 1), mantissa bit 0; exponent 0 is
    subnormal (m / 2)."""
    sign = -1.0 if c & 8 else 1.0
    e, m = (c >> 1) & 3, c & 1
    return sign * (m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1))


def test_fp4_pack_layout():
    # element 2j in the low nibble: codes (1, 9, 15, 0) -> bytes 0x91, 0x0F
    b = O.pack_fp4(np.array([[1, 9, 15, 0]], np.uint8))
    assert b.tolist() == [[0x91, 0x0F]]
    rng = np.random.default_rng(5)
    c = rng.integers(0, 16, size=(3, 64)).astype(np.uint8)
    assert np.array_equal(O.unpack_fp4(O.pack_fp4(c)), c)


def test_fp4_gemm_brute_force():
    # the exact accumulator against a triple loop over field-decoded values
    rng = np.random.default_rng(6)
    ca = rng.integers(0, 16, size=(3, 40)).astype(np.uint8)
    cw = rng.integers(0, 16, size=(4, 40)).astype(np.uint8)
    acc = O.fp4_gemm(ca, cw)
    for m in range(3):
        for n in range(4):
            want = sum(_e2m1_decode_bits(int(ca[m, k])) * _e2m1_decode_bits(int(cw[n, k]))
                       for k in range(40))
            assert acc[m, n] == want
    # products are quarter-integers: the sum is exact, and equals it at the
    # extremes (all +-6: 36 K)
    full = np.full((1, 4096), 7, np.uint8)                  # +6
    neg = np.full((1, 4096), 15, np.uint8)                  # -6
    assert O.fp4_gemm(full, np.vstack([full, neg]))[0].tolist() == [36.0 * 4096, -36.0 * 4096]


def test_fp4_layer_is_lossless_on_grid_inputs():
    # rows that are (scale x e2m1 values) with absmax 6 x scale quantize
    # without error, so with no rotation Y = fp16(X W^T) exactly (float64 sum)
    rng = np.random.default_rng(8)
    grid = np.concatenate([-O.E2M1, O.E2M1])
    K = 64
    x = rng.choice(grid, size=(4, K)) * 0.25
    w = rng.choice(grid, size=(5, K)) * 0.125
    x[:, 0] = 6 * 0.25
    w[:, 0] = -6 * 0.125
    a, ws, acc, y = O.linear_forward_fp4(x, w, O.Rotation(O.NONE))
    assert np.array_equal(y, (x @ w.T).astype(np.float16))
    np.testing.assert_array_equal(acc * 0.25 * 0.125, x @ w.T)
