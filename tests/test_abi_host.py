"""Host-side checks of the C ABI: the library loads, exports every function
include/qr.h declares, and rejects bad arguments before launching anything.
No test here runs a kernel (this file runs without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from tests.conftest import ROOT
from w4a4_rotation_quantized_b200 import _lib as L
from w4a4_rotation_quantized_b200 import build as B

HEADER = os.path.join(ROOT, "include", "qr.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qr_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(L.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {L.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (qr_[a-z0-9_]+)", out))
    assert exported == set(declared_functions())


def test_abi_version_and_status_strings(lib):
    assert L.qr_abi_version() == 6
    for s in range(6):
        assert L.status_string(s) and L.status_string(s) != "unknown status"
    assert L.status_string(99) == "unknown status"


FAKE = 0x10000          # never dereferenced: every call below fails validation first


def _rot(kind, block=0, n1=0, n2=0, clip=1.0, p=FAKE):
    return L.make_rotation(kind, block, p if n1 else 0, n1, p if n2 else 0, n2, 0,
                           L.QR_CHAN_DIVIDE, clip)


@pytest.mark.parametrize("kind,block,n1,n2,K,n_out", [
    (L.QR_ROT_HADAMARD, 4096, 0, 0, 4096, 0),
    (L.QR_ROT_HADAMARD, 4096, 0, 0, 8192, 256),
    (L.QR_ROT_HADAMARD, 256, 0, 0, 256, 0),
    (L.QR_ROT_HADAMARD, 2, 0, 0, 300, 4),
    (L.QR_ROT_GSR, 128, 0, 0, 11008, 0),
    (L.QR_ROT_GSR, 256, 0, 0, 1000, 0),
    (L.QR_ROT_NONE, 0, 0, 0, 33, 0),
    (L.QR_ROT_NONE, 0, 0, 0, 0, 0),
    (L.QR_ROT_KRON, 0, 128, 64, 8192, 0),
    (L.QR_ROT_KRON, 0, 16, 8, 136, 8),
])
def test_packed_k_matches_the_oracle(lib, kind, block, n1, n2, K, n_out):
    names = {L.QR_ROT_NONE: O.NONE, L.QR_ROT_HADAMARD: O.HADAMARD, L.QR_ROT_GSR: O.GSR,
             L.QR_ROT_KRON: O.KRON}
    orot = O.Rotation(names[kind], block=block,
                      P1=np.eye(n1) if n1 else None, P2=np.eye(n2) if n2 else None)
    assert L.qr_packed_k(_rot(kind, block, n1, n2), K, n_out) == O.packed_width(orot, K, n_out)


@pytest.mark.parametrize("rot,K,n_out", [
    (_rot(L.QR_ROT_HADAMARD, 96), 96, 0),          # block not a power of two
    (_rot(L.QR_ROT_HADAMARD, 32768), 32768, 0),    # block too large
    (_rot(L.QR_ROT_GSR, 512), 512, 0),             # GSR block too large
    (_rot(L.QR_ROT_KRON, 0, 128, 64), 8000, 0),    # K != n1*n2
    (_rot(L.QR_ROT_KRON, 0, 128, 128), 16384, 0),  # factors too large
    (_rot(L.QR_ROT_KRON, 0, 6, 8), 48, 0),         # n1 not a multiple of 4
    (_rot(L.QR_ROT_HADAMARD, 64, clip=0.0), 64, 0),
    (_rot(L.QR_ROT_HADAMARD, 64, clip=1.5), 64, 0),
    (_rot(7, 64), 64, 0),                           # unknown kind
    (_rot(L.QR_ROT_NONE), 10, 11),                 # n_out > K
])
def test_packed_k_rejects_bad_descriptors(lib, rot, K, n_out):
    assert L.qr_packed_k(rot, K, n_out) == -1


def _rq(rot, X=FAKE, M=4, K=256, ldx=256, idx=None, n_out=0, codes=FAKE, scales=FAKE, xo=None,
        dbg=None):
    return L.qr_rotate_quant(rot, X, M, K, ldx, idx, n_out, codes, scales, xo, dbg, None,
                             check=False)


def test_rotate_quant_argument_errors(lib):
    h = _rot(L.QR_ROT_HADAMARD, 256)
    assert _rq(h, M=-1) == L.QR_ERR_INVALID_ARG
    assert _rq(h, ldx=100) == L.QR_ERR_INVALID_ARG              # ldx < K
    assert _rq(h, X=None) == L.QR_ERR_INVALID_ARG
    assert _rq(h, codes=None) == L.QR_ERR_INVALID_ARG
    assert _rq(h, n_out=4, idx=None, xo=FAKE) == L.QR_ERR_INVALID_ARG
    assert _rq(h, n_out=4, idx=FAKE, xo=None) == L.QR_ERR_INVALID_ARG
    assert _rq(h, codes=FAKE + 8) == L.QR_ERR_ALIGNMENT
    assert _rq(_rot(L.QR_ROT_HADAMARD, 96)) == L.QR_ERR_UNSUPPORTED
    assert _rq(_rot(L.QR_ROT_HADAMARD, 64, clip=2.0)) == L.QR_ERR_INVALID_ARG
    assert _rq(_rot(L.QR_ROT_NONE), K=40000, ldx=40000) == L.QR_ERR_UNSUPPORTED
    assert _rq(h, M=0) == L.QR_OK                                 # empty: nothing to do
    # random signs: HADAMARD / GSR only, 8-byte aligned
    signed = _rot(L.QR_ROT_HADAMARD, 256)
    signed.signs = FAKE + 4
    assert _rq(signed) == L.QR_ERR_ALIGNMENT
    kron = _rot(L.QR_ROT_KRON, n1=16, n2=16)
    kron.signs = FAKE
    assert _rq(kron) == L.QR_ERR_INVALID_ARG


def _lin(M=16, N=16, Kp=256, a=FAKE, sa=FAKE, w=FAKE, sw=FAKE, xo=None, wo=None, n_out=0,
         Y=FAKE, ldy=None, acc=None):
    return L.qr_w4a4_linear(a, sa, w, sw, M, N, Kp, xo, wo, n_out, Y, N if ldy is None else ldy,
                            acc, None, check=False)


def test_linear_argument_errors(lib):
    assert _lin(Kp=200) == L.QR_ERR_INVALID_ARG                   # K_p % 128
    assert _lin(M=-1) == L.QR_ERR_INVALID_ARG
    assert _lin(ldy=8) == L.QR_ERR_INVALID_ARG
    assert _lin(Y=None) == L.QR_ERR_INVALID_ARG
    assert _lin(a=None) == L.QR_ERR_INVALID_ARG
    assert _lin(n_out=8, xo=None, wo=FAKE) == L.QR_ERR_INVALID_ARG
    assert _lin(n_out=12, xo=FAKE, wo=FAKE) == L.QR_ERR_UNSUPPORTED   # n_out % 8
    assert _lin(Kp=65536 + 128) == L.QR_ERR_UNSUPPORTED
    assert _lin(a=FAKE + 4) == L.QR_ERR_ALIGNMENT
    assert _lin(n_out=8, xo=FAKE + 2, wo=FAKE) == L.QR_ERR_ALIGNMENT
    assert _lin(M=0) == L.QR_OK and _lin(N=0) == L.QR_OK


def test_calibration_argument_errors(lib):
    assert L.qr_select_outliers(FAKE, 8, 0, 8, 1, FAKE, None, check=False) == L.QR_ERR_INVALID_ARG
    assert L.qr_select_outliers(FAKE, 8, 16, 8, 1, FAKE, None, check=False) == L.QR_ERR_INVALID_ARG
    assert L.qr_select_outliers(FAKE, 8, 16, 16, 17, FAKE, None, check=False) == L.QR_ERR_INVALID_ARG
    assert L.qr_select_outliers(FAKE, 8, 20000, 20000, 4, FAKE, None,
                                check=False) == L.QR_ERR_UNSUPPORTED
    assert L.qr_invert_transpose(FAKE, 0, FAKE, FAKE, None, check=False) == L.QR_ERR_INVALID_ARG
    assert L.qr_invert_transpose(FAKE, 200, FAKE, FAKE, None, check=False) == L.QR_ERR_UNSUPPORTED
    assert L.qr_invert_transpose(None, 4, FAKE, FAKE, None, check=False) == L.QR_ERR_INVALID_ARG


def test_asymmetric_entry_points_argument_errors(lib):
    h = _rot(L.QR_ROT_HADAMARD, 256)
    rq = lambda rot, zeros=FAKE, M=4: L.qr_rotate_quant_asym(
        rot, FAKE, M, 256, 256, None, 0, FAKE, FAKE, zeros, None, None, None, check=False)
    assert rq(h, zeros=None) == L.QR_ERR_INVALID_ARG
    assert rq(_rot(L.QR_ROT_KRON, n1=16, n2=16)) == L.QR_ERR_UNSUPPORTED
    assert rq(h, zeros=None, M=0) == L.QR_OK
    sums = lambda N=8, Kp=256, codes=FAKE, out=FAKE: L.qr_weight_code_sums(codes, N, Kp, out, None,
                                                                          check=False)
    assert sums(Kp=100) == L.QR_ERR_INVALID_ARG
    assert sums(out=None) == L.QR_ERR_INVALID_ARG
    assert sums(codes=FAKE + 4) == L.QR_ERR_ALIGNMENT
    assert sums(N=0) == L.QR_OK
    lin = lambda za=FAKE, ws=FAKE: L.qr_w4a4_linear_asym(FAKE, FAKE, za, FAKE, FAKE, ws, 16, 16, 256,
                                                         None, None, 0, FAKE, 16, None, None,
                                                         check=False)
    assert lin(za=None) == L.QR_ERR_INVALID_ARG
    assert lin(ws=None) == L.QR_ERR_INVALID_ARG



def test_kv_quantize_argument_errors(lib):
    # every call here fails validation (or has no tokens): nothing launches
    def kv(q=FAKE, k=FAKE, v=FAKE, tokens=4, heads=4, d=128, g=128, qr=FAKE, kc=FAKE, ks=FAKE,
           kz=FAKE, vc=FAKE, vs=FAKE, vz=FAKE):
        return L.qr_kv_quantize(q, k, v, tokens, heads, d, g, qr, kc, ks, kz, vc, vs, vz, None,
                                check=False)
    assert kv(tokens=-1) == L.QR_ERR_INVALID_ARG
    assert kv(heads=0) == L.QR_ERR_INVALID_ARG
    assert kv(d=96) == L.QR_ERR_UNSUPPORTED
    assert kv(g=192) == L.QR_ERR_UNSUPPORTED            # groups of 128 or 256
    assert kv(g=512, heads=8) == L.QR_ERR_UNSUPPORTED
    assert kv(d=256, g=128) == L.QR_ERR_UNSUPPORTED      # a group must hold whole heads
    assert kv(heads=3, d=128, g=256) == L.QR_ERR_UNSUPPORTED   # width not a multiple of g
    assert kv(qr=None) == L.QR_ERR_INVALID_ARG           # Q without its output
    assert kv(kz=None) == L.QR_ERR_INVALID_ARG           # a partly given K side
    assert kv(v=None) == L.QR_ERR_INVALID_ARG            # V outputs without V
    assert kv(q=FAKE + 2) == L.QR_ERR_ALIGNMENT
    assert kv(tokens=0) == L.QR_OK
    assert kv(q=None, k=None, v=None, qr=None, kc=None, ks=None, kz=None, vc=None, vs=None,
              vz=None) == L.QR_OK


def test_wait_selfcheck_argument_errors(lib):
    # the limit is validated on the host, before any launch
    for bad in (0, 999, 100000001, -5):
        assert L.qr_check_wait_timeout(bad, None, check=False) == L.QR_ERR_INVALID_ARG


def test_int8_entry_points_argument_errors(lib):
    # the 8-bit calls validate like the 4-bit ones; nothing launches here
    h = _rot(L.QR_ROT_HADAMARD, 256)
    def rq8(rot, codes=FAKE, M=4, K=512):
        return L.qr_rotate_quant8(rot, FAKE, M, K, K, None, 0, codes, FAKE, None, None, None,
                                  check=False)
    assert rq8(h, codes=FAKE + 8) == L.QR_ERR_ALIGNMENT
    assert rq8(h, M=-1) == L.QR_ERR_INVALID_ARG
    assert rq8(h, M=0) == L.QR_OK
    assert rq8(_rot(L.QR_ROT_KRON, n1=16, n2=32), K=512) == L.QR_ERR_UNSUPPORTED
    assert L.qr_pack_weights8(h, FAKE, 4, 512, 512, None, 0, None, FAKE, None, None, None,
                              check=False) == L.QR_ERR_INVALID_ARG
    def lin8(Kp=256, a=FAKE, n_out=0, xo=None, wo=None, M=16):
        return L.qr_w8a8_linear(a, FAKE, FAKE, FAKE, M, 16, Kp, xo, wo, n_out, FAKE, 16, None,
                                None, check=False)
    assert lin8(Kp=200) == L.QR_ERR_INVALID_ARG
    assert lin8(a=FAKE + 4) == L.QR_ERR_ALIGNMENT
    assert lin8(n_out=12, xo=FAKE, wo=FAKE) == L.QR_ERR_UNSUPPORTED
    assert lin8(M=0) == L.QR_OK


def test_fp4_entry_points_argument_errors(lib):
    # the e2m1 calls validate like the others, and want 32-byte aligned codes
    h = _rot(L.QR_ROT_HADAMARD, 256)
    def rq4(rot, codes=FAKE, M=4, K=512):
        return L.qr_rotate_quant_fp4(rot, FAKE, M, K, K, None, 0, codes, FAKE, None, None, None,
                                     check=False)
    assert rq4(h, codes=FAKE + 16) == L.QR_ERR_ALIGNMENT
    assert rq4(h, M=-1) == L.QR_ERR_INVALID_ARG
    assert rq4(h, M=0) == L.QR_OK
    assert rq4(_rot(L.QR_ROT_KRON, n1=16, n2=32), K=512) == L.QR_ERR_UNSUPPORTED
    assert L.qr_pack_weights_fp4(h, FAKE, 4, 512, 512, None, 0, None, FAKE, None, None, None,
                                 check=False) == L.QR_ERR_INVALID_ARG
    def lin4(Kp=256, a=FAKE, w=FAKE, M=16):
        return L.qr_fp4_linear(a, FAKE, w, FAKE, M, 16, Kp, None, None, 0, FAKE, 16, None, None,
                               check=False)
    assert lin4(Kp=200) == L.QR_ERR_INVALID_ARG
    assert lin4(a=FAKE + 16) == L.QR_ERR_ALIGNMENT
    assert lin4(w=FAKE + 16) == L.QR_ERR_ALIGNMENT
    assert lin4(M=0) == L.QR_OK


def test_fused_decode_argument_errors(lib):
    # the one-kernel decode step validates both halves' arguments, takes at
    # most 64 tokens and no Kronecker rotation, and wants its barrier words
    h = _rot(L.QR_ROT_HADAMARD, 256)
    def fused(rot=h, M=4, K=512, sync=FAKE, a=FAKE, n_out=0, idx=None, xo=None, wo=None,
              zeros=None, sums=None):
        return L.qr_w4a4_linear_fused(rot, FAKE, M, K, K, idx, n_out, FAKE, FAKE, sums, wo, 16, a,
                                      FAKE, zeros, xo, FAKE, 16, sync, None, check=False)
    assert fused(M=0) == L.QR_OK
    assert fused(M=-1) == L.QR_ERR_INVALID_ARG
    assert fused(M=65) == L.QR_ERR_UNSUPPORTED
    assert fused(sync=None) == L.QR_ERR_INVALID_ARG
    assert fused(sync=FAKE + 4) == L.QR_ERR_ALIGNMENT
    assert fused(a=FAKE + 8) == L.QR_ERR_ALIGNMENT
    assert fused(n_out=8) == L.QR_ERR_INVALID_ARG                 # no outlier list or copies
    assert fused(n_out=4, idx=FAKE, xo=FAKE, wo=FAKE) == L.QR_ERR_UNSUPPORTED   # n_out % 8
    assert fused(zeros=FAKE) == L.QR_ERR_INVALID_ARG              # asymmetric without w_sums
    assert fused(rot=_rot(L.QR_ROT_KRON, n1=16, n2=32)) == L.QR_ERR_UNSUPPORTED
    # the no-alloc form: the same checks, and the scratch's capacity
    def noalloc(rot=h, M=4, K=512, n_out=0, idx=None, wo=None, asym=0, sums=None):
        return L.qr_w4a4_linear_fused_noalloc(rot, FAKE, M, K, K, idx, n_out, FAKE, FAKE, sums, wo,
                                              16, asym, FAKE, 16, None, check=False)
    assert noalloc(M=0) == L.QR_OK
    assert noalloc(M=65) == L.QR_ERR_UNSUPPORTED
    assert noalloc(n_out=8) == L.QR_ERR_INVALID_ARG
    assert noalloc(asym=1) == L.QR_ERR_INVALID_ARG                # asymmetric without w_sums
    assert noalloc(rot=_rot(L.QR_ROT_KRON, n1=16, n2=32)) == L.QR_ERR_UNSUPPORTED
