"""ctypes binding of libqr.so: the C ABI declared in include/qr.h, one Python
function per entry point, same names.  Argument marshalling only -- every
step of the layer runs in the library's CUDA kernels.  There is no fallback:
if the library cannot be loaded, every call raises."""
from __future__ import annotations

import ctypes
import os

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libqr.so")

QR_OK, QR_ERR_INVALID_ARG, QR_ERR_UNSUPPORTED, QR_ERR_ALIGNMENT, QR_ERR_CUDA, QR_ERR_DEVICE = range(6)
QR_ROT_NONE, QR_ROT_HADAMARD, QR_ROT_GSR, QR_ROT_KRON = range(4)
QR_CHAN_DIVIDE, QR_CHAN_MULTIPLY = 0, 1

EXPORTED = ("qr_abi_version", "qr_status_string", "qr_packed_k", "qr_rotate_quant",
            "qr_pack_weights", "qr_w4a4_linear", "qr_select_outliers",
            "qr_invert_transpose", "qr_device_status", "qr_rotate_quant_asym",
            "qr_weight_code_sums", "qr_w4a4_linear_asym", "qr_kv_quantize",
            "qr_check_wait_timeout", "qr_rotate_quant8", "qr_pack_weights8", "qr_w8a8_linear",
            "qr_rotate_quant_fp4", "qr_pack_weights_fp4", "qr_fp4_linear",
            "qr_w4a4_linear_fused", "qr_w4a4_linear_fused_noalloc")

# codes of the device status word (qr_device_status)
QR_DEV_TIMEOUT_GRID_SYNC = 0x106
QR_DEV_TIMEOUT_SELFCHECK = 0x1FF


class QrRotation(ctypes.Structure):
    """Mirror of the C struct qr_rotation."""
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("p1", ctypes.c_void_p),
        ("n1", ctypes.c_int32),
        ("p2", ctypes.c_void_p),
        ("n2", ctypes.c_int32),
        ("chan_scale", ctypes.c_void_p),
        ("chan_mode", ctypes.c_int32),
        ("clip_ratio", ctypes.c_float),
        ("signs", ctypes.c_void_p),
    ]


class QrError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libqr.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with "
                           "`python -m w4a4_rotation_quantized_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    rot_p = ctypes.POINTER(QrRotation)
    sig = {
        "qr_abi_version": (i32, []),
        "qr_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "qr_packed_k": (i64, [rot_p, i64, i32]),
        "qr_rotate_quant": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp, vp]),
        "qr_pack_weights": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp, vp]),
        "qr_w4a4_linear": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp, i32, vp, i64, vp,
                                          vp]),
        "qr_select_outliers": (ctypes.c_int, [vp, i64, i64, i64, i32, vp, vp]),
        "qr_invert_transpose": (ctypes.c_int, [vp, i32, vp, vp, vp]),
        "qr_device_status": (ctypes.c_int, [ctypes.POINTER(i32)]),
        "qr_rotate_quant_asym": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp,
                                                vp, vp]),
        "qr_weight_code_sums": (ctypes.c_int, [vp, i64, i64, vp, vp]),
        "qr_w4a4_linear_asym": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, vp, i32,
                                               vp, i64, vp, vp]),
        "qr_kv_quantize": (ctypes.c_int, [vp, vp, vp, i64, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                          vp, vp]),
        "qr_check_wait_timeout": (ctypes.c_int, [i64, vp]),
        "qr_rotate_quant8": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp, vp]),
        "qr_pack_weights8": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp, vp]),
        "qr_w8a8_linear": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp, i32, vp, i64, vp,
                                          vp]),
        "qr_rotate_quant_fp4": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp,
                                               vp]),
        "qr_pack_weights_fp4": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp,
                                               vp]),
        "qr_fp4_linear": (ctypes.c_int, [vp, vp, vp, vp, i64, i64, i64, vp, vp, i32, vp, i64, vp,
                                         vp]),
        "qr_w4a4_linear_fused": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp,
                                                i64, vp, vp, vp, vp, vp, i64, vp, vp]),
        "qr_w4a4_linear_fused_noalloc": (ctypes.c_int, [rot_p, vp, i64, i64, i64, vp, i32, vp, vp,
                                                        vp, vp, i64, i32, vp, i64, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().qr_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != QR_OK:
        raise QrError(fn, status)


def make_rotation(kind: int, block: int = 0, p1: int = 0, n1: int = 0, p2: int = 0, n2: int = 0,
                  chan_scale: int = 0, chan_mode: int = QR_CHAN_DIVIDE,
                  clip_ratio: float = 1.0, signs: int = 0) -> QrRotation:
    return QrRotation(kind, block, p1 or None, n1, p2 or None, n2, chan_scale or None, chan_mode,
                      clip_ratio, signs or None)


def qr_abi_version() -> int:
    return load().qr_abi_version()


def qr_packed_k(rot: QrRotation, K: int, n_out: int) -> int:
    return load().qr_packed_k(ctypes.byref(rot), K, n_out)


def qr_rotate_quant(rot, X, M, K, ldx, outlier_idx, n_out, codes, scales, x_out, x_rot_debug,
                    stream, *, check=True):
    st = load().qr_rotate_quant(ctypes.byref(rot), X, M, K, ldx, outlier_idx, n_out, codes, scales,
                                x_out, x_rot_debug, stream)
    if check:
        _check("qr_rotate_quant", st)
    return st


def qr_pack_weights(rot_w, W, N, K, ldw, outlier_idx, n_out, w_codes, w_scales, w_out,
                    w_rot_debug, stream, *, check=True):
    st = load().qr_pack_weights(ctypes.byref(rot_w), W, N, K, ldw, outlier_idx, n_out, w_codes,
                                w_scales, w_out, w_rot_debug, stream)
    if check:
        _check("qr_pack_weights", st)
    return st


def qr_w4a4_linear(a_codes, a_scales, w_codes, w_scales, M, N, K_p, x_out, w_out, n_out, Y, ldy,
                   acc_debug, stream, *, check=True):
    st = load().qr_w4a4_linear(a_codes, a_scales, w_codes, w_scales, M, N, K_p, x_out, w_out,
                               n_out, Y, ldy, acc_debug, stream)
    if check:
        _check("qr_w4a4_linear", st)
    return st


def qr_rotate_quant_asym(rot, X, M, K, ldx, outlier_idx, n_out, codes, scales, zeros, x_out,
                         x_rot_debug, stream, *, check=True):
    st = load().qr_rotate_quant_asym(ctypes.byref(rot), X, M, K, ldx, outlier_idx, n_out, codes,
                                     scales, zeros, x_out, x_rot_debug, stream)
    if check:
        _check("qr_rotate_quant_asym", st)
    return st


def qr_weight_code_sums(w_codes, N, K_p, w_sums, stream, *, check=True):
    st = load().qr_weight_code_sums(w_codes, N, K_p, w_sums, stream)
    if check:
        _check("qr_weight_code_sums", st)
    return st


def qr_w4a4_linear_asym(a_codes, a_scales, a_zeros, w_codes, w_scales, w_sums, M, N, K_p, x_out,
                        w_out, n_out, Y, ldy, acc_debug, stream, *, check=True):
    st = load().qr_w4a4_linear_asym(a_codes, a_scales, a_zeros, w_codes, w_scales, w_sums, M, N,
                                    K_p, x_out, w_out, n_out, Y, ldy, acc_debug, stream)
    if check:
        _check("qr_w4a4_linear_asym", st)
    return st


def qr_kv_quantize(Q, K, V, tokens, heads, head_dim, group, q_rot, k_codes, k_scales, k_zeros,
                   v_codes, v_scales, v_zeros, stream, *, check=True):
    st = load().qr_kv_quantize(Q, K, V, tokens, heads, head_dim, group, q_rot, k_codes, k_scales,
                               k_zeros, v_codes, v_scales, v_zeros, stream)
    if check:
        _check("qr_kv_quantize", st)
    return st


def qr_select_outliers(X_calib, T, K, ldx, k, idx_out, stream, *, check=True):
    st = load().qr_select_outliers(X_calib, T, K, ldx, k, idx_out, stream)
    if check:
        _check("qr_select_outliers", st)
    return st


def qr_invert_transpose(P, n, out, info, stream, *, check=True):
    st = load().qr_invert_transpose(P, n, out, info, stream)
    if check:
        _check("qr_invert_transpose", st)
    return st


def qr_device_status() -> int:
    code = ctypes.c_int32(0)
    _check("qr_device_status", load().qr_device_status(ctypes.byref(code)))
    return code.value


def qr_check_wait_timeout(limit_ns: int, stream, *, check=True) -> int:
    st = load().qr_check_wait_timeout(limit_ns, stream)
    if check:
        _check("qr_check_wait_timeout", st)
    return st


def qr_rotate_quant8(rot, X, M, K, ldx, outlier_idx, n_out, codes, scales, x_out, x_rot_debug,
                     stream, *, check=True):
    st = load().qr_rotate_quant8(ctypes.byref(rot), X, M, K, ldx, outlier_idx, n_out, codes,
                                 scales, x_out, x_rot_debug, stream)
    if check:
        _check("qr_rotate_quant8", st)
    return st


def qr_pack_weights8(rot_w, W, N, K, ldw, outlier_idx, n_out, w_codes, w_scales, w_out,
                     w_rot_debug, stream, *, check=True):
    st = load().qr_pack_weights8(ctypes.byref(rot_w), W, N, K, ldw, outlier_idx, n_out, w_codes,
                                 w_scales, w_out, w_rot_debug, stream)
    if check:
        _check("qr_pack_weights8", st)
    return st


def qr_w8a8_linear(a_codes, a_scales, w_codes, w_scales, M, N, K_p, x_out, w_out, n_out, Y, ldy,
                   acc_debug, stream, *, check=True):
    st = load().qr_w8a8_linear(a_codes, a_scales, w_codes, w_scales, M, N, K_p, x_out, w_out,
                               n_out, Y, ldy, acc_debug, stream)
    if check:
        _check("qr_w8a8_linear", st)
    return st


def qr_rotate_quant_fp4(rot, X, M, K, ldx, outlier_idx, n_out, codes, scales, x_out, x_rot_debug,
                        stream, *, check=True):
    st = load().qr_rotate_quant_fp4(ctypes.byref(rot), X, M, K, ldx, outlier_idx, n_out, codes,
                                    scales, x_out, x_rot_debug, stream)
    if check:
        _check("qr_rotate_quant_fp4", st)
    return st


def qr_pack_weights_fp4(rot_w, W, N, K, ldw, outlier_idx, n_out, w_codes, w_scales, w_out,
                        w_rot_debug, stream, *, check=True):
    st = load().qr_pack_weights_fp4(ctypes.byref(rot_w), W, N, K, ldw, outlier_idx, n_out,
                                    w_codes, w_scales, w_out, w_rot_debug, stream)
    if check:
        _check("qr_pack_weights_fp4", st)
    return st


def qr_fp4_linear(a_codes, a_scales, w_codes, w_scales, M, N, K_p, x_out, w_out, n_out, Y, ldy,
                  acc_debug, stream, *, check=True):
    st = load().qr_fp4_linear(a_codes, a_scales, w_codes, w_scales, M, N, K_p, x_out, w_out,
                              n_out, Y, ldy, acc_debug, stream)
    if check:
        _check("qr_fp4_linear", st)
    return st


def qr_w4a4_linear_fused(rot, X, M, K, ldx, outlier_idx, n_out, w_codes, w_scales, w_sums, w_out,
                         N, a_codes, a_scales, a_zeros, x_out, Y, ldy, sync, stream, *,
                         check=True):
    st = load().qr_w4a4_linear_fused(ctypes.byref(rot), X, M, K, ldx, outlier_idx, n_out, w_codes, w_scales,
                                     w_sums, w_out, N, a_codes, a_scales, a_zeros, x_out, Y, ldy,
                                     sync, stream)
    if check:
        _check("qr_w4a4_linear_fused", st)
    return st


def qr_w4a4_linear_fused_noalloc(rot, X, M, K, ldx, outlier_idx, n_out, w_codes, w_scales, w_sums,
                                 w_out, N, asym, Y, ldy, stream, *, check=True):
    st = load().qr_w4a4_linear_fused_noalloc(ctypes.byref(rot), X, M, K, ldx, outlier_idx, n_out,
                                             w_codes, w_scales, w_sums, w_out, N, asym, Y, ldy,
                                             stream)
    if check:
        _check("qr_w4a4_linear_fused_noalloc", st)
    return st
