"""Torch-facing helpers over the C ABI: allocate outputs as torch CUDA tensors,
pass their pointers and the current stream, nothing else.  All arithmetic
runs in libqr.so's kernels."""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

from . import _lib as L

NONE, HADAMARD, GSR, KRON = L.QR_ROT_NONE, L.QR_ROT_HADAMARD, L.QR_ROT_GSR, L.QR_ROT_KRON


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _need_cuda(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


@dataclass
class Rotation:
    """Python-side rotation descriptor; keeps its device tensors alive."""
    kind: int = NONE
    block: int = 1
    p1: Optional[torch.Tensor] = None       # fp32 [n1, n1] (KRON)
    p2: Optional[torch.Tensor] = None       # fp32 [n2, n2]
    chan_scale: Optional[torch.Tensor] = None   # fp32 [n1*n2]
    chan_mode: int = L.QR_CHAN_DIVIDE
    clip_ratio: float = 1.0
    signs: Optional[torch.Tensor] = None    # int8 [K_p] of +-1 (HADAMARD, GSR): R = D B
    _c: Optional[L.QrRotation] = field(default=None, repr=False)

    def c(self) -> L.QrRotation:
        for t in (self.p1, self.p2, self.chan_scale):
            if t is not None:
                _need_cuda(t, torch.float32, "rotation tensor")
                if not t.is_contiguous():
                    raise ValueError("rotation tensors must be contiguous")
        if self.signs is not None:
            _need_cuda(self.signs, torch.int8, "signs")
            if not self.signs.is_contiguous():
                raise ValueError("signs must be contiguous")
        n1 = 0 if self.p1 is None else self.p1.shape[0]
        n2 = 0 if self.p2 is None else self.p2.shape[0]
        self._c = L.make_rotation(self.kind, self.block, _ptr(self.p1) or 0, n1,
                                  _ptr(self.p2) or 0, n2, _ptr(self.chan_scale) or 0,
                                  self.chan_mode, self.clip_ratio, _ptr(self.signs) or 0)
        return self._c


def invert_transpose(p: torch.Tensor) -> torch.Tensor:
    """(P^{-1})^T on the GPU (fp64 Gauss-Jordan); raises if P is singular."""
    _need_cuda(p, torch.float32, "P")
    p = p.contiguous()
    n = p.shape[0]
    out = torch.empty_like(p)
    info = torch.zeros(1, dtype=torch.int32, device=p.device)
    L.qr_invert_transpose(p.data_ptr(), n, out.data_ptr(), info.data_ptr(), _stream())
    if int(info.item()) != 0:
        raise ValueError(f"P is singular (no pivot in column {int(info.item()) - 1})")
    return out


def weight_rotation(rot: Rotation) -> Rotation:
    """The weight-side descriptor matching an activation-side one."""
    if rot.kind != KRON:
        return rot
    return Rotation(KRON, p1=invert_transpose(rot.p1), p2=invert_transpose(rot.p2),
                    chan_scale=rot.chan_scale, chan_mode=L.QR_CHAN_MULTIPLY,
                    clip_ratio=rot.clip_ratio)


def packed_k(rot: Rotation, K: int, n_out: int = 0) -> int:
    kp = L.qr_packed_k(rot.c(), K, n_out)
    if kp < 0:
        raise ValueError("invalid rotation descriptor or sizes")
    return kp


def _rows(fn, rot: Rotation, x: torch.Tensor, outlier_idx, debug: bool, asym: bool = False,
          bits: int = 4):
    _need_cuda(x, torch.float16, "input")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("input must be a 2-D row-major tensor")
    rows, K = x.shape
    n_out = 0 if outlier_idx is None else int(outlier_idx.numel())
    if n_out:
        _need_cuda(outlier_idx, torch.int32, "outlier_idx")
    crot = rot.c()
    kp = L.qr_packed_k(crot, K, n_out)
    if kp < 0:
        raise ValueError("invalid rotation descriptor or sizes")
    dev = x.device
    codes = (torch.empty((rows, kp), dtype=torch.int8, device=dev) if bits == 8
             else torch.empty((rows, kp // 2), dtype=torch.uint8, device=dev))
    scales = torch.empty(rows, dtype=torch.float32, device=dev)
    out16 = torch.empty((rows, n_out), dtype=torch.float16, device=dev) if n_out else None
    dbg = torch.empty((rows, kp), dtype=torch.float32, device=dev) if debug else None
    if asym:
        zeros = torch.empty(rows, dtype=torch.int32, device=dev)
        fn(crot, x.data_ptr(), rows, K, x.stride(0), _ptr(outlier_idx) if n_out else None, n_out,
           codes.data_ptr(), scales.data_ptr(), zeros.data_ptr(), _ptr(out16), _ptr(dbg),
           _stream())
        return codes, scales, zeros, out16, dbg
    fn(crot, x.data_ptr(), rows, K, x.stride(0), _ptr(outlier_idx) if n_out else None, n_out,
       codes.data_ptr(), scales.data_ptr(), _ptr(out16), _ptr(dbg), _stream())
    return codes, scales, out16, dbg


def rotate_quant(x, rot: Rotation, outlier_idx=None, debug: bool = False):
    """Online activation path: (codes, scales, x_out, x_rot or None)."""
    return _rows(L.qr_rotate_quant, rot, x, outlier_idx, debug)


def rotate_quant_asym(x, rot: Rotation, outlier_idx=None, debug: bool = False):
    """Online activation path with QUIK's asymmetric per-token quantizer:
    (codes, scales, zeros, x_out, x_rot or None); x ~= scale * (code - zero)."""
    return _rows(L.qr_rotate_quant_asym, rot, x, outlier_idx, debug, asym=True)


def rotate_quant8(x, rot: Rotation, outlier_idx=None, debug: bool = False):
    """Online activation path with 8-bit codes (QUIK's INT8 layers):
    (codes int8 [rows x K_p], scales, x_out, x_rot or None)."""
    return _rows(L.qr_rotate_quant8, rot, x, outlier_idx, debug, bits=8)


def pack_weights8(w, rot_w: Rotation, outlier_idx=None, debug: bool = False):
    """Offline weight path with 8-bit codes: (codes int8, scales, w_out, w_rot or None)."""
    return _rows(L.qr_pack_weights8, rot_w, w, outlier_idx, debug, bits=8)


def w8a8_linear(a_codes, a_scales, w_codes, w_scales, x_out=None, w_out=None,
                out: Optional[torch.Tensor] = None, acc_debug: bool = False):
    """The 8-bit linear: Y = fp16(acc * sa * sw + x_out w_out^T) for int8 codes;
    returns (Y, acc or None)."""
    M, kp = a_codes.shape
    N = w_codes.shape[0]
    n_out = 0 if x_out is None else x_out.shape[1]
    dev = a_codes.device
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=dev)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev) if acc_debug else None
    L.qr_w8a8_linear(a_codes.data_ptr(), a_scales.data_ptr(), w_codes.data_ptr(),
                     w_scales.data_ptr(), M, N, kp, _ptr(x_out), _ptr(w_out), n_out,
                     y.data_ptr(), y.stride(0), _ptr(acc), _stream())
    return y, acc


def rotate_quant_fp4(x, rot: Rotation, outlier_idx=None, debug: bool = False):
    """Online activation path with e2m1 codes (two per byte, element 2j in
    the low nibble): (codes uint8 [rows x K_p/2], scales, x_out, x_rot or None)."""
    return _rows(L.qr_rotate_quant_fp4, rot, x, outlier_idx, debug)


def pack_weights_fp4(w, rot_w: Rotation, outlier_idx=None, debug: bool = False):
    """Offline weight path with e2m1 codes: (codes, scales, w_out, w_rot or None)."""
    return _rows(L.qr_pack_weights_fp4, rot_w, w, outlier_idx, debug)


def fp4_linear(a_codes, a_scales, w_codes, w_scales, x_out=None, w_out=None,
               out: Optional[torch.Tensor] = None, acc_debug: bool = False):
    """The FP4 linear: Y = fp16(acc * sa * sw + x_out w_out^T) for packed
    e2m1 codes; returns (Y, acc float32 or None)."""
    M, kp2 = a_codes.shape
    N = w_codes.shape[0]
    n_out = 0 if x_out is None else x_out.shape[1]
    dev = a_codes.device
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=dev)
    acc = torch.empty((M, N), dtype=torch.float32, device=dev) if acc_debug else None
    L.qr_fp4_linear(a_codes.data_ptr(), a_scales.data_ptr(), w_codes.data_ptr(),
                    w_scales.data_ptr(), M, N, 2 * kp2, _ptr(x_out), _ptr(w_out), n_out,
                    y.data_ptr(), y.stride(0), _ptr(acc), _stream())
    return y, acc


def weight_code_sums(w_codes: torch.Tensor) -> torch.Tensor:
    """Per weight row, the sum of its packed codes (int32 [N])."""
    N, kp2 = w_codes.shape
    sums = torch.empty(N, dtype=torch.int32, device=w_codes.device)
    L.qr_weight_code_sums(w_codes.data_ptr(), N, 2 * kp2, sums.data_ptr(), _stream())
    return sums


def pack_weights(w, rot_w: Rotation, outlier_idx=None, debug: bool = False):
    """Offline weight path: (codes, scales, w_out, w_rot or None)."""
    return _rows(L.qr_pack_weights, rot_w, w, outlier_idx, debug)


def w4a4_linear(a_codes, a_scales, w_codes, w_scales, x_out=None, w_out=None,
                out: Optional[torch.Tensor] = None, acc_debug: bool = False):
    """Y = fp16(acc * sa * sw + x_out w_out^T); returns (Y, acc or None)."""
    M, kp2 = a_codes.shape
    N = w_codes.shape[0]
    n_out = 0 if x_out is None else x_out.shape[1]
    dev = a_codes.device
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=dev)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev) if acc_debug else None
    L.qr_w4a4_linear(a_codes.data_ptr(), a_scales.data_ptr(), w_codes.data_ptr(),
                     w_scales.data_ptr(), M, N, 2 * kp2, _ptr(x_out), _ptr(w_out), n_out,
                     y.data_ptr(), y.stride(0), _ptr(acc), _stream())
    return y, acc


def w4a4_linear_asym(a_codes, a_scales, a_zeros, w_codes, w_scales, w_sums, x_out=None,
                     w_out=None, out: Optional[torch.Tensor] = None, acc_debug: bool = False):
    """Y = fp16((acc - zero_a w_sums) * sa * sw + x_out w_out^T) for asymmetric
    activation codes; returns (Y, acc or None)."""
    M, kp2 = a_codes.shape
    N = w_codes.shape[0]
    n_out = 0 if x_out is None else x_out.shape[1]
    dev = a_codes.device
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=dev)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev) if acc_debug else None
    L.qr_w4a4_linear_asym(a_codes.data_ptr(), a_scales.data_ptr(), a_zeros.data_ptr(),
                          w_codes.data_ptr(), w_scales.data_ptr(), w_sums.data_ptr(), M, N,
                          2 * kp2, _ptr(x_out), _ptr(w_out), n_out, y.data_ptr(), y.stride(0),
                          _ptr(acc), _stream())
    return y, acc


def w4a4_linear_fused(x, rot: Rotation, outlier_idx, w_codes, w_scales, w_out=None, w_sums=None,
                      asym: bool = False, sync: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, check: bool = True):
    """The decode step in one kernel: rotate + quantize the M <= 64 rows of x
    and multiply them with the packed weights.  Same results as rotate_quant
    (rotate_quant_asym) followed by w4a4_linear (w4a4_linear_asym).  Returns
    (Y, codes, scales, zeros or None, x_out or None), or None when check is
    False and the library answers UNSUPPORTED (the caller then takes the
    two-call path).  `sync` is two int32 words, zero before the first call,
    that calls sharing it must not overlap; a fresh zeroed pair when None."""
    _need_cuda(x, torch.float16, "input")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("input must be a 2-D row-major tensor")
    M, K = x.shape
    N = w_codes.shape[0]
    n_out = 0 if outlier_idx is None else int(outlier_idx.numel())
    crot = rot.c()
    kp = L.qr_packed_k(crot, K, n_out)
    if kp < 0:
        raise ValueError("invalid rotation descriptor or sizes")
    dev = x.device
    codes = torch.empty((M, kp // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(M, dtype=torch.float32, device=dev)
    zeros = torch.empty(M, dtype=torch.int32, device=dev) if asym else None
    x_out = torch.empty((M, n_out), dtype=torch.float16, device=dev) if n_out else None
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=dev)
    if sync is None:
        sync = torch.zeros(2, dtype=torch.int32, device=dev)
    st = L.qr_w4a4_linear_fused(crot, x.data_ptr(), M, K, x.stride(0),
                                _ptr(outlier_idx) if n_out else None, n_out, w_codes.data_ptr(),
                                w_scales.data_ptr(), _ptr(w_sums) if asym else None,
                                _ptr(w_out) if n_out else None, N, codes.data_ptr(),
                                scales.data_ptr(), _ptr(zeros), _ptr(x_out), y.data_ptr(),
                                y.stride(0), sync.data_ptr(), _stream(), check=check)
    if st == L.QR_ERR_UNSUPPORTED and not check:
        return None
    if st != L.QR_OK:
        raise L.QrError("qr_w4a4_linear_fused", st)
    return y, codes, scales, zeros, x_out


def w4a4_linear_fused_noalloc(x, rot: Rotation, outlier_idx, w_codes, w_scales, w_out=None,
                              w_sums=None, asym: bool = False, out: Optional[torch.Tensor] = None):
    """w4a4_linear_fused with its intermediate arrays and barrier words in the
    library's own per-device scratch; returns Y only.  Calls on one device
    share that scratch, so they must not overlap (one stream)."""
    _need_cuda(x, torch.float16, "input")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("input must be a 2-D row-major tensor")
    M, K = x.shape
    N = w_codes.shape[0]
    n_out = 0 if outlier_idx is None else int(outlier_idx.numel())
    y = out if out is not None else torch.empty((M, N), dtype=torch.float16, device=x.device)
    L.qr_w4a4_linear_fused_noalloc(rot.c(), x.data_ptr(), M, K, x.stride(0),
                                   _ptr(outlier_idx) if n_out else None, n_out, w_codes.data_ptr(),
                                   w_scales.data_ptr(), _ptr(w_sums) if asym else None,
                                   _ptr(w_out) if n_out else None, N, 1 if asym else 0,
                                   y.data_ptr(), y.stride(0), _stream())
    return y


def kv_quantize(q: Optional[torch.Tensor], k: Optional[torch.Tensor], v: Optional[torch.Tensor],
                head_dim: int, group: int = 128):
    """The KV-cache step after RoPE: R3 (H_d / sqrt(d) per head) on q and k,
    group-wise asymmetric 4-bit codes for k (after R3) and v.  Inputs are
    fp16 [tokens, heads*head_dim] row-major (any may be None).  Returns
    (q_rot, (k_codes, k_scales, k_zeros), (v_codes, v_scales, v_zeros)),
    None for a part not given."""
    given = [t for t in (q, k, v) if t is not None]
    if not given:
        raise ValueError("nothing to do")
    tokens, width = given[0].shape
    for t in given:
        _need_cuda(t, torch.float16, "input")
        if t.shape != (tokens, width) or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous [tokens, heads*head_dim] tensors")
    if width % head_dim:
        raise ValueError("width must be a multiple of head_dim")
    heads = width // head_dim
    dev = given[0].device
    q_rot = torch.empty_like(q) if q is not None else None

    def side(t):
        if t is None:
            return None
        return (torch.empty((tokens, width // 2), dtype=torch.uint8, device=dev),
                torch.empty((tokens, width // group), dtype=torch.float32, device=dev),
                torch.empty((tokens, width // group), dtype=torch.int32, device=dev))
    ks, vs = side(k), side(v)
    p = lambda tup, i: None if tup is None else tup[i].data_ptr()
    L.qr_kv_quantize(_ptr(q), _ptr(k), _ptr(v), tokens, heads, head_dim, group, _ptr(q_rot),
                     p(ks, 0), p(ks, 1), p(ks, 2), p(vs, 0), p(vs, 1), p(vs, 2), _stream())
    return q_rot, ks, vs


def select_outliers(x_calib: torch.Tensor, k: int) -> torch.Tensor:
    """QUIK calibration: the k columns of largest infinity-norm, ascending."""
    _need_cuda(x_calib, torch.float16, "x_calib")
    T, K = x_calib.shape
    idx = torch.empty(k, dtype=torch.int32, device=x_calib.device)
    L.qr_select_outliers(x_calib.data_ptr(), T, K, x_calib.stride(0), k, idx.data_ptr(),
                         _stream())
    return idx


class QuantizedLinear:
    """A linear layer held as rotated 4-bit (or, with bits=8, 8-bit; with
    fp4=True, e2m1) weights; forward() is the online path."""

    def __init__(self, weight: torch.Tensor, rot: Rotation, outlier_idx=None,
                 asym_activations: bool = False, bits: int = 4, fp4: bool = False,
                 fused_decode: bool = False):
        if bits not in (4, 8) or (bits == 8 and asym_activations):
            raise ValueError("bits must be 4, or 8 with symmetric activations")
        if fp4 and (bits != 4 or asym_activations):
            raise ValueError("fp4 codes are 4-bit with symmetric activations")
        self.rot = rot
        self.rot_w = weight_rotation(rot)
        self.outlier_idx = outlier_idx
        self.asym = asym_activations
        self.bits = bits
        self.fp4 = fp4
        pack = pack_weights_fp4 if fp4 else pack_weights8 if bits == 8 else pack_weights
        self.w_codes, self.w_scales, self.w_out, _ = pack(weight, self.rot_w, outlier_idx)
        self.w_sums = weight_code_sums(self.w_codes) if asym_activations else None
        self.out_features, self.in_features = weight.shape
        # with fused_decode, decode steps (M <= 64 tokens) run as one fused
        # kernel when the library takes the shape; its grid barrier words
        # live here, so forward calls of one layer must not overlap (one
        # stream)
        self.fused_decode = fused_decode and bits == 4 and not fp4 and rot.kind != L.QR_ROT_KRON
        self._sync = torch.zeros(2, dtype=torch.int32, device=weight.device)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if self.fp4:
            codes, scales, x_out, _ = rotate_quant_fp4(x, self.rot, self.outlier_idx)
            y, _ = fp4_linear(codes, scales, self.w_codes, self.w_scales, x_out, self.w_out)
            return y
        if self.bits == 8:
            codes, scales, x_out, _ = rotate_quant8(x, self.rot, self.outlier_idx)
            y, _ = w8a8_linear(codes, scales, self.w_codes, self.w_scales, x_out, self.w_out)
            return y
        if self.fused_decode and x.dim() == 2 and 0 < x.shape[0] <= 64:
            r = w4a4_linear_fused(x, self.rot, self.outlier_idx, self.w_codes, self.w_scales,
                                  self.w_out, self.w_sums, self.asym, self._sync, check=False)
            if r is not None:
                return r[0]
        if self.asym:
            codes, scales, zeros, x_out, _ = rotate_quant_asym(x, self.rot, self.outlier_idx)
            y, _ = w4a4_linear_asym(codes, scales, zeros, self.w_codes, self.w_scales, self.w_sums,
                                    x_out, self.w_out)
            return y
        codes, scales, x_out, _ = rotate_quant(x, self.rot, self.outlier_idx)
        y, _ = w4a4_linear(codes, scales, self.w_codes, self.w_scales, x_out, self.w_out)
        return y

    __call__ = forward


class GraphedLinear:
    """The online path of a QuantizedLinear for a fixed token count, captured
    once as a CUDA graph (rotate + quantize, then the W4A4 GEMM).

    A call copies x into the captured input buffer, replays the graph on the
    current stream and returns the captured output buffer, which the next
    call overwrites.  The replay costs one graph launch instead of two
    kernel launches through Python, which is most of a decode step's time.
    """

    def __init__(self, layer: QuantizedLinear, tokens: int):
        dev = layer.w_codes.device
        self.layer = layer
        self.x = torch.zeros((tokens, layer.in_features), dtype=torch.float16, device=dev)
        layer(self.x)                       # first call: module load, kernel attributes
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            self.y = layer(self.x)
        torch.cuda.synchronize(dev)

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        if tuple(x.shape) != tuple(self.x.shape):
            raise ValueError(f"captured for input shape {tuple(self.x.shape)}, got {tuple(x.shape)}")
        self.x.copy_(x, non_blocking=True)
        self.graph.replay()
        return self.y

