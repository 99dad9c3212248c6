"""B200-native online W4A4 rotated linear layer.

The layer rotates fp16 activations per token (Walsh-Hadamard, grouped
sequency-ordered Walsh, or a Kronecker affine transform), quantizes them to
symmetric 4-bit codes, multiplies the codes with pre-rotated 4-bit weights on
tcgen05 integer tensor cores and dequantizes to fp16, adding the QUIK fp16
outlier product.  The compute lives in libqr.so (include/qr.h); this package
is its ctypes binding plus torch-facing helpers.
"""
from . import _lib  # noqa: F401
from .layer import (GSR, HADAMARD, KRON, NONE, GraphedLinear, QuantizedLinear,  # noqa: F401
                    Rotation,
                    invert_transpose, kv_quantize, pack_weights, packed_k, rotate_quant,
                    pack_weights8, rotate_quant8, rotate_quant_asym, w8a8_linear,
                    fp4_linear, pack_weights_fp4, rotate_quant_fp4,
                    select_outliers, w4a4_linear, w4a4_linear_asym, w4a4_linear_fused,
                    w4a4_linear_fused_noalloc,
                    weight_code_sums,
                    weight_rotation)
