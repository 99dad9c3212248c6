// row_quant.cuh -- per-row quantization helpers shared by the rotate kernels
// and the decode kernel's fused rotate prologue: the round-half-to-even
// nibble packer, the per-row symmetric / asymmetric quantizer parameters, a
// streaming vector load, and the shared-memory Walsh-Hadamard pass used for
// whole rows held in shared memory.
#pragma once

#include <cuda_fp16.h>

#include "qr_device.cuh"

namespace qr {

namespace {

constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

// Byte-permute (PTX prmt): byte i of the result is byte sel[i] of {b, a}.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight consecutive codes round_half_even(v[i] * r) (clamped to +-7 when
// CLIP) packed two per byte, v[0] in the low nibble.  Each fused multiply-add
// with 1.5*2^23 leaves the integer's two's-complement byte in the low byte;
// byte permutes gather the even and the odd codes, and one shift and one
// 3-input logic op interleave their nibbles.
template <bool CLIP>
__device__ __forceinline__ uint32_t quant_word(const float (&v)[8], float r, float c = kRoundMagic,
                                               float lo = kRoundMagic - 7.0f,
                                               float hi = kRoundMagic + 7.0f) {
  uint32_t b[8];
  const uint64_t r2 = f2_pack(r, r), c2 = f2_pack(c, c);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    float t0, t1;
    f2_unpack(f2_fma(f2_pack(v[i], v[i + 1]), r2, c2), t0, t1);
    if (CLIP) {
      t0 = fminf(fmaxf(t0, lo), hi);
      t1 = fminf(fmaxf(t1, lo), hi);
    }
    b[i] = __float_as_uint(t0);
    b[i + 1] = __float_as_uint(t1);
  }
  const uint32_t even = prmt(prmt(b[0], b[2], 0x0040u), prmt(b[4], b[6], 0x4000u), 0x7610u);
  const uint32_t odd = prmt(prmt(b[1], b[3], 0x0040u), prmt(b[5], b[7], 0x4000u), 0x7610u);
  uint32_t w;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(w) : "r"(even), "r"(odd << 4), "r"(0x0F0F0F0Fu));
  return w;   // (even & 0x0F0F0F0F) | ((odd << 4) & ~0x0F0F0F0F)
}

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 u;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
               : "l"(p));
  return u;
}

// Per-row quantizer: codes are the low nibble of fma(v, r, c) clamped to
// [lo, hi] (CLIP).  Symmetric (min-max over [-7, 7]): c = 1.5*2^23, bounds
// +-7.  Asymmetric (QUIK's per-token activations, min-max over [0, 15]
// stored as q - 8): c = 1.5*2^23 + z - 8, bounds [-8, 7], and the kernels
// always clamp.  v are the unnormalized transform outputs; inv_sqrt folds
// the 1/sqrt(b) of the rotation into the scale.
struct RowQ { float r, c, lo, hi; };

__device__ __forceinline__ RowQ sym_row_q(float am, float clip, float inv_sqrt, float* scale_out) {
  if (scale_out != nullptr) *scale_out = __fdividef(clip * (am * inv_sqrt), 7.0f);
  return RowQ{(am > 0.0f) ? __fdividef(7.0f, clip * am) : 0.0f, kRoundMagic, kRoundMagic - 7.0f,
              kRoundMagic + 7.0f};
}

// 8-bit symmetric codes (QUIK's INT8 layers): s = alpha * absmax / 127,
// codes clamped to +-127.
__device__ __forceinline__ RowQ sym_row_q8(float am, float clip, float inv_sqrt, float* scale_out) {
  if (scale_out != nullptr) *scale_out = __fdividef(clip * (am * inv_sqrt), 127.0f);
  return RowQ{(am > 0.0f) ? __fdividef(127.0f, clip * am) : 0.0f, kRoundMagic, kRoundMagic - 127.0f,
              kRoundMagic + 127.0f};
}

__device__ __forceinline__ RowQ asym_row_q(float mn, float mx, float clip, float inv_sqrt,
                                           float* scale_out, int32_t* zero_out) {
  const float lo = clip * mn, hi = clip * mx;
  const float range = hi - lo;
  const float r = range > 0.0f ? 15.0f / range : 0.0f;
  const float z = range > 0.0f ? rintf(-lo * r) : 0.0f;
  if (scale_out != nullptr) {
    *scale_out = range * inv_sqrt / 15.0f;
    *zero_out = static_cast<int32_t>(z) - 8;
  }
  return RowQ{r, kRoundMagic + (z - 8.0f), kRoundMagic - 8.0f, kRoundMagic + 7.0f};
}

// Shared-memory position of row element e: bits 3-4 XOR bits 6-7, so that
// the butterfly passes with strides 8..32 hit 32 distinct banks; groups of 8
// consecutive elements stay contiguous and aligned.
__device__ __forceinline__ int few_swz(int e) { return e ^ (((e >> 6) & 3) << 3); }

// R butterfly stages on index bits [s, s+R) of the row in shared memory;
// thread t of nthr takes every nthr-th group of 2^R elements.  Returns the
// largest |value| this thread wrote.
template <int R>
__device__ __forceinline__ float wht_smem_pass(float* buf, int Kp, int s, int t, int nthr) {
  constexpr int G = 1 << R;
  const int ngroups = Kp >> R;
  const int lowmask = (1 << s) - 1;
  float am = 0.0f;
  for (int g = t; g < ngroups; g += nthr) {
    const int base = (g & lowmask) | ((g >> s) << (s + R));
    float x[G];
    if (R == 3 && s == 0) {                        // 8 contiguous, aligned elements
      const float4 a = *reinterpret_cast<const float4*>(buf + few_swz(base));
      const float4 b = *reinterpret_cast<const float4*>(buf + few_swz(base) + 4);
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
      x[4 % G] = b.x; x[5 % G] = b.y; x[6 % G] = b.z; x[7 % G] = b.w;
    } else {
#pragma unroll
      for (int k = 0; k < G; ++k) x[k] = buf[few_swz(base + (k << s))];
    }
#pragma unroll
    for (int st = 0; st < R; ++st)
#pragma unroll
      for (int k = 0; k < G; ++k)
        if (!(k & (1 << st))) {
          const float a = x[k], b = x[k | (1 << st)];
          x[k] = a + b;
          x[k | (1 << st)] = a - b;
        }
#pragma unroll
    for (int k = 0; k < G; ++k) am = fmaxf(am, fabsf(x[k]));
    if (R == 3 && s == 0) {
      *reinterpret_cast<float4*>(buf + few_swz(base)) = make_float4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<float4*>(buf + few_swz(base) + 4) =
          make_float4(x[4 % G], x[5 % G], x[6 % G], x[7 % G]);
    } else {
#pragma unroll
      for (int k = 0; k < G; ++k) buf[few_swz(base + (k << s))] = x[k];
    }
  }
  return am;
}

}  // namespace

}  // namespace qr
