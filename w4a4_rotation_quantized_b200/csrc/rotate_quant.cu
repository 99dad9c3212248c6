// rotate_quant.cu -- fused rotate + per-row 4-bit quantize + pack.
//
// One pass over HBM per row: read fp16 (optionally gathering the non-outlier
// columns, QUIK "QUIK量化" §1), rotate in fp32, reduce the row absmax,
// quantize with round-half-to-even, pack two codes per byte, store.  The same
// kernels quantize activations online (per token; QuaRot §2 online Hadamard,
// FlatQuant §2.3 fused transform + quantization) and weights offline (per
// output channel; QuaRot §2 stage 1).
//
// Walsh-Hadamard rows (HADAMARD, GSR, NONE = block 1).  A row is cut into
// 256-element chunks; lane l of a warp holds elements [8l, 8l+8) of each of
// its CPW chunks in registers.  Element index bits 0-2 are therefore inside a
// thread, bits 3-7 across lanes, bits 8.. across a warp's chunks, and any
// higher bits across the warps of a row.  The butterfly H_2 is applied on
// bits [0, log2 b) in that order: in registers, by warp shuffles, in
// registers again, and through shared memory only for blocks above
// 256*CPW elements.  The 1/sqrt(b) factor is folded into the scale.  For the
// grouped sequency-ordered rotation ("Grouped Sequency-arranged Rotation",
// 方法详解) the Walsh matrix of a block is its Hadamard matrix with rows
// permuted, and it is symmetric, so output position j of a block takes
// Hadamard output perm(j) = bitrev(gray(j)); the codes are scattered to their
// sequency positions through shared memory before packing.
//
// Kronecker rows (FlatQuant §2.3): x -> vec(P1^T mat(x) P2), two small
// matrix products per row in fp32 on CUDA cores with P1, P2 resident in
// shared memory.
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

#include "qr_device.cuh"
#include "qr_internal.h"
#include "row_quant.cuh"

namespace qr {

namespace {

// Nibble of round_half_even(v * r), optionally clamped to +-7.  Adding
// 1.5*2^23 leaves a float whose unit in the last place is 1, so the single
// rounding of the fused multiply-add is round-to-nearest-even of the exact
// product; the integer then sits in the low mantissa bits, and its low four
// bits are its two's-complement nibble.
template <bool CLIP>
__device__ __forceinline__ uint32_t quant_nibble(float v, float r, float c = kRoundMagic,
                                                 float lo = kRoundMagic - 7.0f,
                                                 float hi = kRoundMagic + 7.0f) {
  float t = fmaf(v, r, c);
  if (CLIP) t = fminf(fmaxf(t, lo), hi);
  return __float_as_uint(t) & 0xFu;
}

__device__ __forceinline__ void row_barrier(int group, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(group + 1), "r"(nthreads) : "memory");
}

// Eight 8-bit codes round_half_even(v[i] * r) (clamped to [lo, hi] when
// CLIP), one byte each, v[0] first: the low byte of each fma with 1.5*2^23
// is the code's two's-complement byte; byte permutes gather them.
template <bool CLIP>
__device__ __forceinline__ uint2 quant_bytes8(const float (&v)[8], float r, float c, float lo,
                                              float hi) {
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
  return make_uint2(prmt(prmt(b[0], b[1], 0x0040u), prmt(b[2], b[3], 0x4000u), 0x7610u),
                    prmt(prmt(b[4], b[5], 0x0040u), prmt(b[6], b[7], 0x4000u), 0x7610u));
}

// One 8-bit code round_half_even(v * r) (clamped to [lo, hi] when CLIP) as
// its two's-complement byte.
template <bool CLIP>
__device__ __forceinline__ uint32_t quant_byte(float v, float r, float c, float lo, float hi) {
  float t = fmaf(v, r, c);
  if (CLIP) t = fminf(fmaxf(t, lo), hi);
  return __float_as_uint(t) & 0xFFu;
}

// Inverse of the binary-reflected Gray code on 8 bits.
__device__ __forceinline__ int gray_inverse(int g) {
  g ^= g >> 1;
  g ^= g >> 2;
  g ^= g >> 4;
  return g;
}

// Builds, in shared memory, kept[e] = the source column of rotated column e
// (0xFFFF = none), from the strictly ascending outlier index list.  Each
// thread takes a contiguous range of source columns: one binary search for
// the outliers before it, then a walk that skips the outliers it meets.
// Malformed lists never write outside [0, Kr).
__device__ void build_kept_table(const int32_t* __restrict__ outlier_idx, int n_out, int K,
                                 int Kr, uint16_t* kept, int32_t* sidx) {
  for (int i = threadIdx.x; i < n_out; i += blockDim.x) sidx[i] = outlier_idx[i];
  for (int e = threadIdx.x; e < Kr; e += blockDim.x) kept[e] = 0xFFFFu;
  __syncthreads();
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int c0 = threadIdx.x * per;
  const int c1 = c0 + per < K ? c0 + per : K;
  if (c0 < c1) {
    int lo = 0, hi = n_out;            // lo = number of outliers < c0
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sidx[mid] < c0) lo = mid + 1; else hi = mid;
    }
    for (int c = c0; c < c1; ++c) {
      if (lo < n_out && sidx[lo] == c) {
        ++lo;
        continue;
      }
      const int pos = c - lo;
      if (pos >= 0 && pos < Kr) kept[pos] = static_cast<uint16_t>(c);
    }
  }
  __syncthreads();
}

struct WhtParams {
  const __half* src;
  int64_t rows, ld;
  int32_t K, Kr, Kp, n_out;
  const int32_t* outlier_idx;
  const int8_t* signs;        // random-sign diagonal [Kp] or null
  int32_t lb;                 // butterflies on in-block index bits [0, lb)
  int32_t nb;                 // blocks per row, Kp >> lb
  int32_t gsr;                // sequency order within blocks
  int32_t vec_ok;             // 16-byte loads allowed (aligned rows, no gather)
  int32_t nt;                 // threads per row group (multiple of 32)
  int32_t rows_per_cta;       // row groups per CTA
  int32_t items;              // items per thread in the register-held phase
  float clip_ratio, inv_sqrt_block;
  uint8_t* codes;
  float* scales;
  int32_t* zeros;             // asymmetric activations: zero points [rows] (null: symmetric)
  __half* out16;
  float* rot_debug;
  int32_t off_buf, buf_bytes, off_red, off_kept, off_idx;   // shared-memory carve-up
  int32_t off_signs;          // the sign diagonal as bits [Kp/8] (signs != null)
  // ring mode: rows stream into shared memory by bulk copies
  int32_t ring_slots, ring_row_bytes, off_ring, off_bars, rows_per_block;
  int32_t* status;
  int32_t bits8;              // 8-bit codes (one int8 per code) instead of nibbles
};

// Loads 8 consecutive rotated-domain elements [e, e+8) of a row as fp32:
// gathered through the kept-column table when outliers are split off,
// zero beyond the Kr real columns.
__device__ __forceinline__ void load8(const WhtParams& p, const __half* srow, const uint16_t* kept,
                                      int e, float (&x)[8]) {
  if (p.n_out == 0 && p.vec_ok && e + 8 <= p.Kr) {
    const uint4 u = ld_stream_v4(srow + e);
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __half22float2(h[q]);
      x[2 * q] = f.x;
      x[2 * q + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ei = e + i;
      float v = 0.0f;
      if (ei < p.Kr) {
        const int c = p.n_out ? static_cast<int>(kept[ei]) : ei;
        if (c < p.K) v = __half2float(srow[c]);
      }
      x[i] = v;
    }
  }
}

// The QUIK outlier columns of a row, copied through unchanged.
__device__ __forceinline__ void copy_outliers(const WhtParams& p, const __half* srow, int64_t row,
                                              int t, int nt) {
  if (p.n_out > 0 && p.out16 != nullptr)
    for (int j = t; j < p.n_out; j += nt) {
      const int c = __ldg(p.outlier_idx + j);
      p.out16[row * p.n_out + j] = (c >= 0 && c < p.K) ? srow[c] : __float2half(0.0f);
    }
}

// Randomized Hadamard.  The CTA first packs the int8 sign diagonal into a
// bitmask in shared memory (bit j of byte i: element 8i + j is negated; only
// the sign bit of each int8 entry is read); then 8 consecutive rotated-domain
// values [e, e+8) flip their sign bits where the diagonal is negative.  The
// flip is exact.
__device__ __forceinline__ void build_sign_bits(const int8_t* signs, int kp, uint8_t* bits) {
  for (int i = threadIdx.x; i < kp / 8; i += blockDim.x) {
    const uint2 d = __ldg(reinterpret_cast<const uint2*>(signs) + i);
    uint32_t b = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      b |= ((d.x >> (8 * j + 7)) & 1u) << j;
      b |= ((d.y >> (8 * j + 7)) & 1u) << (4 + j);
    }
    bits[i] = static_cast<uint8_t>(b);
  }
}

__device__ __forceinline__ void apply_signs8(const uint8_t* bits, int e, float (&x)[8]) {
  const uint32_t b = bits[e >> 3];
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __uint_as_float(__float_as_uint(x[i]) ^ (((b >> i) & 1u) << 31));
}

// Shared-memory position of rotated element e: 8 floats of padding after
// every 2^SH elements (SH = the layout-B stride bits), so that the 8-float
// groups a warp reads in layout B fall in distinct banks while each thread's
// layout-B values stay at constant offsets from one base.
template <int SH>
__device__ __forceinline__ int swz(int e) {
  return e + ((e >> SH) << 3);
}

// Maximum over a row group (any sign).
__device__ __forceinline__ float row_max(float v, float* red, int rg, int t, int nt) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int nw = nt >> 5;
  if (nw > 1) {
    if ((t & 31) == 0) red[t >> 5] = v;
    row_barrier(rg, nt);
    v = -INFINITY;
    for (int w = 0; w < nw; ++w) v = fmaxf(v, red[w]);
  }
  return v;
}

// Reduce a row's absmax over its row group; returns the maximum.
__device__ __forceinline__ float row_absmax(float am, float* red, int rg, int t, int nt) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int nw = nt >> 5;
  if (nw > 1) {
    if ((t & 31) == 0) red[t >> 5] = am;
    row_barrier(rg, nt);
    am = 0.0f;
    for (int w = 0; w < nw; ++w) am = fmaxf(am, red[w]);
  }
  return am;
}

// Sequency output of a block of 2^LB (6 <= LB <= 8) held by a layout-B
// thread (natural in-block index tb_low + 8 j, j < 2^(LB-3)): output word k
// (positions 8k..8k+7) takes Hadamard outputs perm(8k+t) = bitrev(gray(8k+t)),
// whose three low bits do not depend on t, so one thread owns each word.  For
// p_m the bits of a position, the low three bits of perm are
// (p_{LB-1}, p_{LB-2}^p_{LB-1}, p_{LB-3}^p_{LB-2}); the in-register index j
// of perm(8k+t) is a constant of (t, k's free bits) XOR p_{LB-3}.
template <int LB>
__host__ __device__ constexpr int gsr_j_static(int t, int f) {
  // position with p_{LB-3..LB-1} = 0: pos = 8 f + t
  int pos = 8 * f + t;
  int j = 0;
  for (int m = 3; m < LB; ++m) {
    const int i = LB - 1 - m;                       // j bit (m-3) = g_i
    const int gi = ((pos >> i) & 1) ^ ((i + 1 < LB) ? ((pos >> (i + 1)) & 1) : 0);
    j |= gi << (m - 3);
  }
  return j;
}

// Kernel for blocks of 2^LB with LB = 3 + MB + HA >= 4.
//   layout A: a thread holds in-block bits {0,1,2} and the top HA bits
//             (2^(3+HA) values, loaded as 16-byte rows of 8), T_A = 2^MB
//             threads per block;
//   layout B: a thread holds the MB middle bits {3..2+MB} (2^MB values),
//             T_B = 2^(3+HA) threads per block.
// Butterflies run in registers in each layout; one pass through shared
// memory (fp32, swizzled) moves the row from A to B.  OUT: 0 = natural order
// via 8x8 nibble transposes across lanes, 1 = sequency order assembled in a
// thread (HA = 0, 3 <= MB <= 5), 2 = codes scattered through shared memory.
template <int MB, int HA, int ITEMS>
struct AbBounds {
  static constexpr int value = ((8 << HA) <= 64 && (1 << MB) * ITEMS <= 64) ? 512 : 256;
};

template <int MB, int HA, int ITEMS, bool CLIP, int OUT, bool RING>
__global__ void __launch_bounds__(AbBounds<MB, HA, ITEMS>::value) wht_ab_kernel(const WhtParams p) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int LB = 3 + MB + HA;
  constexpr int EA = 8 << HA, TA = 1 << MB;
  constexpr int EB = 1 << MB, TB = 8 << HA;
  extern __shared__ __align__(16) uint8_t smem[];
  const int nt = p.nt;
  const int rg = threadIdx.x / nt;
  const int t = threadIdx.x - rg * nt;
  const int lane = threadIdx.x & 31;
  uint8_t* sbits = smem + p.off_signs;
  if (p.signs != nullptr) {
    build_sign_bits(p.signs, p.Kp, sbits);
    __syncthreads();
  }
  uint16_t* kept = reinterpret_cast<uint16_t*>(smem + p.off_kept);
  if (p.n_out > 0) build_kept_table(p.outlier_idx, p.n_out, p.K, p.Kr, kept,
                                    reinterpret_cast<int32_t*>(smem + p.off_idx));
  float* buf = reinterpret_cast<float*>(smem + p.off_buf + static_cast<size_t>(rg) * p.buf_bytes);
  float* red = reinterpret_cast<float*>(smem + p.off_red) + rg * 32;
  const int items_a = p.nb * TA, items_b = p.nb * TB;

  // Ring mode: the CTA owns rows [row0, row1); a producer warp (after the
  // row groups) streams them into ring slots with bulk copies; row group g
  // takes the CTA's rows g, g+R, ...
  uint64_t* ring_full = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint64_t* ring_empty = ring_full + p.ring_slots;
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(ring_empty + p.ring_slots);
  int64_t row0 = 0, row1 = 0;
  if constexpr (RING) {
    row0 = static_cast<int64_t>(blockIdx.x) * p.rows_per_block;
    row1 = row0 + p.rows_per_block < p.rows ? row0 + p.rows_per_block : p.rows;
    if (threadIdx.x == 0) {
      for (int i = 0; i < p.ring_slots; ++i) {
        mbar_init(&ring_full[i], 1);
        mbar_init(&ring_empty[i], nt / 32);
      }
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncthreads();
    if (rg == p.rows_per_cta) {            // the producer warp
      if (lane == 0) {
        const int n = static_cast<int>(row1 - row0);
        int i = 0;
        bool ok = true;
        for (; i < n; ++i) {
          const int s = i % p.ring_slots;
          const uint32_t ph = (i / p.ring_slots) & 1;
          if (!(ok = mbar_wait_bounded(&ring_empty[s], ph ^ 1, abort_flag, p.status,
                                       kDevTimeoutProducer)))
            break;
          mbar_arrive_expect_tx(&ring_full[s], p.ring_row_bytes);
          bulk_load(smem + p.off_ring + static_cast<size_t>(s) * p.ring_row_bytes,
                    p.src + (row0 + i) * p.ld, p.ring_row_bytes, &ring_full[s]);
        }
        // every copy issued lands before the CTA may exit
        for (int j = (i > p.ring_slots ? i - p.ring_slots : 0); j < i; ++j)
          mbar_wait_bounded(&ring_full[j % p.ring_slots], (j / p.ring_slots) & 1, abort_flag,
                            nullptr, 0, kDrainLimitNs);
      }
      return;
    }
  }
  const int64_t row_first = RING ? row0 + rg : static_cast<int64_t>(blockIdx.x) * p.rows_per_cta + rg;
  const int64_t row_end = RING ? row1 : p.rows;
  const int64_t row_step = RING ? p.rows_per_cta : static_cast<int64_t>(gridDim.x) * p.rows_per_cta;

  for (int64_t row = row_first; row < row_end; row += row_step) {
    const __half* srow = p.src + row * p.ld;
    const __half* ring_row = nullptr;
    int slot = 0;
    if constexpr (RING) {
      const int i = static_cast<int>(row - row0);
      slot = i % p.ring_slots;
      if (!mbar_wait_bounded(&ring_full[slot], (i / p.ring_slots) & 1, abort_flag, p.status,
                             kDevTimeoutWiden))
        break;
      ring_row = reinterpret_cast<const __half*>(smem + p.off_ring +
                                                 static_cast<size_t>(slot) * p.ring_row_bytes);
    } else {
      copy_outliers(p, srow, row, t, nt);
    }

    // ---- phase A: load, butterflies on bits {0,1,2} and the top HA bits
#pragma unroll 1
    for (int w = t; w < items_a; w += nt) {
      const int blk = w >> MB, ta = w & (TA - 1);
      const int e0 = (blk << LB) + 8 * ta;
      float v[EA];
#pragma unroll
      for (int h = 0; h < (1 << HA); ++h) {
        float x[8];
        const int e = e0 + (h << (3 + MB));
        if constexpr (RING) {
          if (e + 8 <= p.Kr) {
            const uint4 u = *reinterpret_cast<const uint4*>(ring_row + e);
            const __half2* hh = reinterpret_cast<const __half2*>(&u);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 f = __half22float2(hh[q]);
              x[2 * q] = f.x;
              x[2 * q + 1] = f.y;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = 0.0f;
          }
        } else {
          load8(p, srow, kept, e, x);
        }
        if (p.signs != nullptr) apply_signs8(sbits, e, x);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[8 * h + i] = x[i];
      }
      wht_stages<0, 3 + HA>(v);
#pragma unroll
      for (int h = 0; h < (1 << HA); ++h) {
        const int e = e0 + (h << (3 + MB));
        float4* d = reinterpret_cast<float4*>(buf + swz<3 + MB>(e));
        d[0] = make_float4(v[8 * h], v[8 * h + 1], v[8 * h + 2], v[8 * h + 3]);
        d[1] = make_float4(v[8 * h + 4], v[8 * h + 5], v[8 * h + 6], v[8 * h + 7]);
      }
    }
    if constexpr (RING) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&ring_empty[slot]);
    }
    row_barrier(rg, nt);

    // ---- phase B: butterflies on the middle bits, absmax
    float v[ITEMS][EB];
    float am = 0.0f;
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
      const int w = t + k * nt;
      const bool ok = w < items_b;
      const int blk = w >> (3 + HA), tb = w & (TB - 1);
      const int e0 = (blk << LB) + (tb & 7) + ((tb >> 3) << (3 + MB));
      const float* bp = buf + swz<3 + MB>(e0);          // e0 + 8j never crosses 2^(3+MB)
#pragma unroll
      for (int j = 0; j < EB; ++j) v[k][j] = ok ? bp[8 * j] : 0.0f;
      wht_stages<0, MB>(v[k]);
#pragma unroll
      for (int j = 0; j < EB; ++j) am = fmaxf(am, fabsf(v[k][j]));
    }
    RowQ q;
    if (p.zeros == nullptr) {
      am = row_absmax(am, red, rg, t, nt);
      q = p.bits8 ? sym_row_q8(am, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr)
                  : sym_row_q(am, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr);
    } else {
      float mx = -INFINITY, mn = INFINITY;
#pragma unroll
      for (int k = 0; k < ITEMS; ++k)
        if (t + k * nt < items_b)
#pragma unroll
          for (int j = 0; j < EB; ++j) {
            mx = fmaxf(mx, v[k][j]);
            mn = fminf(mn, v[k][j]);
          }
      mx = row_max(mx, red, rg, t, nt);
      mn = -row_max(-mn, red + 16, rg, t, nt);
      q = asym_row_q(mn, mx, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr,
                     p.zeros + row);
    }
    const float r = q.r;
    uint8_t* crow = p.codes + row * (p.bits8 ? p.Kp : (p.Kp >> 1));

    if (p.rot_debug != nullptr) {
#pragma unroll
      for (int k = 0; k < ITEMS; ++k) {
        const int w = t + k * nt;
        if (w < items_b) {
          const int blk = w >> (3 + HA), tb = w & (TB - 1);
          const int e0 = (blk << LB) + (tb & 7) + ((tb >> 3) << (3 + MB));
#pragma unroll
          for (int j = 0; j < EB; ++j) {
            int n = (e0 & ((1 << LB) - 1)) + 8 * j;
            if (p.gsr) {
              const int rev = static_cast<int>(__brev(static_cast<unsigned>(n)) >> (32 - LB));
              n = gray_inverse(rev);
            }
            p.rot_debug[row * p.Kp + (blk << LB) + n] = v[k][j] * p.inv_sqrt_block;
          }
        }
      }
    }

    if (p.bits8) {
      // 8-bit codes: one byte each through shared memory at its output
      // position, then copied out in 16-byte pieces
      row_barrier(rg, nt);                 // every thread is done reading buf
      uint8_t* cb = reinterpret_cast<uint8_t*>(buf);
#pragma unroll
      for (int k = 0; k < ITEMS; ++k) {
        const int w = t + k * nt;
        if (w < items_b) {
          const int blk = w >> (3 + HA), tb = w & (TB - 1);
          const int e0 = (blk << LB) + (tb & 7) + ((tb >> 3) << (3 + MB));
#pragma unroll
          for (int j = 0; j < EB; ++j) {
            int n = (e0 & ((1 << LB) - 1)) + 8 * j;
            if (p.gsr) {
              const int rev = static_cast<int>(__brev(static_cast<unsigned>(n)) >> (32 - LB));
              n = gray_inverse(rev);
            }
            cb[(blk << LB) + n] = static_cast<uint8_t>(quant_byte<CLIP>(v[k][j], r, q.c, q.lo, q.hi));
          }
        }
      }
      row_barrier(rg, nt);
      for (int e = 16 * t; e < p.Kp; e += 16 * nt)
        *reinterpret_cast<uint4*>(crow + e) = *reinterpret_cast<const uint4*>(cb + e);
    } else if constexpr (OUT == 0) {
      static_assert(MB >= 3, "nibble transposes need 8 values per lane");
      const int l = lane & 7;
      const uint32_t sel4 = (l & 4) ? 0x3276u : 0x5410u;
      const uint32_t sel2 = (l & 2) ? 0x3715u : 0x6240u;
      const uint32_t rot1 = (l & 1) ? 28u : 4u;
      const uint32_t msk1 = (l & 1) ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
#pragma unroll
      for (int k = 0; k < ITEMS; ++k) {
        const int w = t + k * nt;
        const int blk = w >> (3 + HA), tb = w & (TB - 1);
#pragma unroll
        for (int wb = 0; wb < EB / 8; ++wb) {
          float q8[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) q8[jj] = v[k][8 * wb + jj];
          uint32_t W = quant_word<CLIP>(q8, r, q.c, q.lo, q.hi);
          // Transpose the 8x8 nibble block held by the lanes with tb_low =
          // 0..7: swap 16-bit halves with lane^4, bytes with lane^2 (byte
          // permutes), nibbles with lane^1 (rotate + 3-input logic op).
          W = prmt(W, __shfl_xor_sync(0xffffffffu, W, 4), sel4);
          W = prmt(W, __shfl_xor_sync(0xffffffffu, W, 2), sel2);
          {
            const uint32_t P = __shfl_xor_sync(0xffffffffu, W, 1);
            const uint32_t s4 = __funnelshift_l(P, P, rot1);
            uint32_t nw;
            asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(nw) : "r"(W), "r"(s4), "r"(msk1));
            W = nw;   // (W & msk1) | (s4 & ~msk1)
          }
          if (w < items_b) {
            const int e = (blk << LB) + 8 * (8 * wb + l) + ((tb >> 3) << (3 + MB));
            *reinterpret_cast<uint32_t*>(crow + (e >> 1)) = W;
          }
        }
      }
    } else if constexpr (OUT == 1) {
      static_assert(HA == 0 && MB >= 3 && MB <= 5, "in-thread sequency words");
#pragma unroll
      for (int k = 0; k < ITEMS; ++k) {
        const int w = t + k * nt;
        if (w < items_b) {
          const int blk = w >> 3, tbl = w & 7;
          const int a0 = tbl & 1, a1 = (tbl >> 1) & 1, a2 = (tbl >> 2) & 1;
          const int p1 = a0, p2 = a1 ^ a0, p3 = a2 ^ p2;   // p_{LB-1}, p_{LB-2}, p_{LB-3}
          uint32_t nib[EB];
#pragma unroll
          for (int j = 0; j < EB; ++j) nib[j] = quant_nibble<CLIP>(v[k][j], r, q.c, q.lo, q.hi);
#pragma unroll
          for (int f = 0; f < (1 << (MB - 3)); ++f) {
            const int kw = f | (p3 << (MB - 3)) | (p2 << (MB - 2)) | (p1 << (MB - 1));
            uint32_t W = 0;
#pragma unroll
            for (int tt = 0; tt < 8; ++tt) {
              const int js = gsr_j_static<LB>(tt, f);
              const uint32_t nv = p3 ? nib[js ^ 1] : nib[js];
              W |= nv << (4 * tt);
            }
            *reinterpret_cast<uint32_t*>(crow + (((blk << LB) + 8 * kw) >> 1)) = W;
          }
        }
      }
    } else {
      // codes through shared memory (one byte each), then packed
      row_barrier(rg, nt);                 // every thread is done reading buf
      uint8_t* cb = reinterpret_cast<uint8_t*>(buf);
#pragma unroll
      for (int k = 0; k < ITEMS; ++k) {
        const int w = t + k * nt;
        if (w < items_b) {
          const int blk = w >> (3 + HA), tb = w & (TB - 1);
          const int e0 = (blk << LB) + (tb & 7) + ((tb >> 3) << (3 + MB));
#pragma unroll
          for (int j = 0; j < EB; ++j) {
            int n = (e0 & ((1 << LB) - 1)) + 8 * j;
            if (p.gsr) {
              const int rev = static_cast<int>(__brev(static_cast<unsigned>(n)) >> (32 - LB));
              n = gray_inverse(rev);
            }
            cb[(blk << LB) + n] = static_cast<uint8_t>(quant_nibble<CLIP>(v[k][j], r, q.c, q.lo, q.hi));
          }
        }
      }
      row_barrier(rg, nt);
      for (int e = 8 * t; e < p.Kp; e += 8 * nt) {
        const uint32_t lo = *reinterpret_cast<const uint32_t*>(cb + e);
        const uint32_t hi = *reinterpret_cast<const uint32_t*>(cb + e + 4);
        const uint32_t plo = (lo & 0xFu) | ((lo >> 4) & 0xF0u) | ((lo >> 8) & 0xF00u) |
                             ((lo >> 12) & 0xF000u);
        const uint32_t phi = (hi & 0xFu) | ((hi >> 4) & 0xF0u) | ((hi >> 8) & 0xF00u) |
                             ((hi >> 12) & 0xF000u);
        *reinterpret_cast<uint32_t*>(crow + (e >> 1)) = plo | (phi << 16);
      }
    }
    row_barrier(rg, nt);                   // buf and red are reused by the next row
  }
}

// Blocks of at most 8 (and no rotation): a thread holds ITEMS groups of 8
// consecutive elements, all block bits are inside a thread.
template <int ITEMS, bool CLIP>
__global__ void __launch_bounds__(512) wht_small_kernel(const WhtParams p) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ __align__(16) uint8_t smem[];
  const int nt = p.nt;
  const int rg = threadIdx.x / nt;
  const int t = threadIdx.x - rg * nt;
  uint8_t* sbits = smem + p.off_signs;
  if (p.signs != nullptr) {
    build_sign_bits(p.signs, p.Kp, sbits);
    __syncthreads();
  }
  uint16_t* kept = reinterpret_cast<uint16_t*>(smem + p.off_kept);
  if (p.n_out > 0) build_kept_table(p.outlier_idx, p.n_out, p.K, p.Kr, kept,
                                    reinterpret_cast<int32_t*>(smem + p.off_idx));
  float* red = reinterpret_cast<float*>(smem + p.off_red) + rg * 32;
  const int lb = p.lb;
  const int ngroups = p.Kp >> 3;
  const int64_t row_step = static_cast<int64_t>(gridDim.x) * p.rows_per_cta;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * p.rows_per_cta + rg; row < p.rows;
       row += row_step) {
    const __half* srow = p.src + row * p.ld;
    copy_outliers(p, srow, row, t, nt);
    float v[ITEMS][8];
    float am = 0.0f;
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
      const int g = t + k * nt;
      float x[8];
      if (g < ngroups) {
        load8(p, srow, kept, 8 * g, x);
        if (p.signs != nullptr) apply_signs8(sbits, 8 * g, x);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = 0.0f;
      }
#pragma unroll
      for (int s = 0; s < 3; ++s)
        if (s < lb)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (!(i & (1 << s))) {
              const float a = x[i], b = x[i | (1 << s)];
              x[i] = a + b;
              x[i | (1 << s)] = a - b;
            }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[k][i] = x[i];
        am = fmaxf(am, fabsf(x[i]));
      }
    }
    RowQ q;
    if (p.zeros == nullptr) {
      am = row_absmax(am, red, rg, t, nt);
      q = p.bits8 ? sym_row_q8(am, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr)
                  : sym_row_q(am, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr);
    } else {
      float mx = -INFINITY, mn = INFINITY;
#pragma unroll
      for (int k = 0; k < ITEMS; ++k)
        if (t + k * nt < ngroups)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            mx = fmaxf(mx, v[k][i]);
            mn = fminf(mn, v[k][i]);
          }
      mx = row_max(mx, red, rg, t, nt);
      mn = -row_max(-mn, red + 16, rg, t, nt);
      q = asym_row_q(mn, mx, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr,
                     p.zeros + row);
    }
    const float r = q.r;
    uint8_t* crow = p.codes + row * (p.bits8 ? p.Kp : (p.Kp >> 1));
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
      const int g = t + k * nt;
      if (g < ngroups) {
        uint32_t W = 0, B0 = 0, B1 = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          int pos = i;
          if (p.gsr && lb > 0) {
            const int bm = (1 << lb) - 1;
            const int rev = static_cast<int>(__brev(static_cast<unsigned>(i & bm)) >> (32 - lb));
            pos = (i & ~bm) + gray_inverse(rev);
          }
          if (p.bits8) {
            const uint32_t b = quant_byte<CLIP>(v[k][i], r, q.c, q.lo, q.hi);
            if (pos < 4) B0 |= b << (8 * pos); else B1 |= b << (8 * (pos - 4));
          } else {
            W |= quant_nibble<CLIP>(v[k][i], r, q.c, q.lo, q.hi) << (4 * pos);
          }
          if (p.rot_debug != nullptr) p.rot_debug[row * p.Kp + 8 * g + pos] = v[k][i] * p.inv_sqrt_block;
        }
        if (p.bits8)
          *reinterpret_cast<uint2*>(crow + 8 * g) = make_uint2(B0, B1);
        else
          *reinterpret_cast<uint32_t*>(crow + 4 * g) = W;
      }
    }
    row_barrier(rg, nt);                   // red is reused by the next row
  }
}

// FP4 (e2m1) codes with a per-row scale: s = alpha * absmax / 6; the codes
// are the nearest e2m1 values of x / s (ties to the even mantissa,
// saturating at +-6), the tensor core's own conversion.
__device__ __forceinline__ RowQ sym_row_qf4(float am, float clip, float inv_sqrt, float* scale_out) {
  if (scale_out != nullptr) *scale_out = __fdividef(clip * (am * inv_sqrt), 6.0f);
  return RowQ{(am > 0.0f) ? __fdividef(6.0f, clip * am) : 0.0f, 0.0f, 0.0f, 0.0f};
}

// Two e2m1 codes of (lo * r, hi * r) in one byte, lo in the low nibble.
__device__ __forceinline__ uint32_t e2m1_pair(float lo, float hi, float r) {
  uint32_t b;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(b)
      : "f"(hi * r), "f"(lo * r));
  return b;
}

// Eight consecutive e2m1 codes of v[i] * r packed two per byte, v[0] in the
// low nibble (the layout of quant_word).
__device__ __forceinline__ uint32_t quant_word_fp4(const float (&v)[8], float r) {
  const uint32_t b0 = e2m1_pair(v[0], v[1], r), b1 = e2m1_pair(v[2], v[3], r);
  const uint32_t b2 = e2m1_pair(v[4], v[5], r), b3 = e2m1_pair(v[6], v[7], r);
  return prmt(prmt(b0, b1, 0x0040u), prmt(b2, b3, 0x0040u), 0x5410u);
}

// Three-input maximum / minimum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Stage-0 butterfly of a half2 (lo, hi) straight into fp32: (lo + hi, lo - hi),
// each with one rounding (mixed-precision fma with an fp16 multiplicand).
__device__ __forceinline__ void bfly_h2(uint32_t w, float& y0, float& y1) {
  asm("{\n\t.reg .f16 l, h, one;\n\t.reg .f32 fh, nfh;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "mov.b16 one, 0x3C00;\n\t"
      "cvt.f32.f16 fh, h;\n\t"
      "neg.f32 nfh, fh;\n\t"
      "fma.rn.f32.f16 %0, l, one, fh;\n\t"
      "fma.rn.f32.f16 %1, l, one, nfh;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "r"(w));
}
// Sign flips of a half2 word for elements 2q, 2q+1 from a byte of sign bits.
__device__ __forceinline__ uint32_t sign_mask_h2(uint32_t b, int q) {
  return (((b >> (2 * q)) & 1u) << 15) | (((b >> (2 * q + 1)) & 1u) << 31);
}

// ------------------------------------------------------------------ block-local rows
// Blocks of 2^LB (6 <= LB <= 8): a block never leaves one warp's chunk of
// four blocks, so the change of layout between the two butterfly passes goes
// through a small per-warp shared-memory buffer with __syncwarp only.  A row
// group of W warps holds one row in registers (chunk c of the row is item
// c / W of warp c % W); its one row-wide step is the absmax (or min/max)
// reduction.  Rows stream into a shared-memory ring by bulk copies from a
// producer warp; with QUIK outliers the kept columns are gathered from the
// ring copy through the kept-column table.
//   layout A: lane l holds chunk elements [256 j + 8 l, +8) for each 256-element
//             piece j (in-block bits 0-2 inside the thread);
//   layout B: lane l = 8 b + t holds elements t + 8 m of block b of the chunk
//             (in-block bits 3..LB-1 inside the thread).
template <int LB>
struct BlkGeom {
  static constexpr int kBlock = 1 << LB;
  static constexpr int kVB = 1 << (LB - 3);      // layout-B values per thread per chunk
  static constexpr int kChunk = 4 << LB;         // elements per warp chunk
  static constexpr int kPieces = 1 << (LB - 6);  // layout-A pieces of 8 per thread
  static constexpr int kStride = kBlock + 8;     // floats per block in a warp buffer
  static constexpr int kBufFloats = 4 * kStride;
};

// Warp-buffer position of in-block index q of chunk block b:
// b * kStride + (q ^ (bit 5 of q) << 2).  The 8 floats of padding per block
// put the four blocks of a layout-B read in different banks; swapping the
// 4-float halves of every other 8-float group makes the layout-A 16-byte
// stores conflict-free.  The kernel resolves it into per-lane base offsets.

// Threads per CTA the kernel is compiled for, from its register budget: the
// values one thread holds plus an overhead that grows with them (set where
// the compiler stops spilling).
template <int LB, int CPW>
struct BlkBounds {
  static constexpr int kVals = CPW * BlkGeom<LB>::kVB;
  static constexpr int kRegs = 56 + kVals + (kVals >= 64 ? 24 : 0) + (LB == 6 ? 16 : 0);
  static constexpr int value = ((65536 / kRegs) / 32) * 32 > 1024 ? 1024 : ((65536 / kRegs) / 32) * 32;
};

// Eight rotated-domain elements [e, e+8) of a ring row: straight 16-byte
// loads without outliers, else gathered through the kept-column table; zero
// at and beyond Kr.
__device__ __forceinline__ void blk_load8(const WhtParams& p, const __half* rrow,
                                          const uint16_t* kept, int e, float (&x)[8]) {
  if (e + 8 <= p.Kr) {
    if (p.n_out == 0) {
      const uint4 u = *reinterpret_cast<const uint4*>(rrow + e);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(h[q]);
        x[2 * q] = f.x;
        x[2 * q + 1] = f.y;
      }
    } else {
      const uint4 k = *reinterpret_cast<const uint4*>(kept + e);
      const uint32_t kk[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {     // (a malformed outlier list leaves 0xFFFF: read as 0)
        const uint32_t c0 = kk[q] & 0xFFFFu, c1 = kk[q] >> 16;
        x[2 * q] = c0 < static_cast<uint32_t>(p.K) ? __half2float(rrow[c0]) : 0.0f;
        x[2 * q + 1] = c1 < static_cast<uint32_t>(p.K) ? __half2float(rrow[c1]) : 0.0f;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ei = e + i;
      const int c = ei < p.Kr ? (p.n_out ? static_cast<int>(kept[ei]) : ei) : p.K;
      x[i] = c < p.K ? __half2float(rrow[c]) : 0.0f;
    }
  }
}

// MODE: 0 = symmetric 4-bit, 1 = asymmetric 4-bit, 2 = symmetric 8-bit,
// 3 = e2m1 (FP4).
template <int LB, int CPW, int MODE, bool CLIP>
__global__ void __launch_bounds__(BlkBounds<LB, CPW>::value, 1) wht_blk_kernel(const WhtParams p) {
  using G = BlkGeom<LB>;
  constexpr int VB = G::kVB;
  static_assert(LB >= 6 && LB <= 8, "block-local kernel: blocks of 64..256");
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ __align__(128) uint8_t smem[];
  const int W = p.nt >> 5;                       // warps per row group
  const int groups = p.rows_per_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = warp / W, wr = warp - rg * W;
  uint64_t* ring_full = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint64_t* ring_empty = ring_full + p.ring_slots;
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(ring_empty + p.ring_slots);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * p.rows_per_block;
  const int64_t row1 = row0 + p.rows_per_block < p.rows ? row0 + p.rows_per_block : p.rows;
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ring_slots; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], W);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  uint8_t* sbits = smem + p.off_signs;
  if (p.signs != nullptr) build_sign_bits(p.signs, p.Kp, sbits);
  uint16_t* kept = reinterpret_cast<uint16_t*>(smem + p.off_kept);
  const int32_t* sidx = reinterpret_cast<const int32_t*>(smem + p.off_idx);
  if (p.n_out > 0)   // (synchronizes the CTA)
    build_kept_table(p.outlier_idx, p.n_out, p.K, p.Kr, kept, reinterpret_cast<int32_t*>(smem + p.off_idx));
  __syncthreads();

  if (warp == groups * W) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const int n = static_cast<int>(row1 - row0);
      int i = 0;
      bool ok = true;
      for (; i < n; ++i) {
        const int s = i % p.ring_slots;
        const uint32_t ph = (i / p.ring_slots) & 1;
        if (!(ok = mbar_wait_bounded(&ring_empty[s], ph ^ 1, abort_flag, p.status,
                                     kDevTimeoutProducer)))
          break;
        mbar_arrive_expect_tx(&ring_full[s], p.ring_row_bytes);
        bulk_load(smem + p.off_ring + static_cast<size_t>(s) * p.ring_row_bytes,
                  p.src + (row0 + i) * p.ld, p.ring_row_bytes, &ring_full[s]);
      }
      // every copy issued lands before the CTA may exit
      for (int j = (i > p.ring_slots ? i - p.ring_slots : 0); j < i; ++j)
        mbar_wait_bounded(&ring_full[j % p.ring_slots], (j / p.ring_slots) & 1, abort_flag,
                          nullptr, 0, kDrainLimitNs);
    }
    return;
  }

  float* buf = reinterpret_cast<float*>(smem + p.off_buf) + warp * G::kBufFloats;
  float* red = reinterpret_cast<float*>(smem + p.off_red) + rg * 64;   // [2 rows][16 warps][2]
  const int nchunks = (p.Kp + G::kChunk - 1) / G::kChunk;
  const int nb = p.Kp >> LB;
  const int b = lane >> 3, tl = lane & 7;
  // Layout-A stores: piece j of this lane lands at a_pos + j * (256 >> LB) *
  // kStride (its second half at a_pos2 + ...), the half swap resolved per lane.
  const int qa = (8 * lane) & (G::kBlock - 1);
  const int xa = ((qa >> 5) & 1) << 2;
  const int a_pos = (lane >> (LB - 3)) * G::kStride + qa + xa;
  const int a_pos2 = (lane >> (LB - 3)) * G::kStride + qa + 4 - xa;
  // Layout-B loads: value m sits at b_pos[(m >> 2) & 1] + 8 m.
  const int b_pos0 = b * G::kStride + tl, b_pos1 = b * G::kStride + (tl ^ 4);
  const bool plain = p.n_out == 0 && p.signs == nullptr;   // no gather, no sign flips
  // GSR: the lanes whose sequency words take Hadamard outputs j ^ 1 (the
  // parity of t, see gsr_j_static) get them in place: y[j ^ 1] is the
  // transform of x with odd-j inputs negated, which the first layout-B
  // butterfly absorbs as (x0 + s x1, x0 - s x1) with s = -1.
  const int swap_par = p.gsr ? ((tl ^ (tl >> 1) ^ (tl >> 2)) & 1) : 0;
  const float bsign = swap_par ? -1.0f : 1.0f;
  int par = 0;
  // this group's rows are rg, rg + groups, ...: slot and parity advance by
  // `groups` slots per row (groups <= ring_slots, so one wrap at most)
  int slot = rg;
  uint32_t rph = 0;
  for (int64_t row = row0 + rg; row < row1; row += groups, par ^= 1) {
    if (!mbar_wait_bounded(&ring_full[slot], rph, abort_flag, p.status, kDevTimeoutWiden))
      break;
    const __half* rrow =
        reinterpret_cast<const __half*>(smem + p.off_ring + static_cast<size_t>(slot) * p.ring_row_bytes);
    if (p.n_out > 0 && p.out16 != nullptr)
      for (int j = wr * 32 + lane; j < p.n_out; j += W * 32) {
        const int c = sidx[j];
        p.out16[row * p.n_out + j] = (c >= 0 && c < p.K) ? rrow[c] : __float2half(0.0f);
      }

    // ---- both butterfly passes, one chunk at a time
    float v[CPW][VB];
    float am = 0.0f, mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < CPW; ++c) {
      const int ch = wr + c * W;
      if (ch < nchunks) {                         // warp-uniform
        const int e0 = ch * G::kChunk;
        constexpr int kPieceStride = (256 >> LB) * G::kStride;
        if (plain && e0 + G::kChunk <= p.Kr) {
          // whole chunk of a plain row: no per-piece checks
#pragma unroll
          for (int j = 0; j < G::kPieces; ++j) {
            const uint4 u = *reinterpret_cast<const uint4*>(rrow + e0 + 256 * j + 8 * lane);
            float x[8];
            bfly_h2(u.x, x[0], x[1]); bfly_h2(u.y, x[2], x[3]);
            bfly_h2(u.z, x[4], x[5]); bfly_h2(u.w, x[6], x[7]);
            wht_stages<1, 3>(x);
            *reinterpret_cast<float4*>(buf + a_pos + j * kPieceStride) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4*>(buf + a_pos2 + j * kPieceStride) = make_float4(x[4], x[5], x[6], x[7]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < G::kPieces; ++j) {
            const int e = e0 + 256 * j + 8 * lane;
            float x[8];
            if (p.n_out == 0 && e + 8 <= p.Kr) {
              uint4 u = *reinterpret_cast<const uint4*>(rrow + e);
              if (p.signs != nullptr) {
                const uint32_t sb = sbits[e >> 3];
                u.x ^= sign_mask_h2(sb, 0); u.y ^= sign_mask_h2(sb, 1);
                u.z ^= sign_mask_h2(sb, 2); u.w ^= sign_mask_h2(sb, 3);
              }
              bfly_h2(u.x, x[0], x[1]); bfly_h2(u.y, x[2], x[3]);
              bfly_h2(u.z, x[4], x[5]); bfly_h2(u.w, x[6], x[7]);
              wht_stages<1, 3>(x);
            } else {
              blk_load8(p, rrow, kept, e, x);
              if (p.signs != nullptr && e < p.Kp) apply_signs8(sbits, e, x);
              wht_stages<0, 3>(x);
            }
            *reinterpret_cast<float4*>(buf + a_pos + j * kPieceStride) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4*>(buf + a_pos2 + j * kPieceStride) = make_float4(x[4], x[5], x[6], x[7]);
          }
        }
        __syncwarp();
#pragma unroll
        for (int m = 0; m < VB; ++m) v[c][m] = buf[(((m >> 2) & 1) ? b_pos1 : b_pos0) + 8 * m];
        __syncwarp();                             // before the next chunk's stores
#pragma unroll
        for (int m = 0; m < VB; m += 2) {
          const float x0 = v[c][m], x1 = v[c][m + 1];
          v[c][m] = fmaf(x1, bsign, x0);
          v[c][m + 1] = fmaf(x1, -bsign, x0);
        }
        wht_stages<1, LB - 3>(v[c]);
        if constexpr (MODE == 1) {
          if (ch * 4 + b < nb)
#pragma unroll
            for (int m = 0; m < VB; m += 2) {
              mn = fmin3(mn, v[c][m], v[c][m + 1]);
              mx = fmax3(mx, v[c][m], v[c][m + 1]);
            }
        } else {
#pragma unroll
          for (int m = 0; m < VB; m += 2) am = fmax3(am, fabsf(v[c][m]), fabsf(v[c][m + 1]));
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring_empty[slot]);   // this warp is done with the ring row

    // ---- the row's scale: warp reduction, then across the group's warps
    float* rp = red + par * 32;
    RowQ q;
    if constexpr (MODE == 1) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      }
      if (lane == 0) { rp[2 * wr] = mx; rp[2 * wr + 1] = mn; }
      row_barrier(rg, p.nt);
      mx = lane < W ? rp[2 * lane] : -INFINITY;
      mn = lane < W ? rp[2 * lane + 1] : INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      }
      const bool first = wr == 0 && lane == 0;
      q = asym_row_q(mn, mx, p.clip_ratio, p.inv_sqrt_block, first ? p.scales + row : nullptr,
                     p.zeros + row);
    } else {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      if (lane == 0) rp[wr] = am;
      row_barrier(rg, p.nt);
      am = lane < W ? rp[lane] : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      float* so = (wr == 0 && lane == 0) ? p.scales + row : nullptr;
      q = MODE == 2   ? sym_row_q8(am, p.clip_ratio, p.inv_sqrt_block, so)
          : MODE == 3 ? sym_row_qf4(am, p.clip_ratio, p.inv_sqrt_block, so)
                      : sym_row_q(am, p.clip_ratio, p.inv_sqrt_block, so);
    }
    const float r = q.r;

    // ---- codes
    uint8_t* crow = p.codes + row * (MODE == 2 ? p.Kp : (p.Kp >> 1));
#pragma unroll
    for (int c = 0; c < CPW; ++c) {
      const int ch = wr + c * W;
      if (ch >= nchunks) continue;                // warp-uniform
      const int bg = ch * 4 + b;                  // block of the row
      const bool ok = bg < nb;
      if (p.rot_debug != nullptr && ok) {
#pragma unroll
        for (int m = 0; m < VB; ++m) {
          int n = tl + 8 * (m ^ swap_par);
          if (p.gsr) n = gray_inverse(static_cast<int>(__brev(static_cast<unsigned>(n)) >> (32 - LB)));
          p.rot_debug[row * p.Kp + (bg << LB) + n] = v[c][m] * p.inv_sqrt_block;
        }
      }
      if (p.gsr) {
        // sequency order: one thread owns each 8-position output word
        const int a0 = tl & 1, a1 = (tl >> 1) & 1, a2 = (tl >> 2) & 1;
        const int p1 = a0, p2 = a1 ^ a0, p3 = a2 ^ p2;
#pragma unroll
        for (int f = 0; f < (1 << (LB - 6)); ++f) {
          const int kw = f | (p3 << (LB - 6)) | (p2 << (LB - 5)) | (p1 << (LB - 4));
          float w8[8];
#pragma unroll
          for (int tt = 0; tt < 8; ++tt) {
            const int js = gsr_j_static<LB>(tt, f);
            w8[tt] = v[c][js];                   // (odd-parity lanes hold j ^ 1 here)
          }
          if (ok) {
            if constexpr (MODE == 2)
              *reinterpret_cast<uint2*>(crow + (bg << LB) + 8 * kw) = quant_bytes8<CLIP>(w8, r, q.c, q.lo, q.hi);
            else if constexpr (MODE == 3)
              *reinterpret_cast<uint32_t*>(crow + (((bg << LB) + 8 * kw) >> 1)) = quant_word_fp4(w8, r);
            else
              *reinterpret_cast<uint32_t*>(crow + (((bg << LB) + 8 * kw) >> 1)) =
                  quant_word<CLIP>(w8, r, q.c, q.lo, q.hi);
          }
        }
      } else if constexpr (MODE == 2) {
        if (ok)
#pragma unroll
          for (int m = 0; m < VB; ++m)
            crow[(bg << LB) + tl + 8 * m] = static_cast<uint8_t>(quant_byte<CLIP>(v[c][m], r, q.c, q.lo, q.hi));
      } else {
        // natural order: 8x8 nibble transposes across the 8 lanes of a block
        const uint32_t sel4 = (tl & 4) ? 0x3276u : 0x5410u;
        const uint32_t sel2 = (tl & 2) ? 0x3715u : 0x6240u;
        const uint32_t rot1 = (tl & 1) ? 28u : 4u;
        const uint32_t msk1 = (tl & 1) ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
        uint32_t wd[VB / 8];
#pragma unroll
        for (int wb = 0; wb < VB / 8; ++wb) {
          float q8[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) q8[jj] = v[c][8 * wb + jj];
          wd[wb] = MODE == 3 ? quant_word_fp4(q8, r) : quant_word<CLIP>(q8, r, q.c, q.lo, q.hi);
        }
#pragma unroll
        for (int wb = 0; wb < VB / 8; ++wb) wd[wb] = prmt(wd[wb], __shfl_xor_sync(0xffffffffu, wd[wb], 4), sel4);
#pragma unroll
        for (int wb = 0; wb < VB / 8; ++wb) wd[wb] = prmt(wd[wb], __shfl_xor_sync(0xffffffffu, wd[wb], 2), sel2);
#pragma unroll
        for (int wb = 0; wb < VB / 8; ++wb) {
          const uint32_t P = __shfl_xor_sync(0xffffffffu, wd[wb], 1);
          const uint32_t s4 = __funnelshift_l(P, P, rot1);
          uint32_t nw;
          asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(nw) : "r"(wd[wb]), "r"(s4), "r"(msk1));
          if (ok) *reinterpret_cast<uint32_t*>(crow + (((bg << LB) + 8 * (8 * wb + tl)) >> 1)) = nw;
        }
      }
    }
    slot += groups;
    if (slot >= p.ring_slots) { slot -= p.ring_slots; rph ^= 1; }
  }
}

// ------------------------------------------------------------------ 4096-point rows
// Blocks of 4096, a row group of two warps per block, 64 values per thread:
//   layout A: thread t of a block holds elements 8 t + 512 h + i (h, i < 8),
//             in-block bits 0-2 and 9-11 inside the thread;
//   layout B: thread t holds elements (t & 7) + 8 j + 512 (t >> 3) (j < 64),
//             bits 3-8 inside the thread.
// One pass through the group's fp32 row buffer moves the row from A to B.
// With QUIK outliers the kept columns are gathered from the ring copy of the
// row through the kept-column table.  Compiled for 608 threads (96 registers each): nine row groups per SM,
// which hides more latency than eight at 128 registers.
// In the buffer, element e of a block sits at (e + 8 (e >> 9)) with bit 2
// flipped where bit 5 of e is set: the padding spreads a layout-B read over
// all banks, the flip makes the layout-A 16-byte stores conflict-free.
// Rows stream into a shared-memory ring by bulk copies (one producer warp).
constexpr int kH12Floats = 4096 + 64;

// MODE: 0 = symmetric, 1 = asymmetric (4-bit codes), 2 = e2m1 (FP4);
// natural order.
template <int MODE, bool CLIP>
__global__ void __launch_bounds__(608, 1) wht_h12_kernel(const WhtParams p) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ __align__(128) uint8_t smem[];
  const int nt = p.nt;                          // 64 x blocks per row
  const int groups = p.rows_per_cta;
  const int rg = threadIdx.x / nt, t = threadIdx.x - rg * nt;
  const int lane = threadIdx.x & 31;
  uint64_t* ring_full = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint64_t* ring_empty = ring_full + p.ring_slots;
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(ring_empty + p.ring_slots);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * p.rows_per_block;
  const int64_t row1 = row0 + p.rows_per_block < p.rows ? row0 + p.rows_per_block : p.rows;
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ring_slots; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], nt / 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  uint8_t* sbits = smem + p.off_signs;
  if (p.signs != nullptr) build_sign_bits(p.signs, p.Kp, sbits);
  uint16_t* kept = reinterpret_cast<uint16_t*>(smem + p.off_kept);
  const int32_t* sidx = reinterpret_cast<const int32_t*>(smem + p.off_idx);
  if (p.n_out > 0)   // (synchronizes the CTA)
    build_kept_table(p.outlier_idx, p.n_out, p.K, p.Kr, kept, reinterpret_cast<int32_t*>(smem + p.off_idx));
  __syncthreads();

  if (rg == groups) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const int n = static_cast<int>(row1 - row0);
      int i = 0;
      bool ok = true;
      for (; i < n; ++i) {
        const int s = i % p.ring_slots;
        const uint32_t ph = (i / p.ring_slots) & 1;
        if (!(ok = mbar_wait_bounded(&ring_empty[s], ph ^ 1, abort_flag, p.status,
                                     kDevTimeoutProducer)))
          break;
        mbar_arrive_expect_tx(&ring_full[s], p.ring_row_bytes);
        bulk_load(smem + p.off_ring + static_cast<size_t>(s) * p.ring_row_bytes,
                  p.src + (row0 + i) * p.ld, p.ring_row_bytes, &ring_full[s]);
      }
      for (int j = (i > p.ring_slots ? i - p.ring_slots : 0); j < i; ++j)
        mbar_wait_bounded(&ring_full[j % p.ring_slots], (j / p.ring_slots) & 1, abort_flag,
                          nullptr, 0, kDrainLimitNs);
    }
    return;
  }

  const int blk = t >> 6, tb = t & 63;
  float* buf = reinterpret_cast<float*>(smem + p.off_buf) +
               (static_cast<size_t>(rg) * (nt >> 6) + blk) * kH12Floats;
  float* red = reinterpret_cast<float*>(smem + p.off_red) + rg * 64;   // [2 rows][16 warps][2]
  const int nw = nt >> 5, wr = t >> 5;
  // layout-A stores of group h: a_pos + 520 h (first half), a_pos2 + 520 h
  const int xa = ((tb >> 2) & 1) << 2;
  const int a_pos = 8 * tb + xa, a_pos2 = 8 * tb + 4 - xa;
  // layout-B loads: value j at (bit 2 of j ? b_pos1 : b_pos0) + 8 j
  const int b_pos0 = (tb & 7) + 520 * (tb >> 3), b_pos1 = ((tb & 7) ^ 4) + 520 * (tb >> 3);
  const int eA = blk * 4096 + 8 * tb;           // row element of layout-A group h = 0
  // no outlier gather, no zero tail, no sign flips
  const bool full_plain = p.n_out == 0 && p.K == p.Kp && p.signs == nullptr;
  int par = 0;
  // this group's rows are rg, rg + groups, ...: slot and parity advance by
  // `groups` slots per row (groups <= ring_slots, so one wrap at most)
  int slot = rg;
  uint32_t rph = 0;
  for (int64_t row = row0 + rg; row < row1; row += groups, par ^= 1) {
    if (!mbar_wait_bounded(&ring_full[slot], rph, abort_flag, p.status, kDevTimeoutWiden))
      break;
    const __half* rrow =
        reinterpret_cast<const __half*>(smem + p.off_ring + static_cast<size_t>(slot) * p.ring_row_bytes);
    if (p.n_out > 0 && p.out16 != nullptr)         // QUIK outlier columns, copied through
      for (int j = t; j < p.n_out; j += nt) {
        const int c = sidx[j];
        p.out16[row * p.n_out + j] = (c >= 0 && c < p.K) ? rrow[c] : __float2half(0.0f);
      }

    // ---- phase A: bits 0-2 and 9-11
    float v[64];
    if (full_plain) {
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const uint4 u = *reinterpret_cast<const uint4*>(rrow + eA + 512 * h);
        bfly_h2(u.x, v[8 * h], v[8 * h + 1]); bfly_h2(u.y, v[8 * h + 2], v[8 * h + 3]);
        bfly_h2(u.z, v[8 * h + 4], v[8 * h + 5]); bfly_h2(u.w, v[8 * h + 6], v[8 * h + 7]);
      }
    } else if (p.n_out > 0) {
      // kept columns gathered from the ring copy of the row (zero beyond K_r)
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const int e = eA + 512 * h;
        float x[8];
        blk_load8(p, rrow, kept, e, x);
        if (p.signs != nullptr) apply_signs8(sbits, e, x);
        wht_stages<0, 1>(x);
#pragma unroll
        for (int q = 0; q < 8; ++q) v[8 * h + q] = x[q];
      }
    } else {
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const int e = eA + 512 * h;
      if (e + 8 <= p.K) {
        uint4 u = *reinterpret_cast<const uint4*>(rrow + e);
        if (p.signs != nullptr) {
          const uint32_t sb = sbits[e >> 3];
          u.x ^= sign_mask_h2(sb, 0); u.y ^= sign_mask_h2(sb, 1);
          u.z ^= sign_mask_h2(sb, 2); u.w ^= sign_mask_h2(sb, 3);
        }
        bfly_h2(u.x, v[8 * h], v[8 * h + 1]); bfly_h2(u.y, v[8 * h + 2], v[8 * h + 3]);
        bfly_h2(u.z, v[8 * h + 4], v[8 * h + 5]); bfly_h2(u.w, v[8 * h + 6], v[8 * h + 7]);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[8 * h + q] = 0.0f;
      }
    }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring_empty[slot]);   // this warp is done with the ring row
    wht_stages<1, 6>(v);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      *reinterpret_cast<float4*>(buf + a_pos + 520 * h) = make_float4(v[8 * h], v[8 * h + 1], v[8 * h + 2], v[8 * h + 3]);
      *reinterpret_cast<float4*>(buf + a_pos2 + 520 * h) = make_float4(v[8 * h + 4], v[8 * h + 5], v[8 * h + 6], v[8 * h + 7]);
    }
    row_barrier(rg, nt);

    // ---- phase B: bits 3-8, then the row's scale
#pragma unroll
    for (int j = 0; j < 64; ++j) v[j] = buf[(((j >> 2) & 1) ? b_pos1 : b_pos0) + 8 * j];
    wht_stages<0, 6>(v);
    float* rp = red + par * 32;
    RowQ q;
    if constexpr (MODE == 1) {
      float mn = fmin3(v[0], v[1], v[2]), mx = fmax3(v[0], v[1], v[2]);
#pragma unroll
      for (int j = 3; j < 63; j += 2) {
        mn = fmin3(mn, v[j], v[j + 1]);
        mx = fmax3(mx, v[j], v[j + 1]);
      }
      mn = fminf(mn, v[63]);
      mx = fmaxf(mx, v[63]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      }
      if (lane == 0) { rp[2 * wr] = mx; rp[2 * wr + 1] = mn; }
      row_barrier(rg, nt);
      mx = lane < nw ? rp[2 * lane] : -INFINITY;
      mn = lane < nw ? rp[2 * lane + 1] : INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      }
      q = asym_row_q(mn, mx, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr,
                     p.zeros + row);
    } else {
      float am = 0.0f;
#pragma unroll
      for (int j = 0; j < 64; j += 2) am = fmax3(am, fabsf(v[j]), fabsf(v[j + 1]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      if (lane == 0) rp[wr] = am;
      row_barrier(rg, nt);
      am = lane < nw ? rp[lane] : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      q = MODE == 2 ? sym_row_qf4(am, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr)
                    : sym_row_q(am, p.clip_ratio, p.inv_sqrt_block, t == 0 ? p.scales + row : nullptr);
    }
    const float r = q.r;
    uint8_t* crow = p.codes + row * (p.Kp >> 1);
    const int eB = blk * 4096 + 512 * (tb >> 3);  // row element of this thread's layout-B group
    if (p.rot_debug != nullptr)
#pragma unroll
      for (int j = 0; j < 64; ++j) p.rot_debug[row * p.Kp + eB + (tb & 7) + 8 * j] = v[j] * p.inv_sqrt_block;

    // ---- codes in natural order: 8x8 nibble transposes across the 8 lanes
    // holding one 512-element group
    const int l = tb & 7;
    const uint32_t sel4 = (l & 4) ? 0x3276u : 0x5410u;
    const uint32_t sel2 = (l & 2) ? 0x3715u : 0x6240u;
    const uint32_t rot1 = (l & 1) ? 28u : 4u;
    const uint32_t msk1 = (l & 1) ? 0xF0F0F0F0u : 0x0F0F0F0Fu;
    uint32_t wd[8];
#pragma unroll
    for (int wb = 0; wb < 8; ++wb) {
      float q8[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) q8[jj] = v[8 * wb + jj];
      wd[wb] = MODE == 2 ? quant_word_fp4(q8, r) : quant_word<CLIP>(q8, r, q.c, q.lo, q.hi);
    }
#pragma unroll
    for (int wb = 0; wb < 8; ++wb) wd[wb] = prmt(wd[wb], __shfl_xor_sync(0xffffffffu, wd[wb], 4), sel4);
#pragma unroll
    for (int wb = 0; wb < 8; ++wb) wd[wb] = prmt(wd[wb], __shfl_xor_sync(0xffffffffu, wd[wb], 2), sel2);
#pragma unroll
    for (int wb = 0; wb < 8; ++wb) {
      const uint32_t P = __shfl_xor_sync(0xffffffffu, wd[wb], 1);
      const uint32_t s4 = __funnelshift_l(P, P, rot1);
      uint32_t nw2;
      asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(nw2) : "r"(wd[wb]), "r"(s4), "r"(msk1));
      *reinterpret_cast<uint32_t*>(crow + ((eB + 64 * wb + 8 * l) >> 1)) = nw2;
    }
    row_barrier(rg, nt);                          // the row buffer is reused by the next row
    slot += groups;
    if (slot >= p.ring_slots) { slot -= p.ring_slots; rph ^= 1; }
  }
}

// ------------------------------------------------------------------ few rows

// Few rows (decode): a cluster of CL CTAs per row, each holding a span of
// whole rotation blocks in shared memory.  The kernels above give each row
// one group of threads and keep it in registers, which fills the GPU only
// with many rows; with a handful of tokens a row's latency is the whole
// cost, so here up to CL x 1024 threads on CL SMs share one row and every
// global load is issued up front.  Steps: load the row (vector loads) and
// the outlier indices together; drop the outlier columns of QUIK §1 by a
// binary search of the ascending outlier list, each CTA keeping the kept
// columns whose rotated positions fall in its span; run the Walsh-Hadamard
// butterflies in passes of up to three stages through shared memory, the
// last pass also taking the span's absmax; combine the CL maxima through
// distributed shared memory; then quantize + pack as the other kernels do.
struct FewRowsParams {
  const __half* src;
  int64_t rows, ld;
  int32_t K, Kr, Kp, n_out;
  const int32_t* outlier_idx;
  const int8_t* signs;        // random-sign diagonal [Kp] or null
  int32_t lb, gsr, aligned;
  int32_t cl;                 // CTAs per row (a cluster)
  int32_t span;               // rotated elements per CTA (whole blocks, a multiple of 128)
  int32_t off_bits, off_scan;
  float clip_ratio, inv_sqrt_block;
  uint8_t* codes;
  float* scales;
  int32_t* zeros;             // asymmetric activations: zero points [rows] (null: symmetric)
  __half* out16;
  float* rot_debug;
  int32_t bits8;              // 8-bit codes (one int8 per code) instead of nibbles
};

constexpr int kFewMaxChunks = 4;   // 8-column chunks per thread (K <= 32768 at 1024 threads)

// Maximum over the block (any sign); `sh` holds 32 floats.  Contains two
// __syncthreads.
__device__ __forceinline__ float block_max(float v, float* sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) sh[w] = v;
  __syncthreads();
  float m = -INFINITY;
  for (int i = 0; i < nw; ++i) m = fmaxf(m, sh[i]);
  __syncthreads();
  return m;
}

template <bool CLIP, bool ASYM, bool SIGNS>
__global__ void __launch_bounds__(1024, 1) wht_few_rows_kernel(const FewRowsParams p) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ __align__(16) uint8_t smem[];
  float* buf = reinterpret_cast<float*>(smem);                       // [span], few_swz order
  int* sidx = reinterpret_cast<int*>(smem + p.off_bits);             // the outlier columns
  float* red = reinterpret_cast<float*>(smem + p.off_scan + 128);    // 32 floats
  float* maxima = reinterpret_cast<float*>(smem + p.off_scan + 256); // 2 x CL floats
  const int t = threadIdx.x, nthr = blockDim.x;
  const int64_t row = blockIdx.x / p.cl;
  const int cr = blockIdx.x % p.cl;                                  // rank in the cluster
  const int e_lo = cr * p.span;                                      // this CTA's rotated span
  const int e_hi = min(p.Kp, e_lo + p.span);
  const int nloc = max(0, e_hi - e_lo);
  const int nchunks = (p.K + 7) >> 3;                                // 8 source columns each
  const int cpt = (nchunks + nthr - 1) / nthr;                       // chunks per thread
  const int c0 = t * cpt;                                            // this thread's chunks
  const __half* srow = p.src + row * p.ld;
  // the row's vector loads first; their latency overlaps the outlier work
  uint4 raw[kFewMaxChunks];
#pragma unroll
  for (int q = 0; q < kFewMaxChunks; ++q) {
    const int col0 = 8 * (c0 + q);
    raw[q] = make_uint4(0u, 0u, 0u, 0u);
    if (q < cpt && p.aligned && col0 + 8 <= p.K) raw[q] = ld_stream_v4(srow + col0);
  }
  // `before` = outlier columns left of this thread's first column: a binary
  // search of the (strictly ascending) outlier list staged in shared memory
  int before = 0;
  if (p.n_out > 0) {
    for (int j = t; j < p.n_out; j += nthr) {
      const int c = __ldg(p.outlier_idx + j);
      sidx[j] = c;
      if (p.out16 != nullptr && cr == 0)
        p.out16[row * p.n_out + j] = (c >= 0 && c < p.K) ? srow[c] : __float2half(0.0f);
    }
    __syncthreads();
    int lo = 0, hi = p.n_out;
    const int col_first = 8 * c0;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sidx[mid] < col_first) lo = mid + 1;
      else hi = mid;
    }
    before = lo;
  }
  // scatter the kept columns whose rotated positions are in [e_lo, e_hi);
  // zero the padding beyond the real columns
  for (int e = max(p.Kr, e_lo) + t; e < e_hi; e += nthr) buf[few_swz(e - e_lo)] = 0.0f;
#pragma unroll
  for (int q = 0; q < kFewMaxChunks; ++q) {
    const int c = c0 + q;
    if (q >= cpt || c >= nchunks) continue;
    const int col0 = 8 * c;
    float x[8];
    if (p.aligned && col0 + 8 <= p.K) {
      const __half2* h = reinterpret_cast<const __half2*>(&raw[q]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = (col0 + i < p.K) ? __half2float(srow[col0 + i]) : 0.0f;
    }
    // outlier columns of this chunk: the next entries of the list below col0 + 8
    uint32_t m8 = 0u;
    for (int k = before; k < p.n_out && k < before + 8; ++k) {
      const int d = sidx[k] - col0;
      if (d >= 8) break;
      if (d >= 0) m8 |= 1u << d;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = col0 + i - before;
      if ((m8 >> i) & 1u) {
        ++before;
      } else if (col0 + i < p.K && e < p.Kr && e >= e_lo && e < e_hi) {
        float xv = x[i];
        if (SIGNS && __ldg(p.signs + e) < 0) xv = -xv;
        buf[few_swz(e - e_lo)] = xv;
      }
    }
  }
  __syncthreads();
  float am = 0.0f;
  for (int s = 0; s < p.lb; s += 3) {
    const int r = min(3, p.lb - s);
    if (r == 3) am = wht_smem_pass<3>(buf, nloc, s, t, nthr);
    else if (r == 2) am = wht_smem_pass<2>(buf, nloc, s, t, nthr);
    else am = wht_smem_pass<1>(buf, nloc, s, t, nthr);
    __syncthreads();
  }
  if (p.lb == 0)
    for (int e = t; e < nloc; e += nthr) am = fmaxf(am, fabsf(buf[e]));
  // symmetric: the span's absmax; asymmetric: its max and -min
  float m0 = am, m1 = 0.0f;
  if (ASYM) {
    m0 = -INFINITY;
    m1 = -INFINITY;
    for (int e = t; e < nloc; e += nthr) {
      m0 = fmaxf(m0, buf[e]);
      m1 = fmaxf(m1, -buf[e]);
    }
    m1 = block_max(m1, red);
  }
  m0 = block_max(m0, red);
  if (p.cl > 1) {
    // every CTA of the row stores its span's maxima into every CTA
    if (t < p.cl) {
      const uint32_t dst = mapa_shared(smem_u32(maxima + cr), t);
      asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst), "f"(m0) : "memory");
      if (ASYM) asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst + 32u), "f"(m1) : "memory");
    }
    cluster_sync();
    for (int i = 0; i < p.cl; ++i) {
      m0 = fmaxf(m0, maxima[i]);
      if (ASYM) m1 = fmaxf(m1, maxima[8 + i]);
    }
  }
  const bool lead = t == 0 && cr == 0;
  const RowQ q = ASYM ? asym_row_q(-m1, m0, p.clip_ratio, p.inv_sqrt_block,
                                   lead ? p.scales + row : nullptr, p.zeros + row)
                 : p.bits8 ? sym_row_q8(m0, p.clip_ratio, p.inv_sqrt_block,
                                        lead ? p.scales + row : nullptr)
                           : sym_row_q(m0, p.clip_ratio, p.inv_sqrt_block,
                                       lead ? p.scales + row : nullptr);
  const float r = q.r;
  uint8_t* crow = p.codes + row * (p.bits8 ? p.Kp : (p.Kp >> 1));
  const int bm = (1 << p.lb) - 1;
  for (int g = t; g < (nloc >> 3); g += nthr) {
    const int el = 8 * g;                          // local index of the group
    float v[8];
    if (p.gsr) {
      // sequency position j of a block takes Hadamard output bitrev(gray(j))
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = (el + i) & bm;
        const int nat = static_cast<int>(__brev(static_cast<unsigned>(j ^ (j >> 1))) >> (32 - p.lb));
        v[i] = buf[few_swz(((el + i) & ~bm) + nat)];
      }
    } else {
      const float4 a = *reinterpret_cast<const float4*>(buf + few_swz(el));
      const float4 b = *reinterpret_cast<const float4*>(buf + few_swz(el) + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    if (!ASYM && p.bits8)
      *reinterpret_cast<uint2*>(crow + e_lo + el) = quant_bytes8<CLIP>(v, r, q.c, q.lo, q.hi);
    else
      *reinterpret_cast<uint32_t*>(crow + ((e_lo + el) >> 1)) = quant_word<CLIP>(v, r, q.c, q.lo, q.hi);
    if (p.rot_debug != nullptr)
#pragma unroll
      for (int i = 0; i < 8; ++i) p.rot_debug[row * p.Kp + e_lo + el + i] = v[i] * p.inv_sqrt_block;
  }
}

// ------------------------------------------------------------------ Kronecker

struct KronParams {
  const __half* src;
  int64_t rows, ld;
  int32_t K, Kr, Kp, n_out;
  const int32_t* outlier_idx;
  const float* p1;            // [n1 x n1]
  const float* p2;            // [n2 x n2]
  const float* chan;          // [Kp] or null
  int32_t chan_multiply;
  int32_t n1, n2;
  float clip_ratio;
  uint8_t* codes;
  float* scales;
  __half* out16;
  float* rot_debug;
  int32_t off_p1, off_p2, off_x, off_t, off_red, off_kept, off_idx;
};

// out[i][j] = sum_k A[i][k] B[k][j] for one 4x4 register tile; A i-major
// (row stride lda), B k-major (row stride ldb).
__device__ __forceinline__ void tile4x4_imajor(const float* __restrict__ A, int lda,
                                               const float* __restrict__ B, int ldb, int kdim,
                                               float (&acc)[4][4]) {
  for (int k = 0; k < kdim; k += 4) {
    float a[4][4], b[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 t = *reinterpret_cast<const float4*>(A + r * lda + k);
      a[r][0] = t.x; a[r][1] = t.y; a[r][2] = t.z; a[r][3] = t.w;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float4 t = *reinterpret_cast<const float4*>(B + (k + kk) * ldb);
      b[kk][0] = t.x; b[kk][1] = t.y; b[kk][2] = t.z; b[kk][3] = t.w;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r][kk], b[kk][c], acc[r][c]);
  }
}

// Same with A k-major: A[k][i] at A + k*lda + i.
__device__ __forceinline__ void tile4x4_kmajor(const float* __restrict__ A, int lda,
                                               const float* __restrict__ B, int ldb, int kdim,
                                               float (&acc)[4][4]) {
  for (int k = 0; k < kdim; ++k) {
    const float4 a = *reinterpret_cast<const float4*>(A + k * lda);
    const float4 b = *reinterpret_cast<const float4*>(B + k * ldb);
    const float av[4] = {a.x, a.y, a.z, a.w};
    const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
  }
}

template <bool CLIP>
__global__ void __launch_bounds__(256) kron_rotate_quant_kernel(const KronParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* P1 = reinterpret_cast<float*>(smem + p.off_p1);
  float* P2 = reinterpret_cast<float*>(smem + p.off_p2);
  float* X = reinterpret_cast<float*>(smem + p.off_x);     // x (row-major n1 x n2), later Y
  float* T = reinterpret_cast<float*>(smem + p.off_t);     // X P2
  float* red = reinterpret_cast<float*>(smem + p.off_red);
  const int n1 = p.n1, n2 = p.n2, n = n1 * n2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool gather = p.n_out > 0;
  uint16_t* kept = reinterpret_cast<uint16_t*>(smem + p.off_kept);
  if (gather) build_kept_table(p.outlier_idx, p.n_out, p.K, p.Kr, kept,
                               reinterpret_cast<int32_t*>(smem + p.off_idx));
  for (int i = tid; i < n1 * n1; i += blockDim.x) P1[i] = p.p1[i];
  for (int i = tid; i < n2 * n2; i += blockDim.x) P2[i] = p.p2[i];
  __syncthreads();

  const int tiles_j = n2 / 4;
  const int ntiles = (n1 / 4) * tiles_j;
  for (int64_t row = blockIdx.x; row < p.rows; row += gridDim.x) {
    const __half* srow = p.src + row * p.ld;
    if (gather && p.out16 != nullptr) {
      for (int j = tid; j < p.n_out; j += blockDim.x) {
        const int c = __ldg(p.outlier_idx + j);
        p.out16[row * p.n_out + j] = (c >= 0 && c < p.K) ? srow[c] : __float2half(0.0f);
      }
    }
    for (int e = tid; e < n; e += blockDim.x) {
      const int c = gather ? static_cast<int>(kept[e]) : e;
      float x = (e < p.Kr && c < p.K) ? __half2float(srow[c]) : 0.0f;
      if (p.chan != nullptr) x = p.chan_multiply ? x * p.chan[e] : x / p.chan[e];
      X[e] = x;
    }
    __syncthreads();
    // T = mat(x) P2   (n1 x n2)
    for (int t = tid; t < ntiles; t += blockDim.x) {
      const int i0 = (t / tiles_j) * 4, j0 = (t % tiles_j) * 4;
      float acc[4][4] = {};
      tile4x4_imajor(X + i0 * n2, n2, P2 + j0, n2, n2, acc);
#pragma unroll
      for (int r = 0; r < 4; ++r)
        *reinterpret_cast<float4*>(T + (i0 + r) * n2 + j0) =
            make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    }
    __syncthreads();
    // Y = P1^T T   (n1 x n2), written over X
    float am = 0.0f;
    for (int t = tid; t < ntiles; t += blockDim.x) {
      const int i0 = (t / tiles_j) * 4, j0 = (t % tiles_j) * 4;
      float acc[4][4] = {};
      tile4x4_kmajor(P1 + i0, n1, T + j0, n2, n1, acc);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
#pragma unroll
        for (int c = 0; c < 4; ++c) am = fmaxf(am, fabsf(acc[r][c]));
        *reinterpret_cast<float4*>(X + (i0 + r) * n2 + j0) =
            make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if (lane == 0) red[warp] = am;
    __syncthreads();
    am = 0.0f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) am = fmaxf(am, red[w]);
    const float s = (p.clip_ratio * am) / 7.0f;
    const float r = (am > 0.0f) ? 7.0f / (p.clip_ratio * am) : 0.0f;
    if (tid == 0) p.scales[row] = s;
    uint8_t* crow = p.codes + row * (p.Kp / 2);
    for (int e0 = tid * 8; e0 < n; e0 += blockDim.x * 8) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) word |= quant_nibble<CLIP>(X[e0 + i], r) << (4 * i);
      *reinterpret_cast<uint32_t*>(crow + e0 / 2) = word;
      if (p.rot_debug != nullptr)
#pragma unroll
        for (int i = 0; i < 8; ++i) p.rot_debug[row * p.Kp + e0 + i] = X[e0 + i];
    }
    __syncthreads();   // X, red reused by the next row
  }
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int ilog2(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

template <typename Kernel>
cudaError_t set_smem(Kernel k, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

template <typename Kernel>
cudaError_t launch_rows_kernel(Kernel k, const WhtParams& p, int threads, size_t smem,
                               cudaStream_t s) {
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, smem);
  if (e != cudaSuccess) return e;
  const int64_t want = (p.rows + p.rows_per_cta - 1) / p.rows_per_cta;
  const int64_t cap = static_cast<int64_t>(std::max(per_sm, 1)) * sm_count();
  const int grid = static_cast<int>(std::min(want, cap));
  e = launch_pdl(k, dim3(grid), dim3(threads), smem, s, 1, p);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

// Ring-mode launch: one CTA per SM (at most one per row), contiguous rows.
template <typename Kernel>
cudaError_t launch_ring_kernel(Kernel k, const WhtParams& p, int threads, size_t smem,
                               int grid, cudaStream_t s) {
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k, dim3(grid), dim3(threads), smem, s, 1, p);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

template <int LB, int CPW>
cudaError_t dispatch_blk(int mode, bool clip, const WhtParams& p, int threads, size_t smem, int grid,
                         cudaStream_t s) {
  if (mode == 1) return launch_ring_kernel(wht_blk_kernel<LB, CPW, 1, true>, p, threads, smem, grid, s);
  if (mode == 3) return launch_ring_kernel(wht_blk_kernel<LB, CPW, 3, false>, p, threads, smem, grid, s);
  if (mode == 2)
    return clip ? launch_ring_kernel(wht_blk_kernel<LB, CPW, 2, true>, p, threads, smem, grid, s)
                : launch_ring_kernel(wht_blk_kernel<LB, CPW, 2, false>, p, threads, smem, grid, s);
  return clip ? launch_ring_kernel(wht_blk_kernel<LB, CPW, 0, true>, p, threads, smem, grid, s)
              : launch_ring_kernel(wht_blk_kernel<LB, CPW, 0, false>, p, threads, smem, grid, s);
}

// Thread budget of the block-local kernel instantiation for (lb, cpw).
int blk_bound(int lb, int cpw) {
  switch (lb * 16 + cpw) {
    case 6 * 16 + 4: return BlkBounds<6, 4>::value;
    case 7 * 16 + 2: return BlkBounds<7, 2>::value;
    case 7 * 16 + 4: return BlkBounds<7, 4>::value;
    case 8 * 16 + 1: return BlkBounds<8, 1>::value;
    case 8 * 16 + 2: return BlkBounds<8, 2>::value;
    default: return 0;
  }
}

// Rows of blocks of 64..256 through wht_blk_kernel.  Returns false (nothing
// launched) when the row shape does not fit it.
bool launch_wht_blk(const RowJob& job, WhtParams p, int lb, cudaStream_t stream, qr_status* st) {
  if (lb < 6 || lb > 8 || job.K <= 0 || job.Kp <= 0 || job.rows <= 0 || job.K % 8 != 0 || job.ld % 8 != 0 ||
      reinterpret_cast<uintptr_t>(job.src) % 16 != 0)
    return false;
  p.status = device_status_word();
  if (p.status == nullptr) return false;
  const int chunk = 4 << lb;
  const int nchunks = (job.Kp + chunk - 1) / chunk;
  const int cpw_small = lb == 6 ? 4 : (lb == 7 ? 2 : 1);
  int cpw = (nchunks + cpw_small - 1) / cpw_small <= 16 ? cpw_small : (lb == 6 ? 0 : 2 * cpw_small);
  if (cpw == 0) return false;
  const int W = (nchunks + cpw - 1) / cpw;
  if (W < 1 || W > 16) return false;
  const int bound = blk_bound(lb, cpw);
  const int64_t blocks = std::min<int64_t>(job.rows, sm_count());
  const int64_t per_block = (job.rows + blocks - 1) / blocks;
  const int row_bytes = static_cast<int>(job.K * 2);
  const size_t buf_floats = 4 * static_cast<size_t>((1 << lb) + 8);
  const size_t sign_bytes = p.signs != nullptr ? static_cast<size_t>(job.Kp / 8) : 0;
  int groups = static_cast<int>(std::min<int64_t>(std::min(8, (bound - 32) / (32 * W)), per_block));
  for (; groups >= 1; --groups) {
    size_t off = sizeof(float) * 64 * groups;                                   // red
    p.off_red = 0;
    p.off_buf = static_cast<int32_t>(align_up(off, 16));
    off = p.off_buf + sizeof(float) * buf_floats * W * groups;
    p.off_kept = static_cast<int32_t>(align_up(off, 16));
    if (job.n_out > 0) off = p.off_kept + sizeof(uint16_t) * align_up(job.Kr, 8);
    p.off_idx = static_cast<int32_t>(align_up(off, 16));
    if (job.n_out > 0) off = p.off_idx + sizeof(int32_t) * job.n_out;
    p.off_signs = static_cast<int32_t>(align_up(off, 16));
    off = p.off_signs + sign_bytes;
    p.off_ring = static_cast<int32_t>(align_up(off, 128));
    const int64_t fit = (static_cast<int64_t>(max_smem_optin()) - p.off_ring - 16 * per_block - 16 - 16) /
                        row_bytes;
    int slots = static_cast<int>(std::min<int64_t>(per_block, fit));
    // reused slots each belong to one row group (no parity aliasing)
    if (slots < per_block) slots = slots / groups * groups;
    if (slots < 1) continue;
    p.ring_slots = slots;
    p.ring_row_bytes = row_bytes;
    p.off_bars = static_cast<int32_t>(align_up(p.off_ring + static_cast<size_t>(slots) * row_bytes, 16));
    const size_t smem = p.off_bars + 16 * static_cast<size_t>(slots) + 16;
    p.rows_per_block = static_cast<int32_t>(per_block);
    p.rows_per_cta = groups;
    p.nt = 32 * W;
    const int threads = groups * 32 * W + 32;
    const int grid = static_cast<int>((job.rows + per_block - 1) / per_block);
    const int mode = job.zeros != nullptr ? 1 : job.bits == 8 ? 2 : job.bits == kFp4Codes ? 3 : 0;
    const bool clip = p.clip_ratio < 1.0f;
    cudaError_t e;
    switch (lb * 16 + cpw) {
      case 6 * 16 + 4: e = dispatch_blk<6, 4>(mode, clip, p, threads, smem, grid, stream); break;
      case 7 * 16 + 2: e = dispatch_blk<7, 2>(mode, clip, p, threads, smem, grid, stream); break;
      case 7 * 16 + 4: e = dispatch_blk<7, 4>(mode, clip, p, threads, smem, grid, stream); break;
      case 8 * 16 + 1: e = dispatch_blk<8, 1>(mode, clip, p, threads, smem, grid, stream); break;
      case 8 * 16 + 2: e = dispatch_blk<8, 2>(mode, clip, p, threads, smem, grid, stream); break;
      default: return false;
    }
    *st = e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
    return true;
  }
  return false;
}

// Rows of 4096-point blocks through wht_h12_kernel (4-bit integer or e2m1
// codes, aligned rows, any row count).  Returns false (nothing launched)
// when the shape does not fit it.
bool launch_wht_h12(const RowJob& job, WhtParams p, int lb, cudaStream_t stream, qr_status* st) {
  if (lb != 12 || (job.bits != 4 && job.bits != kFp4Codes) || job.K <= 0 || job.rows <= 0 || job.K % 8 != 0 ||
      job.ld % 8 != 0 || reinterpret_cast<uintptr_t>(job.src) % 16 != 0 || job.Kp % 4096 != 0)
    return false;
  p.status = device_status_word();
  if (p.status == nullptr) return false;
  const int nblk = job.Kp / 4096;
  const int nt = 64 * nblk;
  if (nt + 32 > 608) return false;
  const int64_t blocks = std::min<int64_t>(job.rows, sm_count());
  const int64_t per_block = (job.rows + blocks - 1) / blocks;
  const int row_bytes = static_cast<int>(job.K * 2);
  const size_t sign_bytes = p.signs != nullptr ? static_cast<size_t>(job.Kp / 8) : 0;
  int groups = static_cast<int>(std::min<int64_t>(std::min(9, (608 - 32) / nt), per_block));
  for (; groups >= 1; --groups) {
    p.off_red = 0;
    size_t off = sizeof(float) * 64 * groups;
    p.off_buf = static_cast<int32_t>(align_up(off, 16));
    off = p.off_buf + sizeof(float) * static_cast<size_t>(kH12Floats) * nblk * groups;
    p.off_kept = static_cast<int32_t>(align_up(off, 16));
    if (job.n_out > 0) off = p.off_kept + sizeof(uint16_t) * align_up(job.Kr, 8);
    p.off_idx = static_cast<int32_t>(align_up(off, 16));
    if (job.n_out > 0) off = p.off_idx + sizeof(int32_t) * job.n_out;
    p.off_signs = static_cast<int32_t>(align_up(off, 16));
    off = p.off_signs + sign_bytes;
    p.off_ring = static_cast<int32_t>(align_up(off, 128));
    const int64_t fit = (static_cast<int64_t>(max_smem_optin()) - p.off_ring - 16 * per_block - 16 - 16) /
                        row_bytes;
    int slots = static_cast<int>(std::min<int64_t>(per_block, fit));
    if (slots < per_block) slots = slots / groups * groups;   // reused slots: one group each
    if (slots < 1) continue;
    p.ring_slots = slots;
    p.ring_row_bytes = row_bytes;
    p.off_bars = static_cast<int32_t>(align_up(p.off_ring + static_cast<size_t>(slots) * row_bytes, 16));
    const size_t smem = p.off_bars + 16 * static_cast<size_t>(slots) + 16;
    p.rows_per_block = static_cast<int32_t>(per_block);
    p.rows_per_cta = groups;
    p.nt = nt;
    const int threads = groups * nt + 32;
    const int grid = static_cast<int>((job.rows + per_block - 1) / per_block);
    const bool clip = p.clip_ratio < 1.0f;
    cudaError_t e;
    if (job.bits == kFp4Codes)
      e = launch_ring_kernel(wht_h12_kernel<2, false>, p, threads, smem, grid, stream);
    else if (job.zeros != nullptr)
      e = launch_ring_kernel(wht_h12_kernel<1, true>, p, threads, smem, grid, stream);
    else if (clip)
      e = launch_ring_kernel(wht_h12_kernel<0, true>, p, threads, smem, grid, stream);
    else
      e = launch_ring_kernel(wht_h12_kernel<0, false>, p, threads, smem, grid, stream);
    *st = e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
    return true;
  }
  return false;
}

template <int MB, int HA, int OUT, bool CLIP, bool RING>
cudaError_t dispatch_items(int items, const WhtParams& p, int threads, size_t smem, int grid,
                           cudaStream_t s) {
  constexpr int EB = 1 << MB;
  constexpr int IMAX = (64 / EB) >= 8 ? 8 : ((64 / EB) < 1 ? 1 : 64 / EB);
#define QR_LAUNCH(I)                                                                      \
  return RING ? launch_ring_kernel(wht_ab_kernel<MB, HA, I, CLIP, OUT, RING>, p, threads, \
                                   smem, grid, s)                                         \
              : launch_rows_kernel(wht_ab_kernel<MB, HA, I, CLIP, OUT, RING>, p, threads, smem, s)
  switch (items) {
    case 1: QR_LAUNCH(1);
    case 2:
      if constexpr (IMAX >= 2) { QR_LAUNCH(2); }
      break;
    case 4:
      if constexpr (IMAX >= 4) { QR_LAUNCH(4); }
      break;
    case 8:
      if constexpr (IMAX >= 8) { QR_LAUNCH(8); }
      break;
    default: break;
  }
#undef QR_LAUNCH
  return cudaErrorInvalidValue;
}

template <bool CLIP, bool RING>
cudaError_t dispatch_ab(int lb, int out, int items, const WhtParams& p, int threads, size_t smem,
                        int grid, cudaStream_t s) {
  switch (lb) {
    case 4: return dispatch_items<1, 0, 2, CLIP, RING>(items, p, threads, smem, grid, s);
    case 5: return dispatch_items<2, 0, 2, CLIP, RING>(items, p, threads, smem, grid, s);
    case 6: return out == 1 ? dispatch_items<3, 0, 1, CLIP, RING>(items, p, threads, smem, grid, s)
                            : dispatch_items<3, 0, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 7: return out == 1 ? dispatch_items<4, 0, 1, CLIP, RING>(items, p, threads, smem, grid, s)
                            : dispatch_items<4, 0, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 8: return out == 1 ? dispatch_items<5, 0, 1, CLIP, RING>(items, p, threads, smem, grid, s)
                            : dispatch_items<5, 0, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 9: return dispatch_items<5, 1, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 10: return dispatch_items<5, 2, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 11: return dispatch_items<5, 3, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 12: return dispatch_items<6, 3, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 13: return dispatch_items<6, 4, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    case 14: return dispatch_items<7, 4, 0, CLIP, RING>(items, p, threads, smem, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

template <bool CLIP>
cudaError_t dispatch_small(int items, const WhtParams& p, int threads, size_t smem,
                           cudaStream_t s) {
  switch (items) {
    case 1: return launch_rows_kernel(wht_small_kernel<1, CLIP>, p, threads, smem, s);
    case 2: return launch_rows_kernel(wht_small_kernel<2, CLIP>, p, threads, smem, s);
    case 4: return launch_rows_kernel(wht_small_kernel<4, CLIP>, p, threads, smem, s);
    case 8: return launch_rows_kernel(wht_small_kernel<8, CLIP>, p, threads, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

int pow2_at_least(int v) {
  int r = 1;
  while (r < v) r <<= 1;
  return r;
}

// One CTA per row while the rows do not fill the SMs.
bool few_rows(const RowJob& job) {
  return job.rows <= sm_count() && job.Kp <= 32768 && job.Kp > 0 &&
         (job.K + 7) / 8 <= 1024 * kFewMaxChunks;
}

qr_status launch_wht_few_rows(const RowJob& job, cudaStream_t stream) {
  const qr_rotation& rot = *job.rot;
  FewRowsParams p{};
  p.src = reinterpret_cast<const __half*>(job.src);
  p.rows = job.rows;
  p.ld = job.ld;
  p.K = static_cast<int32_t>(job.K);
  p.Kr = job.Kr;
  p.Kp = job.Kp;
  p.n_out = job.n_out;
  p.outlier_idx = job.outlier_idx;
  p.signs = (rot.kind == QR_ROT_HADAMARD || rot.kind == QR_ROT_GSR) ? rot.signs : nullptr;
  const int block = (rot.kind == QR_ROT_NONE) ? 1 : rot.block;
  p.lb = ilog2(block);
  p.gsr = rot.kind == QR_ROT_GSR;
  p.aligned = (reinterpret_cast<uintptr_t>(job.src) % 16 == 0) && (job.ld % 8 == 0);
  p.clip_ratio = rot.clip_ratio;
  p.inv_sqrt_block = static_cast<float>(1.0 / std::sqrt(static_cast<double>(block)));
  p.codes = job.codes;
  p.scales = job.scales;
  p.zeros = job.zeros;
  p.out16 = reinterpret_cast<__half*>(job.out16);
  p.rot_debug = job.rot_debug;
  p.bits8 = job.bits == 8;
  // CTAs per row: up to 8 (and the SMs left per row), each a span of whole
  // blocks that is a multiple of 128 elements
  const int unit = std::max(1, 128 >> p.lb);                  // blocks per 128 elements
  const int nunits = (job.Kp >> p.lb) / unit;
  const int64_t room = std::max<int64_t>(1, sm_count() / job.rows);
  int cl = 1;
  while (cl * 2 <= 8 && cl * 2 <= nunits && cl * 2 <= room) cl *= 2;
  const int units_per_cta = (nunits + cl - 1) / cl;
  p.cl = cl;
  p.span = units_per_cta * unit << p.lb;
  const int64_t chunks = (job.K + 7) / 8;
  const int64_t want = std::max<int64_t>(p.span / 8, (chunks + kFewMaxChunks - 1) / kFewMaxChunks);
  const int threads = static_cast<int>(std::min<int64_t>(1024, std::max<int64_t>(128, (want + 31) / 32 * 32)));
  if (chunks > static_cast<int64_t>(threads) * kFewMaxChunks) return QR_ERR_UNSUPPORTED;
  size_t off = align_up(sizeof(float) * static_cast<size_t>(p.span), 16);
  p.off_bits = static_cast<int32_t>(off);
  off = align_up(off + sizeof(int32_t) * static_cast<size_t>(std::max(job.n_out, 1)), 16);
  p.off_scan = static_cast<int32_t>(off);
  off += 512;                                  // block maxima, cluster maxima
  if (off > static_cast<size_t>(max_smem_optin())) return QR_ERR_UNSUPPORTED;
  // asymmetric codes always clamp (their bounds are [-8, 7])
  using Kfn = void (*)(FewRowsParams);
  Kfn k;
  if (p.signs != nullptr)
    k = job.zeros != nullptr    ? wht_few_rows_kernel<true, true, true>
        : rot.clip_ratio < 1.0f ? wht_few_rows_kernel<true, false, true>
                                : wht_few_rows_kernel<false, false, true>;
  else
    k = job.zeros != nullptr    ? wht_few_rows_kernel<true, true, false>
        : rot.clip_ratio < 1.0f ? wht_few_rows_kernel<true, false, false>
                                : wht_few_rows_kernel<false, false, false>;
  cudaError_t e = set_smem(k, off);
  if (e != cudaSuccess) return QR_ERR_CUDA;
  e = launch_pdl(k, dim3(static_cast<unsigned>(job.rows * cl)), dim3(static_cast<unsigned>(threads)),
                 off, stream, static_cast<unsigned>(cl), p);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

qr_status launch_wht_rows(const RowJob& job, cudaStream_t stream) {
  const qr_rotation& rot = *job.rot;
  WhtParams p{};
  p.src = reinterpret_cast<const __half*>(job.src);
  p.rows = job.rows;
  p.ld = job.ld;
  p.K = static_cast<int32_t>(job.K);
  p.Kr = job.Kr;
  p.Kp = job.Kp;
  p.n_out = job.n_out;
  p.outlier_idx = job.outlier_idx;
  p.signs = (rot.kind == QR_ROT_HADAMARD || rot.kind == QR_ROT_GSR) ? rot.signs : nullptr;
  const int block = (rot.kind == QR_ROT_NONE) ? 1 : rot.block;
  const int lb = ilog2(block);
  p.lb = lb;
  p.nb = job.Kp >> lb;
  p.gsr = rot.kind == QR_ROT_GSR;
  p.vec_ok = job.n_out == 0 && (reinterpret_cast<uintptr_t>(job.src) % 16 == 0) && (job.ld % 8 == 0);
  p.clip_ratio = rot.clip_ratio;
  p.inv_sqrt_block = static_cast<float>(1.0 / std::sqrt(static_cast<double>(block)));
  p.codes = job.codes;
  p.scales = job.scales;
  p.zeros = job.zeros;
  p.out16 = reinterpret_cast<__half*>(job.out16);
  p.rot_debug = job.rot_debug;
  p.bits8 = job.bits == 8;
  if (job.Kp > 32768) return QR_ERR_UNSUPPORTED;
  {
    qr_status st = QR_OK;
    if (launch_wht_blk(job, p, lb, stream, &st)) return st;
    if (launch_wht_h12(job, p, lb, stream, &st)) return st;
    if (job.bits == kFp4Codes) return QR_ERR_UNSUPPORTED;   // e2m1 codes: those two kernels only
  }

  const bool small = lb <= 3;
  int items_total, imax;
  int out = 0;
  int ea = 8, eb = 1;
  if (small) {
    items_total = std::max(1, job.Kp / 8);
    imax = 8;
  } else {
    const int mb = (lb <= 8) ? lb - 3 : (lb == 9 || lb == 10 || lb == 11) ? 5 : (lb == 14 ? 7 : 6);
    const int ha = lb - 3 - mb;
    items_total = p.nb * (8 << ha);
    ea = 8 << ha;
    eb = 1 << mb;
    imax = std::min(8, std::max(1, 64 / eb));
    out = (lb <= 5) ? 2 : (p.gsr ? 1 : 0);
  }
  int nt = std::max(32, (((items_total + imax - 1) / imax) + 31) / 32 * 32);
  if (nt > 512) return QR_ERR_UNSUPPORTED;
  int items = pow2_at_least((items_total + nt - 1) / nt);
  if (items > imax) return QR_ERR_UNSUPPORTED;
  int R = std::max(1, std::min(8, 256 / nt));
  if (job.rows < R) R = static_cast<int>(std::max<int64_t>(job.rows, 1));
  p.nt = nt;
  p.items = items;
  p.rows_per_cta = R;

  size_t off = 0;
  p.off_red = static_cast<int32_t>(off);
  off = align_up(off + sizeof(float) * 32 * R, 16);
  p.off_buf = static_cast<int32_t>(off);
  // fp32 row buffer with the layout-B padding: 8 floats after every 8*eb
  // elements (swz<3 + MB>), plus 8 spare
  p.buf_bytes = small ? 0 : static_cast<int32_t>(align_up(sizeof(float) * (job.Kp + job.Kp / eb + 8), 16));
  off += static_cast<size_t>(p.buf_bytes) * R;
  p.off_kept = static_cast<int32_t>(off);
  if (job.n_out > 0) off = align_up(off + sizeof(uint16_t) * job.Kr, 16);
  p.off_idx = static_cast<int32_t>(off);
  if (job.n_out > 0) off = align_up(off + sizeof(int32_t) * job.n_out, 16);
  const size_t sign_bytes = p.signs != nullptr ? static_cast<size_t>(job.Kp / 8) : 0;
  p.off_signs = static_cast<int32_t>(off);
  off = align_up(off + sign_bytes, 16);
  if (off > static_cast<size_t>(max_smem_optin())) return QR_ERR_UNSUPPORTED;

  p.status = device_status_word();
  // Ring mode: aligned rows without an outlier gather stream into shared
  // memory by bulk copies, all of a CTA's rows in flight at once when they fit.
  bool ring = !small && job.n_out == 0 && p.vec_ok && (job.K % 8 == 0) && job.K > 0 &&
              p.status != nullptr;
  int grid = 0;
  if (ring) {
    const int64_t blocks = std::min<int64_t>(job.rows, sm_count());
    const int64_t per_block = (job.rows + blocks - 1) / blocks;
    const int row_bytes = static_cast<int>(job.K * 2);
    const int max_groups = std::max(1, std::min(8, (512 - 32) / nt));
    const int bound = (ea <= 64 && eb * items <= 64) ? 512 : 256;   // the kernel's launch bound
    int groups = static_cast<int>(std::min<int64_t>(max_groups, per_block));
    while (groups > 1 && groups * nt + 32 > bound) --groups;
    // layout: red | row-group buffers | ring slots | barriers
    size_t roff = 0, buf_off = 0;
    int slots = 0;
    for (; groups >= 1; --groups) {
      roff = align_up(sizeof(float) * 32 * groups, 16);
      buf_off = roff;
      roff = align_up(roff + static_cast<size_t>(p.buf_bytes) * groups, 128);
      const int64_t fit = (static_cast<int64_t>(max_smem_optin()) - static_cast<int64_t>(roff) -
                           16 * per_block - 16 - 1024 - static_cast<int64_t>(sign_bytes)) / row_bytes;
      slots = static_cast<int>(std::min<int64_t>(per_block, fit));
      // Reused slots must each belong to one row group (a slot count that is a
      // multiple of the groups): a group then never waits on a slot more than
      // one phase past its own last use of it, so parity waits cannot alias.
      if (slots < per_block) slots = slots / groups * groups;
      if (slots >= 1) break;
    }
    if (groups >= 1 && slots >= 1 && groups * nt + 32 <= bound) {
      p.off_red = 0;
      p.off_buf = static_cast<int32_t>(buf_off);
      p.off_kept = p.off_idx = 0;                                // no outlier gather here
      p.ring_slots = slots;
      p.ring_row_bytes = row_bytes;
      p.off_ring = static_cast<int32_t>(roff);
      p.off_bars = static_cast<int32_t>(align_up(roff + static_cast<size_t>(slots) * row_bytes, 16));
      p.rows_per_block = static_cast<int32_t>(per_block);
      p.rows_per_cta = groups;                                   // row groups
      off = p.off_bars + 16 * static_cast<size_t>(slots) + 16;
      p.off_signs = static_cast<int32_t>(align_up(off, 16));
      off = p.off_signs + sign_bytes;
      grid = static_cast<int>((job.rows + per_block - 1) / per_block);
    } else {
      ring = false;
    }
  }
  const int threads = ring ? p.rows_per_cta * nt + 32 : R * nt;
  const bool clip = rot.clip_ratio < 1.0f || job.zeros != nullptr;   // asymmetric codes clamp
  cudaError_t e;
  if (small)
    e = clip ? dispatch_small<true>(items, p, threads, off, stream)
             : dispatch_small<false>(items, p, threads, off, stream);
  else if (ring)
    e = clip ? dispatch_ab<true, true>(lb, out, items, p, threads, off, grid, stream)
             : dispatch_ab<false, true>(lb, out, items, p, threads, off, grid, stream);
  else
    e = clip ? dispatch_ab<true, false>(lb, out, items, p, threads, off, 0, stream)
             : dispatch_ab<false, false>(lb, out, items, p, threads, off, 0, stream);
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

qr_status launch_kron_rows(const RowJob& job, cudaStream_t stream) {
  const qr_rotation& rot = *job.rot;
  KronParams p{};
  p.src = reinterpret_cast<const __half*>(job.src);
  p.rows = job.rows;
  p.ld = job.ld;
  p.K = static_cast<int32_t>(job.K);
  p.Kr = job.Kr;
  p.Kp = job.Kp;
  p.n_out = job.n_out;
  p.outlier_idx = job.outlier_idx;
  p.p1 = rot.p1;
  p.p2 = rot.p2;
  p.chan = rot.chan_scale;
  p.chan_multiply = rot.chan_mode == QR_CHAN_MULTIPLY;
  p.n1 = rot.n1;
  p.n2 = rot.n2;
  p.clip_ratio = rot.clip_ratio;
  p.codes = job.codes;
  p.scales = job.scales;
  p.out16 = reinterpret_cast<__half*>(job.out16);
  p.rot_debug = job.rot_debug;
  const size_t n1 = rot.n1, n2 = rot.n2;
  size_t off = 0;
  p.off_p1 = static_cast<int32_t>(off); off = align_up(off + 4 * n1 * n1, 16);
  p.off_p2 = static_cast<int32_t>(off); off = align_up(off + 4 * n2 * n2, 16);
  p.off_x = static_cast<int32_t>(off);  off = align_up(off + 4 * n1 * n2, 16);
  p.off_t = static_cast<int32_t>(off);  off = align_up(off + 4 * n1 * n2, 16);
  p.off_red = static_cast<int32_t>(off); off = align_up(off + 4 * 32, 16);
  p.off_kept = static_cast<int32_t>(off);
  if (job.n_out > 0) off = align_up(off + sizeof(uint16_t) * job.Kr, 16);
  p.off_idx = static_cast<int32_t>(off);
  if (job.n_out > 0) off = align_up(off + sizeof(int32_t) * job.n_out, 16);
  if (off > static_cast<size_t>(max_smem_optin())) return QR_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(std::min<int64_t>(job.rows, 4 * static_cast<int64_t>(sm_count())));
  cudaError_t e;
  if (rot.clip_ratio < 1.0f) {
    e = set_smem(kron_rotate_quant_kernel<true>, off);
    if (e == cudaSuccess) kron_rotate_quant_kernel<true><<<grid, 256, off, stream>>>(p);
  } else {
    e = set_smem(kron_rotate_quant_kernel<false>, off);
    if (e == cudaSuccess) kron_rotate_quant_kernel<false><<<grid, 256, off, stream>>>(p);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

// KV-cache groups: one warp per group of G = 32 E consecutive values (a
// token's heads are contiguous, so a group holds G / D whole heads).  Lane L
// holds elements [E L, E L + E): R3's butterflies over the bits below
// log2(D) run in registers (element bits) and by xor shuffles (lane bits);
// the group's min and max come from two warp reductions; the asymmetric
// 4-bit codes use the same fma-and-clamp as the row kernels, with 1/sqrt(D)
// folded into the scale; each lane stores its E nibbles (E / 2 bytes, a
// coalesced 32 E / 2-byte row per warp) and lane 0 the scale and zero point.
constexpr int kKvBatch = 4;

template <int E, bool ROT>
__global__ void __launch_bounds__(256) kv_group_quant_kernel(const __half* __restrict__ src,
                                                             int64_t groups, int head_bits,
                                                             float inv_sqrt, uint8_t* codes,
                                                             float* scales, int32_t* zeros) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int G = 32 * E;
  constexpr int LE = E == 4 ? 2 : 3;
  static_assert(E == 4 || E == 8, "groups of 128 or 256");
  using V = typename std::conditional<E == 4, uint2, uint4>::type;
  using C = typename std::conditional<E == 4, uint16_t, uint32_t>::type;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  // kKvBatch groups per warp and iteration: their loads are issued together,
  // so that enough bytes are in flight to cover the memory latency
  for (int64_t g0 = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * kKvBatch;
       g0 < groups; g0 += nwarps * kKvBatch) {
    V raws[kKvBatch];
#pragma unroll
    for (int u = 0; u < kKvBatch; ++u)
      if (g0 + u < groups) raws[u] = *reinterpret_cast<const V*>(src + (g0 + u) * G + lane * E);
#pragma unroll
    for (int u = 0; u < kKvBatch; ++u) {
      const int64_t g = g0 + u;
      if (g >= groups) break;                        // uniform over the warp
      const V raw = raws[u];
      const __half* h = reinterpret_cast<const __half*>(&raw);
      float x[E];
#pragma unroll
      for (int j = 0; j < E; ++j) x[j] = __half2float(h[j]);
      if (ROT) {
        // head_dim >= 32 (qr_kv_quantize rejects smaller heads), so
        // head_bits >= 5 > LE: every element bit is a butterfly stage.
#pragma unroll
        for (int b = 0; b < LE; ++b)
#pragma unroll
            for (int j = 0; j < E; ++j)
              if (!(j & (1 << b))) {
                const float a = x[j], c = x[j | (1 << b)];
                x[j] = a + c;
                x[j | (1 << b)] = a - c;
              }
#pragma unroll
        for (int lb = 0; lb < 5; ++lb)
          if (LE + lb < head_bits) {
            const bool upper = (lane >> lb) & 1;
#pragma unroll
            for (int j = 0; j < E; ++j) {
              const float o = __shfl_xor_sync(0xffffffffu, x[j], 1 << lb);
              x[j] = upper ? o - x[j] : x[j] + o;
            }
          }
      }
      float mx = x[0], mn = x[0];
#pragma unroll
      for (int j = 1; j < E; ++j) {
        mx = fmaxf(mx, x[j]);
        mn = fminf(mn, x[j]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      }
      const RowQ q = asym_row_q(mn, mx, 1.0f, inv_sqrt, lane == 0 ? scales + g : nullptr, zeros + g);
      C packed = 0;
#pragma unroll
      for (int j = 0; j < E; ++j)
        packed |= static_cast<C>(quant_nibble<true>(x[j], q.r, q.c, q.lo, q.hi) << (4 * j));
      *reinterpret_cast<C*>(codes + g * (G / 2) + lane * (E / 2)) = packed;
    }
  }
}

}  // namespace

// Group-wise asymmetric KV-cache codes over rows of `group` (128 or 256)
// contiguous values, R3 (the Hadamard of head_dim, a power of two dividing
// the group) applied first when `rotate`.
qr_status launch_kv_group_quant(const uint16_t* src, int64_t groups, int group, int head_dim,
                                bool rotate, uint8_t* codes, float* scales, int32_t* zeros,
                                cudaStream_t stream) {
  if (groups == 0) return QR_OK;
  int hb = 0;
  while ((1 << hb) < head_dim) ++hb;
  const float inv_sqrt = rotate ? static_cast<float>(1.0 / std::sqrt(static_cast<double>(head_dim)))
                                : 1.0f;
  const int64_t blocks = std::min<int64_t>((groups + 8 * kKvBatch - 1) / (8 * kKvBatch),
                                           static_cast<int64_t>(sm_count()) * 8);
  const auto* x = reinterpret_cast<const __half*>(src);
  cudaError_t e;
  if (group == 128)
    e = rotate ? launch_pdl(kv_group_quant_kernel<4, true>, dim3(static_cast<unsigned>(blocks)),
                            dim3(256), 0, stream, 1, x, groups, hb, inv_sqrt, codes, scales, zeros)
               : launch_pdl(kv_group_quant_kernel<4, false>, dim3(static_cast<unsigned>(blocks)),
                            dim3(256), 0, stream, 1, x, groups, hb, inv_sqrt, codes, scales, zeros);
  else if (group == 256)
    e = rotate ? launch_pdl(kv_group_quant_kernel<8, true>, dim3(static_cast<unsigned>(blocks)),
                            dim3(256), 0, stream, 1, x, groups, hb, inv_sqrt, codes, scales, zeros)
               : launch_pdl(kv_group_quant_kernel<8, false>, dim3(static_cast<unsigned>(blocks)),
                            dim3(256), 0, stream, 1, x, groups, hb, inv_sqrt, codes, scales, zeros);
  else
    return QR_ERR_UNSUPPORTED;
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

qr_status launch_rotate_quant(const RowJob& job, cudaStream_t stream) {
  if (job.rows == 0) return QR_OK;
  if (job.bits == 8 && (job.rot->kind == QR_ROT_KRON || job.zeros != nullptr))
    return QR_ERR_UNSUPPORTED;
  if (job.bits == kFp4Codes)
    return (job.rot->kind == QR_ROT_KRON || job.zeros != nullptr) ? QR_ERR_UNSUPPORTED
                                                                   : launch_wht_rows(job, stream);
  if (job.rot->kind == QR_ROT_KRON)
    return kron_tc_supported(job) ? launch_kron_tc(job, stream) : launch_kron_rows(job, stream);
  // (The row-group kernels at one row per CTA lose to the one-row-per-
  // cluster kernel on decode-sized jobs: 12.9 us against 7.2 us for 64
  // QUIK rows, one SM carrying a row's load latency and both passes.)
  return few_rows(job) ? launch_wht_few_rows(job, stream) : launch_wht_rows(job, stream);
}

}  // namespace qr
