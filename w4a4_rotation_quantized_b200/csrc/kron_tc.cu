// kron_tc.cu -- FlatQuant's Kronecker affine transform on fifth-generation
// tensor cores, fused with per-token 4-bit quantization.
//
// FlatQuant ("LLM量化新篇章：...FlatQuant的平坦之道", §2.3 and 模型架构):
// each row x (n1*n2 channels) is scaled per channel and transformed by two
// small matrices, Y = P1^T mat(x / c) P2, then quantized per token; the page
// fuses the two small matmuls with the quantization into one kernel.
//
// Shapes: n1 = 128, n2 = 64; mat(x) = X [128 x 64], row a = x[64a .. 64a+63].
// Per token, two stages on tcgen05 MMAs (M = 128, fp32 accumulators in TMEM):
//   stage 1  T = X P2        A = X (TMEM, lane a), B = [P2 hi | P2 lo] (smem)
//   stage 2  Y = P1^T T      A = P1^T (TMEM, lane c), B = [T_0 | T_1] (smem)
// fp16 operands carry 11 bits, so every operand v is split into hi = fp16(v)
// and lo = fp16(v - hi).  Stage 1 puts P2's hi and lo side by side along N
// (N = 128): the MMAs with X_hi and X_lo give all four cross terms in two
// column halves that the converter adds.  Stage 2 takes two tokens side by
// side along N (N = 128) and sums P1hi.Thi + P1hi.Tlo + P1lo.Thi (the dropped
// lo.lo term is ~2^-22 of each product).  With A in TMEM an M128 K16 MMA
// takes max(64, N/2) clocks (measured), so a token costs 8 + 12 MMAs of 64
// clocks.
//
// Range: each token is scaled by a power of two sigma that puts max|x/c|
// in [2^7, 2^8), and P1, P2 by powers of two that put their largest entries
// in [1, 2).  Then no fp16 operand overflows (|T| < 2^15) and the lo parts of
// everything that matters at the 1e-5 row-norm level stay normal fp16
// numbers, for any fp16 input.  The scale factors are exact, so the codes
// equal those of the unscaled arithmetic and the scale is divided back out.
//
// Warp roles (one CTA of 17 warps per SM, persistent over pairs of tokens):
//   warp 0      TMEM allocation, and one thread issuing every MMA
//   warps 1-8   loaders: x -> x/c -> per-token max -> sigma -> hi/lo -> TMEM
//               (16 lanes x 4 threads per row, so each warp load touches 8
//               rows of 64 contiguous bytes; the K order inside a row is
//               permuted to the store layout and P2's rows follow it)
//   warps 9-16  converters (stage-1 accumulators -> hi/lo T tiles in smem)
//               and the epilogue (absmax over the token, codes, scale)
// The prologue stages P1, P2 and c in shared memory with bulk copies.  MMA
// issue order, per pair p: S1(2p), S2(p-1) first half, S1(2p+1), S2(p-1)
// second half, so that the converters' work on one token overlaps the tensor
// core's work on another.  Every wait is bounded.
#include <cuda_fp16.h>

#include <algorithm>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

constexpr int kN1 = 128, kN2 = 64;
constexpr int kLoadWarps = 8, kPostWarps = 8;
constexpr int kThreadsTc = 32 * (1 + kLoadWarps + kPostWarps);     // 544
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
constexpr int kXSlots = 8;              // per-token max exchange slots

// TMEM columns (512 allocated)
constexpr uint32_t kColA1 = 0;          // 2 slots x (X hi 32 | X lo 32)
constexpr uint32_t kColD1 = 128;        // stage 1: [x P2hi | x P2lo], 128 fp32
constexpr uint32_t kColP1 = 256;        // P1^T hi 64 | lo 64
constexpr uint32_t kColD2 = 384;        // stage 2: two tokens x 64 fp32

// shared memory (byte offsets from a 1 KB-aligned base)
constexpr int kBp2Bytes = 128 * 128;    // 128 rows (n) x 64 fp16 (K), SW128 K-major
constexpr int kTokT = 128 * 128;        // one token's T, hi or lo: 128 K-rows x 64 fp16
constexpr int kB2Slot = 4 * kTokT;      // T hi (2 tokens) | T lo (2 tokens)
constexpr int off_bp2 = 0;
constexpr int off_b2 = off_bp2 + kBp2Bytes;
constexpr int off_bar = off_b2 + 2 * kB2Slot;
// barriers (8 bytes each)
constexpr int kBarXFull = 0, kBarXEmpty = 2, kBarD1Full = 4, kBarD1Empty = 5,
              kBarB2Full = 6, kBarB2Empty = 8, kBarD2Full = 10, kBarD2Empty = 11,
              kBarXMax = 12, kBarYMax = 12 + kXSlots, kBarDrain = kBarYMax + 4,
              kBarPrologue = kBarDrain + 1, kNumBars = kBarPrologue + 1;
constexpr int off_redx = off_bar + 8 * kNumBars;            // float [kXSlots][8]
constexpr int off_redy = off_redx + 4 * kXSlots * 8;        // float [2][2][4]
constexpr int off_pmax = off_redy + 4 * 16;                 // float [warps][2]
constexpr int off_misc = off_pmax + 8 * (kThreadsTc / 32);    // tmem slot, abort flag
constexpr int kSmemTc = off_misc + 16 + 1024;

struct KronTcParams {
  const __half* src;
  int64_t rows, ld;
  const float* p1;          // [128 x 128] row-major
  const float* p2;          // [64 x 64]
  const float* chan;        // [8192] or null
  int32_t chan_multiply;
  float clip_ratio;
  uint8_t* codes;
  float* scales;
  float* rot_debug;
  int32_t* status;
};

// byte offset of 16-byte chunk j of row r in a 128-byte-swizzled tile whose
// rows are 128 bytes (8-row atoms of 1 KB)
__device__ __forceinline__ int sw128(int r, int j) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Stores two blocks of 8 consecutive 32-bit columns of 16 TMEM lanes (lanes
// taddr.lane .. +15) in the MMA accumulator-fragment order: thread 4g + c
// holds, for block k, registers 4k..4k+3 = (lane g, col 8k+2c), (lane g,
// col 8k+2c+1), (lane g+8, col 8k+2c), (lane g+8, col 8k+2c+1).
__device__ __forceinline__ void tmem_st_16x256b_x2(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.16x256b.x2.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}

// A power of two f with f * m in [2^e, 2^(e+1)) for finite m > 0; 1 otherwise.
__device__ __forceinline__ float pow2_normalizer(float m, int e) {
  const uint32_t bits = __float_as_uint(m);
  const int ex = static_cast<int>((bits >> 23) & 0xFFu);
  if (!(m > 0.0f) || ex == 0xFF) return 1.0f;
  const int f = min(254, max(1, e + 254 - ex));
  return __uint_as_float(static_cast<uint32_t>(f) << 23);
}

// K order of stage 1: the MMA's K index kk (TMEM column kk/2 of a row)
// holds x[a][perm_b(kk)], so that thread c of a row group loads the
// contiguous b ranges [8c, 8c+8) and [32+8c, 32+8c+8) and stores them with
// the 16x256b layout (block k, register pair e, half hf).
__host__ __device__ __forceinline__ int perm_b(int kk) {
  const int k = kk >> 4, c = (kk >> 2) & 3, e = (kk >> 1) & 1, hf = kk & 1;
  return 32 * (k >> 1) + 8 * c + 4 * (k & 1) + 2 * e + hf;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Kind::f16 instruction descriptors: D f32, A/B f16, M = 128, N = 128; A from
// TMEM, B K-major (stage 1) or MN-major (stage 2, bit 16).
constexpr uint32_t kIdescS1 = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescS2 = kIdescS1 | (1u << 16);

// lo = v - fp16(v) for both halves of a packed hi pair, one mixed-precision
// fma each (hi * -1 + v, exact), packed to fp16.
__device__ __forceinline__ uint32_t split_lo(uint32_t hi, float v0, float v1) {
  float l0, l1;
  asm("{\n\t.reg .f16 h0, h1, m1;\n\t"
      "mov.b32 {h0, h1}, %2;\n\t"
      "mov.b16 m1, 0xBC00;\n\t"
      "fma.rn.f32.f16 %0, h0, m1, %3;\n\t"
      "fma.rn.f32.f16 %1, h1, m1, %4;\n\t}"
      : "=f"(l0), "=f"(l1)
      : "r"(hi), "f"(v0), "f"(v1));
  return pack_h2(l0, l1);
}

// hi / lo fp16 pairs of two fp32 values: 2 conversions and 2 fmas.
__device__ __forceinline__ void split_pair(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  hi = pack_h2(v0, v1);
  lo = split_lo(hi, v0, v1);
}

// Byte-permute: byte i of the result is byte sel[i] of {b, a}.
__device__ __forceinline__ uint32_t prmt_b(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight codes round_half_even(y[i] * r) (clamped to +-7 when CLIP), two per
// byte, y[0] in the low nibble: fma with 1.5*2^23 leaves each code's
// two's-complement byte in the low byte; byte permutes gather the even and
// odd codes and one 3-input logic op interleaves their nibbles.
template <bool CLIP>
__device__ __forceinline__ uint32_t code_word(const uint32_t* y, float r) {
  uint32_t b[8];
  const uint64_t r2 = f2_pack(r, r), c2 = f2_pack(kMagic, kMagic);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    float t0, t1;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(y[i]), __uint_as_float(y[i + 1])), r2, c2), t0, t1);
    if (CLIP) {
      t0 = fminf(fmaxf(t0, kMagic - 7.0f), kMagic + 7.0f);
      t1 = fminf(fmaxf(t1, kMagic - 7.0f), kMagic + 7.0f);
    }
    b[i] = __float_as_uint(t0);
    b[i + 1] = __float_as_uint(t1);
  }
  const uint32_t even = prmt_b(prmt_b(b[0], b[2], 0x0040u), prmt_b(b[4], b[6], 0x4000u), 0x7610u);
  const uint32_t odd = prmt_b(prmt_b(b[1], b[3], 0x0040u), prmt_b(b[5], b[7], 0x4000u), 0x7610u);
  uint32_t w;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(w) : "r"(even), "r"(odd << 4), "r"(0x0F0F0F0Fu));
  return w;
}

template <bool CLIP>
__global__ void __launch_bounds__(kThreadsTc, 1) kron_tc_kernel(const KronTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + off_bar);
  volatile float* red_x = reinterpret_cast<volatile float*>(smem + off_redx);
  volatile float* red_y = reinterpret_cast<volatile float*>(smem + off_redy);
  float* pmax = reinterpret_cast<float*>(smem + off_pmax);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_misc);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + off_misc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this CTA's pairs of tokens: pair P = blockIdx.x + i * gridDim.x holds rows
  // 2P and 2P + 1; an odd row count leaves the last pair one token short
  const int64_t npairs = (p.rows + 1) >> 1;
  const int np = static_cast<int>((npairs - 1 - blockIdx.x) / gridDim.x + 1);
  const bool short_tail =
      (p.rows & 1) && (blockIdx.x + static_cast<int64_t>(np - 1) * gridDim.x == npairs - 1);
  const int ntok = 2 * np - (short_tail ? 1 : 0);
  auto row_of = [&](int t) -> int64_t {
    return 2 * (blockIdx.x + static_cast<int64_t>(t >> 1) * gridDim.x) + (t & 1);
  };

  // the prologue stages P1, P2 and c in the (not yet used) T-tile region
  float* sp1 = reinterpret_cast<float*>(smem + off_b2);                 // 64 KB
  float* sp2 = reinterpret_cast<float*>(smem + off_b2 + 65536);         // 16 KB
  float* sc = reinterpret_cast<float*>(smem + off_b2 + 81920);          // 32 KB
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kBarXFull + i], kLoadWarps);
      mbar_init(&bars[kBarXEmpty + i], 1);
      mbar_init(&bars[kBarB2Full + i], 2 * kPostWarps);
      mbar_init(&bars[kBarB2Empty + i], 1);
    }
    mbar_init(&bars[kBarD1Full], 1);
    mbar_init(&bars[kBarD1Empty], kPostWarps);
    mbar_init(&bars[kBarD2Full], 1);
    mbar_init(&bars[kBarD2Empty], kPostWarps);
    for (int i = 0; i < kXSlots; ++i) mbar_init(&bars[kBarXMax + i], kLoadWarps);
    for (int i = 0; i < 4; ++i) mbar_init(&bars[kBarYMax + i], 4);
    mbar_init(&bars[kBarDrain], 1);
    mbar_init(&bars[kBarPrologue], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  grid_dep_wait();
  grid_dep_launch();
  __syncthreads();
  if (threadIdx.x == 32) {
    const uint32_t bytes = 65536 + 16384 + (p.chan != nullptr ? 32768 : 0);
    mbar_arrive_expect_tx(&bars[kBarPrologue], bytes);
    for (int i = 0; i < 4; ++i)
      bulk_load(reinterpret_cast<uint8_t*>(sp1) + 16384 * i,
                reinterpret_cast<const uint8_t*>(p.p1) + 16384 * i, 16384, &bars[kBarPrologue]);
    bulk_load(sp2, p.p2, 16384, &bars[kBarPrologue]);
    if (p.chan != nullptr)
      for (int i = 0; i < 2; ++i)
        bulk_load(reinterpret_cast<uint8_t*>(sc) + 16384 * i,
                  reinterpret_cast<const uint8_t*>(p.chan) + 16384 * i, 16384, &bars[kBarPrologue]);
  }
  bool ok = mbar_wait_bounded(&bars[kBarPrologue], 0, abort_flag, p.status, kDevTimeoutProducer);

  // ---- prologue: power-of-two normalizers of P1 and P2
  {
    float m1a = 0.0f, m1b = 0.0f, m2 = 0.0f;
    for (int i = threadIdx.x; i < kN1 * kN1 / 4; i += kThreadsTc) {
      const float4 v = reinterpret_cast<const float4*>(sp1)[i];
      m1a = fmaxf(m1a, fmaxf(fabsf(v.x), fabsf(v.y)));
      m1b = fmaxf(m1b, fmaxf(fabsf(v.z), fabsf(v.w)));
    }
    for (int i = threadIdx.x; i < kN2 * kN2 / 4; i += kThreadsTc) {
      const float4 v = reinterpret_cast<const float4*>(sp2)[i];
      m2 = fmaxf(m2, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    const float m1 = warp_max(fmaxf(m1a, m1b));
    m2 = warp_max(m2);
    if (lane == 0) {
      pmax[2 * warp] = m1;
      pmax[2 * warp + 1] = m2;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  float rho1, rho2;
  {
    float m1 = 0.0f, m2 = 0.0f;
    for (int w = 0; w < kThreadsTc / 32; ++w) {
      m1 = fmaxf(m1, pmax[2 * w]);
      m2 = fmaxf(m2, pmax[2 * w + 1]);
    }
    rho1 = pow2_normalizer(m1, 0);
    rho2 = pow2_normalizer(m2, 0);
  }
  const int q = warp & 3;                              // TMEM lane quadrant
  const uint32_t quad_off = static_cast<uint32_t>(32 * q) << 16;
  float cf[32];                                        // loaders: channel factors
  float cfmax = 0.0f;
  if (warp >= 1 && warp <= kLoadWarps) {
    const int h = (warp - 1) >> 2;
    // P1^T (rows c = lane row, K = a in [64h, 64h+64)) -> TMEM, hi | lo
    const int c = 32 * q + lane;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t hw[16], lw[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int a = 64 * h + 32 * hf + 2 * j;
        split_pair(sp1[a * kN1 + c] * rho1, sp1[(a + 1) * kN1 + c] * rho1, hw[j], lw[j]);
      }
      tmem_st_32x32b_x16(tmem + quad_off + kColP1 + 32 * h + 16 * hf, hw);
      tmem_st_32x32b_x16(tmem + quad_off + kColP1 + 64 + 32 * h + 16 * hf, lw);
    }
    // channel factors of the 32 values this thread loads per token: rows
    // g and g+8 of its 16-lane half, b in [8c', 8c'+8) and [32+8c', 32+8c'+8)
    const int g = lane >> 2, cq = lane & 3;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int a = 32 * q + 16 * h + g + 8 * rr;
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float f = 1.0f;
          if (p.chan != nullptr) {
            const float cv = sc[a * kN2 + 32 * u + 8 * cq + e];
            f = p.chan_multiply ? cv : __frcp_rn(cv);    // = 1/c, correctly rounded
          }
          cf[16 * rr + 8 * u + e] = f;
          cfmax = fmaxf(cfmax, fabsf(f));
        }
    }
    tmem_st_wait();
  } else if (warp > kLoadWarps) {
    // [P2 hi | P2 lo] as stage 1's B: row n, K index kk holds P2[perm_b(kk)][n % 64]
    const int idx = threadIdx.x - 32 * (1 + kLoadWarps);
#pragma unroll 1
    for (int cid = idx; cid < 128 * 8; cid += 32 * kPostWarps) {
      const int n = cid & 127, ch = cid >> 7, d = n & 63;
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        split_pair(sp2[perm_b(8 * ch + 2 * e) * kN2 + d] * rho2,
                   sp2[perm_b(8 * ch + 2 * e + 1) * kN2 + d] * rho2, hi[e], lo[e]);
      const uint32_t* w = (n < 64) ? hi : lo;
      *reinterpret_cast<uint4*>(smem + off_bp2 + sw128(n, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();                                     // the staging region is free again
  tc_fence_after();
  if (*abort_flag) ok = false;

  auto wait = [&](int b, uint32_t parity, int32_t code) -> bool {
    return mbar_wait_bounded(&bars[b], parity, abort_flag, p.status, code);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t bp2 = smem_u32(smem + off_bp2);
      // S1(t) then, from t = 2, one half of S2 of pair t/2 - 1
      for (int t = 0; t < 2 * np && ok; ++t) {
        if (t < ntok) {
          const int j = t & 1;
          if (!(ok = wait(kBarXFull + j, (t >> 1) & 1, kDevTimeoutMma))) break;
          if (t >= 1 && !(ok = wait(kBarD1Empty, (t - 1) & 1, kDevTimeoutMma))) break;
          tc_fence_after();
          const uint32_t a = tmem + kColA1 + 64 * j;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f16_ts(tmem + kColD1, a + 8 * k, smem_desc_kmajor(bp2 + 32 * k, 128), kIdescS1, k > 0);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f16_ts(tmem + kColD1, a + 32 + 8 * k, smem_desc_kmajor(bp2 + 32 * k, 128), kIdescS1, 1);
          mma_commit(&bars[kBarXEmpty + j]);
          mma_commit(&bars[kBarD1Full]);
        }
        const bool last = (t == 2 * np - 1);
        for (int rep = 0; rep < (last ? 3 : 1) && ok; ++rep) {
          // after S1(t): S2 half (t & 1) of pair t/2 - 1; after the last
          // token also both halves of the last pair
          const int pr = last ? (rep == 0 ? (t >> 1) - 1 : np - 1) : (t >> 1) - 1;
          const int half = last ? (rep == 0 ? 1 : rep - 1) : (t & 1);
          if (pr < 0) continue;
          const int sl = pr & 1;
          if (half == 0) {
            if (!(ok = wait(kBarB2Full + sl, (pr >> 1) & 1, kDevTimeoutMma))) break;
            if (pr >= 1 && !(ok = wait(kBarD2Empty, (pr - 1) & 1, kDevTimeoutMma))) break;
            tc_fence_after();
          }
          const uint32_t bh = smem_u32(smem + off_b2 + sl * kB2Slot), bl = bh + 2 * kTokT;
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) {
            const int s = 4 * half + s4;
            const uint64_t dh = smem_desc_mn_sw128(bh + 2048 * s, kTokT);
            const uint64_t dl = smem_desc_mn_sw128(bl + 2048 * s, kTokT);
            mma_f16_ts(tmem + kColD2, tmem + kColP1 + 8 * s, dh, kIdescS2, s > 0);
            mma_f16_ts(tmem + kColD2, tmem + kColP1 + 8 * s, dl, kIdescS2, 1);
            mma_f16_ts(tmem + kColD2, tmem + kColP1 + 64 + 8 * s, dh, kIdescS2, 1);
          }
          if (half == 1) {
            mma_commit(&bars[kBarB2Empty + sl]);
            mma_commit(&bars[kBarD2Full]);
          }
        }
      }
      mma_commit(&bars[kBarDrain]);
      mbar_wait_bounded(&bars[kBarDrain], 0, abort_flag, p.status, kDevTimeoutDrain,
                        kDrainLimitNs);
    }
  } else if (warp <= kLoadWarps) {
    // ------------------------------------------------------------ loaders
    const int h = (warp - 1) >> 2, wi = warp - 1;
    const int g = lane >> 2, cq = lane & 3;
    const int a0 = 32 * q + 16 * h + g;                // rows a0 and a0 + 8
    const uint32_t lanes16 = static_cast<uint32_t>(32 * q + 16 * h) << 16;
    auto load = [&](uint4 (&b)[4], int t) {
      const __half* base = p.src + row_of(t) * p.ld;
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int u = 0; u < 2; ++u)
          b[2 * rr + u] = __ldg(reinterpret_cast<const uint4*>(
              base + (a0 + 8 * rr) * kN2 + 32 * u + 8 * cq));
    };
    // This warp's bound of max|x/c| for token t (its max|x| times its largest
    // channel factor), posted to the token's exchange slot.  The normalizer
    // sigma of a token keeps sigma |x/c| below 2^8 and is within a factor
    // max(c)/min(c) of tight.
    auto post_max = [&](const uint4 (&b)[4], int t) {
      __half2 m0 = __habs2(reinterpret_cast<const __half2*>(&b[0])[0]);
      __half2 m1 = __habs2(reinterpret_cast<const __half2*>(&b[1])[0]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = (i < 2 ? 1 : 0); e < 4; ++e) {
          const __half2 v = __habs2(reinterpret_cast<const __half2*>(&b[i])[e]);
          if ((i + e) & 1) m1 = __hmax2(m1, v); else m0 = __hmax2(m0, v);
        }
      const float2 mf = __half22float2(__hmax2(m0, m1));
      const float m = warp_max(fmaxf(mf.x, mf.y) * cfmax);
      const int xs = t & (kXSlots - 1);
      if (lane == 0) {
        red_x[xs * 8 + wi] = m;
        mbar_arrive(&bars[kBarXMax + xs]);
      }
    };
    uint4 cur[4], nxt[4];
    if (ok) {
      load(cur, 0);
      if (ntok > 1) load(nxt, 1);
      post_max(cur, 0);
    }
    for (int t = 0; t < ntok && ok; ++t) {
      const int xs = t & (kXSlots - 1);
      if (!(ok = wait(kBarXMax + xs, (t >> 3) & 1, kDevTimeoutProducer))) break;
      const float mx = fmaxf(fmaxf(fmaxf(red_x[xs * 8 + 0], red_x[xs * 8 + 1]),
                                   fmaxf(red_x[xs * 8 + 2], red_x[xs * 8 + 3])),
                             fmaxf(fmaxf(red_x[xs * 8 + 4], red_x[xs * 8 + 5]),
                                   fmaxf(red_x[xs * 8 + 6], red_x[xs * 8 + 7])));
      const float sg = pow2_normalizer(mx, 7);
      // registers of the 16x256b stores: block k, lane half rr, column pair
      // e: K indices 16k + 4cq + 2e + {0, 1} of row a0 + 8rr, i.e. b =
      // 32(k>>1) + 8cq + 4(k&1) + 2e + {0, 1}: elements 4(k&1) + 2e, +1 of
      // load cur[2rr + (k>>1)].  Two stores of two blocks each.
      const uint32_t col = tmem + lanes16 + kColA1 + 64 * (t & 1);
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        uint32_t hw[8], lw[8];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int k = 2 * k2 + kk;
              const int li = 2 * rr + (k >> 1), el = 4 * (k & 1) + 2 * e;
              const float2 f = __half22float2(reinterpret_cast<const __half2*>(&cur[li])[el >> 1]);
              const int ci = 8 * li + el;
              float v0, v1;
              f2_unpack(f2_fma(f2_pack(f.x, f.y), f2_pack(cf[ci] * sg, cf[ci + 1] * sg),
                               f2_pack(0.0f, 0.0f)), v0, v1);
              split_pair(v0, v1, hw[4 * kk + 2 * rr + e], lw[4 * kk + 2 * rr + e]);
            }
        if (k2 == 0 && t >= 2 &&
            !(ok = wait(kBarXEmpty + (t & 1), ((t >> 1) - 1) & 1, kDevTimeoutProducer)))
          break;
        if (k2 == 0) tc_fence_after();
        tmem_st_16x256b_x2(col + 16 * k2, hw);
        tmem_st_16x256b_x2(col + 32 + 16 * k2, lw);
      }
      if (!ok) break;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarXFull + (t & 1)]);
      // rotate the prefetch buffers, fetch token t + 2, post token t + 1's max
#pragma unroll
      for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
      if (t + 2 < ntok) load(nxt, t + 2);
      if (t + 1 < ntok) post_max(cur, t + 1);
    }
  } else {
    // ------------------------------------------------------------ converters + epilogue
    const int h = (warp - 1 - kLoadWarps) >> 2;
    const int r = 32 * q + lane;                       // TMEM lane: row a, then row c
    for (int t = 0; t < 2 * np && ok; ++t) {
      const int pr = t >> 1, j = t & 1, sl = pr & 1;
      if (t < ntok) {
        // ---- convert token t: T = D1[:, :64] + D1[:, 64:] -> hi/lo T tiles
        if (!(ok = wait(kBarD1Full, t & 1, kDevTimeoutWiden))) break;
        tc_fence_after();
        uint32_t u[32], w[32];
        tmem_ld_32x32b_x32(tmem + quad_off + kColD1 + 32 * h, u);
        tmem_ld_32x32b_x32(tmem + quad_off + kColD1 + 64 + 32 * h, w);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarD1Empty]);
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float t0, t1;
          f2_unpack(f2_add(f2_pack(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1])),
                           f2_pack(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]))),
                    t0, t1);
          split_pair(t0, t1, hw[i], lw[i]);
        }
        if (j == 0 && pr >= 2 &&
            !(ok = wait(kBarB2Empty + sl, ((pr >> 1) - 1) & 1, kDevTimeoutWiden)))
          break;
        uint8_t* th = smem + off_b2 + sl * kB2Slot + j * kTokT;
        uint8_t* tl = th + 2 * kTokT;
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4) {
          const int ch = 4 * h + m4;
          *reinterpret_cast<uint4*>(th + sw128(r, ch)) =
              make_uint4(hw[4 * m4], hw[4 * m4 + 1], hw[4 * m4 + 2], hw[4 * m4 + 3]);
          *reinterpret_cast<uint4*>(tl + sw128(r, ch)) =
              make_uint4(lw[4 * m4], lw[4 * m4 + 1], lw[4 * m4 + 2], lw[4 * m4 + 3]);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarB2Full + sl]);   // a short pair's missing token too
      // ---- after the second token of pair pr: the epilogue of pair pr - 1,
      // and after the last token that of the last pair
      const int nepi = (t == 2 * np - 1) ? 2 : (j == 1 ? 1 : 0);
      for (int ie = 0; ie < nepi && ok; ++ie) {
        const int ep = (ie == 0) ? pr - 1 : np - 1;
        if (ep < 0) continue;
        const int te = 2 * ep + h;                       // this warp's token
        if (!(ok = wait(kBarD2Full, ep & 1, kDevTimeoutEpilogue))) break;
        tc_fence_after();
        uint32_t y[64];
        tmem_ld_32x32b_x32(tmem + quad_off + kColD2 + 64 * h,
                           *reinterpret_cast<uint32_t(*)[32]>(&y[0]));
        tmem_ld_32x32b_x32(tmem + quad_off + kColD2 + 64 * h + 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&y[32]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarD2Empty]);
        if (te >= ntok) continue;                        // the missing token of a short pair
        float am8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) am8[i] = fabsf(__uint_as_float(y[i]));
#pragma unroll
        for (int i = 8; i < 64; ++i) am8[i & 7] = fmaxf(am8[i & 7], fabsf(__uint_as_float(y[i])));
        float am = fmaxf(fmaxf(fmaxf(am8[0], am8[1]), fmaxf(am8[2], am8[3])),
                         fmaxf(fmaxf(am8[4], am8[5]), fmaxf(am8[6], am8[7])));
        am = warp_max(am);
        const int ys = ep & 1;
        if (lane == 0) {
          red_y[(ys * 2 + h) * 4 + q] = am;
          mbar_arrive(&bars[kBarYMax + 2 * ys + h]);
        }
        if (!(ok = wait(kBarYMax + 2 * ys + h, (ep >> 1) & 1, kDevTimeoutEpilogue))) break;
        am = fmaxf(fmaxf(red_y[(ys * 2 + h) * 4 + 0], red_y[(ys * 2 + h) * 4 + 1]),
                   fmaxf(red_y[(ys * 2 + h) * 4 + 2], red_y[(ys * 2 + h) * 4 + 3]));
        // the token's normalizer, from the loaders' exchange slot (still
        // intact: the loaders reuse it only eight tokens later)
        const int xs = te & (kXSlots - 1);
        if (!(ok = wait(kBarXMax + xs, (te >> 3) & 1, kDevTimeoutEpilogue))) break;
        const float mx = fmaxf(fmaxf(fmaxf(red_x[xs * 8 + 0], red_x[xs * 8 + 1]),
                                     fmaxf(red_x[xs * 8 + 2], red_x[xs * 8 + 3])),
                               fmaxf(fmaxf(red_x[xs * 8 + 4], red_x[xs * 8 + 5]),
                                     fmaxf(red_x[xs * 8 + 6], red_x[xs * 8 + 7])));
        const float unscale = (1.0f / pow2_normalizer(mx, 7)) * (1.0f / rho1) * (1.0f / rho2);
        const float rcp = (am > 0.0f) ? 7.0f / (p.clip_ratio * am) : 0.0f;
        const int64_t row = row_of(te);
        if (r == 0) p.scales[row] = ((p.clip_ratio * am) / 7.0f) * unscale;
        uint32_t wd[8];
#pragma unroll
        for (int jw = 0; jw < 8; ++jw) wd[jw] = code_word<CLIP>(&y[8 * jw], rcp);
        uint4* cdst = reinterpret_cast<uint4*>(p.codes + row * (kN1 * kN2 / 2) + r * 32);
        cdst[0] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        cdst[1] = make_uint4(wd[4], wd[5], wd[6], wd[7]);
        if (p.rot_debug != nullptr) {
          float4* dd = reinterpret_cast<float4*>(p.rot_debug + row * (kN1 * kN2) + r * 64);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            dd[i] = make_float4(__uint_as_float(y[4 * i]) * unscale,
                                __uint_as_float(y[4 * i + 1]) * unscale,
                                __uint_as_float(y[4 * i + 2]) * unscale,
                                __uint_as_float(y[4 * i + 3]) * unscale);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool kron_tc_supported(const RowJob& job) {
  const qr_rotation& rot = *job.rot;
  return rot.n1 == kN1 && rot.n2 == kN2 && job.n_out == 0 && job.Kp == kN1 * kN2 &&
         job.zeros == nullptr && (reinterpret_cast<uintptr_t>(job.src) % 16 == 0) &&
         (reinterpret_cast<uintptr_t>(rot.p1) % 16 == 0) &&
         (reinterpret_cast<uintptr_t>(rot.p2) % 16 == 0) &&
         (reinterpret_cast<uintptr_t>(rot.chan_scale) % 16 == 0) &&
         (job.ld % 8 == 0) && (reinterpret_cast<uintptr_t>(job.codes) % 16 == 0) &&
         (job.rot_debug == nullptr || reinterpret_cast<uintptr_t>(job.rot_debug) % 16 == 0);
}

qr_status launch_kron_tc(const RowJob& job, cudaStream_t stream) {
  const qr_rotation& rot = *job.rot;
  if (job.rows == 0) return QR_OK;
  KronTcParams p{};
  p.src = reinterpret_cast<const __half*>(job.src);
  p.rows = job.rows;
  p.ld = job.ld;
  p.p1 = rot.p1;
  p.p2 = rot.p2;
  p.chan = rot.chan_scale;
  p.chan_multiply = rot.chan_mode == QR_CHAN_MULTIPLY;
  p.clip_ratio = rot.clip_ratio;
  p.codes = job.codes;
  p.scales = job.scales;
  p.rot_debug = job.rot_debug;
  p.status = device_status_word();
  if (p.status == nullptr) return QR_ERR_CUDA;
  const int64_t npairs = (job.rows + 1) / 2;
  const int grid = static_cast<int>(std::min<int64_t>(npairs, sm_count()));
  cudaError_t e;
  if (rot.clip_ratio < 1.0f) {
    e = cudaFuncSetAttribute(kron_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
    if (e == cudaSuccess)
      e = launch_pdl(kron_tc_kernel<true>, dim3(grid), dim3(kThreadsTc), kSmemTc, stream, 1, p);
  } else {
    e = cudaFuncSetAttribute(kron_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
    if (e == cudaSuccess)
      e = launch_pdl(kron_tc_kernel<false>, dim3(grid), dim3(kThreadsTc), kSmemTc, stream, 1, p);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
