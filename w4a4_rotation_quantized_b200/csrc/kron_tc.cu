// kron_tc.cu -- FlatQuant's Kronecker affine transform on fifth-generation
// tensor cores, fused with per-token 4-bit quantization.
//
// FlatQuant ("LLM量化新篇章：...FlatQuant的平坦之道", §2.3 and 模型架构):
// each row x (n1*n2 channels) is scaled per channel and transformed by two
// small matrices, Y = P1^T mat(x / c) P2, then quantized per token; the page
// fuses the two small matmuls with the quantization into one kernel.
//
// Here, per token, with mat(x) = X [128 x 64] (row a = x[64a .. 64a+63]):
//   stage 1  T  = X P2        MMA M = a (128), N = d (64), K = b (64)
//   stage 2  Y  = P1^T T      MMA M = c (128), N = d (64), K = a (128)
// Stage 2's B operand is T read "MN-major" (row a of T holds the 64 d's
// contiguously), so each thread writes its own TMEM row of T straight back to
// shared memory without a transpose.  fp16 operands carry ~11 bits; every
// fp32 operand is split into hi = fp16(v) and lo = fp16(v - hi), and each
// product is hi*hi + hi*lo + lo*hi accumulated in fp32 (relative error about
// 2^-22), which keeps the rotated rows well inside 1e-5 of the row norm.
//
// One CTA of 128 threads per SM, persistent over tokens; thread i owns TMEM
// lane i (row a in stage 1, row c in stage 2).  Supports n1 = 128, n2 = 64,
// no outlier split, 16-byte aligned rows; other shapes use the CUDA-core
// kernel.
#include <cuda_fp16.h>

#include <algorithm>

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

constexpr int kN1 = 128, kN2 = 64;
constexpr int kThreadsTc = 128;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23

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

// shared-memory carve-up (bytes, 1024-aligned regions)
constexpr int kA1 = kN1 * kN2 * 2;           // X hi or lo: 128 rows x 128 B
constexpr int kB1 = kN2 * kN2 * 2;           // P2^T hi or lo: 64 rows x 128 B
constexpr int kA2 = kN1 * kN1 * 2;           // P1^T hi or lo: two K-halves of 128 x 128 B
constexpr int kB2 = kN1 * kN2 * 2;           // T hi or lo: 128 K-rows x 128 B (MN-major)
constexpr int off_a1h = 0, off_a1l = off_a1h + kA1;
constexpr int off_b1h = off_a1l + kA1, off_b1l = off_b1h + kB1;
constexpr int off_a2h = off_b1l + kB1, off_a2l = off_a2h + kA2;
constexpr int off_b2h = off_a2l + kA2, off_b2l = off_b2h + kB2;
constexpr int off_bar = off_b2l + kB2;
constexpr int off_red = off_bar + 32;
constexpr int kSmemTc = off_red + 64 + 1024;

// byte offset of 16-byte chunk j of row r in a 128-byte-swizzled tile whose
// rows are 128 bytes (8-row atoms of 1 KB)
__device__ __forceinline__ int sw128(int r, int j) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Splits 8 fp32 values into fp16 hi and lo parts (hi = fp16(v), lo = fp16(v - hi)).
__device__ __forceinline__ void split8(const float (&v)[8], uint4& hi, uint4& lo) {
  float h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) h[i] = __half2float(__float2half_rn(v[i]));
  hi = make_uint4(pack_h2(h[0], h[1]), pack_h2(h[2], h[3]), pack_h2(h[4], h[5]),
                  pack_h2(h[6], h[7]));
  lo = make_uint4(pack_h2(v[0] - h[0], v[1] - h[1]), pack_h2(v[2] - h[2], v[3] - h[3]),
                  pack_h2(v[4] - h[4], v[5] - h[5]), pack_h2(v[6] - h[6], v[7] - h[7]));
}

// Descriptors: K-major SW128 (rows of 128 bytes, SBO 1 KB) and MN-major
// SW128 (128-byte rows along N, 8 K-rows per 1 KB atom, SBO 1 KB).
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t addr) {
  const uint64_t start = (addr >> 4) & 0x3FFFu;
  const uint64_t lbo = (8192u >> 4);          // stride between 64-wide N atoms (one atom here)
  const uint64_t sbo = (1024u >> 4);
  return start | (lbo << 16) | (sbo << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptors: D f32, A/B f16, M=128, N=64;
// stage 2 reads B MN-major (bit 16).
constexpr uint32_t kIdescS1 = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescS2 = kIdescS1 | (1u << 16);

template <bool CLIP>
__global__ void __launch_bounds__(kThreadsTc, 1) kron_tc_kernel(const KronTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + off_bar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 16);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + off_bar + 20);
  float* red = reinterpret_cast<float*>(smem + off_red);
  const int i = threadIdx.x;                 // = TMEM lane = row a / row c
  const int warp = i >> 5, lane = i & 31;

  // ---- constants: P2^T (rows d, K = b) and P1^T (rows c, K = a), hi/lo
  if (i < kN2) {
    for (int j = 0; j < 8; ++j) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = p.p2[(8 * j + e) * kN2 + i];     // P2[b][d = i]
      uint4 hi, lo;
      split8(v, hi, lo);
      *reinterpret_cast<uint4*>(smem + off_b1h + sw128(i, j)) = hi;
      *reinterpret_cast<uint4*>(smem + off_b1l + sw128(i, j)) = lo;
    }
  }
  for (int j = 0; j < 16; ++j) {                                         // a = 8j .. 8j+7
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = p.p1[(8 * j + e) * kN1 + i];      // P1[a][c = i]
    uint4 hi, lo;
    split8(v, hi, lo);
    const int half = j >> 3, jj = j & 7;
    *reinterpret_cast<uint4*>(smem + off_a2h + half * (kA2 / 2) + sw128(i, jj)) = hi;
    *reinterpret_cast<uint4*>(smem + off_a2l + half * (kA2 / 2) + sw128(i, jj)) = lo;
  }
  // per-thread channel factors of the 64 channels this thread owns (a = i)
  float cf[64];
#pragma unroll
  for (int b = 0; b < 64; ++b) {
    float c = 1.0f;
    if (p.chan != nullptr) {
      const float cv = p.chan[i * 64 + b];
      c = p.chan_multiply ? cv : 1.0f / cv;
    }
    cf[b] = c;
  }
  if (i == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t d1 = tmem, d2 = tmem + 64;

  uint32_t phase = 0;
  bool ok = true;
  // prefetch of this thread's 64 halves of the first token
  uint4 nx[8];
  int64_t row = blockIdx.x;
  if (row < p.rows) {
    const uint4* src = reinterpret_cast<const uint4*>(p.src + row * p.ld + i * 64);
#pragma unroll
    for (int q = 0; q < 8; ++q) nx[q] = __ldg(src + q);
  }
  for (; row < p.rows && ok; row += gridDim.x) {
    // ---- X row a = i, scaled, split, into the stage-1 A tiles
    uint4 cx[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) cx[q] = nx[q];
    const int64_t next = row + gridDim.x;
    if (next < p.rows) {
      const uint4* src = reinterpret_cast<const uint4*>(p.src + next * p.ld + i * 64);
#pragma unroll
      for (int q = 0; q < 8; ++q) nx[q] = __ldg(src + q);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const __half2* h = reinterpret_cast<const __half2*>(&cx[q]);
      float v[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        v[2 * e] = f.x * cf[8 * q + 2 * e];
        v[2 * e + 1] = f.y * cf[8 * q + 2 * e + 1];
      }
      uint4 hi, lo;
      split8(v, hi, lo);
      *reinterpret_cast<uint4*>(smem + off_a1h + sw128(i, q)) = hi;
      *reinterpret_cast<uint4*>(smem + off_a1l + sw128(i, q)) = lo;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- stage 1: T = X P2  (hi*hi + hi*lo + lo*hi)
    if (i == 0) {
      tc_fence_after();
      const uint32_t a_h = smem_u32(smem + off_a1h), a_l = smem_u32(smem + off_a1l);
      const uint32_t b_h = smem_u32(smem + off_b1h), b_l = smem_u32(smem + off_b1l);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t o = 32 * s;
        mma_f16(d1, smem_desc_kmajor(a_h + o, 128), smem_desc_kmajor(b_h + o, 128), kIdescS1, s > 0);
        mma_f16(d1, smem_desc_kmajor(a_h + o, 128), smem_desc_kmajor(b_l + o, 128), kIdescS1, 1);
        mma_f16(d1, smem_desc_kmajor(a_l + o, 128), smem_desc_kmajor(b_h + o, 128), kIdescS1, 1);
      }
      mma_commit(bar);
    }
    if (!(ok = mbar_wait_bounded(bar, phase, abort_flag, p.status, kDevTimeoutMma))) break;
    phase ^= 1;
    tc_fence_after();
    // ---- T row a = i (64 fp32) -> hi/lo, MN-major stage-2 B tiles
    {
      uint32_t t[64];
      uint32_t (&t0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&t[0]);
      uint32_t (&t1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&t[32]);
      tmem_ld_32x32b_x32(d1 + lane_off, t0);
      tmem_ld_32x32b_x32(d1 + lane_off + 32, t1);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(t[8 * j + e]);
        uint4 hi, lo;
        split8(v, hi, lo);
        *reinterpret_cast<uint4*>(smem + off_b2h + sw128(i, j)) = hi;
        *reinterpret_cast<uint4*>(smem + off_b2l + sw128(i, j)) = lo;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- stage 2: Y = P1^T T  (K = a in 8 steps of 16)
    if (i == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t ao = (s >> 2) * (kA2 / 2) + 32 * (s & 3);
        const uint32_t bo = 2048 * s;
        const uint64_t ah = smem_desc_kmajor(smem_u32(smem + off_a2h) + ao, 128);
        const uint64_t al = smem_desc_kmajor(smem_u32(smem + off_a2l) + ao, 128);
        const uint64_t bh = desc_mn_sw128(smem_u32(smem + off_b2h) + bo);
        const uint64_t bl = desc_mn_sw128(smem_u32(smem + off_b2l) + bo);
        mma_f16(d2, ah, bh, kIdescS2, s > 0);
        mma_f16(d2, ah, bl, kIdescS2, 1);
        mma_f16(d2, al, bh, kIdescS2, 1);
      }
      mma_commit(bar);
    }
    if (!(ok = mbar_wait_bounded(bar, phase, abort_flag, p.status, kDevTimeoutMma))) break;
    phase ^= 1;
    tc_fence_after();
    // ---- Y row c = i: absmax over the token, quantize, pack, store
    uint32_t y[64];
    uint32_t (&y0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&y[0]);
    uint32_t (&y1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&y[32]);
    tmem_ld_32x32b_x32(d2 + lane_off, y0);
    tmem_ld_32x32b_x32(d2 + lane_off + 32, y1);
    tmem_ld_wait();
    float am = 0.0f;
#pragma unroll
    for (int j = 0; j < 64; ++j) am = fmaxf(am, fabsf(__uint_as_float(y[j])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if (lane == 0) red[warp] = am;
    tc_fence_before();
    __syncthreads();
    am = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float s = (p.clip_ratio * am) / 7.0f;
    const float r = (am > 0.0f) ? 7.0f / (p.clip_ratio * am) : 0.0f;
    if (i == 0) p.scales[row] = s;
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float t = fmaf(__uint_as_float(y[8 * j + e]), r, kMagic);
        if (CLIP) t = fminf(fmaxf(t, kMagic - 7.0f), kMagic + 7.0f);
        word |= (__float_as_uint(t) & 0xFu) << (4 * e);
      }
      w[j] = word;
    }
    uint4* cdst = reinterpret_cast<uint4*>(p.codes + row * (kN1 * kN2 / 2) + i * 32);
    cdst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    cdst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    if (p.rot_debug != nullptr) {
      float* dd = p.rot_debug + row * (kN1 * kN2) + i * 64;
#pragma unroll
      for (int j = 0; j < 64; ++j) dd[j] = __uint_as_float(y[j]);
    }
    __syncthreads();     // red, A1, B2 are reused by the next token
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

bool kron_tc_supported(const RowJob& job) {
  const qr_rotation& rot = *job.rot;
  return rot.n1 == kN1 && rot.n2 == kN2 && job.n_out == 0 && job.Kp == kN1 * kN2 &&
         (reinterpret_cast<uintptr_t>(job.src) % 16 == 0) && (job.ld % 8 == 0) &&
         (reinterpret_cast<uintptr_t>(job.codes) % 16 == 0);
}

qr_status launch_kron_tc(const RowJob& job, cudaStream_t stream) {
  const qr_rotation& rot = *job.rot;
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
  const int grid = static_cast<int>(std::min<int64_t>(job.rows, sm_count()));
  cudaError_t e;
  if (rot.clip_ratio < 1.0f) {
    e = cudaFuncSetAttribute(kron_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
    if (e == cudaSuccess) kron_tc_kernel<true><<<grid, kThreadsTc, kSmemTc, stream>>>(p);
  } else {
    e = cudaFuncSetAttribute(kron_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
    if (e == cudaSuccess) kron_tc_kernel<false><<<grid, kThreadsTc, kSmemTc, stream>>>(p);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? QR_OK : QR_ERR_CUDA;
}

}  // namespace qr
