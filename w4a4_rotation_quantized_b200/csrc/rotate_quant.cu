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

#include "qr_device.cuh"
#include "qr_internal.h"

namespace qr {

namespace {

constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

// Nibble of round_half_even(v * r), optionally clamped to +-7.  Adding
// 1.5*2^23 leaves a float whose unit in the last place is 1, so the single
// rounding of the fused multiply-add is round-to-nearest-even of the exact
// product; the integer then sits in the low mantissa bits, and its low four
// bits are its two's-complement nibble.
template <bool CLIP>
__device__ __forceinline__ uint32_t quant_nibble(float v, float r) {
  float t = fmaf(v, r, kRoundMagic);
  if (CLIP) t = fminf(fmaxf(t, kRoundMagic - 7.0f), kRoundMagic + 7.0f);
  return __float_as_uint(t) & 0xFu;
}

__device__ __forceinline__ void row_barrier(int group, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(group + 1), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 u;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
               : "l"(p));
  return u;
}

// Inverse of the binary-reflected Gray code on 8 bits.
__device__ __forceinline__ int gray_inverse(int g) {
  g ^= g >> 1;
  g ^= g >> 2;
  g ^= g >> 4;
  return g;
}

struct WhtParams {
  const __half* src;
  int64_t rows, ld;
  int32_t K, Kr, Kp, n_out;
  const int32_t* outlier_idx;
  int32_t log_block;          // butterflies on index bits [0, log_block)
  int32_t gsr;                // sequency order within blocks (log_block <= 8)
  int32_t vec_ok;             // 16-byte loads allowed (aligned, no gather)
  int32_t warps_per_row, rows_per_cta;
  float clip_ratio, inv_sqrt_block;
  uint8_t* codes;
  float* scales;
  __half* out16;
  float* rot_debug;
  // shared memory carve-up (byte offsets)
  int32_t off_red, off_xbuf, off_gsr, off_kept, off_idx;
};

// Builds, in shared memory, kept[e] = the source column of rotated column e
// (0xFFFF = none), from the strictly ascending outlier index list.  Malformed
// lists never write outside [0, Kr).
__device__ void build_kept_table(const int32_t* __restrict__ outlier_idx, int n_out, int K,
                                 int Kr, uint16_t* kept, int32_t* sidx) {
  for (int i = threadIdx.x; i < n_out; i += blockDim.x) sidx[i] = outlier_idx[i];
  for (int e = threadIdx.x; e < Kr; e += blockDim.x) kept[e] = 0xFFFFu;
  __syncthreads();
  for (int c = threadIdx.x; c < K; c += blockDim.x) {
    int lo = 0, hi = n_out;            // lo = number of outliers < c
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sidx[mid] < c) lo = mid + 1; else hi = mid;
    }
    const bool is_out = lo < n_out && sidx[lo] == c;
    const int pos = c - lo;
    if (!is_out && pos >= 0 && pos < Kr) kept[pos] = static_cast<uint16_t>(c);
  }
  __syncthreads();
}

template <int CPW, bool CLIP>
__global__ void __launch_bounds__(256) wht_rotate_quant_kernel(const WhtParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int W = p.warps_per_row;
  const int rg = warp / W;
  const int wr = warp - rg * W;
  const bool gather = p.n_out > 0;

  uint16_t* kept = reinterpret_cast<uint16_t*>(smem + p.off_kept);
  if (gather) build_kept_table(p.outlier_idx, p.n_out, p.K, p.Kr, kept,
                               reinterpret_cast<int32_t*>(smem + p.off_idx));

  const int64_t row = static_cast<int64_t>(blockIdx.x) * p.rows_per_cta + rg;
  if (rg >= p.rows_per_cta || row >= p.rows) return;
  const __half* srow = p.src + row * p.ld;
  const int nthr_row = W * 32;

  // QUIK outlier columns, copied through unchanged.
  if (gather && p.out16 != nullptr) {
    for (int j = wr * 32 + lane; j < p.n_out; j += nthr_row) {
      const int c = __ldg(p.outlier_idx + j);
      p.out16[row * p.n_out + j] = (c >= 0 && c < p.K) ? srow[c] : __float2half(0.0f);
    }
  }

  // ---- load (gather + zero padding), fp16 -> fp32
  float v[CPW][8];
#pragma unroll
  for (int j = 0; j < CPW; ++j) {
    const int e0 = (wr * CPW + j) * 256 + lane * 8;
    if (!gather && p.vec_ok && e0 + 8 <= p.Kr) {
      const uint4 u = ld_stream_v4(srow + e0);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(h[q]);
        v[j][2 * q] = f.x;
        v[j][2 * q + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i;
        float x = 0.0f;
        if (e < p.Kr) {
          const int c = gather ? static_cast<int>(kept[e]) : e;
          if (c < p.K) x = __half2float(srow[c]);
        }
        v[j][i] = x;
      }
    }
  }

  const int lb = p.log_block;
  // ---- butterflies on bits 0..2 (inside a thread)
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    if (s < lb) {
#pragma unroll
      for (int j = 0; j < CPW; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (!(i & (1 << s))) {
            const float a = v[j][i], b = v[j][i | (1 << s)];
            v[j][i] = a + b;
            v[j][i | (1 << s)] = a - b;
          }
    }
  }
  // ---- bits 3..7 (across lanes): lower half keeps a+b, upper half a-b
#pragma unroll
  for (int s = 3; s < 8; ++s) {
    if (s < lb) {
      const int m = 1 << (s - 3);
      const float sg = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
      for (int j = 0; j < CPW; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float o = __shfl_xor_sync(0xffffffffu, v[j][i], m);
          v[j][i] = fmaf(sg, v[j][i], o);
        }
    }
  }
  // ---- bits 8 .. 8+log2(CPW)-1 (across this thread's chunks)
#pragma unroll
  for (int t = 0; (1 << t) < CPW; ++t) {
    if (8 + t < lb) {
#pragma unroll
      for (int j = 0; j < CPW; ++j)
        if (!(j & (1 << t))) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = v[j][i], b = v[j | (1 << t)][i];
            v[j][i] = a + b;
            v[j | (1 << t)][i] = a - b;
          }
        }
    }
  }
  // ---- remaining bits: across the warps of the row, through shared memory
  {
    constexpr int LC = (CPW >= 16) ? 4 : (CPW >= 8) ? 3 : (CPW >= 4) ? 2 : (CPW >= 2) ? 1 : 0;
    float* xb = reinterpret_cast<float*>(smem + p.off_xbuf) + static_cast<size_t>(rg) * W * CPW * 256;
    for (int t = 0; 8 + LC + t < lb; ++t) {
      float* mine = xb + static_cast<size_t>(wr) * CPW * 256;
      float* peer = xb + static_cast<size_t>(wr ^ (1 << t)) * CPW * 256;
#pragma unroll
      for (int j = 0; j < CPW; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) mine[(j * 8 + i) * 32 + lane] = v[j][i];
      row_barrier(rg, nthr_row);
      const bool upper = (wr >> t) & 1;
#pragma unroll
      for (int j = 0; j < CPW; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float o = peer[(j * 8 + i) * 32 + lane];
          v[j][i] = upper ? (o - v[j][i]) : (v[j][i] + o);
        }
      row_barrier(rg, nthr_row);
    }
  }

  // ---- row absmax
  float am = 0.0f;
#pragma unroll
  for (int j = 0; j < CPW; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(v[j][i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  if (W > 1) {
    float* red = reinterpret_cast<float*>(smem + p.off_red) + rg * W;
    if (lane == 0) red[wr] = am;
    row_barrier(rg, nthr_row);
    am = 0.0f;
    for (int w = 0; w < W; ++w) am = fmaxf(am, red[w]);
  }

  // s = alpha * max|x'| / 7 with x' = (unscaled butterfly output) / sqrt(b);
  // the codes use the unscaled values times r = 7 / (alpha * max).
  const float s = (p.clip_ratio * (am * p.inv_sqrt_block)) / 7.0f;
  const float r = (am > 0.0f) ? 7.0f / (p.clip_ratio * am) : 0.0f;
  if (wr == 0 && lane == 0) p.scales[row] = s;

  uint8_t* crow = p.codes + row * (p.Kp / 2);
  if (!p.gsr) {
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int e0 = (wr * CPW + j) * 256 + lane * 8;
      if (e0 < p.Kp) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) word |= quant_nibble<CLIP>(v[j][i], r) << (4 * i);
        *reinterpret_cast<uint32_t*>(crow + e0 / 2) = word;
        if (p.rot_debug != nullptr) {
          float* d = p.rot_debug + row * p.Kp + e0;
#pragma unroll
          for (int i = 0; i < 8; ++i) d[i] = v[j][i] * p.inv_sqrt_block;
        }
      }
    }
  } else {
    // Natural Hadamard position q of a chunk -> sequency output position.
    const int bmask = (1 << lb) - 1;
    int pos[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = lane * 8 + i;
      const int n = q & bmask;
      const int rev = lb ? static_cast<int>(__brev(static_cast<unsigned>(n)) >> (32 - lb)) : 0;
      pos[i] = (q & ~bmask) + gray_inverse(rev);
    }
    uint8_t* g = smem + p.off_gsr + static_cast<size_t>(rg) * p.Kp;
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int c0 = (wr * CPW + j) * 256;
      if (c0 + lane * 8 < p.Kp) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          g[c0 + pos[i]] = static_cast<uint8_t>(quant_nibble<CLIP>(v[j][i], r));
          if (p.rot_debug != nullptr)
            p.rot_debug[row * p.Kp + c0 + pos[i]] = v[j][i] * p.inv_sqrt_block;
        }
      }
    }
    row_barrier(rg, nthr_row);
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int e0 = (wr * CPW + j) * 256 + lane * 8;
      if (e0 < p.Kp) {
        const uint32_t lo = *reinterpret_cast<const uint32_t*>(g + e0);
        const uint32_t hi = *reinterpret_cast<const uint32_t*>(g + e0 + 4);
        const uint32_t plo = (lo & 0xFu) | ((lo >> 4) & 0xF0u) | ((lo >> 8) & 0xF00u) |
                             ((lo >> 12) & 0xF000u);
        const uint32_t phi = (hi & 0xFu) | ((hi >> 4) & 0xF0u) | ((hi >> 8) & 0xF00u) |
                             ((hi >> 12) & 0xF000u);
        *reinterpret_cast<uint32_t*>(crow + e0 / 2) = plo | (phi << 16);
      }
    }
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

template <int CPW, bool CLIP>
cudaError_t launch_wht(const WhtParams& p, int grid, int threads, size_t smem, cudaStream_t s) {
  auto k = wht_rotate_quant_kernel<CPW, CLIP>;
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  k<<<grid, threads, smem, s>>>(p);
  return cudaGetLastError();
}

template <bool CLIP>
cudaError_t dispatch_cpw(int cpw, const WhtParams& p, int grid, int threads, size_t smem,
                         cudaStream_t s) {
  switch (cpw) {
    case 1: return launch_wht<1, CLIP>(p, grid, threads, smem, s);
    case 2: return launch_wht<2, CLIP>(p, grid, threads, smem, s);
    case 4: return launch_wht<4, CLIP>(p, grid, threads, smem, s);
    case 8: return launch_wht<8, CLIP>(p, grid, threads, smem, s);
    default: return launch_wht<16, CLIP>(p, grid, threads, smem, s);
  }
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
  const int block = (rot.kind == QR_ROT_NONE) ? 1 : rot.block;
  p.log_block = ilog2(block);
  p.gsr = rot.kind == QR_ROT_GSR;
  p.vec_ok = job.n_out == 0 && (reinterpret_cast<uintptr_t>(job.src) % 16 == 0) && (job.ld % 8 == 0);
  p.clip_ratio = rot.clip_ratio;
  p.inv_sqrt_block = static_cast<float>(1.0 / std::sqrt(static_cast<double>(block)));
  p.codes = job.codes;
  p.scales = job.scales;
  p.out16 = reinterpret_cast<__half*>(job.out16);
  p.rot_debug = job.rot_debug;

  // Chunks per warp: enough registers to hold a whole block up to 4096
  // elements, and no more than 8 warps per row unless the row is long.
  const int chunks = (job.Kp + 255) / 256;
  int cpw = 1;
  if (p.log_block > 8) cpw = std::min(16, 1 << (p.log_block - 8));
  while (cpw < 16 && (chunks + cpw - 1) / cpw > 8) cpw *= 2;
  const int W = std::max(1, (chunks + cpw - 1) / cpw);
  if (W > 8 || job.Kp > 32768) return QR_ERR_UNSUPPORTED;
  const bool cross = p.log_block > 8 + ilog2(cpw);
  int R = cross ? 1 : std::max(1, 8 / W);
  if (job.rows < R) R = static_cast<int>(std::max<int64_t>(job.rows, 1));
  p.warps_per_row = W;
  p.rows_per_cta = R;

  size_t off = 0;
  p.off_red = static_cast<int32_t>(off);
  off = align_up(off + sizeof(float) * R * W, 16);
  p.off_xbuf = static_cast<int32_t>(off);
  if (cross) off = align_up(off + sizeof(float) * static_cast<size_t>(R) * W * cpw * 256, 16);
  p.off_gsr = static_cast<int32_t>(off);
  if (p.gsr) off = align_up(off + static_cast<size_t>(R) * job.Kp, 16);
  p.off_kept = static_cast<int32_t>(off);
  if (job.n_out > 0) off = align_up(off + sizeof(uint16_t) * job.Kr, 16);
  p.off_idx = static_cast<int32_t>(off);
  if (job.n_out > 0) off = align_up(off + sizeof(int32_t) * job.n_out, 16);
  if (off > static_cast<size_t>(max_smem_optin())) return QR_ERR_UNSUPPORTED;

  const int64_t grid64 = (job.rows + R - 1) / R;
  if (grid64 > 0x7FFFFFFF) return QR_ERR_UNSUPPORTED;
  const int threads = R * W * 32;
  const bool clip = rot.clip_ratio < 1.0f;
  cudaError_t e = clip ? dispatch_cpw<true>(cpw, p, static_cast<int>(grid64), threads, off, stream)
                       : dispatch_cpw<false>(cpw, p, static_cast<int>(grid64), threads, off, stream);
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

}  // namespace

qr_status launch_rotate_quant(const RowJob& job, cudaStream_t stream) {
  if (job.rows == 0) return QR_OK;
  if (job.rot->kind == QR_ROT_KRON) return launch_kron_rows(job, stream);
  return launch_wht_rows(job, stream);
}

}  // namespace qr
